"""Full-size layer shapes on the GPU, checked on sampled outputs the oracle computes one by one.

The 7B FFN pair (with 0.1% outliers, 4096 tokens, r=64) and the 70B shapes run in
the same launch configuration as every other call.  The oracle encodes each whole
weight (about a minute for a 70B FFN matrix), then checks sampled Y columns, sampled
dX columns, and U, G, dA and dB in full; dA and dB come from the oracle's own chain
(u = X A^T, g = dY B), never from the GPU's saved factors.
"""
import numpy as np
import pytest
import torch

import bit_quantized_base_nf4_b200 as q
from bit_quantized_base_nf4_b200 import synthetic as syn
from oracle import nf4_oracle as O

pytestmark = pytest.mark.gpu

DEV = "cuda"
GROUP_W = O.BLOCK * O.GROUP          # weights per double-quant group


def _assert_tol(got, ref, what):
    nw, rw = O.rel_errors(got, ref)
    assert nw <= O.NORMWISE_TOL and rw <= O.ROWWISE_TOL, f"{what}: normwise {nw:.3e} rowwise {rw:.3e}"


def _np(t):
    return t.detach().cpu().numpy()


class Layer:
    def __init__(self, case: syn.LayerCase, with_bwd=True):
        self.case = case
        c = case
        self.W = c.weight()
        self.w = q.NF4Weight.empty(c.N, c.K)
        q.qlora_quantize_nf4_dq(self.W.to(DEV), self.w)
        self.X, self.A, self.B = c.x().to(DEV), c.lora_a().to(DEV), c.lora_b().to(DEV)
        self.ws = torch.empty(q.qlora_workspace_bytes(c.M, c.N, c.K, c.r), dtype=torch.uint8, device=DEV)
        self.Y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV)
        self.U = torch.empty(c.M, c.r, dtype=torch.bfloat16, device=DEV)
        q.qlora_lora_linear_fwd(self.w, self.X, self.A, self.B, c.r, c.scaling, self.Y, self.U, self.ws)
        if with_bwd:
            self.dY = c.dy().to(DEV)
            self.dX = torch.empty(c.M, c.K, dtype=torch.bfloat16, device=DEV)
            self.G = torch.empty(c.M, c.r, dtype=torch.bfloat16, device=DEV)
            q.qlora_lora_linear_bwd_dx(self.w, self.dY, self.A, self.B, c.r, c.scaling, self.dX, self.G, self.ws)
            self.dA = torch.empty(c.r, c.K, dtype=torch.float32, device=DEV)
            self.dB = torch.empty(c.N, c.r, dtype=torch.float32, device=DEV)
            q.qlora_lora_grad_AB(self.X, self.dY, self.U, self.G, c.r, c.scaling, self.dA, self.dB)
        q.qlora_sync_status()


def _check_full(layer: Layer, seed: int):
    """Full encode by the oracle: sampled Y columns, sampled dX columns, full U, G, dA, dB."""
    c = layer.case
    ref = O.quantize_nf4_dq(layer.W.numpy())
    assert np.array_equal(_np(layer.w.codes), ref["codes"])
    assert np.array_equal(_np(layer.w.scales), ref["scales"])
    assert np.array_equal(_np(layer.w.scales2).view(np.uint32), ref["scales2"].view(np.uint32))
    Wd = O.dequant(ref["codes"], ref["scales"], ref["scales2"]).reshape(c.N, c.K)
    rng = np.random.default_rng(seed)
    X, A, B, dY = (t.cpu() for t in (layer.X, layer.A, layer.B, layer.dY))
    rows = np.sort(rng.choice(c.N, 40, replace=False))
    Yref = O.lora_linear_fwd_rows(Wd, X, A, B, c.scaling, rows)
    _assert_tol(_np(layer.Y.float())[:, rows], Yref, f"{c.name} Y[:, sample]")
    cols = np.sort(rng.choice(c.K, 40, replace=False))
    dXref, gref = O.lora_linear_bwd_dx(Wd[:, cols], dY, A.float().numpy()[:, cols], B, c.scaling)
    _assert_tol(_np(layer.dX.float())[:, cols], dXref, f"{c.name} dX[:, sample]")
    _, uref = O.lora_linear_fwd(np.zeros((1, c.K)), X, A, B, c.scaling)
    _, gfull = O.lora_linear_bwd_dx(np.zeros((c.N, 1)), dY, A.float().numpy()[:, :1], B, c.scaling)
    _assert_tol(_np(layer.U.float()), uref, f"{c.name} U")
    _assert_tol(_np(layer.G.float()), gfull, f"{c.name} G")
    dAref, dBref = O.lora_grad_ab(X, dY, uref, gfull, c.scaling)
    _assert_tol(_np(layer.dA), dAref, f"{c.name} dA")
    _assert_tol(_np(layer.dB), dBref, f"{c.name} dB")


@pytest.mark.parametrize("idx", [0, 1], ids=["up-11008x4096", "down-4096x11008"])
def test_7b_ffn_full_size_sampled(idx):
    layer = Layer(syn.ffn7b_cases()[idx])
    _check_full(layer, 10 + idx)


def test_70b_attention_full_size_sampled():
    layer = Layer(syn.l70b_cases()[0])
    _check_full(layer, 20)


@pytest.mark.parametrize("idx", [1, 2], ids=["up-28672x8192", "down-8192x28672"])
def test_70b_ffn_full_size_sampled(idx):
    """Forward and backward of the 70B FFN matrices at 4096 tokens, r = 64."""
    layer = Layer(syn.l70b_cases()[idx])
    _check_full(layer, 30 + idx)
