"""Full-size layer shapes on the GPU, checked on sampled outputs the oracle computes one by one.

The 7B FFN pair (with 0.1% outliers, 4096 tokens, r=64) and the 70B shapes run in
the same launch configuration as every other call.
- The oracle encodes the whole weight where that stays within seconds.
- For the 70B FFN matrices it encodes only the 256-block groups that cover the
  sampled rows. A group is a contiguous run of 16384 weights, so encoding those runs
  on their own reproduces the full encode of them.
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


def _sampled_rows_oracle(W: torch.Tensor, rows, w_gpu: q.NF4Weight):
    """Oracle dequant of the given W rows by encoding the groups that cover them; also checks
    the GPU's codes, u8 scales and fp32 steps of those groups bit for bit."""
    N, K = W.shape
    flat = W.reshape(-1)
    codes_gpu, scales_gpu, s2_gpu = _np(w_gpu.codes), _np(w_gpu.scales), _np(w_gpu.scales2)
    out = np.empty((len(rows), K), np.float32)
    for i, r in enumerate(rows):
        lo, hi = r * K, (r + 1) * K
        g0, g1 = lo // GROUP_W, (hi - 1) // GROUP_W
        start, stop = g0 * GROUP_W, min((g1 + 1) * GROUP_W, N * K)
        ref = O.quantize_nf4_dq(flat[start:stop].numpy())
        assert np.array_equal(codes_gpu[start // 2:stop // 2], ref["codes"]), f"codes of row {r}"
        assert np.array_equal(scales_gpu[start // 64:stop // 64], ref["scales"]), f"scales of row {r}"
        assert np.array_equal(s2_gpu[g0:g1 + 1].view(np.uint32), ref["scales2"].view(np.uint32)), f"steps of row {r}"
        wd = O.dequant(ref["codes"], ref["scales"], ref["scales2"])
        out[i] = wd[lo - start:hi - start]
    return out


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
    _assert_tol(_np(layer.U.float()), uref, f"{c.name} U")
    _assert_tol(_np(layer.G.float()), gref, f"{c.name} G")
    dAref, dBref = O.lora_grad_ab(X, dY, layer.U.float().cpu(), layer.G.float().cpu(), c.scaling)
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
def test_70b_ffn_full_size_sampled_rows(idx):
    """Forward only; the oracle encodes just the groups of 24 sampled rows."""
    c = syn.l70b_cases()[idx]
    layer = Layer(c, with_bwd=False)
    rng = np.random.default_rng(30 + idx)
    rows = np.sort(np.concatenate([[0, c.N - 1], rng.choice(np.arange(1, c.N - 1), 22, replace=False)]))
    Wrows = _sampled_rows_oracle(layer.W, rows, layer.w)
    X, A, B = (t.cpu() for t in (layer.X, layer.A, layer.B))
    Yref = O.lora_linear_fwd_rows(Wrows, X, A, B[rows], c.scaling, np.arange(len(rows)))
    _assert_tol(_np(layer.Y.float())[:, rows], Yref, f"{c.name} Y[:, sample]")
