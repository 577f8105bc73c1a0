"""The Q8_0 route on the GPU against the oracle ("Training LoRA directly on GGUF
quantized weights" page, sections 1.1 and 2.2).

Encode and dequant are compared bit for bit with quantize_q8_0 / dequant_q8_0; the
layer (forward with the int8 x fp16-scale dequant in the GEMM main loop, dX with the
transposed dequant, dA and dB from the rank-r kernels) within the usual tolerance, with
the adapter term checked element by element and dA/dB from the oracle's own chain."""
import numpy as np
import pytest
import torch

import bit_quantized_base_nf4_b200 as q
from bit_quantized_base_nf4_b200 import synthetic as syn
from oracle import nf4_oracle as O

from test_gpu_parity import assert_adapter_term

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _assert_tol(got, ref, what):
    nw, rw = O.rel_errors(got, ref)
    assert nw <= O.NORMWISE_TOL and rw <= O.ROWWISE_TOL, f"{what}: normwise {nw:.3e} rowwise {rw:.3e}"


def _upload(ref, n_out, n_in):
    w = q.Q80Weight.empty(n_out, n_in, device=DEV)
    w.q.copy_(torch.from_numpy(np.ascontiguousarray(ref["q"])))
    w.d.copy_(torch.from_numpy(np.ascontiguousarray(ref["d"])))
    return w


def _weight(n_out, n_in, seed):
    W = syn.with_outliers(syn.normal_f32((n_out, n_in), 0.02, seed), 1e-3, 10.0, seed + 1)
    W[1, :64] = 0.0                        # all-zero blocks: d = 0, q = 0
    W[2, 32:64] *= 1e-7                    # a block whose scale is an fp16 subnormal
    W[3, 5] = 0.5                          # a block whose max is far above the rest
    return W


@pytest.mark.parametrize("n_out,n_in,seed", [(40, 704, 601), (256, 4096, 602), (7, 64, 603)])
def test_q8_0_encode_and_dequant_bit_exact(n_out, n_in, seed):
    W = _weight(n_out, n_in, seed) if n_out > 3 else syn.normal_f32((n_out, n_in), 0.02, seed)
    ref = O.quantize_q8_0(W.numpy())
    w = q.Q80Weight.empty(n_out, n_in, device=DEV)
    q.qlora_quantize_q8_0(W.to(DEV), w)
    q.qlora_sync_status()
    assert np.array_equal(w.q.cpu().numpy(), ref["q"]), "int8 codes differ"
    assert np.array_equal(w.d.cpu().numpy().view(np.uint16), ref["d"].view(np.uint16)), "fp16 scales differ"
    assert q.qlora_q8_0_packed_bytes(n_out * n_in) == O.q8_0_packed_bytes(n_out * n_in)
    want = O.dequant_q8_0(ref["q"], ref["d"])
    wo = _upload(ref, n_out, n_in)
    for dtype in (torch.float32, torch.bfloat16):
        out = torch.empty(n_out, n_in, dtype=dtype, device=DEV)
        q.qlora_dequant_q8_0(wo, out)
        q.qlora_sync_status()
        exp = want if dtype == torch.float32 else O.bf16_round(want)
        assert np.array_equal(out.float().cpu().numpy().reshape(-1).view(np.uint32), exp.view(np.uint32)), \
            f"{dtype} dequant differs"


CASES = [
    syn.LayerCase("q8-m1-n4096-k4096-r8", M=1, N=4096, K=4096, r=8, alpha=16.0, seed=611),
    syn.LayerCase("q8-m48-n2048-k1024-r64", M=48, N=2048, K=1024, r=64, alpha=128.0, seed=612),
    syn.LayerCase("q8-m300-n320-k576-r16", M=300, N=320, K=576, r=16, alpha=32.0, seed=613),
    syn.LayerCase("q8-m512-n1024-k2048-r0", M=512, N=1024, K=2048, r=0, alpha=0.0, seed=614),
]


class Q8Run:
    def __init__(self, c):
        self.c = c
        ref = O.quantize_q8_0(_weight(c.N, c.K, c.seed).numpy())
        self.Wd = O.dequant_q8_0(ref["q"], ref["d"]).reshape(c.N, c.K)
        self.w = _upload(ref, c.N, c.K)
        self.X, self.dY = c.x().to(DEV), c.dy().to(DEV)
        self.A = c.lora_a().to(DEV) if c.r else None
        self.B = c.lora_b().to(DEV) if c.r else None
        self.ws = torch.empty(q.qlora_workspace_bytes(c.M, c.N, c.K, c.r), dtype=torch.uint8, device=DEV)
        self.Y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV)
        self.dX = torch.empty(c.M, c.K, dtype=torch.bfloat16, device=DEV)
        self.U = torch.empty(c.M, c.r, dtype=torch.bfloat16, device=DEV) if c.r else None
        self.G = torch.empty(c.M, c.r, dtype=torch.bfloat16, device=DEV) if c.r else None
        q.qlora_q8_0_lora_linear_fwd(self.w, self.X, self.A, self.B, c.r, c.scaling, self.Y, self.U, self.ws)
        q.qlora_q8_0_lora_linear_bwd_dx(self.w, self.dY, self.A, self.B, c.r, c.scaling, self.dX, self.G, self.ws)
        if c.r:
            self.dA = torch.empty(c.r, c.K, dtype=torch.float32, device=DEV)
            self.dB = torch.empty(c.N, c.r, dtype=torch.float32, device=DEV)
            q.qlora_lora_grad_AB(self.X, self.dY, self.U, self.G, c.r, c.scaling, self.dA, self.dB)
        q.qlora_sync_status()


@pytest.mark.parametrize("c", CASES, ids=[c.name for c in CASES])
def test_q8_0_layer_matches_oracle(c):
    run = Q8Run(c)
    X, dY = run.X.cpu(), run.dY.cpu()
    A = run.A.cpu() if c.r else None
    B = run.B.cpu() if c.r else None
    Yref, uref = O.lora_linear_fwd(run.Wd, X, A, B, c.scaling)
    dXref, gref = O.lora_linear_bwd_dx(run.Wd, dY, A, B, c.scaling)
    _assert_tol(run.Y.float().cpu(), Yref, "Y")
    _assert_tol(run.dX.float().cpu(), dXref, "dX")
    if not c.r:
        return
    _assert_tol(run.U.float().cpu(), uref, "U")
    _assert_tol(run.G.float().cpu(), gref, "G")
    dAref, dBref = O.lora_grad_ab(X, dY, uref, gref, c.scaling)
    _assert_tol(run.dA.cpu(), dAref, "dA")
    _assert_tol(run.dB.cpu(), dBref, "dB")
    # the adapter term alone, element by element
    Y0 = torch.empty_like(run.Y)
    dX0 = torch.empty_like(run.dX)
    q.qlora_q8_0_lora_linear_fwd(run.w, run.X, None, None, 0, 0.0, Y0, None, run.ws)
    q.qlora_q8_0_lora_linear_bwd_dx(run.w, run.dY, None, None, 0, 0.0, dX0, None, run.ws)
    q.qlora_sync_status()
    lora_ref, _ = O.lora_linear_fwd(np.zeros((c.N, c.K)), X, A, B, c.scaling)
    dlora_ref, _ = O.lora_linear_bwd_dx(np.zeros((c.N, c.K)), dY, A, B, c.scaling)
    assert_adapter_term(run.Y.float().cpu().numpy(), Y0.float().cpu().numpy(), lora_ref, "Y adapter")
    assert_adapter_term(run.dX.float().cpu().numpy(), dX0.float().cpu().numpy(), dlora_ref, "dX adapter")


def test_q8_0_full_size_7b_attention_sampled():
    """The 7B attention projection at 2048 tokens, r = 8: sampled Y and dX columns."""
    c = syn.attn7b_case()
    W = c.weight()
    w = q.Q80Weight.empty(c.N, c.K, device=DEV)
    q.qlora_quantize_q8_0(W.to(DEV), w)
    X, A, B, dY = (t.to(DEV) for t in (c.x(), c.lora_a(), c.lora_b(), c.dy()))
    ws = torch.empty(q.qlora_workspace_bytes(c.M, c.N, c.K, c.r), dtype=torch.uint8, device=DEV)
    Y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV)
    dX = torch.empty(c.M, c.K, dtype=torch.bfloat16, device=DEV)
    q.qlora_q8_0_lora_linear_fwd(w, X, A, B, c.r, c.scaling, Y, None, ws)
    q.qlora_q8_0_lora_linear_bwd_dx(w, dY, A, B, c.r, c.scaling, dX, None, ws)
    q.qlora_sync_status()
    ref = O.quantize_q8_0(W.numpy())
    assert np.array_equal(w.q.cpu().numpy(), ref["q"])
    Wd = O.dequant_q8_0(ref["q"], ref["d"]).reshape(c.N, c.K)
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(c.N, 48, replace=False))
    Xc, Ac, Bc, dYc = X.cpu(), A.cpu(), B.cpu(), dY.cpu()
    Yref = O.lora_linear_fwd_rows(Wd, Xc, Ac, Bc, c.scaling, rows)
    _assert_tol(Y.float().cpu().numpy()[:, rows], Yref, "Y[:, sample]")
    cols = np.sort(rng.choice(c.K, 48, replace=False))
    dXref, _ = O.lora_linear_bwd_dx(Wd[:, cols], dYc, Ac.float().numpy()[:, cols], Bc, c.scaling)
    _assert_tol(dX.float().cpu().numpy()[:, cols], dXref, "dX[:, sample]")
