"""The FP4 quant type on the GPU against the oracle.

The kernels are those of NF4; only the 16 levels (and the encode thresholds) come
from the weight's quant type.  Encode and dequant are compared bit for bit; the
layer within the usual tolerance on the pair, split-K and small-M paths; the merge
from an NF4 base into an FP4 result bit for bit."""
import numpy as np
import pytest
import torch

import bit_quantized_base_nf4_b200 as q
from bit_quantized_base_nf4_b200 import synthetic as syn
from oracle import nf4_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
FP4 = q.QLORA_QT_FP4


def _assert_tol(got, ref, what):
    nw, rw = O.rel_errors(got, ref)
    assert nw <= O.NORMWISE_TOL and rw <= O.ROWWISE_TOL, f"{what}: normwise {nw:.3e} rowwise {rw:.3e}"


def _upload(ref, n_out, n_in, quant_type):
    w = q.NF4Weight.empty(n_out, n_in, device=DEV, quant_type=quant_type)
    w.codes.copy_(torch.from_numpy(np.ascontiguousarray(ref["codes"])))
    w.scales.copy_(torch.from_numpy(np.ascontiguousarray(ref["scales"])))
    w.scales2.copy_(torch.from_numpy(np.ascontiguousarray(ref["scales2"])))
    return w


@pytest.mark.parametrize("n_out,n_in,seed", [(72, 576, 401), (512, 1024, 402)])
def test_fp4_encode_and_dequant_bit_exact(n_out, n_in, seed):
    W = syn.with_outliers(syn.normal_f32((n_out, n_in), 0.02, seed), 1e-3, 10.0, seed + 1)
    W[1, :64] = 0.0                                     # an all-zero block
    book = O.fp4_codebook()
    ref = O.quantize_variant(W.numpy(), book=book)
    w = q.NF4Weight.empty(n_out, n_in, device=DEV, quant_type=FP4)
    q.qlora_quantize_nf4_dq(W.to(DEV), w)
    q.qlora_sync_status()
    assert np.array_equal(w.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(w.scales.cpu().numpy(), ref["scales"])
    assert np.array_equal(w.scales2.cpu().numpy().view(np.uint32), ref["scales2"].view(np.uint32))
    # dequant of the oracle's packed weight
    wo = _upload(ref, n_out, n_in, FP4)
    out = torch.empty(n_out, n_in, dtype=torch.float32, device=DEV)
    q.qlora_dequant(wo, out)
    q.qlora_sync_status()
    want = O.dequant_variant(ref["codes"], ref["scales"], ref["scales2"], book=book)
    assert np.array_equal(out.cpu().numpy().reshape(-1).view(np.uint32), want.view(np.uint32))


LAYER_CASES = [
    syn.LayerCase("fp4-pair-m300-n320-k576-r16", M=300, N=320, K=576, r=16, alpha=32.0, seed=411),
    syn.LayerCase("fp4-split-m40-n384-k2048-r8", M=40, N=384, K=2048, r=8, alpha=16.0, seed=412),
    syn.LayerCase("fp4-small-m4-n1024-k4096-r8", M=4, N=1024, K=4096, r=8, alpha=16.0, seed=413),
]


@pytest.mark.parametrize("c", LAYER_CASES, ids=[c.name for c in LAYER_CASES])
def test_fp4_layer_matches_oracle(c):
    book = O.fp4_codebook()
    ref = O.quantize_variant(c.weight().numpy(), book=book)
    Wd = O.dequant_variant(ref["codes"], ref["scales"], ref["scales2"], book=book).reshape(c.N, c.K)
    w = _upload(ref, c.N, c.K, FP4)
    X, A, B, dY = c.x(), c.lora_a(), c.lora_b(), c.dy()
    ws = torch.empty(q.qlora_workspace_bytes(c.M, c.N, c.K, c.r), dtype=torch.uint8, device=DEV)
    Y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV)
    dX = torch.empty(c.M, c.K, dtype=torch.bfloat16, device=DEV)
    q.qlora_lora_linear_fwd(w, X.to(DEV), A.to(DEV), B.to(DEV), c.r, c.scaling, Y, None, ws)
    q.qlora_lora_linear_bwd_dx(w, dY.to(DEV), A.to(DEV), B.to(DEV), c.r, c.scaling, dX, None, ws)
    q.qlora_sync_status()
    Yref, _ = O.lora_linear_fwd(Wd, X, A, B, c.scaling)
    dXref, _ = O.lora_linear_bwd_dx(Wd, dY, A, B, c.scaling)
    _assert_tol(Y.float().cpu(), Yref, "Y")
    _assert_tol(dX.float().cpu(), dXref, "dX")


def test_merge_nf4_base_into_fp4():
    n_out, n_in, r, s, seed = 128, 1024, 8, 2.0, 421
    ref = O.quantize_nf4_dq(syn.normal_f32((n_out, n_in), 0.02, seed).numpy())
    A = syn.normal_bf16((r, n_in), 1.0 / n_in, seed + 1)
    B = syn.normal_bf16((n_out, r), 0.01, seed + 2)
    w = _upload(ref, n_out, n_in, q.QLORA_QT_NF4)
    out = q.NF4Weight.empty(n_out, n_in, device=DEV, quant_type=FP4)
    scratch = torch.empty(n_out, n_in, dtype=torch.float32, device=DEV)
    q.qlora_lora_merge_requant(w, A.to(DEV), B.to(DEV), r, s, scratch, out)
    q.qlora_sync_status()
    m = O.lora_merge_bf16(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, A.float().numpy(),
                          B.float().numpy(), s)
    want = O.quantize_variant(m, book=O.fp4_codebook())
    assert np.array_equal(out.codes.cpu().numpy(), want["codes"])
    assert np.array_equal(out.scales.cpu().numpy(), want["scales"])
    assert np.array_equal(out.scales2.cpu().numpy().view(np.uint32), want["scales2"].view(np.uint32))
