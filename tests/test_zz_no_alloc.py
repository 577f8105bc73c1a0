"""qlora_lora_linear_fwd_static_ws: the forward with the library's static device scratch.

Its results are compared with qlora_lora_linear_fwd (caller workspace) within the
tests' tolerance, on two calls in a row, through the C ABI.  The file is named to
be collected last, and it passes both alone in a fresh process and after the
other tests.
"""
import ctypes

import pytest
import torch

import bit_quantized_base_nf4_b200 as q
from bit_quantized_base_nf4_b200 import _capi
from bit_quantized_base_nf4_b200 import synthetic as syn
from oracle import nf4_oracle as O

DEV = "cuda"

CASES = [
    # CTA-pair forward (M >= 64), ragged in every dimension
    syn.LayerCase("pair-m300-n320-k576-r16", M=300, N=320, K=576, r=16, alpha=32.0, seed=201),
    # 32 tokens: single-CTA forward with a split-K accumulator in the scratch
    syn.LayerCase("split-m32-n512-k2048-r8", M=32, N=512, K=2048, r=8, alpha=16.0, seed=202),
    # 4 tokens: the small-M kernel, which needs no scratch
    syn.LayerCase("decode-m4-n512-k2048-r8", M=4, N=512, K=2048, r=8, alpha=16.0, seed=205),
    # no adapter
    syn.LayerCase("base-only-m64-n256-k512", M=64, N=256, K=512, r=0, alpha=0.0, seed=203),
    # 7B attention projection at 2048 tokens, rank 8
    syn.LayerCase("attn7b-m2048-r8", M=2048, N=4096, K=4096, r=8, alpha=16.0, seed=204),
]


def _assert_tol(got, ref, what):
    nw, rw = O.rel_errors(got.float().cpu().numpy(), ref.float().cpu().numpy())
    assert nw <= O.NORMWISE_TOL and rw <= O.ROWWISE_TOL, f"{what}: normwise {nw:.3e} rowwise {rw:.3e}"


def _call_static(lib, w_c, X, M, A, B, r, scaling, Y, U):
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = lib.qlora_lora_linear_fwd_static_ws(ctypes.byref(w_c), vp(X), M, vp(A), vp(B), r, scaling, vp(Y), vp(U),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    _capi.check("qlora_lora_linear_fwd_static_ws", st)


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c.name for c in CASES])
def test_static_scratch_forward_matches_workspace_forward(case):
    lib = _capi.load()
    M, N, K, r = case.M, case.N, case.K, case.r
    w = q.NF4Weight.empty(N, K)
    q.qlora_quantize_nf4_dq(case.weight().to(DEV), w)
    X = case.x().to(DEV)
    A = case.lora_a().to(DEV) if r else None
    B = case.lora_b().to(DEV) if r else None

    # the existing entry point, with a caller workspace
    ws = torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=DEV)
    Y_ref = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    U_ref = torch.empty(M, r, dtype=torch.bfloat16, device=DEV) if r else None
    q.qlora_lora_linear_fwd(w, X, A, B, r, case.scaling, Y_ref, U_ref, ws)
    q.qlora_sync_status()

    # outputs of both static calls, filled with NaN so unwritten elements fail
    Ys = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    Us = [torch.full((M, r), float("nan"), dtype=torch.bfloat16, device=DEV) if r else None for _ in range(2)]
    w_c = w.c_struct()
    # the first call on the device does the scratch look-up; count device memory after it
    _call_static(lib, w_c, X, M, A, B, r, case.scaling, Ys[0], Us[0])
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    torch_allocs = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
    _call_static(lib, w_c, X, M, A, B, r, case.scaling, Ys[1], Us[1])
    q.qlora_sync_status()
    assert torch.cuda.mem_get_info()[0] == free_before, "device memory changed across the call"
    assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == torch_allocs

    for i in range(2):
        assert torch.isfinite(Ys[i].float()).all(), f"call {i}: Y has unwritten or non-finite elements"
        _assert_tol(Ys[i], Y_ref, f"{case.name} call {i} Y")
        if r:
            assert torch.isfinite(Us[i].float()).all()
            _assert_tol(Us[i], U_ref, f"{case.name} call {i} U_save")


def test_static_scratch_rejects_oversize_before_any_device_work():
    """Sizes whose scratch need exceeds QLORA_STATIC_SCRATCH_BYTES fail on the host."""
    lib = _capi.load()
    w = _capi.Nf4WeightC(4096, 4096, 0x1000, 0x2000, 0x3000)
    X, A, B, Y = (ctypes.c_void_p(a) for a in (0x10000, 0x20000, 0x30000, 0x40000))
    # rank buffers of 6 * M * r bytes: 16384 tokens at r = 128 need 12 MiB
    st = lib.qlora_lora_linear_fwd_static_ws(ctypes.byref(w), X, 16384, A, B, 128, 1.0, Y, None, None)
    assert st == 4, _capi.STATUS_NAMES.get(st, st)
    msg = lib.qlora_last_error().decode()
    assert "static scratch holds %d" % _capi.QLORA_STATIC_SCRATCH_BYTES in msg, msg
    # the first size past the limit at r = 128: 10923 * 128 * 6 bytes = 8 MiB + 256
    st = lib.qlora_lora_linear_fwd_static_ws(ctypes.byref(w), X, 10923, A, B, 128, 1.0, Y, None, None)
    assert st == 4, _capi.STATUS_NAMES.get(st, st)
    assert "needs %d bytes" % (10923 * 128 * 6) in lib.qlora_last_error().decode()
    # argument rules are those of the workspace forward
    assert lib.qlora_lora_linear_fwd_static_ws(ctypes.byref(w), X, 0, A, B, 8, 1.0, Y, None, None) == 2
    assert lib.qlora_lora_linear_fwd_static_ws(ctypes.byref(w), X, 16, A, B, 12, 1.0, Y, None, None) == 2
