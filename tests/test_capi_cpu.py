"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
declared symbol, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_quantized_base_nf4_b200 import _capi
from bit_quantized_base_nf4_b200 import build as libbuild
from oracle import nf4_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return _capi.load()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-zA-Z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = _declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
        assert n in _capi.SIGNATURES, f"{n} has no ctypes signature"


def test_codebook_matches_oracle_bit_for_bit(lib):
    buf = (ctypes.c_float * 16)()
    assert lib.qlora_nf4_codebook(buf) == 0
    got = np.frombuffer(buf, dtype=np.float32)
    ref = O.nf4_codebook()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert lib.qlora_nf4_codebook(None) == 1


@pytest.mark.parametrize("n", [64, 16384, 16384 + 64, 4096 * 4096, 11008 * 4096, 28672 * 8192])
def test_packed_bytes_matches_closed_form(lib, n):
    assert lib.qlora_packed_bytes(n) == O.packed_bytes(n)


def test_packed_bytes_rejects_bad_sizes(lib):
    assert lib.qlora_packed_bytes(0) == 0 and lib.qlora_packed_bytes(65) == 0 and lib.qlora_packed_bytes(-64) == 0


def test_workspace_bytes_covers_adapter_buffer(lib):
    for (M, N, K, r) in [(16, 256, 512, 8), (2048, 4096, 4096, 8), (4096, 11008, 4096, 64), (1, 4096, 4096, 8)]:
        ws = lib.qlora_workspace_bytes(M, N, K, r)
        assert ws >= M * r * 2 and ws % 256 == 0
    assert lib.qlora_workspace_bytes(0, 1, 1, 8) == 0


@pytest.mark.parametrize("fmt,block,dq", [(0, 64, True), (1, 128, True), (2, 64, False), (3, 128, False),
                                          (4, 64, True), (5, 128, True)])
def test_packed_bytes_of_every_format_matches_closed_form(lib, fmt, block, dq):
    for n in (128, 16384 * 3, 4096 * 4096, 28672 * 8192):
        assert lib.qlora_packed_bytes_fmt(n, fmt) == O.packed_bytes_variant(n, block=block, dq=dq)
    assert lib.qlora_packed_bytes_fmt(64 * 3, 1) == 0          # not a multiple of 128
    assert lib.qlora_packed_bytes_fmt(128, 6) == 0             # no double quant + codes after it
    assert lib.qlora_packed_bytes_fmt(128, 8) == 0             # unknown flag


def test_q8_0_sizes_and_validation(lib):
    for n in (32, 4096 * 4096, 3_800_000_000 // 32 * 32):
        assert lib.qlora_q8_0_packed_bytes(n) == O.q8_0_packed_bytes(n)
    assert lib.qlora_q8_0_packed_bytes(48) == 0
    w = _capi.Q80WeightC(256, 96, 0x1000, 0x2000)          # n_in not a multiple of 64
    assert lib.qlora_quantize_q8_0(ctypes.c_void_p(0x4000), ctypes.byref(w), None) == 2
    w = _capi.Q80WeightC(256, 512, 0x1004, 0x2000)
    assert lib.qlora_dequant_q8_0(ctypes.byref(w), ctypes.c_void_p(0x4000), 0, None) == 3
    w = _capi.Q80WeightC(256, 512, 0x1000, 0x2000)
    X, A, B, Y = (ctypes.c_void_p(a) for a in (0x10000, 0x20000, 0x30000, 0x40000))
    assert lib.qlora_q8_0_lora_linear_fwd(ctypes.byref(w), X, 16, A, B, 12, 2.0, Y, None, None, 0, None) == 2
    assert lib.qlora_q8_0_lora_linear_bwd_dx(ctypes.byref(w), X, 64, A, B, 8, 2.0, Y, None, None, 0, None) == 4


def test_format_flags_are_validated(lib):
    X, Y = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000)
    ws = ctypes.c_void_p(0x30000)
    for fmt, n_in, code, msg in ((8, 512, 1, "format"), (6, 512, 1, "format"), (1, 576, 2, "multiple of the block")):
        w = _w(n_in=n_in)
        w.format = fmt
        st = lib.qlora_lora_linear_fwd(ctypes.byref(w), X, 16, None, None, 0, 0.0, Y, None, ws, 1 << 20, None)
        assert st == code and msg in _err(lib), (fmt, st, _err(lib))
    # without double quantization the second-level buffer may be NULL
    w = _w(scales2=0)
    w.format = 2
    st = lib.qlora_dequant(ctypes.byref(w), Y, 0, None)
    assert st not in (1, 2, 3), _err(lib)       # passes validation (fails later only for want of a GPU)
    w.format = 0
    assert lib.qlora_dequant(ctypes.byref(w), Y, 0, None) == 1


def test_wait_limit_range_is_checked_on_the_host(lib):
    # out-of-range limits are refused before any device call
    assert lib.qlora_set_wait_limit_ns(10) == 1
    assert "outside" in _err(lib)
    assert lib.qlora_set_wait_limit_ns(10**12) == 1


def _w(n_out=256, n_in=512, codes=0x1000, scales=0x2000, scales2=0x3000):
    return _capi.Nf4WeightC(n_out, n_in, codes, scales, scales2)


def _err(lib):
    return lib.qlora_last_error().decode()


def test_validation_rejects_before_launch(lib):
    st = lib.qlora_quantize_nf4_dq(ctypes.c_void_p(0x4000), None, None)
    assert st == 1 and "NULL" in _err(lib)
    w = _w(n_in=100)
    assert lib.qlora_quantize_nf4_dq(ctypes.c_void_p(0x4000), ctypes.byref(w), None) == 2
    assert "multiple of the block (64)" in _err(lib)
    w = _w(codes=0x1001)
    assert lib.qlora_dequant(ctypes.byref(w), ctypes.c_void_p(0x4000), 0, None) == 3
    w = _w()
    assert lib.qlora_dequant(ctypes.byref(w), ctypes.c_void_p(0x4000), 2, None) == 1
    # rank rules
    X, A, B, Y = (ctypes.c_void_p(a) for a in (0x10000, 0x20000, 0x30000, 0x40000))
    ws = ctypes.c_void_p(0x50000)
    for r in (4, 12, 136):
        assert lib.qlora_lora_linear_fwd(ctypes.byref(w), X, 16, A, B, r, 2.0, Y, None, ws, 1 << 20, None) == 2
    assert lib.qlora_lora_linear_fwd(ctypes.byref(w), X, 16, None, B, 8, 2.0, Y, None, ws, 1 << 20, None) == 1
    assert lib.qlora_lora_linear_fwd(ctypes.byref(w), X, 0, A, B, 8, 2.0, Y, None, ws, 1 << 20, None) == 2
    assert lib.qlora_lora_linear_fwd(ctypes.byref(w), X, 16, A, B, 8, float("nan"), Y, None, ws, 1 << 20,
                                     None) == 1
    # workspace too small / missing (64 tokens: the adapter's rank buffers live in the workspace)
    assert lib.qlora_lora_linear_fwd(ctypes.byref(w), X, 64, A, B, 8, 2.0, Y, None, ws, 8, None) == 4
    assert lib.qlora_lora_linear_fwd(ctypes.byref(w), X, 64, A, B, 8, 2.0, Y, None, None, 0, None) == 4
    assert lib.qlora_lora_linear_bwd_dx(ctypes.byref(w), X, 64, A, B, 8, 2.0, Y, None, ws, 8, None) == 4

    # misaligned activations
    assert lib.qlora_lora_linear_fwd(ctypes.byref(w), ctypes.c_void_p(0x10002), 16, A, B, 8, 2.0, Y, None, ws,
                                     1 << 20, None) == 3
    # merge + requantize argument rules
    sc = ctypes.c_void_p(0x80000)
    w2 = _w(n_out=128)
    assert lib.qlora_lora_merge_requant(ctypes.byref(w), A, B, 8, 2.0, sc, ctypes.byref(w2), None) == 2
    assert "shape" in _err(lib)
    assert lib.qlora_lora_merge_requant(ctypes.byref(w), A, B, 12, 2.0, sc, ctypes.byref(w), None) == 2
    assert lib.qlora_lora_merge_requant(ctypes.byref(w), None, B, 8, 2.0, sc, ctypes.byref(w), None) == 1
    assert lib.qlora_lora_merge_requant(ctypes.byref(w), A, B, 8, 2.0, None, ctypes.byref(w), None) == 1
    assert lib.qlora_lora_merge_requant(ctypes.byref(w), A, B, 8, 2.0, ctypes.c_void_p(0x80004), ctypes.byref(w),
                                        None) == 3
    # grad_AB argument rules
    dA, dB = ctypes.c_void_p(0x60000), ctypes.c_void_p(0x70000)
    assert lib.qlora_lora_grad_AB(X, Y, A, B, 16, 256, 512, 8, 2.0, dA, None, 0, None) == 1
    assert lib.qlora_lora_grad_AB(X, Y, A, B, 16, 256, 512, 6, 2.0, dA, dB, 0, None) == 2
    assert lib.qlora_lora_grad_AB(X, Y, A, B, 16, 256, 512, 8, 2.0, dA, dB, 3, None) == 1


def test_weight_descriptor_layout_and_quant_type(lib):
    # the C side pins the same layout with a static_assert
    assert ctypes.sizeof(_capi.Nf4WeightC) == 48 and _capi.Nf4WeightC.quant_type.offset == 40
    w = _w()
    w.quant_type = 2
    assert lib.qlora_dequant(ctypes.byref(w), ctypes.c_void_p(0x4000), 0, None) == 1
    assert "quant_type" in _err(lib)
    assert lib.qlora_quantize_nf4_dq(ctypes.c_void_p(0x4000), ctypes.byref(w), None) == 1


def test_codebooks_match_oracle_bit_for_bit(lib):
    for qt, book in ((0, O.nf4_codebook()), (1, O.fp4_codebook())):
        buf = (ctypes.c_float * 16)()
        assert lib.qlora_codebook(qt, buf) == 0
        assert np.array_equal(np.array(list(buf), np.float32).view(np.uint32), book.view(np.uint32))
    buf = (ctypes.c_float * 16)()
    assert lib.qlora_codebook(2, buf) == 1
    assert lib.qlora_codebook(0, None) == 1


def test_binding_refuses_missing_library(tmp_path):
    saved = _capi._lib
    try:
        _capi._lib = None
        with pytest.raises(ImportError):
            _capi.load(str(tmp_path / "absent.so"))
    finally:
        _capi._lib = saved
