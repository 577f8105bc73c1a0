"""ctypes declarations of the C ABI in include/qlora_nf4.h (loads libqlora_nf4.so)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLORA_OK = 0
QLORA_STATIC_SCRATCH_BYTES = 8 << 20   # the header's QLORA_STATIC_SCRATCH_BYTES
STATUS_NAMES = {0: "QLORA_OK", 1: "QLORA_ERR_ARG", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGN",
                4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_CUDA", 6: "QLORA_ERR_TIMEOUT",
                7: "QLORA_ERR_UNSUPPORTED"}

# every symbol the header declares, with (restype, argtypes)
_vp, _i64, _int, _f32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


class Nf4WeightC(ctypes.Structure):
    _fields_ = [("n_out", ctypes.c_int64), ("n_in", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("scales2", ctypes.c_void_p), ("quant_type", ctypes.c_int32),
                ("format", ctypes.c_int32)]


QT_NF4, QT_FP4 = 0, 1
FMT_BLOCK128, FMT_NO_DQ, FMT_CODES_AFTER_DQ = 1, 2, 4


_WP = ctypes.POINTER(Nf4WeightC)


class Q80WeightC(ctypes.Structure):
    _fields_ = [("n_out", ctypes.c_int64), ("n_in", ctypes.c_int64), ("q", ctypes.c_void_p), ("d", ctypes.c_void_p)]


_QP = ctypes.POINTER(Q80WeightC)

SIGNATURES = {
    "qlora_packed_bytes": (_sz, [_i64]),
    "qlora_packed_bytes_fmt": (_sz, [_i64, ctypes.c_int32]),
    "qlora_nf4_codebook": (_int, [ctypes.POINTER(ctypes.c_float)]),
    "qlora_codebook": (_int, [_int, ctypes.POINTER(ctypes.c_float)]),
    "qlora_quantize_nf4_dq": (_int, [_vp, _WP, _vp]),
    "qlora_dequant": (_int, [_WP, _vp, _int, _vp]),
    "qlora_lora_merge_requant": (_int, [_WP, _vp, _vp, _int, _f32, _vp, _WP, _vp]),
    "qlora_workspace_bytes": (_sz, [_i64, _i64, _i64, _int]),
    "qlora_lora_linear_fwd": (_int, [_WP, _vp, _i64, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_lora_linear_fwd_static_ws": (_int, [_WP, _vp, _i64, _vp, _vp, _int, _f32, _vp, _vp, _vp]),
    "qlora_lora_linear_bwd_dx": (_int, [_WP, _vp, _i64, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_lora_grad_AB": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _f32, _vp, _vp, _int, _vp]),
    "qlora_sync_status": (_int, [_vp]),
    "qlora_last_error": (ctypes.c_char_p, []),
    "qlora_set_wait_limit_ns": (_int, [ctypes.c_uint64]),
    "qlora_q8_0_packed_bytes": (_sz, [_i64]),
    "qlora_quantize_q8_0": (_int, [_vp, _QP, _vp]),
    "qlora_dequant_q8_0": (_int, [_QP, _vp, _int, _vp]),
    "qlora_q8_0_lora_linear_fwd": (_int, [_QP, _vp, _i64, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_q8_0_lora_linear_bwd_dx": (_int, [_QP, _vp, _i64, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_probe_wait_timeout": (_int, [_vp]),
}

_lib = None


class QloraError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} -> {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library; raises if it has not been built (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m bit_quantized_base_nf4_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def check(fn: str, status: int) -> None:
    if status != QLORA_OK:
        msg = load().qlora_last_error().decode(errors="replace")
        raise QloraError(fn, status, msg)
