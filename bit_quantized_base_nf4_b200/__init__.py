"""B200 (sm_100a) frozen-base NF4 + double-quant LoRA linear layer.

A thin Python binding over the C ABI of libqlora_nf4.so (include/qlora_nf4.h).
The functions below carry the C names and only marshal torch tensors to raw
device pointers and sizes; every step of the computation runs in the
library's CUDA kernels.  If the library is missing, importing the binding
functions raises: there is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _capi

__all__ = ["NF4Weight", "QLORA_QT_NF4", "QLORA_QT_FP4", "QLORA_FMT_BLOCK128", "QLORA_FMT_NO_DQ",
           "QLORA_FMT_CODES_AFTER_DQ", "qlora_packed_bytes", "qlora_packed_bytes_fmt", "qlora_nf4_codebook",
           "qlora_codebook",
           "qlora_quantize_nf4_dq", "qlora_dequant",
           "qlora_lora_merge_requant",
           "qlora_workspace_bytes", "qlora_lora_linear_fwd", "qlora_lora_linear_fwd_static_ws",
           "qlora_lora_linear_bwd_dx", "qlora_lora_grad_AB",
           "qlora_sync_status", "qlora_set_wait_limit_ns", "qlora_probe_wait_timeout", "Q80Weight",
           "qlora_q8_0_packed_bytes", "qlora_quantize_q8_0", "qlora_dequant_q8_0", "qlora_q8_0_lora_linear_fwd",
           "qlora_q8_0_lora_linear_bwd_dx", "QloraError"]

QloraError = _capi.QloraError


def _lib():
    return _capi.load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, dtype, shape, name):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous cuda {dtype} {tuple(shape)}, got {t.dtype} "
                         f"{tuple(t.shape)} on {t.device}")


QLORA_QT_NF4, QLORA_QT_FP4 = _capi.QT_NF4, _capi.QT_FP4
QLORA_FMT_BLOCK128, QLORA_FMT_NO_DQ, QLORA_FMT_CODES_AFTER_DQ = (_capi.FMT_BLOCK128, _capi.FMT_NO_DQ,
                                                                 _capi.FMT_CODES_AFTER_DQ)


@dataclass
class NF4Weight:
    """Packed 4-bit weight: device buffers owned by this object (codes, first-level scales,
    second-level steps), the quant type whose 16 levels the codes index (NF4 by default, or
    FP4) and the storage format of the scales (QLORA_FMT_* flags, 0 = blocks of 64 with
    double quantization).  Without double quantization `scales` holds float32 absmaxes and
    `scales2` is an empty tensor."""
    n_out: int
    n_in: int
    codes: torch.Tensor
    scales: torch.Tensor
    scales2: torch.Tensor
    quant_type: int = QLORA_QT_NF4
    format: int = 0

    @classmethod
    def empty(cls, n_out: int, n_in: int, device="cuda", quant_type: int = QLORA_QT_NF4,
              format: int = 0) -> "NF4Weight":
        numel = n_out * n_in
        nb = numel // (128 if format & QLORA_FMT_BLOCK128 else 64)
        if format & QLORA_FMT_NO_DQ:
            scales = torch.empty(nb, dtype=torch.float32, device=device)
            scales2 = torch.empty(0, dtype=torch.float32, device=device)
        else:
            scales = torch.empty(nb, dtype=torch.uint8, device=device)
            scales2 = torch.empty((nb + 255) // 256, dtype=torch.float32, device=device)
        return cls(n_out, n_in, torch.empty(numel // 2, dtype=torch.uint8, device=device), scales, scales2,
                   int(quant_type), int(format))

    def c_struct(self) -> _capi.Nf4WeightC:
        s2 = self.scales2.data_ptr() if self.scales2.numel() else None
        return _capi.Nf4WeightC(self.n_out, self.n_in, self.codes.data_ptr(), self.scales.data_ptr(), s2,
                                int(self.quant_type), int(self.format))


def qlora_packed_bytes(numel: int) -> int:
    return int(_lib().qlora_packed_bytes(int(numel)))


def qlora_packed_bytes_fmt(numel: int, format: int) -> int:
    return int(_lib().qlora_packed_bytes_fmt(int(numel), int(format)))


def qlora_nf4_codebook() -> list[float]:
    buf = (ctypes.c_float * 16)()
    _capi.check("qlora_nf4_codebook", _lib().qlora_nf4_codebook(buf))
    return list(buf)


def qlora_codebook(quant_type: int) -> list[float]:
    buf = (ctypes.c_float * 16)()
    _capi.check("qlora_codebook", _lib().qlora_codebook(int(quant_type), buf))
    return list(buf)


def qlora_quantize_nf4_dq(W: torch.Tensor, weight: NF4Weight, stream=None) -> None:
    _need(W, torch.float32, (weight.n_out, weight.n_in), "W")
    s = weight.c_struct()
    _capi.check("qlora_quantize_nf4_dq", _lib().qlora_quantize_nf4_dq(_ptr(W), ctypes.byref(s), _stream(stream)))


def qlora_dequant(weight: NF4Weight, out: torch.Tensor, stream=None) -> None:
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out must be float32 or bfloat16")
    _need(out, out.dtype, (weight.n_out, weight.n_in), "out")
    s = weight.c_struct()
    _capi.check("qlora_dequant", _lib().qlora_dequant(ctypes.byref(s), _ptr(out), int(out.dtype == torch.bfloat16),
                                                      _stream(stream)))


def qlora_lora_merge_requant(weight: NF4Weight, A, B, r: int, scaling: float, W_scratch: torch.Tensor,
                             out: NF4Weight, stream=None) -> None:
    """Merge the adapter into the base and quantize again into `out` (may be `weight`);
    W_scratch is a float32 [n_out, n_in] device tensor that receives the merged base."""
    _need(W_scratch, torch.float32, (weight.n_out, weight.n_in), "W_scratch")
    if (out.n_out, out.n_in) != (weight.n_out, weight.n_in):
        raise ValueError("out must have the shape of weight")
    if r:
        _need(A, torch.bfloat16, (r, weight.n_in), "A")
        _need(B, torch.bfloat16, (weight.n_out, r), "B")
    s_in, s_out = weight.c_struct(), out.c_struct()
    _capi.check("qlora_lora_merge_requant",
                _lib().qlora_lora_merge_requant(ctypes.byref(s_in), _ptr(A) if r else None, _ptr(B) if r else None,
                                                int(r), float(scaling), _ptr(W_scratch), ctypes.byref(s_out),
                                                _stream(stream)))


def qlora_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(_lib().qlora_workspace_bytes(int(M), int(N), int(K), int(r)))


def qlora_lora_linear_fwd(weight: NF4Weight, X, A, B, r: int, scaling: float, Y, U_save=None, ws=None,
                          stream=None) -> None:
    M = X.shape[0]
    _need(X, torch.bfloat16, (M, weight.n_in), "X")
    _need(Y, torch.bfloat16, (M, weight.n_out), "Y")
    if r:
        _need(A, torch.bfloat16, (r, weight.n_in), "A")
        _need(B, torch.bfloat16, (weight.n_out, r), "B")
    if U_save is not None:
        _need(U_save, torch.bfloat16, (M, r), "U_save")
    s = weight.c_struct()
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _capi.check("qlora_lora_linear_fwd", _lib().qlora_lora_linear_fwd(
        ctypes.byref(s), _ptr(X), M, _ptr(A), _ptr(B), int(r), float(scaling), _ptr(Y), _ptr(U_save), _ptr(ws),
        wsb, _stream(stream)))


def qlora_lora_linear_fwd_static_ws(weight: NF4Weight, X, A, B, r: int, scaling: float, Y, U_save=None,
                                    stream=None) -> None:
    """qlora_lora_linear_fwd with the library's static device scratch (no workspace argument)."""
    M = X.shape[0]
    _need(X, torch.bfloat16, (M, weight.n_in), "X")
    _need(Y, torch.bfloat16, (M, weight.n_out), "Y")
    if r:
        _need(A, torch.bfloat16, (r, weight.n_in), "A")
        _need(B, torch.bfloat16, (weight.n_out, r), "B")
    if U_save is not None:
        _need(U_save, torch.bfloat16, (M, r), "U_save")
    s = weight.c_struct()
    _capi.check("qlora_lora_linear_fwd_static_ws", _lib().qlora_lora_linear_fwd_static_ws(
        ctypes.byref(s), _ptr(X), M, _ptr(A), _ptr(B), int(r), float(scaling), _ptr(Y), _ptr(U_save),
        _stream(stream)))


def qlora_lora_linear_bwd_dx(weight: NF4Weight, dY, A, B, r: int, scaling: float, dX, G_save=None, ws=None,
                             stream=None) -> None:
    M = dY.shape[0]
    _need(dY, torch.bfloat16, (M, weight.n_out), "dY")
    _need(dX, torch.bfloat16, (M, weight.n_in), "dX")
    if r:
        _need(A, torch.bfloat16, (r, weight.n_in), "A")
        _need(B, torch.bfloat16, (weight.n_out, r), "B")
    if G_save is not None:
        _need(G_save, torch.bfloat16, (M, r), "G_save")
    s = weight.c_struct()
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _capi.check("qlora_lora_linear_bwd_dx", _lib().qlora_lora_linear_bwd_dx(
        ctypes.byref(s), _ptr(dY), M, _ptr(A), _ptr(B), int(r), float(scaling), _ptr(dX), _ptr(G_save), _ptr(ws),
        wsb, _stream(stream)))


def qlora_lora_grad_AB(X, dY, U, G, r: int, scaling: float, dA, dB, accumulate: bool = False,
                       stream=None) -> None:
    M, K = X.shape
    N = dY.shape[1]
    _need(X, torch.bfloat16, (M, K), "X")
    _need(dY, torch.bfloat16, (M, N), "dY")
    _need(U, torch.bfloat16, (M, r), "U")
    _need(G, torch.bfloat16, (M, r), "G")
    _need(dA, torch.float32, (r, K), "dA")
    _need(dB, torch.float32, (N, r), "dB")
    _capi.check("qlora_lora_grad_AB", _lib().qlora_lora_grad_AB(
        _ptr(X), _ptr(dY), _ptr(U), _ptr(G), M, N, K, int(r), float(scaling), _ptr(dA), _ptr(dB),
        int(bool(accumulate)), _stream(stream)))


def qlora_sync_status(stream=None) -> None:
    _capi.check("qlora_sync_status", _lib().qlora_sync_status(_stream(stream)))


def qlora_set_wait_limit_ns(ns: int) -> None:
    """Time after which a kernel pipeline wait gives up on the current device (default 2e9 ns)."""
    _capi.check("qlora_set_wait_limit_ns", _lib().qlora_set_wait_limit_ns(int(ns)))


def qlora_probe_wait_timeout(stream=None) -> None:
    """Enqueue the self-test kernel whose wait runs out; the next sync reports QLORA_ERR_TIMEOUT."""
    _capi.check("qlora_probe_wait_timeout", _lib().qlora_probe_wait_timeout(_stream(stream)))


# ----------------------------------------------------------------------------- Q8_0 route

@dataclass
class Q80Weight:
    """Q8_0 weight: int8 codes [n_out, n_in] and an fp16 scale per 32 weights (device)."""
    n_out: int
    n_in: int
    q: torch.Tensor
    d: torch.Tensor

    @classmethod
    def empty(cls, n_out: int, n_in: int, device="cuda") -> "Q80Weight":
        return cls(n_out, n_in, torch.empty(n_out * n_in, dtype=torch.int8, device=device),
                   torch.empty(n_out * n_in // 32, dtype=torch.float16, device=device))

    def c_struct(self) -> _capi.Q80WeightC:
        return _capi.Q80WeightC(self.n_out, self.n_in, self.q.data_ptr(), self.d.data_ptr())


def qlora_q8_0_packed_bytes(numel: int) -> int:
    return int(_lib().qlora_q8_0_packed_bytes(int(numel)))


def qlora_quantize_q8_0(W: torch.Tensor, weight: Q80Weight, stream=None) -> None:
    _need(W, torch.float32, (weight.n_out, weight.n_in), "W")
    s = weight.c_struct()
    _capi.check("qlora_quantize_q8_0", _lib().qlora_quantize_q8_0(_ptr(W), ctypes.byref(s), _stream(stream)))


def qlora_dequant_q8_0(weight: Q80Weight, out: torch.Tensor, stream=None) -> None:
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out must be float32 or bfloat16")
    _need(out, out.dtype, (weight.n_out, weight.n_in), "out")
    s = weight.c_struct()
    _capi.check("qlora_dequant_q8_0", _lib().qlora_dequant_q8_0(ctypes.byref(s), _ptr(out),
                                                                int(out.dtype == torch.bfloat16), _stream(stream)))


def qlora_q8_0_lora_linear_fwd(weight: Q80Weight, X, A, B, r: int, scaling: float, Y, U_save=None, ws=None,
                               stream=None) -> None:
    M = X.shape[0]
    _need(X, torch.bfloat16, (M, weight.n_in), "X")
    _need(Y, torch.bfloat16, (M, weight.n_out), "Y")
    if r:
        _need(A, torch.bfloat16, (r, weight.n_in), "A")
        _need(B, torch.bfloat16, (weight.n_out, r), "B")
    if U_save is not None:
        _need(U_save, torch.bfloat16, (M, r), "U_save")
    s = weight.c_struct()
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _capi.check("qlora_q8_0_lora_linear_fwd", _lib().qlora_q8_0_lora_linear_fwd(
        ctypes.byref(s), _ptr(X), M, _ptr(A), _ptr(B), int(r), float(scaling), _ptr(Y), _ptr(U_save), _ptr(ws),
        wsb, _stream(stream)))


def qlora_q8_0_lora_linear_bwd_dx(weight: Q80Weight, dY, A, B, r: int, scaling: float, dX, G_save=None, ws=None,
                                  stream=None) -> None:
    M = dY.shape[0]
    _need(dY, torch.bfloat16, (M, weight.n_out), "dY")
    _need(dX, torch.bfloat16, (M, weight.n_in), "dX")
    if r:
        _need(A, torch.bfloat16, (r, weight.n_in), "A")
        _need(B, torch.bfloat16, (weight.n_out, r), "B")
    if G_save is not None:
        _need(G_save, torch.bfloat16, (M, r), "G_save")
    s = weight.c_struct()
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _capi.check("qlora_q8_0_lora_linear_bwd_dx", _lib().qlora_q8_0_lora_linear_bwd_dx(
        ctypes.byref(s), _ptr(dY), M, _ptr(A), _ptr(B), int(r), float(scaling), _ptr(dX), _ptr(G_save), _ptr(ws),
        wsb, _stream(stream)))
