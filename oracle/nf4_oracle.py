"""CPU oracle for the QLoRA frozen-base NF4 linear layer (test infrastructure).

This module is TEST INFRASTRUCTURE.  Only the tests, the smoke check and the
bench's CPU-baseline leg may import it; the library never does.  It is a
plain, slow restatement of what the pages describe, in float64 unless a step
is defined in float32, and it shares no code, table or constant with the CUDA
library.

Pages cited (title, then section):

* "Course notes: LLM basics and quantized fine-tuning" (lqnn.cn/news/228537)
* "Quantized vs. non-quantized weights" (kwkr.cn/news/627310)
* "QLoRA double quantization and block-wise quantization memory"
  (news.rkmt.cn/news/4821)
* "5.8 QLoRA: 4-bit base + 16-bit sticky notes" (llm-training-guide, qlora)
* "Training LoRA directly on GGUF quantized weights" (cf-1.com/news/5705389)

Readings adopted where the pages are silent:

* NF4 levels: 8 positive and 7 negative normal quantiles with the offset
  delta = ((1 - 1/30) + (1 - 1/32)) / 2, each half divided by
  Phi^-1(delta), plus an exact zero, sorted ascending (index 7 is 0).
* Blocks of 64 run over the row-major flattened weight; groups of 256
  blocks (16384 weights) for the second level.  A ragged last group uses the
  blocks that exist.
* First level: absmax a_b, normalised value RN32(w / a_b), nearest level
  with ties to the lower index; a_b = 0 gives code 7.
* Packing: element 2j in the low nibble of byte j, element 2j+1 in the high
  nibble.
* Second level: d_g = RN32(max_b a_b / 255), q_b = clamp(rint_even(RN32(a_b /
  d_g)), 0, 255); d_g = 0 gives q_b = 0.
* Dequant: s_b = RN32(q_b * d_g), w' = RN32(c[code] * s_b).
* Layer: Y = X W'^T + s (X A^T) B^T, dX = dY W' + s (dY B) A,
  dA = s (dY B)^T X, dB = s dY^T (X A^T), no gradient for W0.
* Merge: m = bf16(RN32(bf16(w') + s sum_j B[n, j] A[j, k])), sum and product in
  float64 with j ascending, then the NF4 + double-quant encode of m.
* Format variants: block 64 or 128; double quantization on or off (fp32 absmax
  per block); codes against a_b or against the dequantized scale; FP4 levels =
  the E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 divided by 6, both signs.
* Q8_0: blocks of 32, d = fp16(max|w| / 127), q = clamp(rint_even(w / d), -127,
  127), w' = q d.

Parity status: every function here is pinned by a ``-m "not gpu"`` test in
tests/test_oracle_pins.py against a fact other than itself (a printed worked
example, a closed form, an invariant, brute force or an independent
quantile routine).  The NF4 level VALUES agree with other NF4 codebooks only
through the construction reading above: the pages print no level values, so
agreement with any third-party table is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64          # first-level block ("QLoRA double quantization ..." page, §1.2)
GROUP = 256         # second-level block of scales (same page, §2.2)
GROUP_WEIGHTS = BLOCK * GROUP


# ---------------------------------------------------------------------------
# Affine INT8 quantization ("Quantized vs. non-quantized weights" page, §2.1)
# ---------------------------------------------------------------------------

def affine_params(rmin: float, rmax: float, qmin: int = 0, qmax: int = 255):
    """scale = (rmax - rmin) / (qmax - qmin), zero_point = round(-rmin / scale) + qmin, in float64.

    round() is round-half-to-even (Python's), the one rounding the page leaves open.
    """
    scale = (float(rmax) - float(rmin)) / float(qmax - qmin)
    zp = int(round(-float(rmin) / scale)) + qmin
    return scale, zp


def affine_quant(r, scale: float, zp: int, qmin: int = 0, qmax: int = 255):
    """q = clamp(round(r / scale) + zp) (§2.1 forward formula)."""
    r = np.asarray(r, dtype=np.float64)
    return np.clip(np.rint(r / scale) + zp, qmin, qmax).astype(np.int64)


def affine_dequant(q, scale: float, zp: int):
    """r = scale * (q - zp) (§2.1 inverse formula)."""
    return float(scale) * (np.asarray(q, dtype=np.float64) - zp)


def symmetric_params(rmin: float, rmax: float):
    """Symmetric INT8: zero_point 0, scale = max(|rmin|, |rmax|) / 127 (§2.1)."""
    return max(abs(float(rmin)), abs(float(rmax))) / 127.0, 0


# ---------------------------------------------------------------------------
# Storage accounting ("QLoRA double quantization ..." page, §1.3 and §2.3;
# "5.8 QLoRA" page, "three parts that make it work")
# ---------------------------------------------------------------------------

def packed_bytes(numel: int) -> int:
    """Bytes of the packed NF4+DQ weight: 4-bit codes, one u8 scale per 64, one fp32 per 256 scales."""
    n = int(numel)
    nblocks = n // BLOCK
    return n // 2 + nblocks + 4 * ((nblocks + GROUP - 1) // GROUP)


def constant_bits_per_param(block: int = BLOCK, group: int = GROUP, dq: bool = True) -> float:
    """Quantization-constant overhead per weight: 8/64 + 32/(64*256) with DQ, 32/64 without."""
    if dq:
        return 8.0 / block + 32.0 / (block * group)
    return 32.0 / block


# ---------------------------------------------------------------------------
# NF4 levels ("5.8 QLoRA" page, "three parts": NF4 places its 16 levels by
# the normal distribution, dense near zero; "Quantized vs. non-quantized"
# page, §4.2; "QLoRA double quantization ..." page, §3.3)
# ---------------------------------------------------------------------------

def normal_cdf(x: float) -> float:
    """Phi(x) = erfc(-x / sqrt 2) / 2 (textbook identity; libm erfc)."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def normal_ppf(p: float) -> float:
    """Phi^-1(p) by bisection on normal_cdf until the bracket stops shrinking.

    For p > 1/2 it returns -Phi^-1(1 - p) (1 - p is exact there), so the
    bisection always runs in the lower tail where erfc keeps full relative
    precision.
    """
    if not 0.0 < p < 1.0:
        raise ValueError("p must lie in (0, 1)")
    if p > 0.5:
        return -normal_ppf(1.0 - p)
    lo, hi = -40.0, 0.0
    while True:
        mid = 0.5 * (lo + hi)
        if mid <= lo or mid >= hi:
            return mid
        if normal_cdf(mid) < p:
            lo = mid
        else:
            hi = mid


NF4_DELTA = 0.5 * ((1.0 - 1.0 / (2 * 15)) + (1.0 - 1.0 / (2 * 16)))


def nf4_levels_f64() -> np.ndarray:
    """16 NF4 levels in float64, ascending, with exact -1, 0, +1."""
    top = normal_ppf(NF4_DELTA)
    pos = [normal_ppf(0.5 + j * (NF4_DELTA - 0.5) / 8) / top for j in range(1, 9)]
    neg = [-normal_ppf(0.5 + j * (NF4_DELTA - 0.5) / 7) / top for j in range(1, 8)]
    levels = sorted(neg + [0.0] + pos)
    return np.array(levels, dtype=np.float64)


def nf4_codebook() -> np.ndarray:
    """The stored codebook: each float64 level rounded to nearest float32."""
    return nf4_levels_f64().astype(np.float32)


def nearest_code(nvals: np.ndarray, book: np.ndarray | None = None) -> np.ndarray:
    """Index of the nearest level for each float32 value, exact ties to the lower index.

    Distances are taken in float64 on the float32 inputs; np.argmin returns
    the first minimum, which is the lower index on an exact tie.  Where a table
    holds the same value twice (the FP4 table's -0 and +0), a value strictly above
    it takes the higher copy.  That follows from the format, not from a tie rule:
    an E2M1 number has a sign bit, and round-to-nearest keeps the sign of a
    strictly positive (negative) value that rounds to zero, giving +0 (-0).  A
    value that is exactly zero carries no sign here and takes the lower index,
    the rule of every other exact tie.
    """
    if book is None:
        book = nf4_codebook()
    v = np.asarray(nvals, dtype=np.float32).astype(np.float64)
    c = book.astype(np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    flat_v, flat_o = v.reshape(-1), out.reshape(-1)
    step = 1 << 20
    for s in range(0, flat_v.size, step):
        d = np.abs(flat_v[s:s + step, None] - c[None, :])
        flat_o[s:s + step] = np.argmin(d, axis=1).astype(np.uint8)
    dup = np.nonzero(c[1:] == c[:-1])[0]
    for k in dup:
        up = (flat_o == k) & (flat_v > c[k])
        flat_o[up] = k + 1
    return out


# ---------------------------------------------------------------------------
# Encode: block absmax + NF4 codes + double quantization of the scales
# ("QLoRA double quantization ..." page, §1.2, §1.3, §2.2, §2.3; "5.8 QLoRA"
# page, double quantization paragraph)
# ---------------------------------------------------------------------------

def block_absmax(w: np.ndarray) -> np.ndarray:
    """a_b = max |w| over each block of 64 consecutive weights (float32, exact)."""
    return np.max(np.abs(np.asarray(w, np.float32).reshape(-1, BLOCK)), axis=1)


def normalise(w: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """RN32(w / a_b): float64 quotient rounded once to float32; 0 where a_b = 0."""
    blocks = np.asarray(w, np.float32).reshape(-1, BLOCK).astype(np.float64)
    a = absmax.astype(np.float64)[:, None]
    safe = np.where(a == 0.0, 1.0, a)
    out = (blocks / safe).astype(np.float32)
    out[np.broadcast_to(a == 0.0, out.shape)] = 0.0
    return out


def double_quant(absmax: np.ndarray):
    """Second level: per group of 256 scales d_g = RN32(max/255), q_b = clamp(rint(RN32(a_b/d_g)))."""
    a = np.asarray(absmax, np.float32)
    nb = a.size
    ng = (nb + GROUP - 1) // GROUP
    d = np.zeros(ng, dtype=np.float32)
    q = np.zeros(nb, dtype=np.uint8)
    for g in range(ng):
        seg = a[g * GROUP:(g + 1) * GROUP]
        c2 = float(seg.max())
        dg = np.float32(c2 / 255.0)
        d[g] = dg
        if dg == 0.0:
            continue
        ratio = (seg.astype(np.float64) / float(dg)).astype(np.float32)
        q[g * GROUP:(g + 1) * GROUP] = np.clip(np.rint(ratio), 0, 255).astype(np.uint8)
    return q, d


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: element 2j in bits 0-3, element 2j+1 in bits 4-7."""
    c = np.asarray(codes, np.uint8).reshape(-1)
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0x0F
    out[1::2] = p >> 4
    return out


def quantize_nf4_dq(w: np.ndarray) -> dict:
    """Full encode of a float32 weight whose element count is a multiple of 64."""
    w = np.asarray(w, np.float32).reshape(-1)
    if w.size % BLOCK:
        raise ValueError("numel must be a multiple of 64")
    absmax = block_absmax(w)
    codes = nearest_code(normalise(w, absmax)).reshape(-1)
    q, d = double_quant(absmax)
    return {"codes": pack_codes(codes), "scales": q, "scales2": d,
            "absmax": absmax, "codes_unpacked": codes}


# ---------------------------------------------------------------------------
# Format variants ("QLoRA double quantization ..." page, §3.1 block size 64 or
# 128, §3.2 the double-quantization switch, §3.3 quant type nf4 or fp4; §1.3
# and §2.3 for the storage they cost)
# ---------------------------------------------------------------------------

def fp4_levels_f64() -> np.ndarray:
    """FP4 levels (reading: the pages name fp4 but print no values).  The 4-bit float
    with one sign, two exponent and one mantissa bit (E2M1) has magnitudes 0, 0.5, 1,
    1.5, 2, 3, 4, 6; divided by 6 so that the largest is 1, both signs, ascending:
    index 7 is -0 and index 8 is +0."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    return np.array([-m / 6.0 for m in reversed(mags)] + [m / 6.0 for m in mags], dtype=np.float64)
    # a zero normalised value takes index 7 and a positive one below 1/24 takes index 8
    # (nearest_code: the sign of a zero follows the sign of the value)


def fp4_codebook() -> np.ndarray:
    return fp4_levels_f64().astype(np.float32)


def packed_bytes_variant(numel: int, block: int = BLOCK, dq: bool = True) -> int:
    """4-bit codes plus the scales: u8 per block and fp32 per 256 blocks with double
    quantization, fp32 per block without."""
    n = int(numel)
    nb = n // block
    if dq:
        return n // 2 + nb + 4 * ((nb + GROUP - 1) // GROUP)
    return n // 2 + 4 * nb


def quantize_variant(w: np.ndarray, block: int = BLOCK, dq: bool = True, codes_after_dq: bool = False,
                     book: np.ndarray | None = None) -> dict:
    """Blockwise 4-bit encode with the format's switches.

    block: weights per first-level block; dq: double-quantize the block absmaxes
    (u8 q_b + one fp32 d_g per 256 blocks) or keep them as fp32; codes_after_dq: take
    the codes against the dequantized scale s_b = RN32(q_b d_g) instead of the absmax
    a_b (normalised values above 1 then go to the end levels); book: the 16 levels in
    float32, NF4 by default.  The steps are those of quantize_nf4_dq otherwise."""
    w = np.asarray(w, np.float32).reshape(-1)
    if w.size % block:
        raise ValueError("numel must be a multiple of the block")
    blocks = w.reshape(-1, block)
    a = np.max(np.abs(blocks), axis=1)
    out = {"absmax": a}
    scale = a
    if dq:
        q, d = double_quant(a)
        out["scales"], out["scales2"] = q, d
        if codes_after_dq:
            scale = dequant_scales(q, d)
    else:
        out["scales"] = a.copy()
    sc = scale.astype(np.float64)[:, None]
    safe = np.where(sc == 0.0, 1.0, sc)
    n = (blocks.astype(np.float64) / safe).astype(np.float32)
    n[np.broadcast_to(sc == 0.0, n.shape)] = 0.0
    codes = nearest_code(n, book).reshape(-1)
    out["codes"] = pack_codes(codes)
    out["codes_unpacked"] = codes
    return out


def dequant_variant(codes, scales, scales2=None, block: int = BLOCK, book: np.ndarray | None = None) -> np.ndarray:
    """w' = RN32(c[code] s_b) with s_b = RN32(q_b d_g) (scales2 given) or the fp32
    absmax itself (double quantization off)."""
    c = unpack_codes(codes)
    s = dequant_scales(scales, scales2) if scales2 is not None else np.asarray(scales, np.float32)
    if book is None:
        book = nf4_codebook()
    vals = book.astype(np.float64)[c].reshape(-1, block) * s.astype(np.float64)[:, None]
    return vals.astype(np.float32).reshape(-1)


# ---------------------------------------------------------------------------
# Q8_0 block format ("Training LoRA directly on GGUF quantized weights" page,
# §1.1: 32 weights share one fp16 scale, a little over one byte per weight;
# §2.2: blockwise dequant inside the GEMM or a one-shot dequant to bf16).
# Reading: symmetric int8 per block as in the "Quantized vs. non-quantized
# weights" page, §2.1: d = fp16(max|w| / 127), q = clamp(rint_even(w / d),
# -127, 127), w' = q * d; a block of zeros has d = 0 and q = 0.
# ---------------------------------------------------------------------------

Q8_BLOCK = 32


def q8_0_packed_bytes(numel: int) -> int:
    """32 int8 values plus one fp16 scale per block: 34 bytes per 32 weights."""
    return (int(numel) // Q8_BLOCK) * (Q8_BLOCK + 2)


def quantize_q8_0(w: np.ndarray) -> dict:
    """Blockwise symmetric int8: the fp16 scale of each block of 32 and the int8 values."""
    w = np.asarray(w, np.float32).reshape(-1)
    if w.size % Q8_BLOCK:
        raise ValueError("numel must be a multiple of 32")
    blocks = w.reshape(-1, Q8_BLOCK).astype(np.float64)
    d = (np.max(np.abs(blocks), axis=1) / 127.0).astype(np.float16)
    d64 = d.astype(np.float64)[:, None]
    safe = np.where(d64 == 0.0, 1.0, d64)
    q = np.clip(np.rint(blocks / safe), -127, 127)
    q[np.broadcast_to(d64 == 0.0, q.shape)] = 0
    return {"q": q.astype(np.int8).reshape(-1), "d": d}


def dequant_q8_0(q: np.ndarray, d: np.ndarray) -> np.ndarray:
    """w' = q * d, exact in float32 (an 8-bit integer times an 11-bit fp16 significand)."""
    qb = np.asarray(q, np.int8).reshape(-1, Q8_BLOCK).astype(np.float64)
    return (qb * np.asarray(d, np.float16).astype(np.float64)[:, None]).astype(np.float32).reshape(-1)


def dequant_scales(q: np.ndarray, d: np.ndarray) -> np.ndarray:
    """s_b = RN32(q_b * d_g); the float64 product of an 8-bit and a 24-bit value is exact."""
    q = np.asarray(q, np.uint8)
    g = np.arange(q.size) // GROUP
    return (q.astype(np.float64) * np.asarray(d, np.float32)[g].astype(np.float64)).astype(np.float32)


def dequant(codes: np.ndarray, q: np.ndarray, d: np.ndarray, numel: int | None = None) -> np.ndarray:
    """w' = RN32(c[code] * s_b) as float32 (the product is exact in float64, then one rounding)."""
    c = unpack_codes(codes)
    if numel is not None:
        c = c[:numel]
    s = dequant_scales(q, d)
    book = nf4_codebook().astype(np.float64)
    vals = book[c].reshape(-1, BLOCK) * s.astype(np.float64)[:, None]
    return vals.astype(np.float32).reshape(-1)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), returned as float32."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


# ---------------------------------------------------------------------------
# Frozen-base LoRA linear layer ("Training LoRA directly on GGUF quantized
# weights" page, §2.1 formula h = W0 x + (B A) x and §3.2 module with
# scaling = alpha / r; "Course notes" page, LoRA section W' = W + B A)
# ---------------------------------------------------------------------------

def _f64(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().to("cpu").float().numpy()
    return np.asarray(t, dtype=np.float64)


def lora_linear_fwd(w_deq, x, a, b, scaling: float):
    """Y = X W'^T + s (X A^T) B^T in float64; returns (Y, u) with u = X A^T."""
    W, X = _f64(w_deq), _f64(x)
    Y = X @ W.T
    u = None
    if a is not None and b is not None and _f64(a).size:
        u = X @ _f64(a).T
        Y = Y + float(scaling) * (u @ _f64(b).T)
    return Y, u


def lora_linear_bwd_dx(w_deq, dy, a, b, scaling: float):
    """dX = dY W' + s (dY B) A (chain rule through the frozen base and the adapter); returns (dX, g)."""
    W, dY = _f64(w_deq), _f64(dy)
    dX = dY @ W
    g = None
    if a is not None and b is not None and _f64(a).size:
        g = dY @ _f64(b)
        dX = dX + float(scaling) * (g @ _f64(a))
    return dX, g


def lora_grad_ab(x, dy, u, g, scaling: float):
    """dA = s g^T X  [r, K] and dB = s dY^T u  [N, r]; W0 receives no gradient."""
    X, dY, U, G = _f64(x), _f64(dy), _f64(u), _f64(g)
    return float(scaling) * (G.T @ X), float(scaling) * (dY.T @ U)


def lora_linear_fwd_rows(w_deq, x, a, b, scaling: float, rows):
    """Selected output columns n (rows of W0) of Y, for sampled checks at full size."""
    W = _f64(w_deq)[rows]
    X = _f64(x)
    Y = X @ W.T
    if a is not None and b is not None and _f64(a).size:
        Y = Y + float(scaling) * ((X @ _f64(a).T) @ _f64(b)[rows].T)
    return Y


# ---------------------------------------------------------------------------
# Tolerance used for every floating-point output (the layer's stated bar)
# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# Merging the adapter back into the quantized base ("Course notes" page, §3.3:
# dequantize W to BF16, merge at high precision, quantize again; "Training LoRA
# directly on GGUF quantized weights" page, §3.3 and §4.3: merge the dequantized
# base and the LoRA into bf16, then rerun the quantization, with one rounding in
# the merge and one in the requantization; merge formula W' = W + B A from the
# "Course notes" page, §3.2)
# ---------------------------------------------------------------------------

def lora_merge_bf16(codes, q, d, n_out: int, n_in: int, a, b, scaling: float) -> np.ndarray:
    """The merged base as float32 holding bf16 values:
    m = bf16(RN32(bf16(w') + s * sum_j B[n, j] A[j, k])).

    The dequantized base is taken to bf16 first (the pages' "dequantize to BF16").
    The adapter product and the add are done in float64 ("high precision"), j in
    ascending order; bf16 x bf16 products are exact in float64.  The float64 sum is
    rounded to float32 and then to bf16, the precision the merged base is kept in.
    a [r, K] and b [N, r] are the bf16 adapter factors (any r >= 0)."""
    w = dequant(codes, q, d, n_out * n_in).reshape(n_out, n_in)
    return lora_merge_bf16_deq(w, a, b, scaling)


def lora_merge_bf16_deq(w, a, b, scaling: float) -> np.ndarray:
    """lora_merge_bf16 from an already dequantized float32 base w [N, K] (any storage
    format of the packed weight: the steps after the dequant are the same)."""
    w = np.asarray(w, np.float32)
    n_out, n_in = w.shape
    wb = bf16_round(w).astype(np.float64)
    acc = np.zeros((n_out, n_in), np.float64)
    a64, b64 = _f64(a), _f64(b)
    for j in range(a64.shape[0] if a64.size else 0):
        acc = acc + np.outer(b64[:, j], a64[j, :])
    m = wb + np.float64(np.float32(scaling)) * acc
    return bf16_round(m.astype(np.float32))


def lora_merge_requant(codes, q, d, n_out: int, n_in: int, a, b, scaling: float) -> dict:
    """W'' = quant(merged base): the NF4 + double-quant encode of lora_merge_bf16."""
    return quantize_nf4_dq(lora_merge_bf16(codes, q, d, n_out, n_in, a, b, scaling))


def rel_errors(got, ref):
    """(normwise ||got-ref||_F/||ref||_F, max over rows of max|err| / max(max|ref_row|, 1e-6))."""
    G, R = _f64(got), _f64(ref)
    if G.shape != R.shape:
        raise ValueError(f"shape mismatch {G.shape} vs {R.shape}")
    if R.size == 0:
        return 0.0, 0.0
    diff = G - R
    nrm = np.linalg.norm(R)
    normwise = float(np.linalg.norm(diff) / nrm) if nrm > 0 else float(np.linalg.norm(diff))
    R2 = R.reshape(R.shape[0], -1) if R.ndim > 1 else R.reshape(1, -1)
    D2 = diff.reshape(R2.shape)
    rowmax = np.maximum(np.max(np.abs(R2), axis=1), 1e-6)
    rowwise = float(np.max(np.max(np.abs(D2), axis=1) / rowmax))
    return normwise, rowwise


NORMWISE_TOL = 1e-2
ROWWISE_TOL = 2e-2


def within_tolerance(got, ref) -> bool:
    nw, rw = rel_errors(got, ref)
    return nw <= NORMWISE_TOL and rw <= ROWWISE_TOL
