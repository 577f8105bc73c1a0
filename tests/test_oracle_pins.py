"""Pins of the CPU oracle against facts other than itself (no GPU needed).

Each test names what it pins: a value printed on a page, a closed form, an
invariant of the construction, brute force on a tiny input, or an independent
routine.  A plausible slip in the oracle (wrong nibble order, dropped LoRA
term, transposed operand, wrong rounding, wrong group index) fails at least
one of them.
"""
import json
import math
import os
import statistics
import struct

import numpy as np
import pytest

from oracle import nf4_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------- INT8 example

def test_int8_worked_example_printed_values():
    g = _golden("int8_worked_example.json")
    scale, zp = O.affine_params(g["rmin"], g["rmax"], g["qmin"], g["qmax"])
    assert round(scale, g["printed_scale_decimals"]) == g["printed_scale"]
    assert zp == g["printed_zero_point"]
    q0 = int(O.affine_quant([0.0], scale, zp)[0])
    assert q0 == g["printed_zero_point"]
    assert float(O.affine_dequant([q0], scale, zp)[0]) == g["zero_round_trips_to"]
    # range ends land on the integer range ends
    assert O.affine_quant([g["rmin"], g["rmax"]], scale, zp).tolist() == [0, 255]


def test_int8_example_needs_float64():
    # 2 / (4/255) is exactly 127.5 in float64 (zp 128 under half-even or half-away),
    # but 127.49999 in float32, which would give 127: the helper must run in float64.
    s32 = np.float32(4.0) / np.float32(255.0)
    assert int(np.rint(np.float32(2.0) / s32)) == 127
    assert 2.0 / (4.0 / 255.0) == 127.5
    assert O.affine_params(-2.0, 2.0)[1] == 128


def test_symmetric_int8_scale():
    scale, zp = O.symmetric_params(-0.5, 2.0)
    assert zp == 0 and scale == 2.0 / 127.0


# --------------------------------------------------------------- accounting

def test_constant_overhead_closed_form_and_printed_figures():
    g = _golden("dq_accounting.json")
    p, tol = g["printed"], g["relative_tolerance"]
    n = g["params_7b"]

    def close(key, value):
        assert abs(value - p[key]) <= tol.get(key, 1e-9) * abs(p[key]), (key, value, p[key])

    bits = O.constant_bits_per_param()
    assert bits == 8 / 64 + 32 / (64 * 256) == 0.126953125
    close("bits_per_param_dq", bits)
    assert O.constant_bits_per_param(dq=False) == p["bits_per_param_fp32_scale_only"]
    assert 64 / 64 == p["bits_per_param_scale_plus_zp_fp32"]          # 8 B (scale+zp) per 64
    close("dq_saving_bits_per_param", O.constant_bits_per_param(dq=False) - bits)
    close("blocks_7b", n / 64)
    close("groups_7b", n / 64 / 256)
    close("first_level_fp32_scales_gb", n / 64 * 4 / 1e9)
    close("first_level_u8_scales_gb", n / 64 / 1e9)
    close("second_level_mb", 4 * n / (64 * 256) / 1e6)
    assert n / 64 * 8 / 1e9 == p["constants_no_dq_gb"]
    close("constants_dq_gb", (n / 64 + 4 * n / 16384) / 1e9)
    assert n * 4 / 8 / 1e9 == p["weights_4bit_gb"]
    assert n * 4 / 8 / 1e9 + p["constants_no_dq_gb"] == p["total_no_dq_gb"]
    total_dq = O.packed_bytes(int(n)) / 1e9
    close("total_dq_gb", total_dq)
    close("reduction_percent", 100 * (p["total_no_dq_gb"] - total_dq) / p["total_no_dq_gb"])


@pytest.mark.parametrize("n", [64, 128, 16384, 16384 + 64, 3 * 16384 - 64, 4096 * 4096, 11008 * 4096])
def test_packed_bytes_closed_form(n):
    assert O.packed_bytes(n) == n // 2 + n // 64 + 4 * math.ceil(n / 16384)
    q = O.quantize_nf4_dq(np.linspace(-1, 1, n, dtype=np.float32)) if n <= 65536 else None
    if q is not None:
        assert q["codes"].nbytes + q["scales"].nbytes + q["scales2"].nbytes == O.packed_bytes(n)


# --------------------------------------------------------------- normal quantiles

def _as241(p):
    """Wichura's AS241 (PPND16), written out independently of the oracle's bisection."""
    q = p - 0.5
    if abs(q) <= 0.425:
        r = 0.180625 - q * q
        num = (((((((2509.0809287301226727 * r + 33430.575583588128105) * r + 67265.770927008700853) * r
                   + 45921.953931549871457) * r + 13731.693765509461125) * r + 1971.5909503065514427) * r
                + 133.14166789178437745) * r + 3.387132872796366608)
        den = (((((((5226.495278852545925 * r + 28729.085735721942674) * r + 39307.89580009271061) * r
                   + 21213.794301586595867) * r + 5394.1960214247511077) * r + 687.1870074920579083) * r
                + 42.313330701600911252) * r + 1.0)
        return q * num / den
    r = p if q < 0 else 1.0 - p
    r = math.sqrt(-math.log(r))
    if r <= 5.0:
        r -= 1.6
        num = (((((((7.7454501427834140764e-4 * r + 0.0227238449892691845833) * r + 0.24178072517745061177) * r
                   + 1.27045825245236838258) * r + 3.64784832476320460504) * r + 5.7694972214606914055) * r
                + 4.6303378461565452959) * r + 1.42343711074968357734)
        den = (((((((1.05075007164441684324e-9 * r + 5.475938084995344946e-4) * r + 0.0151986665636164571966) * r
                   + 0.14810397642748007459) * r + 0.68976733498510000455) * r + 1.6763848301838038494) * r
                + 2.05319162663775882187) * r + 1.0)
    else:
        r -= 5.0
        num = (((((((2.01033439929228813265e-7 * r + 2.71155556874348757815e-5) * r + 0.0012426609473880784386) * r
                   + 0.026532189526576123093) * r + 0.29656057182850489123) * r + 1.7848265399172913358) * r
                + 5.4637849111641143699) * r + 6.6579046435011037772)
        den = (((((((2.04426310338993978564e-15 * r + 1.4215117583164458887e-7) * r + 1.8463183175100546818e-5) * r
                   + 7.868691311456132591e-4) * r + 0.0148753612908506148525) * r + 0.13692988092273580531) * r
                + 0.59983220655588793769) * r + 1.0)
    x = num / den
    return -x if q < 0 else x


def test_normal_ppf_textbook_values():
    assert abs(O.normal_ppf(0.5)) < 1e-15          # bisection resolves to within an ulp of the flat CDF
    assert abs(O.normal_ppf(0.975) - 1.959963984540054) < 1e-14
    assert abs(O.normal_ppf(0.8413447460685429) - 1.0) < 1e-14          # Phi(1)
    assert abs(O.normal_ppf(0.022750131948179195) + 2.0) < 1e-13       # Phi(-2)
    for p in (0.6, 0.9, 0.99, 0.9677083333333334):
        assert O.normal_ppf(1 - p) == pytest.approx(-O.normal_ppf(p), abs=1e-14)


def test_normal_ppf_against_two_independent_routines():
    nd = statistics.NormalDist()
    ps = np.concatenate([np.linspace(0.501, 0.999, 97), [0.5 + j * (O.NF4_DELTA - 0.5) / 8 for j in range(1, 9)],
                         [0.5 + j * (O.NF4_DELTA - 0.5) / 7 for j in range(1, 8)]])
    for p in ps:
        x = O.normal_ppf(float(p))
        assert abs(x - _as241(float(p))) <= 4e-15 * max(1.0, abs(x))
        assert abs(x - nd.inv_cdf(float(p))) <= 4e-15 * max(1.0, abs(x))


# --------------------------------------------------------------- NF4 codebook

def test_codebook_invariants():
    c = O.nf4_codebook()
    assert c.dtype == np.float32 and c.size == 16
    assert c[0] == -1.0 and c[7] == 0.0 and c[15] == 1.0
    assert np.all(np.diff(c.astype(np.float64)) > 0)
    assert (c < 0).sum() == 7 and (c > 0).sum() == 8
    # dense near zero, sparse in the tails: gaps grow away from zero on both sides
    lv = O.nf4_levels_f64()
    pos_gaps = np.diff(lv[7:])
    neg_gaps = -np.diff(lv[:8][::-1])
    assert np.all(np.diff(pos_gaps) > 0) and np.all(np.diff(neg_gaps) > 0)


def test_codebook_levels_carry_equal_probability_mass():
    # each half's levels sit at equally spaced probabilities of N(0,1): the
    # "each level gets about the same number of weights" property, checked
    # with the stdlib normal CDF (not the oracle's).
    lv = O.nf4_levels_f64()
    delta = ((1 - 1 / 30) + (1 - 1 / 32)) / 2           # offset of the construction reading
    top = statistics.NormalDist().inv_cdf(delta)
    cdf = statistics.NormalDist().cdf
    pos = [cdf(v * top) - 0.5 for v in lv[8:]]
    neg = [0.5 - cdf(v * top) for v in lv[:7][::-1]]
    assert np.allclose(np.diff([0.0] + pos), (delta - 0.5) / 8, rtol=0, atol=1e-13)
    assert np.allclose(np.diff([0.0] + neg), (delta - 0.5) / 7, rtol=0, atol=1e-13)
    # the two halves follow one formula: the n=8 half at j and the n=7 half at j' coincide when j/8 = j'/7
    assert lv[15] == -lv[0] == 1.0


# --------------------------------------------------------------- code selection

def _thresholds(book):
    mids = (book[:-1].astype(np.float64) + book[1:].astype(np.float64)) / 2.0   # exact in float64
    t = mids.astype(np.float32)
    up = t.astype(np.float64) <= mids
    t[up] = np.nextafter(t[up], np.float32(np.inf))
    return t


def test_nearest_code_matches_threshold_rule_around_every_midpoint():
    book = O.nf4_codebook()
    T = _thresholds(book)
    vals = []
    for t in T:
        v = t
        for _ in range(70):
            v = np.nextafter(v, np.float32(-np.inf))
        for _ in range(140):
            vals.append(v)
            v = np.nextafter(v, np.float32(np.inf))
    vals = np.array(vals, dtype=np.float32)
    got = O.nearest_code(vals)
    rule = (vals[:, None] >= T[None, :]).sum(axis=1)
    assert np.array_equal(got, rule.astype(np.uint8))


def test_nearest_code_exact_ties_go_to_lower_index():
    book = O.nf4_codebook()
    # midpoints that are exactly representable in float32: next to the zero level
    m67 = np.float32(book[6] / 2)
    m78 = np.float32(book[8] / 2)
    assert float(m67) == (float(book[6]) + 0.0) / 2 and float(m78) == (0.0 + float(book[8])) / 2
    assert O.nearest_code(np.array([m67, m78], np.float32)).tolist() == [6, 7]


def test_nearest_code_brute_force_python():
    rng = np.random.default_rng(7)
    book = [float(x) for x in O.nf4_codebook()]
    vals = rng.uniform(-1, 1, 2000).astype(np.float32)
    got = O.nearest_code(vals)
    for v, g in zip(vals, got):
        d = [abs(float(v) - b) for b in book]
        best = min(range(16), key=lambda i: (d[i], i))
        assert best == g


# --------------------------------------------------------------- encode / DQ / dequant

def test_pack_order_low_nibble_first():
    assert O.pack_codes(np.array([1, 2, 3, 4], np.uint8)).tolist() == [0x21, 0x43]
    assert O.unpack_codes(np.array([0x21, 0x43], np.uint8)).tolist() == [1, 2, 3, 4]


def _exact_weights(n_blocks, rng, exps):
    """Weights that NF4+DQ reproduces exactly: each block's absmax is 255 * 2^e and every
    weight is RN32(c[j] * absmax), with the block max present."""
    book = O.nf4_codebook().astype(np.float64)
    codes = rng.integers(0, 16, size=(n_blocks, 64))
    codes[:, 0] = rng.choice([0, 15], size=n_blocks)
    a = 255.0 * np.ldexp(1.0, exps)
    w = (book[codes] * a[:, None]).astype(np.float32)
    return w.reshape(-1), codes.reshape(-1).astype(np.uint8)


def test_encode_dequant_round_trip_exact_on_representable_weights():
    rng = np.random.default_rng(1)
    nb = 3 * 256 + 17                      # three full DQ groups and a ragged tail
    exps = np.repeat(rng.integers(-12, -2, size=4), 256)[:nb]   # one absmax per DQ group
    w, codes = _exact_weights(nb, rng, exps)
    q = O.quantize_nf4_dq(w)
    assert np.array_equal(q["codes_unpacked"], codes)
    assert np.all(q["scales"] == 255)
    assert np.array_equal(q["scales2"], np.ldexp(1.0, exps[::256]).astype(np.float32))
    back = O.dequant(q["codes"], q["scales"], q["scales2"])
    assert np.array_equal(back, w)
    # the block maximum always takes an end code
    assert set(q["codes_unpacked"].reshape(-1, 64)[:, 0].tolist()) <= {0, 15}


def test_dq_brute_force_over_all_256_levels():
    rng = np.random.default_rng(3)
    a = rng.uniform(0, 3.0, size=256 + 100).astype(np.float32)
    a[5] = 0.0
    q, d = O.double_quant(a)
    assert d.size == 2
    for g in range(2):
        seg = a[g * 256:(g + 1) * 256]
        assert d[g] == np.float32(float(seg.max()) / 255.0)
        assert q[g * 256 + int(np.argmax(seg))] == 255
        for i, ab in enumerate(seg):
            ratio = np.float32(float(ab) / float(d[g]))
            # brute force: q minimises |q - ratio| over all 256 levels, ties to even
            cands = sorted(range(256), key=lambda k: (abs(k - float(ratio)), k % 2))
            assert q[g * 256 + i] == cands[0]
    assert q[5] == 0


def test_dq_groups_are_independent():
    w = np.zeros(2 * 16384, np.float32)
    w[0] = 1.0
    w[16384] = 1000.0
    w[16384 + 64] = 1.0
    q = O.quantize_nf4_dq(w)
    assert q["scales2"][0] == np.float32(1.0 / 255) and q["scales2"][1] == np.float32(1000.0 / 255)
    assert q["scales"][0] == 255 and q["scales"][256] == 255 and q["scales"][257] == 0
    assert np.all(q["scales"][1:256] == 0)


def test_zero_weight_gives_code7_and_zero_scales():
    q = O.quantize_nf4_dq(np.zeros(16384 + 128, np.float32))
    assert np.all(q["codes_unpacked"] == 7)
    assert np.all(q["scales"] == 0) and np.all(q["scales2"] == 0)
    assert np.all(O.dequant(q["codes"], q["scales"], q["scales2"]) == 0)


def test_power_of_two_scaling_invariance():
    rng = np.random.default_rng(11)
    w = (rng.standard_normal(16384 * 2) * 0.02).astype(np.float32)
    a = O.quantize_nf4_dq(w)
    b = O.quantize_nf4_dq(w * np.float32(8.0))
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    assert np.array_equal(a["scales2"] * 8, b["scales2"])


def test_round_trip_error_bound():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(16384 * 3) * 0.02).astype(np.float32)
    w[rng.choice(w.size, 50, replace=False)] *= 10
    q = O.quantize_nf4_dq(w)
    back = O.dequant(q["codes"], q["scales"], q["scales2"]).astype(np.float64)
    lv = O.nf4_levels_f64()
    half_gap = float(np.max(np.diff(O.nf4_codebook().astype(np.float64)))) / 2
    a = q["absmax"].astype(np.float64)
    s = O.dequant_scales(q["scales"], q["scales2"]).astype(np.float64)
    bound = np.repeat(a * half_gap + np.abs(a - s), 64) * (1 + 1e-6) + 1e-30
    assert np.all(np.abs(w.astype(np.float64) - back) <= bound)
    assert abs(lv[0]) == 1.0


# --------------------------------------------------------------- layer maths

def _case(M=5, N=6, K=128, r=8, seed=0):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K))
    X = rng.standard_normal((M, K))
    A = rng.standard_normal((r, K)) / K
    B = rng.standard_normal((N, r)) * 0.01
    dY = rng.standard_normal((M, N))
    return W, X, A, B, dY


def test_matmul_is_the_textbook_sum():
    W, X, A, B, _ = _case(M=3, N=4, K=64, r=2)
    Y, u = O.lora_linear_fwd(W, X, A, B, 2.0)
    for m in range(3):
        for n in range(4):
            base = sum(X[m, k] * W[n, k] for k in range(64))
            lora = sum(B[n, j] * sum(A[j, k] * X[m, k] for k in range(64)) for j in range(2))
            assert abs(Y[m, n] - (base + 2.0 * lora)) < 1e-12


def test_b_zero_gives_the_base_output():
    W, X, A, B, _ = _case()
    Y0, _ = O.lora_linear_fwd(W, X, None, None, 2.0)
    Yb, _ = O.lora_linear_fwd(W, X, A, np.zeros_like(B), 2.0)
    assert np.array_equal(Y0, Yb)
    Yl, u = O.lora_linear_fwd(np.zeros_like(W), X, A, B, 2.0)
    assert np.allclose(Yl, 2.0 * (X @ A.T) @ B.T, rtol=0, atol=1e-15)


def test_adjoint_identity_and_lora_directional_derivatives():
    W, X, A, B, dY = _case(M=7, N=9, K=192, r=16, seed=4)
    s = 2.0
    Y, u = O.lora_linear_fwd(W, X, A, B, s)
    dX, g = O.lora_linear_bwd_dx(W, dY, A, B, s)
    dA, dB = O.lora_grad_ab(X, dY, u, g, s)
    L = lambda Xv, Av, Bv: float(np.sum(dY * O.lora_linear_fwd(W, Xv, Av, Bv, s)[0]))
    rng = np.random.default_rng(9)
    E = rng.standard_normal(X.shape)
    # Y is linear in X, A and B separately, so these differences are exact up to rounding
    assert abs((L(X + E, A, B) - L(X, A, B)) - float(np.sum(dX * E))) < 1e-8 * abs(L(X, A, B)) + 1e-9
    EA = rng.standard_normal(A.shape)
    assert abs((L(X, A + EA, B) - L(X, A, B)) - float(np.sum(dA * EA))) < 1e-9
    EB = rng.standard_normal(B.shape)
    assert abs((L(X, A, B + EB) - L(X, A, B)) - float(np.sum(dB * EB))) < 1e-9
    # base-only adjoint: <dY, X W^T> = <dY W, X>
    assert abs(np.sum(dY * (X @ W.T)) - np.sum((dY @ W) * X)) < 1e-9


def test_rows_helper_matches_full_forward():
    W, X, A, B, _ = _case(M=4, N=10, K=64, r=8, seed=2)
    Y, _ = O.lora_linear_fwd(W, X, A, B, 1.5)
    rows = np.array([0, 3, 9])
    assert np.allclose(O.lora_linear_fwd_rows(W, X, A, B, 1.5, rows), Y[:, rows], rtol=0, atol=1e-13)


def test_tolerance_metric():
    ref = np.array([[1.0, -2.0], [0.0, 0.0]])
    got = ref + np.array([[0.01, 0.0], [0.0, 0.0]])
    nw, rw = O.rel_errors(got, ref)
    assert nw == pytest.approx(0.01 / math.sqrt(5))
    assert rw == pytest.approx(0.01 / 2.0)
    assert O.within_tolerance(got, ref)
    assert not O.within_tolerance(ref * 1.05, ref)


def test_bf16_round_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9], np.float32)
    assert O.bf16_round(x).tolist() == [1.0, 1.0, 1.0 + 2 ** -6, 1.0]


# --------------------------------------------------------------- exact-arithmetic pins of each rounding

from fractions import Fraction


def _rn32_exact(fr: Fraction) -> np.float32:
    """Nearest float32 to an exact rational, ties to even (brute force over the neighbours)."""
    c = np.float32(float(fr))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    def key(v):
        bits = int(np.array(v, np.float32).view(np.uint32))
        return (abs(Fraction(float(v)) - fr), bits & 1)
    return min(cands, key=key)


def test_normalise_is_correctly_rounded_division():
    rng = np.random.default_rng(21)
    w = (rng.standard_normal(64 * 40) * 0.02).astype(np.float32)
    a = O.block_absmax(w)
    n = O.normalise(w, a).reshape(-1)
    for i in range(0, w.size, 7):
        exact = Fraction(float(w[i])) / Fraction(float(a[i // 64]))
        assert n[i] == _rn32_exact(exact)


def test_dq_ratio_and_products_are_correctly_rounded():
    rng = np.random.default_rng(22)
    a = rng.uniform(1e-4, 0.3, size=300).astype(np.float32)
    q, d = O.double_quant(a)
    for g in range(2):
        seg = a[g * 256:(g + 1) * 256]
        assert d[g] == _rn32_exact(Fraction(float(seg.max())) / 255)
        for i in range(0, seg.size, 5):
            r = _rn32_exact(Fraction(float(seg[i])) / Fraction(float(d[g])))
            k = int(np.floor(float(r)))
            frac = Fraction(float(r)) - k
            expect = k + (1 if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and k % 2 == 1) else 0)
            assert q[g * 256 + i] == min(max(expect, 0), 255)
    s = O.dequant_scales(q, d)
    book = O.nf4_codebook()
    for b in range(0, s.size, 9):
        assert s[b] == _rn32_exact(Fraction(int(q[b])) * Fraction(float(d[b // 256])))
    codes = np.tile(np.arange(16, dtype=np.uint8), 300 * 4)
    w = O.dequant(O.pack_codes(codes), q, d)
    for i in range(0, w.size, 37):
        assert w[i] == _rn32_exact(Fraction(float(book[codes[i]])) * Fraction(float(s[i // 64])))


# ------------------------------------------------ LoRA merge and requantize

def _f32_rn(x):
    """IEEE float32 round-to-nearest of a Python float, through struct packing."""
    return struct.unpack("<f", struct.pack("<f", x))[0]


def _bf16_rn(x):
    """bfloat16 round-to-nearest-even of a float32 value, on its bit pattern as an int."""
    u = struct.unpack("<I", struct.pack("<f", x))[0]
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return struct.unpack("<f", struct.pack("<I", u & 0xFFFFFFFF))[0]


def _merge_case(n_out, n_in, r, seed, w_std=0.02):
    rng = np.random.default_rng(seed)
    W = rng.normal(0, w_std, (n_out, n_in)).astype(np.float32)
    ref = O.quantize_nf4_dq(W)
    A = O.bf16_round(rng.normal(0, 1.0 / n_in, (r, n_in)).astype(np.float32))
    B = O.bf16_round(rng.normal(0, 0.01, (n_out, r)).astype(np.float32))
    return ref, A, B


def test_merge_brute_force_python():
    # pins lora_merge_bf16 by pure-Python loops: per element, the bf16 base, the
    # float64 sum over j in ascending order, then float32 and bf16 rounding by struct
    n_out, n_in, r, s = 8, 64, 8, 2.0
    ref, A, B = _merge_case(n_out, n_in, r, seed=71)
    got = O.lora_merge_bf16(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, A, B, s)
    book = [float(v) for v in O.nf4_codebook()]
    for n in range(n_out):
        for k in range(n_in):
            e = n * n_in + k
            byte = int(ref["codes"][e // 2])
            code = (byte & 15) if e % 2 == 0 else (byte >> 4)
            blk = e // 64
            sb = _f32_rn(float(ref["scales"][blk]) * float(ref["scales2"][blk // 256]))
            w = _f32_rn(book[code] * sb)
            acc = 0.0
            for j in range(r):
                acc = acc + float(B[n, j]) * float(A[j, k])
            want = _bf16_rn(_f32_rn(_bf16_rn(w) + float(np.float32(s)) * acc))
            assert float(got[n, k]) == want, (n, k)


def test_merge_rank_one_single_row_closed_form():
    # B = unit column at row n0: only row n0 moves, by bf16(RN32(bf16(w') + s a_k))
    n_out, n_in, s, n0 = 16, 128, 0.75, 5
    ref, _, _ = _merge_case(n_out, n_in, 1, seed=72)
    rng = np.random.default_rng(73)
    a = O.bf16_round(rng.normal(0, 0.05, (1, n_in)).astype(np.float32))
    b = np.zeros((n_out, 1), np.float32)
    b[n0, 0] = 1.0
    got = O.lora_merge_bf16(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, a, b, s)
    base = O.bf16_round(O.dequant(ref["codes"], ref["scales"], ref["scales2"])).reshape(n_out, n_in)
    others = np.arange(n_out) != n0
    assert np.array_equal(got[others], base[others])
    for k in range(n_in):
        assert float(got[n0, k]) == _bf16_rn(_f32_rn(float(base[n0, k]) + s * float(a[0, k])))


def test_merge_of_zero_base_is_the_exact_adapter_product():
    # W0 = 0 encodes to code 7 and zero scales, so the base dequantizes to 0; with
    # power-of-two factors s B A is exact in bf16, the merge returns it unchanged and
    # the requantization equals the plain encode of s B A
    n_out, n_in, r, s = 32, 256, 8, 0.5
    ref = O.quantize_nf4_dq(np.zeros((n_out, n_in), np.float32))
    rng = np.random.default_rng(74)
    A = (2.0 ** rng.integers(-6, 0, (r, n_in))).astype(np.float32) * rng.choice([-1, 1], (r, n_in))
    B = np.zeros((n_out, r), np.float32)
    B[np.arange(n_out), rng.integers(0, r, n_out)] = (2.0 ** rng.integers(-4, 0, n_out)).astype(np.float32)
    prod = s * B.astype(np.float64) @ A.astype(np.float64)
    got = O.lora_merge_bf16(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, A, B, s)
    assert np.array_equal(got.astype(np.float64), prod)
    out = O.lora_merge_requant(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, A, B, s)
    direct = O.quantize_nf4_dq(prod.astype(np.float32))
    for key in ("codes", "scales", "scales2"):
        assert np.array_equal(out[key], direct[key])


def test_merge_close_to_float64_definition():
    # the merged base is W' + s B A up to the bf16 roundings (two, each 2^-9 relative)
    n_out, n_in, r, s = 64, 512, 16, 2.0
    ref, A, B = _merge_case(n_out, n_in, r, seed=75)
    got = O.lora_merge_bf16(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, A, B, s).astype(np.float64)
    w = O.dequant(ref["codes"], ref["scales"], ref["scales2"]).reshape(n_out, n_in).astype(np.float64)
    exact = w + s * B.astype(np.float64) @ A.astype(np.float64)
    assert np.all(np.abs(got - exact) <= np.abs(w) * 2.0 ** -8 + np.abs(exact) * 2.0 ** -8 + 1e-30)
    # the adapter term is really in it: with factors large enough that s B A is far
    # above the bf16 rounding of the base, the merged change is s B A
    # (at the realistic adapter scale the two are comparable, the merge loss the
    # GGUF page warns about)
    rng = np.random.default_rng(77)
    A2 = O.bf16_round(rng.normal(0, 1.0 / 16, (r, n_in)).astype(np.float32))
    B2 = O.bf16_round(rng.normal(0, 0.1, (n_out, r)).astype(np.float32))
    got2 = O.lora_merge_bf16(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, A2, B2, s).astype(np.float64)
    delta = got2 - O.bf16_round(w.astype(np.float32)).astype(np.float64)
    lora = s * B2.astype(np.float64) @ A2.astype(np.float64)
    assert np.linalg.norm(delta - lora) < 0.05 * np.linalg.norm(lora)


def test_merge_requant_round_trip_bound():
    # the requantized merge obeys the encode's per-block bound around the merged base
    n_out, n_in, r, s = 64, 512, 8, 2.0
    ref, A, B = _merge_case(n_out, n_in, r, seed=76)
    m = O.lora_merge_bf16(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, A, B, s).reshape(-1)
    out = O.lora_merge_requant(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, A, B, s)
    back = O.dequant(out["codes"], out["scales"], out["scales2"]).astype(np.float64)
    a = out["absmax"].astype(np.float64)
    sb = O.dequant_scales(out["scales"], out["scales2"]).astype(np.float64)
    half_gap = float(np.max(np.diff(O.nf4_codebook().astype(np.float64)))) / 2
    bound = np.repeat(a * half_gap + np.abs(a - sb), 64) * (1 + 1e-6) + 1e-30
    assert np.all(np.abs(back - m.astype(np.float64)) <= bound)


# ------------------------------------------------------- format variants

def _brute_encode(w, block, book, scale_of_block):
    """Pure-Python blockwise encode: nearest level (first index on ties) of RN32(w / scale)."""
    lv = [float(v) for v in book]
    codes = []
    for b in range(len(w) // block):
        sc = scale_of_block(b)
        for x in w[b * block:(b + 1) * block]:
            n = 0.0 if sc == 0.0 else _f32_rn(float(x) / sc)
            best, bd = 0, abs(n - lv[0])
            for k in range(1, 16):
                dk = abs(n - lv[k])
                if dk < bd:
                    best, bd = k, dk
            codes.append(best)
    return codes


def test_variant_defaults_reduce_to_the_nf4_dq_encode():
    w = (np.random.default_rng(81).standard_normal(16384 * 2 + 640) * 0.02).astype(np.float32)
    a, b = O.quantize_variant(w), O.quantize_nf4_dq(w)
    for key in ("codes", "scales", "scales2"):
        assert np.array_equal(a[key], b[key])
    assert np.array_equal(O.dequant_variant(a["codes"], a["scales"], a["scales2"]),
                          O.dequant(b["codes"], b["scales"], b["scales2"]))


@pytest.mark.parametrize("block,dq", [(128, True), (128, False), (64, False)])
def test_variant_encode_brute_force_python(block, dq):
    w = (np.random.default_rng(82).standard_normal(block * 6) * 0.02).astype(np.float32)
    w[: block] = 0.0                       # an all-zero block
    got = O.quantize_variant(w, block=block, dq=dq)
    absmax = [max(abs(float(x)) for x in w[b * block:(b + 1) * block]) for b in range(6)]
    want = _brute_encode(w.tolist(), block, O.nf4_codebook(), lambda b: absmax[b])
    assert got["codes_unpacked"].tolist() == want
    if not dq:
        assert got["scales"].tolist() == [np.float32(a) for a in absmax]


def test_codes_after_dq_brute_force_python():
    w = (np.random.default_rng(83).standard_normal(64 * 300) * 0.02).astype(np.float32)
    got = O.quantize_variant(w, codes_after_dq=True)
    q, d = got["scales"], got["scales2"]
    sb = [_f32_rn(float(q[b]) * float(d[b // 256])) for b in range(300)]
    want = _brute_encode(w.tolist(), 64, O.nf4_codebook(), lambda b: sb[b])
    assert got["codes_unpacked"].tolist() == want
    # the same scales as the default encode; only codes near a threshold move
    base = O.quantize_nf4_dq(w)
    assert np.array_equal(q, base["scales"]) and np.array_equal(d, base["scales2"])
    moved = np.mean(got["codes_unpacked"] != base["codes_unpacked"])
    assert 0 < moved < 0.1


def test_variant_dq_off_round_trip_exact_on_representable_weights():
    # w = c_k * a with a power-of-two absmax: fp32 absmax kept exactly, codes exact
    rng = np.random.default_rng(84)
    book = O.nf4_codebook()
    for block in (64, 128):
        codes = rng.integers(0, 16, size=block * 8).astype(np.uint8)
        codes[::block] = 15                 # the absmax element of each block is +1 * a
        a = (2.0 ** rng.integers(-12, -2, size=8)).astype(np.float32)
        w = (book[codes].reshape(-1, block).astype(np.float64) * a[:, None]).astype(np.float32).reshape(-1)
        got = O.quantize_variant(w, block=block, dq=False)
        assert np.array_equal(got["codes_unpacked"], codes)
        assert np.array_equal(O.dequant_variant(got["codes"], got["scales"], None, block=block), w)


def test_variant_storage_closed_forms():
    n = 4096 * 11008
    for block, dq in ((64, True), (128, True), (64, False), (128, False)):
        assert O.packed_bytes_variant(n, block, dq) * 8 == pytest.approx(
            n * (4 + O.constant_bits_per_param(block=block, dq=dq)), rel=1e-6)
    assert O.packed_bytes_variant(n) == O.packed_bytes(n)
    # halving the block doubles the constants; DQ off costs 32/64 = 0.5 bit per weight at 64
    assert O.constant_bits_per_param(block=64, dq=False) == 0.5
    assert O.constant_bits_per_param(block=128, dq=False) == 0.25


def test_fp4_table_invariants():
    book = O.fp4_codebook()
    assert book.size == 16 and np.all(np.diff(book.astype(np.float64)) >= 0)
    assert book[0] == -1.0 and book[15] == 1.0 and book[7] == 0.0 and book[8] == 0.0
    assert np.signbit(book[7]) and not np.signbit(book[8])
    assert np.array_equal(book[::-1], -book)
    # every level times 6 is an E2M1 magnitude: 0, 0.5, 1, 1.5, 2, 3, 4, 6
    assert sorted({abs(float(v)) * 6 for v in O.fp4_levels_f64()}) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    # a zero normalised value takes -0, a tiny positive one +0, a tiny negative one -0
    got = O.nearest_code(np.array([0.0, 1e-30, -1e-30, 1.0 / 24], np.float32), book).tolist()
    assert got[:3] == [7, 8, 7]


def test_fp4_nearest_code_matches_threshold_rule_around_every_midpoint():
    # the threshold rule: T_k = smallest float32 strictly above the exact midpoint of
    # levels k, k+1 (the +0 copy gets the smallest positive float32) and
    # code = #{k : n >= T_k}; it agrees with the oracle's nearest-level rule
    book = O.fp4_codebook()
    lv = book.astype(np.float64)
    T = []
    for k in range(15):
        mid = (lv[k] + lv[k + 1]) / 2
        t = np.float32(mid)
        if float(t) <= mid:
            t = np.nextafter(t, np.float32(np.inf))
        T.append(float(t))
    assert all(a <= b for a, b in zip(T, T[1:]))
    vals = []
    for k in range(15):
        t = np.float32(T[k])
        for step in range(-3, 4):
            v = t
            for _ in range(abs(step)):
                v = np.nextafter(v, np.float32(np.inf if step > 0 else -np.inf))
            vals.append(v)
    vals = np.array(vals + [0.0, -0.0, 1.0, -1.0], np.float32)
    want = [sum(1 for t in T if float(v) >= t) for v in vals]
    assert O.nearest_code(vals, book).tolist() == want


def _rms_error(w, **kw):
    book = kw.get("book")
    block = kw.get("block", 64)
    q = O.quantize_variant(w, **kw)
    back = O.dequant_variant(q["codes"], q["scales"], q.get("scales2") if kw.get("dq", True) else None,
                             block=block, book=book)
    return float(np.sqrt(np.mean((back.astype(np.float64) - w.astype(np.float64)) ** 2)))


def test_pages_claims_on_normal_weights():
    # "QLoRA double quantization ..." page: larger blocks raise the quantization error
    # (§3.1); double quantization barely changes it (§3.2); nf4 fits normal weights
    # better than fp4 (§3.3)
    w = (np.random.default_rng(85).standard_normal(16384 * 8) * 0.02).astype(np.float32)
    e64 = _rms_error(w)
    e128 = _rms_error(w, block=128)
    e64_nodq = _rms_error(w, dq=False)
    efp4 = _rms_error(w, book=O.fp4_codebook())
    assert e128 > e64
    assert abs(e64 - e64_nodq) < 0.02 * e64_nodq
    assert efp4 > 1.05 * e64


# ------------------------------------------------------------------- Q8_0

def test_q8_0_storage_matches_the_page_figures():
    # GGUF page §1.1: a little over one byte per weight; a 3.8B model of 7.6 GB in bf16
    # is about 4 GB in Q8_0
    n = 3_800_000_000 // 32 * 32
    assert O.q8_0_packed_bytes(n) / n == 34 / 32
    assert 2 * n / 1e9 == pytest.approx(7.6, abs=0.01)
    assert O.q8_0_packed_bytes(n) / 1e9 == pytest.approx(4.0, abs=0.05)


def test_q8_0_brute_force_python():
    rng = np.random.default_rng(91)
    w = (rng.standard_normal(32 * 20) * 0.02).astype(np.float32)
    w[:32] = 0.0
    got = O.quantize_q8_0(w)
    for b in range(20):
        blk = [float(x) for x in w[b * 32:(b + 1) * 32]]
        d = float(np.float16(max(abs(x) for x in blk) / 127.0))
        assert float(got["d"][b]) == d
        for i, x in enumerate(blk):
            if d == 0.0:
                want = 0
            else:
                t = x / d
                fl = math.floor(t)
                frac = t - fl
                want = fl + (1 if frac > 0.5 or (frac == 0.5 and fl % 2 == 1) else 0)
                want = max(-127, min(127, want))
            assert int(got["q"][b * 32 + i]) == want


def test_q8_0_float32_quotient_decides_like_the_exact_one():
    # The kernels divide in float32 (IEEE, correctly rounded) before rounding to an
    # integer; the oracle divides in float64.  Rounding is monotonic and a half-integer
    # k + 1/2 below 128 is a float32, so RN32(w / d) reaches it only when w / d equals
    # it: both precisions round every quotient to the same integer.  Checked here on
    # weights at and one or two float32 steps around every half-integer tie.
    rng = np.random.default_rng(93)
    for _ in range(3000):
        d = float(np.float16(rng.uniform(1e-5, 2e-3)))
        k = int(rng.integers(-128, 127))
        w0 = np.float32((k + 0.5) * d)
        ws = [w0]
        for _ in range(2):
            ws = [np.nextafter(ws[0], np.float32(-1))] + ws + [np.nextafter(ws[-1], np.float32(1))]
        for w in ws:
            t64 = float(w) / d
            t32 = float(np.float32(t64))
            assert np.rint(t64) == np.rint(t32), (w, d)


def test_q8_0_round_trip_bound_and_exact_values():
    rng = np.random.default_rng(92)
    w = (rng.standard_normal(32 * 512) * 0.02).astype(np.float32)
    g = O.quantize_q8_0(w)
    back = O.dequant_q8_0(g["q"], g["d"]).astype(np.float64)
    d = np.repeat(g["d"].astype(np.float64), 32)
    # half a step, plus the clamp at 127 when fp16 rounded the scale down
    assert np.all(np.abs(back - w) <= d * 0.5 + np.abs(w) * 2.0 ** -10 + 1e-30)
    # integers times a representable scale come back exactly
    d0 = np.float16(2.0 ** -9)
    q0 = rng.integers(-127, 128, size=32 * 8)
    q0[::32] = 127
    w0 = (q0.astype(np.float64) * float(d0)).astype(np.float32)
    g0 = O.quantize_q8_0(w0)
    assert np.array_equal(g0["q"].astype(np.int64), q0) and np.all(g0["d"] == d0)
    assert np.array_equal(O.dequant_q8_0(g0["q"], g0["d"]), w0)
