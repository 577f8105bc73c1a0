"""Storage formats of the first-level scales on the GPU against the oracle.

The "QLoRA double quantization and block-wise quantization memory" page, sections 3.1
and 3.2, lets the block size be 64 or 128 and double quantization be on or off; the
oracle's quantize_variant / dequant_variant restate those choices, and its reading
"codes against the double-quantized scale" is the third switch.  Encode and dequant
are compared bit for bit in every combination, for NF4 and FP4 levels; the layer
(forward and dX on the CTA-pair, split-K and small-M shapes) within the usual
tolerance; the merge bit for bit across formats."""
import numpy as np
import pytest
import torch

import bit_quantized_base_nf4_b200 as q
from bit_quantized_base_nf4_b200 import synthetic as syn
from oracle import nf4_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
B128, NODQ, AFTER = q.QLORA_FMT_BLOCK128, q.QLORA_FMT_NO_DQ, q.QLORA_FMT_CODES_AFTER_DQ
FORMATS = [0, B128, NODQ, B128 | NODQ, AFTER, B128 | AFTER]
FMT_IDS = ["b64-dq", "b128-dq", "b64-nodq", "b128-nodq", "b64-dq-after", "b128-dq-after"]


def _variant_kwargs(fmt, book):
    return dict(block=128 if fmt & B128 else 64, dq=not (fmt & NODQ), codes_after_dq=bool(fmt & AFTER), book=book)


def _book(qt):
    return O.fp4_codebook() if qt == q.QLORA_QT_FP4 else O.nf4_codebook()


def _assert_tol(got, ref, what):
    nw, rw = O.rel_errors(got, ref)
    assert nw <= O.NORMWISE_TOL and rw <= O.ROWWISE_TOL, f"{what}: normwise {nw:.3e} rowwise {rw:.3e}"


def _upload(ref, n_out, n_in, qt, fmt):
    w = q.NF4Weight.empty(n_out, n_in, device=DEV, quant_type=qt, format=fmt)
    w.codes.copy_(torch.from_numpy(np.ascontiguousarray(ref["codes"])))
    w.scales.copy_(torch.from_numpy(np.ascontiguousarray(ref["scales"])))
    if not fmt & NODQ:
        w.scales2.copy_(torch.from_numpy(np.ascontiguousarray(ref["scales2"])))
    return w


def _weight(n_out, n_in, seed):
    W = syn.with_outliers(syn.normal_f32((n_out, n_in), 0.02, seed), 1e-3, 10.0, seed + 1)
    W[1, :128] = 0.0                       # an all-zero block (both block sizes)
    W[2, :128] *= 1e-4                     # a block far below its group's max: q_b = 0 while a_b > 0
    return W


def _dequant_ref(ref, fmt, qt):
    kw = _variant_kwargs(fmt, _book(qt))
    return O.dequant_variant(ref["codes"], ref["scales"], None if fmt & NODQ else ref["scales2"],
                             block=kw["block"], book=kw["book"])


@pytest.mark.parametrize("qt", [q.QLORA_QT_NF4, q.QLORA_QT_FP4], ids=["nf4", "fp4"])
@pytest.mark.parametrize("fmt", FORMATS, ids=FMT_IDS)
def test_encode_and_dequant_bit_exact(fmt, qt):
    # 72 x 640: 720 blocks of 64 (2.8 groups) or 360 of 128 (1.4 groups); 40 x 704 adds an
    # odd number of 64-blocks (a half-filled last warp step) where the format allows it
    shapes = [(72, 640, 501)] + ([(40, 704, 502)] if not fmt & B128 else [(48, 1152, 503)])
    for n_out, n_in, seed in shapes:
        W = _weight(n_out, n_in, seed)
        ref = O.quantize_variant(W.numpy(), **_variant_kwargs(fmt, _book(qt)))
        w = q.NF4Weight.empty(n_out, n_in, device=DEV, quant_type=qt, format=fmt)
        q.qlora_quantize_nf4_dq(W.to(DEV), w)
        q.qlora_sync_status()
        assert np.array_equal(w.codes.cpu().numpy(), ref["codes"]), "codes differ"
        if fmt & NODQ:
            assert np.array_equal(w.scales.cpu().numpy().view(np.uint32), ref["scales"].view(np.uint32))
        else:
            assert np.array_equal(w.scales.cpu().numpy(), ref["scales"]), "u8 scales differ"
            assert np.array_equal(w.scales2.cpu().numpy().view(np.uint32), ref["scales2"].view(np.uint32))
        assert q.qlora_packed_bytes_fmt(n_out * n_in, fmt) == O.packed_bytes_variant(
            n_out * n_in, block=128 if fmt & B128 else 64, dq=not fmt & NODQ)
        want = _dequant_ref(ref, fmt, qt)
        wo = _upload(ref, n_out, n_in, qt, fmt)
        for dtype in (torch.float32, torch.bfloat16):
            out = torch.empty(n_out, n_in, dtype=dtype, device=DEV)
            q.qlora_dequant(wo, out)
            q.qlora_sync_status()
            exp = want if dtype == torch.float32 else O.bf16_round(want)
            assert np.array_equal(out.float().cpu().numpy().reshape(-1).view(np.uint32), exp.view(np.uint32)), \
                f"{dtype} dequant differs"


LAYER_CASES = [
    syn.LayerCase("fmt-pair-m300-n320-k640-r16", M=300, N=320, K=640, r=16, alpha=32.0, seed=511),
    syn.LayerCase("fmt-split-m40-n384-k2048-r8", M=40, N=384, K=2048, r=8, alpha=16.0, seed=512),
    syn.LayerCase("fmt-small-m4-n1024-k4096-r8", M=4, N=1024, K=4096, r=8, alpha=16.0, seed=513),
]


@pytest.mark.parametrize("fmt", [B128, NODQ, B128 | NODQ], ids=["b128-dq", "b64-nodq", "b128-nodq"])
@pytest.mark.parametrize("c", LAYER_CASES, ids=[c.name for c in LAYER_CASES])
def test_layer_matches_oracle(c, fmt):
    qt = q.QLORA_QT_NF4
    ref = O.quantize_variant(c.weight().numpy(), **_variant_kwargs(fmt, _book(qt)))
    Wd = _dequant_ref(ref, fmt, qt).reshape(c.N, c.K)
    w = _upload(ref, c.N, c.K, qt, fmt)
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


@pytest.mark.parametrize("fmt_in,fmt_out", [(B128 | NODQ, 0), (0, B128), (NODQ, AFTER)],
                         ids=["b128nodq-to-default", "default-to-b128", "nodq-to-after"])
def test_merge_across_formats_bit_exact(fmt_in, fmt_out):
    n_out, n_in, r, s, seed = 96, 1024, 8, 2.0, 521
    qt = q.QLORA_QT_NF4
    ref = O.quantize_variant(syn.normal_f32((n_out, n_in), 0.02, seed).numpy(), **_variant_kwargs(fmt_in, _book(qt)))
    A = syn.normal_bf16((r, n_in), 1.0 / n_in, seed + 1)
    B = syn.normal_bf16((n_out, r), 0.01, seed + 2)
    w = _upload(ref, n_out, n_in, qt, fmt_in)
    out = q.NF4Weight.empty(n_out, n_in, device=DEV, quant_type=qt, format=fmt_out)
    scratch = torch.empty(n_out, n_in, dtype=torch.float32, device=DEV)
    q.qlora_lora_merge_requant(w, A.to(DEV), B.to(DEV), r, s, scratch, out)
    q.qlora_sync_status()
    m = O.lora_merge_bf16_deq(_dequant_ref(ref, fmt_in, qt).reshape(n_out, n_in), A.float().numpy(),
                              B.float().numpy(), s)
    want = O.quantize_variant(m, **_variant_kwargs(fmt_out, _book(qt)))
    assert np.array_equal(out.codes.cpu().numpy(), want["codes"])
    if fmt_out & NODQ:
        assert np.array_equal(out.scales.cpu().numpy().view(np.uint32), want["scales"].view(np.uint32))
    else:
        assert np.array_equal(out.scales.cpu().numpy(), want["scales"])
        assert np.array_equal(out.scales2.cpu().numpy().view(np.uint32), want["scales2"].view(np.uint32))
