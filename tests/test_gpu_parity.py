"""CUDA path vs the CPU oracle, element by element, through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

import bit_quantized_base_nf4_b200 as q
from bit_quantized_base_nf4_b200 import synthetic as syn
from oracle import nf4_oracle as O

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _encode_gpu(W: torch.Tensor) -> q.NF4Weight:
    w = q.NF4Weight.empty(W.shape[0], W.shape[1])
    q.qlora_quantize_nf4_dq(W.to(DEV).contiguous(), w)
    q.qlora_sync_status()
    return w


def _np(t):
    return t.detach().cpu().numpy()


def _assert_tol(got, ref, what):
    nw, rw = O.rel_errors(got, ref)
    assert nw <= O.NORMWISE_TOL and rw <= O.ROWWISE_TOL, f"{what}: normwise {nw:.3e} rowwise {rw:.3e}"


def bf16_half_ulp(v):
    """Upper bound of |x - bf16(x)| for an x that rounded to the bfloat16 value v: half a
    unit in the last place of v's binade (8 significant bits)."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 2.0 ** -133)


def assert_adapter_term(with_adapter, without, ref, what):
    """Element-by-element check of the adapter term hidden in a bf16 output.

    with_adapter = bf16(acc + t) and without = bf16(acc) come from two calls that form the
    same fp32 base sum acc (the adapter is the last contraction stage, or the epilogue's
    last add), so their float64 difference is t up to the two roundings.  Each element
    must satisfy |(with - without) - ref| <= 2e-2 max_j |ref_ij| (the row-wise bar applied
    to the adapter term alone) + both half-ulps + 2^-16 of the row's output scale (fp32
    reassociation where a split contraction adds partial sums atomically)."""
    Yw, Y0, R = (np.asarray(t, np.float64) for t in (with_adapter, without, ref))
    rowmax = np.maximum(np.max(np.abs(R), axis=1, keepdims=True), 1e-6)
    outmax = np.max(np.abs(Y0), axis=1, keepdims=True)
    bound = O.ROWWISE_TOL * rowmax + bf16_half_ulp(Yw) + bf16_half_ulp(Y0) + 2.0 ** -16 * outmax
    err = np.abs((Yw - Y0) - R)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements off; worst excess "
                           f"{float(np.max(err - bound)):.3e} at {np.unravel_index(np.argmax(err - bound), err.shape)}")


# ----------------------------------------------------------------- encode / dequant (bit-exact)

def _weights_for_encode():
    out = []
    out.append(("tiny-256x512", syn.tiny_case().weight()))
    out.append(("ragged-320x576", syn.normal_f32((320, 576), 0.02, 11)))          # 11.25 DQ groups
    out.append(("one-group-1000x64", syn.normal_f32((1000, 64), 0.02, 12)))
    w = syn.with_outliers(syn.normal_f32((512, 1024), 0.02, 13), 1e-3, 10.0, 14)
    w[3, :64] = 0.0                                                                # an all-zero block
    w[5, :] = 0.0                                                                  # all-zero row
    out.append(("outliers-zeros-512x1024", w))
    # values sitting exactly on and next to the code midpoints (tie rule)
    book = O.nf4_codebook().astype(np.float64)
    mids = ((book[:-1] + book[1:]) / 2).astype(np.float32)
    vals = np.concatenate([mids, np.nextafter(mids, np.float32(-2)), np.nextafter(mids, np.float32(2)),
                           book.astype(np.float32)])
    blk = np.zeros((64, 64), np.float32)
    for i in range(64):
        blk[i, :] = np.resize(np.roll(vals, i), 64)
        blk[i, 0] = 1.0                                                            # absmax 1 -> n = w exactly
    out.append(("midpoints-64x64", torch.from_numpy(blk)))
    return out


@pytest.mark.parametrize("name,W", _weights_for_encode(), ids=[n for n, _ in _weights_for_encode()])
def test_encode_and_dequant_bit_exact(name, W):
    ref = O.quantize_nf4_dq(W.numpy())
    w = _encode_gpu(W)
    assert np.array_equal(_np(w.codes), ref["codes"]), "codes differ"
    assert np.array_equal(_np(w.scales), ref["scales"]), "u8 scales differ"
    assert np.array_equal(_np(w.scales2).view(np.uint32), ref["scales2"].view(np.uint32)), "fp32 steps differ"
    deq_ref = O.dequant(ref["codes"], ref["scales"], ref["scales2"]).reshape(W.shape)
    out32 = torch.empty(W.shape, dtype=torch.float32, device=DEV)
    q.qlora_dequant(w, out32)
    out16 = torch.empty(W.shape, dtype=torch.bfloat16, device=DEV)
    q.qlora_dequant(w, out16)
    q.qlora_sync_status()
    assert np.array_equal(_np(out32).view(np.uint32), deq_ref.view(np.uint32)), "fp32 dequant differs"
    assert np.array_equal(_np(out16.float()).view(np.uint32), O.bf16_round(deq_ref).view(np.uint32)), \
        "bf16 dequant differs"


def test_encode_full_size_7b_ffn_with_outliers_bit_exact():
    case = syn.ffn7b_cases()[0]
    W = case.weight()
    ref = O.quantize_nf4_dq(W.numpy())
    w = _encode_gpu(W)
    assert np.array_equal(_np(w.codes), ref["codes"])
    assert np.array_equal(_np(w.scales), ref["scales"])
    assert np.array_equal(_np(w.scales2).view(np.uint32), ref["scales2"].view(np.uint32))


# ----------------------------------------------------------------- layer (tolerance vs float64)

class Run:
    """Encode + forward + backward of one case on the GPU, with the oracle's references."""

    def __init__(self, case: syn.LayerCase, with_bwd=True):
        self.case = case
        W = case.weight()
        self.ref = O.quantize_nf4_dq(W.numpy())
        self.Wd = O.dequant(self.ref["codes"], self.ref["scales"], self.ref["scales2"]).reshape(case.N, case.K)
        self.w = _encode_gpu(W)
        self.X = case.x().to(DEV)
        r = case.r
        self.A = case.lora_a().to(DEV) if r else None
        self.B = case.lora_b().to(DEV) if r else None
        M, N, K = case.M, case.N, case.K
        ws_bytes = q.qlora_workspace_bytes(M, N, K, r)
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
        self.Y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
        self.U = torch.empty(M, r, dtype=torch.bfloat16, device=DEV) if r else None
        q.qlora_lora_linear_fwd(self.w, self.X, self.A, self.B, r, case.scaling, self.Y, self.U, self.ws)
        if with_bwd:
            self.dY = case.dy().to(DEV)
            self.dX = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
            self.G = torch.empty(M, r, dtype=torch.bfloat16, device=DEV) if r else None
            q.qlora_lora_linear_bwd_dx(self.w, self.dY, self.A, self.B, r, case.scaling, self.dX, self.G, self.ws)
            if r:
                self.dA = torch.empty(r, K, dtype=torch.float32, device=DEV)
                self.dB = torch.empty(N, r, dtype=torch.float32, device=DEV)
                q.qlora_lora_grad_AB(self.X, self.dY, self.U, self.G, r, case.scaling, self.dA, self.dB)
        q.qlora_sync_status()


CASES = [
    syn.tiny_case(),
    syn.LayerCase("ragged-m300-n320-k576-r16", M=300, N=320, K=576, r=16, alpha=32.0, seed=101),
    syn.LayerCase("base-only-m64-n384-k1024", M=64, N=384, K=1024, r=0, alpha=0.0, seed=102),
    syn.LayerCase("r64-m512-n256-k2048", M=512, N=256, K=2048, r=64, alpha=128.0, seed=103),
    syn.LayerCase("r128-m100-n136-k320", M=100, N=136, K=320, r=128, alpha=256.0, seed=104),
    syn.LayerCase("decode-m1-n4096-k4096-r8", M=1, N=4096, K=4096, r=8, alpha=16.0, seed=105),
    syn.LayerCase("decode-m4-n1024-k11008-r8", M=4, N=1024, K=11008, r=8, alpha=16.0, seed=106),
    syn.LayerCase("decode-m16-n2048-k4096-r8", M=16, N=2048, K=4096, r=8, alpha=16.0, seed=107),
    # small-M kernel edges: 12 tokens (second token tile partly empty), ragged last unit
    # (200 = 6 x 32 + 8 rows) and ragged last stage (11 of 16 blocks)
    syn.LayerCase("decode-m12-n200-k704-r16", M=12, N=200, K=704, r=16, alpha=32.0, seed=109),
    # one unit of 8 rows, one 64-k block
    syn.LayerCase("decode-m1-n8-k64-r8", M=1, N=8, K=64, r=8, alpha=16.0, seed=114),
    # 4104 = 128 x 32 + 8 rows: the last unit's 136 scale bytes end in an 8-byte tail
    syn.LayerCase("decode-m9-n4104-k1088-r16", M=9, N=4104, K=1088, r=16, alpha=32.0, seed=115),
    # 300 units: two or three per CTA (scale buffers reused, adapter product kept)
    syn.LayerCase("decode-m3-n9600-k1024-r16", M=3, N=9600, K=1024, r=16, alpha=32.0, seed=116),
    # longest rows on the small-M path (512 blocks of 64)
    syn.LayerCase("decode-m2-n256-k32768-r8", M=2, N=256, K=32768, r=8, alpha=16.0, seed=117),
    # rows longer than that: tensor-core path
    syn.LayerCase("small-m4-n256-k33792-r8", M=4, N=256, K=33792, r=8, alpha=16.0, seed=118),
    # adapter rank above the small-M kernel's limit: tensor-core path
    syn.LayerCase("decode-m1-n4096-k4096-r32", M=1, N=4096, K=4096, r=32, alpha=64.0, seed=110),
    # the 7B down projection at full size, 16 tokens, base only
    syn.LayerCase("decode-m16-n4096-k11008-r0", M=16, N=4096, K=11008, r=0, alpha=0.0, seed=111),
    # adapter rank above the small-M kernel's limit: split-K tensor-core path
    syn.LayerCase("small-m8-n256-k1024-r64", M=8, N=256, K=1024, r=64, alpha=128.0, seed=112),
    # between the small-M kernel and the CTA-pair kernels: split-K tensor-core path
    syn.LayerCase("small-m40-n384-k2048-r8", M=40, N=384, K=2048, r=8, alpha=16.0, seed=113),
    syn.LayerCase("m600-n512-k768-r8-2tiles", M=600, N=512, K=768, r=8, alpha=16.0, seed=108),
    # dX on CTA pairs with the contraction split 28 ways (448 stages of 64 n, two pairs of k)
    syn.LayerCase("dxsplit-m48-n28672-k512-r64", M=48, N=28672, K=512, r=64, alpha=128.0, seed=119),
    # one token, 16 pairs of k, ragged n (4104 = 64 x 64 + 8)
    syn.LayerCase("dxsplit-m1-n4104-k4096-r16", M=1, N=4104, K=4096, r=16, alpha=32.0, seed=120),
]


@pytest.fixture(scope="module", params=CASES, ids=[c.name for c in CASES])
def run(request):
    return Run(request.param)


def test_forward_matches_oracle(run):
    c = run.case
    Yref, uref = O.lora_linear_fwd(run.Wd, run.X.cpu(), run.A.cpu() if c.r else None,
                                   run.B.cpu() if c.r else None, c.scaling)
    _assert_tol(run.Y.float().cpu(), Yref, "Y")
    if c.r:
        _assert_tol(run.U.float().cpu(), uref, "U")


def test_backward_dx_matches_oracle(run):
    c = run.case
    dXref, gref = O.lora_linear_bwd_dx(run.Wd, run.dY.cpu(), run.A.cpu() if c.r else None,
                                       run.B.cpu() if c.r else None, c.scaling)
    _assert_tol(run.dX.float().cpu(), dXref, "dX")
    if c.r:
        _assert_tol(run.G.float().cpu(), gref, "G")


def test_adapter_grads_match_oracle(run):
    """dA and dB against the oracle's own chain: u = X A^T from its forward, g = dY B from
    its backward, then dA = s g^T X and dB = s dY^T u, all in float64 from the inputs."""
    c = run.case
    if not c.r:
        pytest.skip("no adapter")
    X, A, B, dY = (t.cpu() for t in (run.X, run.A, run.B, run.dY))
    _, uref = O.lora_linear_fwd(run.Wd, X, A, B, c.scaling)
    _, gref = O.lora_linear_bwd_dx(run.Wd, dY, A, B, c.scaling)
    dAref, dBref = O.lora_grad_ab(X, dY, uref, gref, c.scaling)
    _assert_tol(run.dA.cpu(), dAref, "dA")
    _assert_tol(run.dB.cpu(), dBref, "dB")


def test_grad_kernel_alone_on_oracle_factors(run):
    """qlora_lora_grad_AB given the oracle's u and g (rounded to bf16 on the host, the
    precision the call takes) against the oracle's products of those same factors."""
    c = run.case
    if not c.r:
        pytest.skip("no adapter")
    X, A, B, dY = (t.cpu() for t in (run.X, run.A, run.B, run.dY))
    _, uref = O.lora_linear_fwd(run.Wd, X, A, B, c.scaling)
    _, gref = O.lora_linear_bwd_dx(run.Wd, dY, A, B, c.scaling)
    u16 = torch.from_numpy(O.bf16_round(uref.astype(np.float32))).to(torch.bfloat16)
    g16 = torch.from_numpy(O.bf16_round(gref.astype(np.float32))).to(torch.bfloat16)
    dA = torch.empty(c.r, c.K, dtype=torch.float32, device=DEV)
    dB = torch.empty(c.N, c.r, dtype=torch.float32, device=DEV)
    q.qlora_lora_grad_AB(run.X, run.dY, u16.to(DEV), g16.to(DEV), c.r, c.scaling, dA, dB)
    q.qlora_sync_status()
    dAref, dBref = O.lora_grad_ab(X, dY, u16.float(), g16.float(), c.scaling)
    _assert_tol(dA.cpu(), dAref, "dA (kernel alone)")
    _assert_tol(dB.cpu(), dBref, "dB (kernel alone)")


def test_adapter_branch_separately(run):
    """The adapter term is about 1 % of Y and of dX, under the layer tolerance: check it on
    its own, element by element, against the oracle's s (X A^T) B^T and s (dY B) A."""
    c = run.case
    if not c.r:
        pytest.skip("no adapter")
    Y0 = torch.empty_like(run.Y)
    q.qlora_lora_linear_fwd(run.w, run.X, None, None, 0, 0.0, Y0, None, run.ws)
    dX0 = torch.empty_like(run.dX)
    q.qlora_lora_linear_bwd_dx(run.w, run.dY, None, None, 0, 0.0, dX0, None, run.ws)
    q.qlora_sync_status()
    X, A, B, dY = (t.cpu() for t in (run.X, run.A, run.B, run.dY))
    lora_ref, _ = O.lora_linear_fwd(np.zeros((c.N, c.K)), X, A, B, c.scaling)
    dlora_ref, _ = O.lora_linear_bwd_dx(np.zeros((c.N, c.K)), dY, A, B, c.scaling)
    assert_adapter_term(run.Y.float().cpu().numpy(), Y0.float().cpu().numpy(), lora_ref, f"{c.name} Y adapter")
    assert_adapter_term(run.dX.float().cpu().numpy(), dX0.float().cpu().numpy(), dlora_ref, f"{c.name} dX adapter")


def test_b_zero_gives_base_output_bitwise():
    c = syn.LayerCase("bzero-m200-n256-k512-r8", M=200, N=256, K=512, r=8, alpha=16.0, seed=201)
    r = Run(c, with_bwd=False)
    Y0 = torch.empty_like(r.Y)
    q.qlora_lora_linear_fwd(r.w, r.X, None, None, 0, 0.0, Y0, None, r.ws)
    Yb = torch.empty_like(r.Y)
    q.qlora_lora_linear_fwd(r.w, r.X, r.A, torch.zeros_like(r.B), 8, c.scaling, Yb, None, r.ws)
    q.qlora_sync_status()
    assert torch.equal(Y0, Yb)


def test_zero_base_gives_adapter_only():
    c = syn.LayerCase("wzero-m64-n256-k512-r16", M=64, N=256, K=512, r=16, alpha=32.0, seed=202)
    w = _encode_gpu(torch.zeros(c.N, c.K))
    assert int(w.scales.max()) == 0 and float(w.scales2.abs().max()) == 0.0
    assert bool((w.codes == 0x77).all())
    X, A, B = c.x().to(DEV), c.lora_a().to(DEV), c.lora_b().to(DEV)
    ws = torch.empty(q.qlora_workspace_bytes(c.M, c.N, c.K, c.r), dtype=torch.uint8, device=DEV)
    Y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV)
    q.qlora_lora_linear_fwd(w, X, A, B, c.r, c.scaling, Y, None, ws)
    q.qlora_sync_status()
    ref = c.scaling * (X.cpu().double() @ A.cpu().double().T) @ B.cpu().double().T
    _assert_tol(Y.float().cpu(), ref.numpy(), "Y (adapter only)")


def test_full_size_7b_attention_sampled():
    """The bench workload at full size (M=2048, N=K=4096, r=8): sampled output columns of Y and dX."""
    c = syn.attn7b_case()
    r = Run(c)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(c.N, 48, replace=False))
    X, A, B, dY = (t.cpu() for t in (r.X, r.A, r.B, r.dY))
    Yref = O.lora_linear_fwd_rows(r.Wd, X, A, B, c.scaling, rows)
    _assert_tol(r.Y.float().cpu().numpy()[:, rows], Yref, "Y[:, sample]")
    cols = np.sort(rng.choice(c.K, 48, replace=False))
    dXref, _ = O.lora_linear_bwd_dx(r.Wd[:, cols], dY, A.float().numpy()[:, cols], B, c.scaling)
    _assert_tol(r.dX.float().cpu().numpy()[:, cols], dXref, "dX[:, sample]")
    _, uref = O.lora_linear_fwd(np.zeros((1, c.K)), X, A, B, c.scaling)
    _, gref = O.lora_linear_bwd_dx(np.zeros((c.N, 1)), dY, A[:, :1], B, c.scaling)
    dAref, dBref = O.lora_grad_ab(X, dY, uref, gref, c.scaling)
    _assert_tol(r.dA.cpu(), dAref, "dA")
    _assert_tol(r.dB.cpu(), dBref, "dB")


def test_grad_accumulate_adds():
    c = syn.LayerCase("acc-m128-n256-k512-r8", M=128, N=256, K=512, r=8, alpha=16.0, seed=203)
    r = Run(c)
    dA2, dB2 = r.dA.clone(), r.dB.clone()
    q.qlora_lora_grad_AB(r.X, r.dY, r.U, r.G, c.r, c.scaling, dA2, dB2, accumulate=True)
    q.qlora_sync_status()
    # partial sums are added with float atomics, so the order (and the last bits) may differ
    for got, one in ((dA2, r.dA), (dB2, r.dB)):
        scale = float(one.abs().max())
        torch.testing.assert_close(got, 2 * one, rtol=1e-4, atol=1e-5 * scale)
