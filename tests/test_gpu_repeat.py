"""Repeated calls on the 70B-shape matrices return the same bits every time.

Each output element of the forward and of dX is one fixed sum taken in a fixed order (the
contraction runs stage by stage into one accumulator per element), so calls on the same
inputs must agree bit for bit.  A call that differs has a tile whose operands were
overwritten, or read before they were complete: the kind of fault that a parity check on
sampled outputs can miss.  The L2 is flushed between calls, so no call replays operands
that the previous one left in the cache.

With the adapter (r > 0) the rank-r factor (U or G) is summed over the tokens with
atomic fp32 additions, whose order varies, so its bf16 rounding, and through it a few
output elements, may move by a rounding step.  Those calls must agree within 2^-7 of each
element's value plus 2^-8 of the output's root mean square (for elements near zero,
where the adapter term's change dominates); a corrupted tile is off by far more
(tenths, on values near 1).
"""
import pytest
import torch

import bit_quantized_base_nf4_b200 as q

pytestmark = pytest.mark.gpu

DEV = "cuda"
M = 4096
SHAPES = [(8192, 8192), (28672, 8192), (8192, 28672)]   # attention, FFN up, FFN down
CALLS_DX = 16
CALLS_FWD = 8


@pytest.fixture(scope="module")
def flush():
    return torch.empty(256 << 20, dtype=torch.uint8, device=DEV)


def _inputs(N, K, r, seed, M=M):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    w = q.NF4Weight.empty(N, K)
    q.qlora_quantize_nf4_dq(torch.randn(N, K, generator=g, device=DEV) * 0.015, w)
    X = torch.randn(M, K, generator=g, device=DEV).to(torch.bfloat16)
    dY = torch.randn(M, N, generator=g, device=DEV).to(torch.bfloat16)
    A = (torch.randn(r, K, generator=g, device=DEV) / K ** 0.5).to(torch.bfloat16) if r else None
    B = (torch.randn(N, r, generator=g, device=DEV) * 0.01).to(torch.bfloat16) if r else None
    ws = torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=DEV)
    return w, X, dY, A, B, ws


def _repeat(call, out, calls, flush, exact):
    ref = torch.empty_like(out)
    call(ref)
    q.qlora_sync_status()
    bad = []
    for i in range(calls):
        flush.fill_(i)
        out.zero_()
        call(out)
        q.qlora_sync_status()
        if exact:
            if not torch.equal(out, ref):
                bad.append((i, int((out != ref).sum())))
        else:
            rf = ref.float()
            floor = 2.0 ** -8 * float(rf.square().mean().sqrt())
            far = (out.float() - rf).abs() > rf.abs() * 2.0 ** -7 + floor
            if bool(far.any()):
                bad.append((i, int(far.sum())))
    assert not bad, f"calls that differ from the first one (call, elements): {bad}"


@pytest.mark.parametrize("N,K,r", [s + (0,) for s in SHAPES] + [(8192, 8192, 64)])
def test_dx_repeats_bit_exact(N, K, r, flush):
    w, X, dY, A, B, ws = _inputs(N, K, r, 11)
    out = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
    _repeat(lambda o: q.qlora_lora_linear_bwd_dx(w, dY, A, B, r, 2.0 if r else 0.0, o, None, ws), out, CALLS_DX,
            flush, exact=r == 0)


@pytest.mark.parametrize("N,K,r", [s + (0,) for s in SHAPES] + [(8192, 8192, 64)])
def test_fwd_repeats_bit_exact(N, K, r, flush):
    w, X, dY, A, B, ws = _inputs(N, K, r, 12)
    out = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    _repeat(lambda o: q.qlora_lora_linear_fwd(w, X, A, B, r, 2.0 if r else 0.0, o, None, ws), out, CALLS_FWD, flush,
            exact=r == 0)


@pytest.mark.parametrize("N,K,m", [(4096, 11008, 1), (11008, 4096, 16), (4096, 4096, 4)])
def test_small_m_forward_repeats_bit_exact(N, K, m, flush):
    """The small-M forward keeps every partial sum in its CTA (the adapter's U included), so
    its results are exact repeats too."""
    r = 8
    w, X, dY, A, B, ws = _inputs(N, K, r, 13, M=m)
    out = torch.empty(m, N, dtype=torch.bfloat16, device=DEV)
    _repeat(lambda o: q.qlora_lora_linear_fwd(w, X, A, B, r, 2.0, o, None, ws), out, CALLS_FWD, flush, exact=True)


@pytest.mark.parametrize("N,K", [(8192, 8192), (8192, 28672)])
def test_q8_0_dx_repeats_bit_exact(N, K, flush):
    """The Q8_0 route's dX, on the same pair-tile kernels, repeats bit for bit as well."""
    g = torch.Generator(device=DEV)
    g.manual_seed(14)
    w = q.Q80Weight.empty(N, K)
    q.qlora_quantize_q8_0(torch.randn(N, K, generator=g, device=DEV) * 0.015, w)
    dY = torch.randn(M, N, generator=g, device=DEV).to(torch.bfloat16)
    ws = torch.empty(q.qlora_workspace_bytes(M, N, K, 0), dtype=torch.uint8, device=DEV)
    out = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
    _repeat(lambda o: q.qlora_q8_0_lora_linear_bwd_dx(w, dY, None, None, 0, 0.0, o, None, ws), out, CALLS_DX, flush,
            exact=True)


@pytest.mark.parametrize("N,K", [(8192, 8192), (28672, 8192)])
def test_q8_0_fwd_repeats_bit_exact(N, K, flush):
    """The Q8_0 route's forward repeats bit for bit."""
    g = torch.Generator(device=DEV)
    g.manual_seed(15)
    w = q.Q80Weight.empty(N, K)
    q.qlora_quantize_q8_0(torch.randn(N, K, generator=g, device=DEV) * 0.015, w)
    X = torch.randn(M, K, generator=g, device=DEV).to(torch.bfloat16)
    ws = torch.empty(q.qlora_workspace_bytes(M, N, K, 0), dtype=torch.uint8, device=DEV)
    out = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    _repeat(lambda o: q.qlora_q8_0_lora_linear_fwd(w, X, None, None, 0, 0.0, o, None, ws), out, CALLS_DX, flush,
            exact=True)
