"""LoRA merge + requantize on the GPU against the oracle.

Both sides start from the oracle's encode of a seeded weight (uploaded to the
device), so no oracle input comes from the CUDA path.  The merged base (the float32
scratch) and the requantized codes, block scales and group steps must match the
oracle bit for bit: the merge fixes every rounding (bf16 base, float64 adapter sum
with j ascending, float32 then bf16), so each code decision is taken in the same
precision on both sides."""
import numpy as np
import pytest
import torch

import bit_quantized_base_nf4_b200 as q
from bit_quantized_base_nf4_b200 import synthetic as syn
from oracle import nf4_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # name, n_out, n_in, r, scaling, seed
    ("ragged-72x576-r16", 72, 576, 16, 2.0, 301),       # 41472 weights: 2.53 second-level groups
    ("r0-128x1024", 128, 1024, 0, 0.0, 302),             # no adapter: requantize bf16(w')
    ("r64-1024x4096", 1024, 4096, 64, 2.0, 304),
    ("attn7b-4096x4096-r8", 4096, 4096, 8, 2.0, 303),    # the 7B attention projection
]


def _upload(ref, n_out, n_in):
    w = q.NF4Weight.empty(n_out, n_in, device=DEV)
    w.codes.copy_(torch.from_numpy(np.ascontiguousarray(ref["codes"])))
    w.scales.copy_(torch.from_numpy(np.ascontiguousarray(ref["scales"])))
    w.scales2.copy_(torch.from_numpy(np.ascontiguousarray(ref["scales2"])))
    return w


def _setup(n_out, n_in, r, seed):
    W = syn.normal_f32((n_out, n_in), 0.02, seed).numpy()
    ref = O.quantize_nf4_dq(W)
    A = syn.normal_bf16((r, n_in), 1.0 / n_in, seed + 1) if r else None
    B = syn.normal_bf16((n_out, r), 0.01, seed + 2) if r else None
    return ref, A, B


def _check(out, scratch, ref, A, B, n_out, n_in, r, s):
    empty = np.zeros((0, n_in), np.float32), np.zeros((n_out, 0), np.float32)
    a, b = (A.float().numpy(), B.float().numpy()) if r else empty
    m = O.lora_merge_bf16(ref["codes"], ref["scales"], ref["scales2"], n_out, n_in, a, b, s)
    assert np.array_equal(scratch.cpu().numpy().view(np.uint32), m.view(np.uint32)), "merged base"
    want = O.quantize_nf4_dq(m)
    assert np.array_equal(out.codes.cpu().numpy(), want["codes"]), "codes"
    assert np.array_equal(out.scales.cpu().numpy(), want["scales"]), "block scales"
    assert np.array_equal(out.scales2.cpu().numpy().view(np.uint32), want["scales2"].view(np.uint32)), "steps"


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_merge_requant_bit_exact(case):
    _, n_out, n_in, r, s, seed = case
    ref, A, B = _setup(n_out, n_in, r, seed)
    w = _upload(ref, n_out, n_in)
    out = q.NF4Weight.empty(n_out, n_in, device=DEV)
    scratch = torch.empty(n_out, n_in, dtype=torch.float32, device=DEV)
    q.qlora_lora_merge_requant(w, A.to(DEV) if r else None, B.to(DEV) if r else None, r, s, scratch, out)
    q.qlora_sync_status()
    _check(out, scratch, ref, A, B, n_out, n_in, r, s)


def test_merge_requant_in_place():
    n_out, n_in, r, s, seed = 256, 1024, 8, 2.0, 305
    ref, A, B = _setup(n_out, n_in, r, seed)
    w = _upload(ref, n_out, n_in)
    scratch = torch.empty(n_out, n_in, dtype=torch.float32, device=DEV)
    q.qlora_lora_merge_requant(w, A.to(DEV), B.to(DEV), r, s, scratch, w)
    q.qlora_sync_status()
    _check(w, scratch, ref, A, B, n_out, n_in, r, s)
