"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each one."""
import numpy as np
import pytest

from oracle import nf4_oracle as O
import tests.test_oracle_pins as P


def _pack_high_first(codes):
    c = np.asarray(codes, np.uint8).reshape(-1)
    return (c[1::2] | (c[0::2] << 4)).astype(np.uint8)


def _normalise_by_reciprocal(w, absmax):
    blocks = np.asarray(w, np.float32).reshape(-1, 64)
    with np.errstate(divide="ignore"):
        inv = (np.float32(1.0) / absmax.astype(np.float32)).astype(np.float32)
    inv[~np.isfinite(inv)] = 0
    return (blocks * inv[:, None]).astype(np.float32)


def _bwd_without_lora(w_deq, dy, a, b, scaling):
    dX = O._f64(dy) @ O._f64(w_deq)
    g = O._f64(dy) @ O._f64(b)
    return dX, g


def _dq_floor(absmax):
    q, d = _orig_dq(absmax)
    a = np.asarray(absmax, np.float32)
    g = np.arange(a.size) // 256
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (a.astype(np.float64) / d[g].astype(np.float64)).astype(np.float32)
    q2 = np.where(d[g] == 0, 0, np.clip(np.floor(r), 0, 255)).astype(np.uint8)
    return q2, d


_orig_dq = O.double_quant
_orig_delta = O.NF4_DELTA


def _merge_without_bf16_base(codes, q, d, n_out, n_in, a, b, scaling):
    w = O.dequant(codes, q, d, n_out * n_in).reshape(n_out, n_in).astype(np.float64)
    acc = np.zeros((n_out, n_in))
    a64, b64 = O._f64(a), O._f64(b)
    for j in range(a64.shape[0] if a64.size else 0):
        acc = acc + np.outer(b64[:, j], a64[j, :])
    return O.bf16_round((w + np.float64(np.float32(scaling)) * acc).astype(np.float32))


def _merge_with_bt(codes, q, d, n_out, n_in, a, b, scaling):
    # adapter factors swapped in the product (A B instead of B A, shapes permitting)
    wb = O.bf16_round(O.dequant(codes, q, d, n_out * n_in).reshape(n_out, n_in)).astype(np.float64)
    b64 = O._f64(b)
    a64 = O._f64(a)
    prod = (b64[:, ::-1] @ a64) if a64.size else 0.0
    return O.bf16_round((wb + np.float64(np.float32(scaling)) * prod).astype(np.float32))

MUTATIONS = [
    ("pack_codes", _pack_high_first, P.test_encode_dequant_round_trip_exact_on_representable_weights),
    ("normalise", _normalise_by_reciprocal, P.test_normalise_is_correctly_rounded_division),
    ("lora_linear_bwd_dx", _bwd_without_lora, P.test_adjoint_identity_and_lora_directional_derivatives),
    ("double_quant", _dq_floor, P.test_dq_brute_force_over_all_256_levels),
    ("NF4_DELTA", 0.9677083, P.test_codebook_levels_carry_equal_probability_mass),
    ("lora_merge_bf16", _merge_without_bf16_base, P.test_merge_brute_force_python),
    ("lora_merge_bf16", _merge_with_bt, P.test_merge_close_to_float64_definition),
]


@pytest.mark.parametrize("name,replacement,pin", MUTATIONS, ids=[f"{m[0]}-{m[2].__name__}" for m in MUTATIONS])
def test_pin_catches_planted_mistake(monkeypatch, name, replacement, pin):
    monkeypatch.setattr(O, name, replacement)
    with pytest.raises(AssertionError):
        pin()
