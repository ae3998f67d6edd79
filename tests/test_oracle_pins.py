"""The oracle checked against what the pages and the mathematics fix (CPU only)."""

import types

import numpy as np
import pytest

import pins
from oracle import c_oracle
from oracle import reference as R


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_numpy_oracle_pin(check):
    check(R)


def _c_impl():
    ns = types.SimpleNamespace(**{k: getattr(R, k) for k in dir(R) if not k.startswith("_")})
    ns.decode = c_oracle.decode
    return ns


C_DECODE_CHECKS = [
    pins.check_p3_block_table_walk,
    pins.check_permutation_invariance,
    pins.check_matches_contiguous_sdpa,
    pins.check_single_token_is_v,
    pins.check_zero_query_is_mean,
    pins.check_equal_keys_is_mean,
    pins.check_dominant_key,
    pins.check_empty_context_is_zero,
]


@pytest.mark.parametrize("check", C_DECODE_CHECKS, ids=lambda c: c.__name__)
def test_c_oracle_pin(check):
    check(_c_impl())


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_c_oracle_equals_numpy_oracle(dtype):
    ctxs = [1, 15, 16, 17, 37, 64, 130]
    q, kc, vc, bt, cl = pins._rand_case(21, len(ctxs), 8, 2, 64, ctxs, NB=40, dtype=dtype)
    a = R.decode(q, kc, vc, bt, cl, 0.125, dtype, 2)
    b = c_oracle.decode(q, kc, vc, bt, cl, 0.125, dtype, 2)
    assert np.abs(a - b).max() < 1e-12
    pairs = [(6, 7), (0, 0), (3, 4)]
    c = c_oracle.decode_pairs(pairs, q, kc, vc, bt, cl, 0.125, dtype, 2)
    for k, (bb, hh) in enumerate(pairs):
        assert np.array_equal(c[k], b[bb, hh])


def test_c_oracle_half_conversion_all_finite_patterns():
    """Every finite binary16 pattern survives the C oracle's upcast exactly (n = 1 -> out = V)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    finite = bits[np.isfinite(vals)]
    D = 64
    n = len(finite) // D
    v = finite[: n * D].view(np.float16).reshape(n, 1, 1, D)
    vc = np.zeros((n, 1, 16, D), dtype=np.float16)
    vc[:, :, :1, :] = v
    kc = np.zeros_like(vc)
    q = np.zeros((n, 1, D), dtype=np.float16)
    bt = np.arange(n, dtype=np.int32)[:, None]
    out = c_oracle.decode(q, kc, vc, bt, np.ones(n, np.int32), 1.0, "f16", 1)
    assert np.array_equal(out[:, 0, :], v[:, 0, 0, :].astype(np.float64))


def test_bf16_upcast_known_patterns():
    pat = np.array([0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F, 0x0000, 0x8000], dtype=np.uint16)
    expect = [1.0, -1.0, 3.140625, 2.0 ** -133, 3.3895313892515355e38, 0.0, -0.0]
    got = R.to_f64(pat, "bf16")
    assert list(got) == expect


def test_c_oracle_rejects_out_of_pool_block():
    q, kc, vc, bt, cl = pins._rand_case(22, 2, 2, 1, 16, [5, 20], NB=4)
    bt[1, 1] = 4
    with pytest.raises(IndexError):
        c_oracle.decode(q, kc, vc, bt, cl, 1.0, "f32", 1)
    with pytest.raises(IndexError):
        R.decode(q, kc, vc, bt, cl, 1.0, "f32", 1)
