"""Pins of the oracle's fp16 rounding against numpy's binary16 conversion.

numpy rounds float32 -> float16 to nearest-even; the directed roundings are
derived from it with ``nextafter``: round-down(x) is the nearest value when that
is <= x, else the next fp16 below it (and symmetrically for round-up).  The
oracle's routines are written from the IEEE 754 binary16 definition instead.
"""
import numpy as np
import pytest

from oracle import oracle as O


def _sample_fp32(n_rand: int = 1 << 20, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    # every sign/exponent combination, with structured and random mantissas
    hi = np.arange(1 << 9, dtype=np.uint32) << 23
    mants = np.concatenate([
        np.array([0, 1, 0x1000, 0xFFF, 0x1001, 0x2000, 0x3000, 0x7FFFFF, 0x7FE000,
                  0x7FF000, 0x400000, 0x401000], dtype=np.uint32),
        rng.integers(0, 1 << 23, size=64, dtype=np.uint32),
    ])
    structured = (hi[:, None] | mants[None, :]).ravel()
    rand = rng.integers(0, 1 << 32, size=n_rand, dtype=np.uint64).astype(np.uint32)
    # dense sampling around the binary16 range (exponents 100..145)
    e = rng.integers(100, 146, size=n_rand, dtype=np.uint32)
    m = rng.integers(0, 1 << 23, size=n_rand, dtype=np.uint32)
    s = rng.integers(0, 2, size=n_rand, dtype=np.uint32) << 31
    near = s | (e << 23) | m
    bits = np.concatenate([structured, rand, near])
    x = bits.view(np.float32)
    return x[~np.isnan(x)]


def _numpy_directed(x: np.ndarray):
    with np.errstate(over="ignore"):
        rn = x.astype(np.float16)
    xd = x.astype(np.float64)
    rnd = rn.astype(np.float64)
    down = np.where(rnd > xd, np.nextafter(rn, np.float16(-np.inf)), rn)
    up = np.where(rnd < xd, np.nextafter(rn, np.float16(np.inf)), rn)
    return rn, down.astype(np.float16), up.astype(np.float16)


def test_round_nearest_down_up_match_numpy():
    x = _sample_fp32()
    rn, down, up = _numpy_directed(x)
    got_rn = O.f16_round_array(x, "nearest")
    got_dn = O.f16_round_array(x, "down")
    got_up = O.f16_round_array(x, "up")
    # compare as values (so +0/-0 from different but equal routes are not an issue
    # for nearest) and as bits for the directed modes on non-zero results
    np.testing.assert_array_equal(got_rn.view(np.float16).astype(np.float64),
                                  rn.astype(np.float64))
    np.testing.assert_array_equal(got_dn.view(np.float16).astype(np.float64),
                                  down.astype(np.float64))
    np.testing.assert_array_equal(got_up.view(np.float16).astype(np.float64),
                                  up.astype(np.float64))


@pytest.mark.parametrize("x,down,up", [
    (1.0, 0x3C00, 0x3C00),
    (1.0001, 0x3C00, 0x3C01),
    (-1.0001, 0xBC01, 0xBC00),
    (65504.0, 0x7BFF, 0x7BFF),
    (65505.0, 0x7BFF, 0x7C00),          # above the largest finite: up -> +inf
    (-65505.0, 0xFC00, 0xFBFF),
    (1e-30, 0x0000, 0x0001),            # below the smallest subnormal
    (-1e-30, 0x8001, 0x8000),
    (2.0 ** -24, 0x0001, 0x0001),       # smallest subnormal, exact
    (2.0 ** -14, 0x0400, 0x0400),       # smallest normal, exact
    (3.0 * 2.0 ** -26, 0x0000, 0x0001),
])
def test_directed_rounding_fixed_points(x, down, up):
    assert O.f16_round_down(x) == down
    assert O.f16_round_up(x) == up


def test_f16_grid_values_are_fixed_points():
    # every finite fp16 value maps to itself in all three modes
    h = np.arange(1 << 16, dtype=np.uint16)
    v = h.view(np.float16)
    ok = np.isfinite(v)
    x = v[ok].astype(np.float32)
    for mode in ("down", "up", "nearest"):
        got = O.f16_round_array(x, mode).view(np.float16).astype(np.float64)
        np.testing.assert_array_equal(got, x.astype(np.float64))
