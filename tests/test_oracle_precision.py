"""Pins of the oracle's rounding to the 16-bit factor formats (oracle/precision.py).

Two independent implementations of the same roundings serve as references: torch's
float32 -> float16 / bfloat16 conversions and numpy's float64 -> float16 cast, both
round-to-nearest-even.  Closed forms fix the ties, the subnormal grid and overflow.
"""

import numpy as np
import pytest
import torch

from oracle import precision as P


def _spread_float32(rng, n, lo_exp, hi_exp):
    """float32 values whose magnitudes cover 2^lo_exp .. 2^hi_exp, both signs, plus
    exact ties of the 16-bit grids (few significant bits)."""
    mant = rng.uniform(1.0, 2.0, size=n)
    ex = rng.integers(lo_exp, hi_exp, size=n)
    x = np.ldexp(mant, ex) * rng.choice([-1.0, 1.0], size=n)
    # ties: k + 1/2 grid steps for odd and even k, k of 8 bits (bf16) and 11 bits (fp16)
    k8 = rng.integers(1 << 7, 1 << 8, size=n // 4)
    k11 = rng.integers(1 << 10, 1 << 11, size=n // 4)
    ties = np.concatenate([np.ldexp(k8 + 0.5, rng.integers(-20, 4, size=n // 4)),
                           np.ldexp(k11 + 0.5, rng.integers(-20, 1, size=n // 4))])
    return np.concatenate([x, ties, -ties]).astype(np.float32)


@pytest.mark.parametrize("fmt,dtype,lo,hi", [("f16", torch.float16, -30, 17),
                                              ("bf16", torch.bfloat16, -140, 128)])
def test_rounding_equals_torch_conversion(fmt, dtype, lo, hi):
    rng = np.random.default_rng(0)
    x32 = _spread_float32(rng, 200_000, lo, hi)
    ref = torch.from_numpy(x32).to(dtype).double().numpy()
    got = P.round_nearest(x32.astype(np.float64), fmt)
    np.testing.assert_array_equal(got, ref)


def test_fp16_rounding_equals_numpy_from_float64():
    rng = np.random.default_rng(1)
    x = np.ldexp(rng.uniform(1, 2, 100_000), rng.integers(-27, 16, 100_000)) * rng.choice([-1, 1], 100_000)
    with np.errstate(over="ignore"):   # values from 65520 up become inf in both
        ref = x.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(P.round_nearest(x, "f16"), ref)


def test_closed_forms():
    r16 = lambda v: float(P.round_nearest(v, "f16"))   # noqa: E731
    rb = lambda v: float(P.round_nearest(v, "bf16"))   # noqa: E731
    # ties to even at 1: the grid above 1 has spacing 2^-10 (fp16), 2^-7 (bf16)
    assert r16(1 + 2.0 ** -11) == 1.0
    assert r16(1 + 3 * 2.0 ** -11) == 1 + 2.0 ** -9
    assert r16(1 + 2.0 ** -11 + 2.0 ** -30) == 1 + 2.0 ** -10
    assert rb(1 + 2.0 ** -8) == 1.0
    assert rb(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert rb(-(1 + 3 * 2.0 ** -8)) == -(1 + 2.0 ** -6)
    # fp16 range: largest finite 65504, the rounding threshold to infinity 65520
    assert r16(65504.0) == 65504.0
    assert r16(65519.9) == 65504.0
    assert r16(65520.0) == np.inf and r16(-1e6) == -np.inf
    # subnormal grid: spacing 2^-24 (fp16), 2^-133 (bf16); half the spacing ties to 0
    assert r16(2.0 ** -24) == 2.0 ** -24
    assert r16(2.0 ** -25) == 0.0
    assert r16(1.5 * 2.0 ** -25) == 2.0 ** -24
    assert rb(2.0 ** -133) == 2.0 ** -133 and rb(2.0 ** -134) == 0.0
    assert P.max_finite("bf16") == float(torch.finfo(torch.bfloat16).max)
    assert P.max_finite("f16") == float(torch.finfo(torch.float16).max)
    assert P.unit_roundoff("f16") == 2.0 ** -11 and P.unit_roundoff("bf16") == 2.0 ** -8


def test_error_bound_and_ulp():
    rng = np.random.default_rng(2)
    x = rng.normal(size=50_000) * 10.0 ** rng.uniform(-4, 4, size=50_000)
    for fmt in ("f16", "bf16"):
        r = P.round_nearest(x, fmt)
        normal = (np.abs(x) >= 2.0 ** P.FORMATS[fmt][1]) & (np.abs(x) <= P.max_finite(fmt))
        assert np.all(np.abs(r - x)[normal] <= P.unit_roundoff(fmt) * np.abs(x[normal]))
        fin = np.isfinite(r)
        assert np.all(np.abs(r - x)[fin] <= 0.5 * P.ulp(x[fin], fmt))
        # the grid spacing is the distance to the next member above a grid point
        g = np.abs(r[(r != 0) & np.isfinite(r)])
        up = g + P.ulp(g, fmt)
        assert np.array_equal(P.round_nearest(up, fmt), up)
        assert np.all(P.round_nearest(g + 0.49 * P.ulp(g, fmt), fmt) == g)
