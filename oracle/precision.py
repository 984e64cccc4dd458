"""Rounding to the 16-bit factor formats, float64 (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

SEED figures & tables (thelatestinai.com), Table 9 (and the 16-bit rows of
Table 4): the shallow state's factors can be kept in fp16 or bf16, rounded when a
compression writes them, to nearest or stochastically.  Round-to-nearest is written
out here from the two formats' definitions:

  fp16 (IEEE 754 binary16): 11 significant bits; normal numbers 2^e (1 + f 2^-10)
      with e in [-14, 15]; below 2^-14 the subnormal grid of spacing 2^-24;
      largest finite value (2 - 2^-10) 2^15 = 65504.
  bf16 (bfloat16): float32's exponent range with 8 significant bits; normal
      numbers 2^e (1 + f 2^-7), e in [-126, 127]; subnormal spacing 2^-133;
      largest finite value (2 - 2^-7) 2^127.

A real x is rounded to the nearest member of the format's grid; a tie goes to the
member whose last significand bit is 0 (even); a magnitude that rounds past the
largest finite value becomes infinite.  The grid spacing at x (one unit in the
last place) is 2^(max(e, e_min) - p + 1), e = floor(log2 |x|), p the significant
bits.  Unit roundoff u = 2^-p: |round(x) - x| <= u |x| for x in the normal range.
"""

from __future__ import annotations

import numpy as np

# name -> (significant bits p, smallest normal exponent e_min, largest exponent e_max)
FORMATS = {"f16": (11, -14, 15), "bf16": (8, -126, 127)}


def unit_roundoff(fmt: str) -> float:
    p, _, _ = FORMATS[fmt]
    return 2.0 ** (-p)


def max_finite(fmt: str) -> float:
    p, _, emax = FORMATS[fmt]
    return (2.0 - 2.0 ** (1 - p)) * 2.0 ** emax


def ulp(x, fmt: str) -> np.ndarray:
    """Grid spacing of the format at |x| (at x = 0: the subnormal spacing)."""
    p, emin, _ = FORMATS[fmt]
    a = np.abs(np.asarray(x, dtype=np.float64))
    _, ex = np.frexp(a)                    # a = m 2^ex, m in [0.5, 1)
    e = np.where(a > 0, ex - 1, emin)      # a in [2^e, 2^(e+1))
    return np.ldexp(1.0, np.maximum(e, emin) - p + 1)


def round_nearest(x, fmt: str) -> np.ndarray:
    """x rounded to the nearest value of fmt, ties to even (float64 result)."""
    x = np.asarray(x, dtype=np.float64)
    step = ulp(x, fmt)
    # |x| / step has at most p + 1 integer bits: the division is exact (step is a
    # power of two) and np.rint rounds half to even
    r = np.rint(np.abs(x) / step) * step
    r = np.where(r > max_finite(fmt), np.inf, r)
    return np.copysign(r, x)
