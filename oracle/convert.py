"""End-of-prefill conversion of a dense state to sink + rank R, float64 (oracle).

SEED figures & tables (thelatestinai.com), Figure 1(a) and Table 1: at the end
of the prefill, the states left by x_1..x_{N-1} are compressed to the shallow
form.  SEED summary (picx.dev), Lemma 1: splitting each value along v̄
decomposes the state into the sink coefficient a and the content C.  For a dense
state that reads as the projection on v̄:

    a = S v̄ / ||v̄||^2,   C = S - a v̄^T   (so C v̄ = 0),

and the content is stored as its best rank-R approximation, the top-R SVD of C
with Sigma^{1/2} on each side.  If rank(C) < R the missing columns are zero
(singular values at rounding level count as zero, the numerical-rank rule).
"""

from __future__ import annotations

import numpy as np

from .compress import numerical_sqrt_sigma
from .factored import sink_coefficient


def convert(S, vbar, R: int):
    """Dense S (n, d_k, d_v) -> (a (n, d_k), U (n, d_k, R), V (n, d_v, R), s of C)."""
    a = sink_coefficient(S, vbar)
    C = S - a[:, :, None] * vbar[:, None, :]
    X, s, Yt = np.linalg.svd(C, full_matrices=False)
    r = min(R, s.shape[-1])
    sq = numerical_sqrt_sigma(s, S.shape[1:])[:, :r]
    U = np.zeros((S.shape[0], S.shape[1], R))
    V = np.zeros((S.shape[0], S.shape[2], R))
    U[:, :, :r] = X[:, :, :r] * sq[:, None, :]
    V[:, :, :r] = np.swapaxes(Yt[:, :r, :], 1, 2) * sq[:, None, :]
    return a, U, V, s
