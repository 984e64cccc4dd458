"""Periodic compression of the factors back to rank R, float64 (oracle).

What it computes: the best rank-R approximation of the content U V^T, the only
approximation of the method.  SEED summary (picx.dev), "Open-Loop Error Bound
(Corollary 4)" (the compression error that the bound integrates), and SEED
figures & tables (thelatestinai.com), Figure 1(b) (the factors return to rank R
once every W steps) and Table 1.  The sink a v̄^T is never touched: it is carried
exactly, outside the truncation (SEED commentary (sungsoo.github.io), "2. Exact
factored update").

Two functions:
  truncate_product  the plain definition: SVD of the d_k x d_v product U V^T,
                    keep the top R triplets (Eckart-Young).
  truncate_qr_core  the stated mechanism: QR of U and V, the (R+W) x (R+W) core
                    M = R_u R_v^T, its SVD, and U' = Q_u X_R, V' = Q_v Y_R.
Both split Sigma_R^{1/2} onto each side (a balanced gauge; the pages leave the
split open and only U V^T is ever compared).  Singular values at rounding level
(numerical rank) give zero columns.  Both return the full list of
singular values so callers can read the tail and the gap at R.
"""

from __future__ import annotations

import numpy as np


def numerical_sqrt_sigma(s, dims):
    """sqrt(s) with singular values at or below max(dims) * eps64 * s_1 set to zero.

    The standard numerical-rank rule: such values are rounding noise of exact
    zeros, their singular vectors are arbitrary, and a rank-deficient content
    keeps zero columns in their place.
    """
    tol = max(dims) * np.finfo(np.float64).eps * s[:, :1]
    return np.sqrt(np.where(s > tol, s, 0.0))


def _pad_cols(X, R):
    if X.shape[-1] >= R:
        return X[..., :R]
    pad = np.zeros(X.shape[:-1] + (R - X.shape[-1],))
    return np.concatenate([X, pad], axis=-1)


def truncate_product(U, V, R: int):
    """Top-R SVD of U V^T.  U (n, d_k, c), V (n, d_v, c) -> (U' (n,d_k,R), V' (n,d_v,R), s)."""
    A = np.einsum("nir,njr->nij", U, V)
    X, s, Yt = np.linalg.svd(A, full_matrices=False)
    r = min(R, s.shape[-1])
    sq = numerical_sqrt_sigma(s, A.shape[1:])[:, :r]
    Up = _pad_cols(X[:, :, :r] * sq[:, None, :], R)
    Vp = _pad_cols(np.swapaxes(Yt[:, :r, :], 1, 2) * sq[:, None, :], R)
    return Up, Vp, s


def truncate_qr_core(U, V, R: int):
    """QR of U and V, SVD of the small core R_u R_v^T, top-R reconstruction.

    Returns (U', V', s) with s the singular values of the core (= those of U V^T).
    """
    Qu, Ru = np.linalg.qr(U)          # (n, d_k, p), (n, p, c)
    Qv, Rv = np.linalg.qr(V)
    M = Ru @ np.swapaxes(Rv, 1, 2)    # (n, p_u, p_v)
    X, s, Yt = np.linalg.svd(M, full_matrices=False)
    r = min(R, s.shape[-1])
    sq = numerical_sqrt_sigma(s, (U.shape[1], V.shape[1]))[:, :r]
    Up = _pad_cols(Qu @ X[:, :, :r] * sq[:, None, :], R)
    Vp = _pad_cols(Qv @ np.swapaxes(Yt[:, :r, :], 1, 2) * sq[:, None, :], R)
    return Up, Vp, s


def tail_norm(s, R: int):
    """sqrt(sum_{i>R} s_i^2): the Frobenius error of the rank-R truncation."""
    return np.sqrt(np.sum(s[:, R:] ** 2, axis=-1))


def rel_gap(s, R: int):
    """(s_R - s_{R+1}) / s_1 at the truncation point (1 where there is no s_{R+1})."""
    if s.shape[-1] <= R:
        return np.ones(s.shape[0])
    top = np.where(s[:, 0] > 0, s[:, 0], 1.0)
    return (s[:, R - 1] - s[:, R]) / top
