"""Energies of a factored state (test infrastructure), by their plain definitions.

SEED figures & tables (thelatestinai.com), Figure 3 (f)-(g) and Figure 12 (f): a
state S = a vbar^T + U V^T splits into the sink a vbar^T and the content U V^T; the
pages report the sink's share of ||S||_F^2, the Frobenius norms of both parts, and
the share of the content energy beyond rank R.  Everything here is formed from the
explicit d_k x d_v matrices in float64.
"""

from __future__ import annotations

import numpy as np


def energies(a, U, V, vbar) -> np.ndarray:
    """Per unit (leading axis): [||a vbar^T||_F^2, ||U V^T||_F^2, 2 <a vbar^T, U V^T>_F,
    ||a vbar^T + U V^T||_F^2] from the explicit matrices (U the true columns)."""
    a, U, V, vbar = (np.asarray(x, dtype=np.float64) for x in (a, U, V, vbar))
    sink = np.einsum("ni,nj->nij", a, vbar)
    content = np.einsum("nir,njr->nij", U, V)
    S = sink + content
    return np.stack([np.sum(sink ** 2, axis=(1, 2)), np.sum(content ** 2, axis=(1, 2)),
                     2.0 * np.sum(sink * content, axis=(1, 2)), np.sum(S ** 2, axis=(1, 2))], axis=1)


def sink_share(e) -> np.ndarray:
    """The sink's share of the state's energy, from energies() rows."""
    e = np.asarray(e, dtype=np.float64)
    return e[:, 0] / np.where(e[:, 3] > 0, e[:, 3], 1.0)


def content_beyond_rank(e, sigma_kept) -> np.ndarray:
    """Share of the content energy (rows [1] + [2] of energies()) that the singular
    values kept at rank R (sigma_kept, [n][R]) do not hold."""
    e = np.asarray(e, dtype=np.float64)
    c = e[:, 1] + e[:, 2]
    kept = np.sum(np.asarray(sigma_kept, dtype=np.float64) ** 2, axis=1)
    return (c - kept) / np.where(c > 0, c, 1.0)


def spectra(a, U, V, vbar):
    """Per unit: the singular values of the state S = a vbar^T + U V^T and of the content
    C = U V^T (U the true columns), each descending, from the explicit d_k x d_v matrices
    (numpy SVD, float64).  SEED figures & tables, Figure 3 (e): the spectra of the state
    and of the content, divided by the head's top singular value (sigma_S[:, :1]);
    Figure 13 (a): the energy share of the state's i-th singular direction,
    sigma_S_i^2 / sum_j sigma_S_j^2.  Returns (sigma_S, sigma_C)."""
    a, U, V, vbar = (np.asarray(x, dtype=np.float64) for x in (a, U, V, vbar))
    C = np.einsum("nir,njr->nij", U, V)
    S = np.einsum("ni,nj->nij", a, vbar) + C
    return np.linalg.svd(S, compute_uv=False), np.linalg.svd(C, compute_uv=False)


def top_output_cosine(a, U, V, vbar):
    """|cos| between each head's top output direction v* and vbar (SEED figures & tables,
    Figure 3 (h); Figure 13 (c) compares v* across prompts).  The read-out o = S^T q lies
    in the span of the right singular vectors of S, so the top output direction is the
    right singular vector of the largest singular value.  Also returns the relative gap
    (sigma_1 - sigma_2) / sigma_1, which bounds how well v* is defined."""
    a, U, V, vbar = (np.asarray(x, dtype=np.float64) for x in (a, U, V, vbar))
    S = np.einsum("ni,nj->nij", a, vbar) + np.einsum("nir,njr->nij", U, V)
    _, s, Wt = np.linalg.svd(S)
    vstar = Wt[:, 0, :]
    cos = np.abs(np.einsum("nj,nj->n", vstar, vbar)) / np.linalg.norm(vbar, axis=1)
    top = np.where(s[:, 0] > 0, s[:, 0], 1.0)
    gap = (s[:, 0] - s[:, 1]) / top if s.shape[1] > 1 else np.ones(s.shape[0])
    return cos, gap


def energy_rank(sigma, frac: float) -> np.ndarray:
    """Smallest k such that the k largest singular values hold at least `frac` of the
    energy sum_i sigma_i^2 (SEED figures & tables, Figure 13 (d): the rank holding 90%
    and 99% of the content's energy); 0 for a zero matrix."""
    s2 = np.sort(np.asarray(sigma, dtype=np.float64) ** 2, axis=-1)[..., ::-1]
    tot = s2.sum(axis=-1)
    cum = np.cumsum(s2, axis=-1)
    k = np.sum(cum < frac * tot[..., None], axis=-1) + 1
    return np.where(tot > 0, k, 0).astype(np.int64)
