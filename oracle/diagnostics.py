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
