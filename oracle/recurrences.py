"""Dense per-head recurrences in float64 (oracle; test infrastructure).

Orientation: the state S of one head is d_k x d_v, a token writes the outer
product k v^T, and the read-out is o = S^T q.

  Gated DeltaNet  S+ = g (I - beta k k^T) S + beta k v^T
  KDA             S+ = (I - beta k k^T) Diag(alpha) S + beta k v^T
  Mamba-2         S+ = alpha S + Delta k v^T

The three forms are the ones named in "Shallow Encoding Emits Deep Memories"
(SEED summary (picx.dev), "Exact Update (Lemma 2)": the factored form is closed
under Gated DeltaNet, Kimi Delta Attention and Mamba-2).  Lemma 1 on the same
page writes each as S_t = Phi_t S_{t-1} + beta_t kappa_t v_t^T; for Gated
DeltaNet Phi = g (I - beta k k^T), for KDA Phi = (I - beta k k^T) Diag(alpha),
for Mamba-2 Phi = alpha I with the write coefficient Delta in place of beta.
Mamba-2's orientation (d_k = d_B = 128, d_v = d_x = 64) is the one given by
SEED figures & tables (thelatestinai.com), Table 17.

All functions are batched over a leading unit axis: S (n, d_k, d_v), k and q
(n, d_k), v (n, d_v), scalar coefficients (n,), KDA alpha (n, d_k).
"""

from __future__ import annotations

import numpy as np

from workloads import FORM_GDN, FORM_KDA, FORM_MAMBA2, philox


def _outer(x, y):
    return x[:, :, None] * y[:, None, :]


def gdn_step(S, k, v, g, beta):
    """Gated DeltaNet: S+ = g (S - beta k (k^T S)) + beta k v^T."""
    g = np.asarray(g, dtype=np.float64)[:, None, None]
    beta = np.asarray(beta, dtype=np.float64)[:, None, None]
    kS = np.einsum("ni,nij->nj", k, S)
    return g * (S - beta * _outer(k, kS)) + beta * _outer(k, v)


def kda_step(S, k, v, alpha, beta):
    """Kimi Delta Attention: S+ = (I - beta k k^T) Diag(alpha) S + beta k v^T."""
    beta = np.asarray(beta, dtype=np.float64)[:, None, None]
    DS = alpha[:, :, None] * S
    kDS = np.einsum("ni,nij->nj", k, DS)
    return DS - beta * _outer(k, kDS) + beta * _outer(k, v)


def mamba2_step(S, k, v, alpha, delta):
    """Mamba-2: S+ = alpha S + Delta k v^T (k = B_t, v = x_t)."""
    alpha = np.asarray(alpha, dtype=np.float64)[:, None, None]
    delta = np.asarray(delta, dtype=np.float64)[:, None, None]
    return alpha * S + delta * _outer(k, v)


def dense_step(form: int, S, k, v, alpha, beta):
    """One dense step of ``form``; ``beta`` is Delta for Mamba-2."""
    if form == FORM_GDN:
        return gdn_step(S, k, v, alpha, beta)
    if form == FORM_KDA:
        return kda_step(S, k, v, alpha, beta)
    if form == FORM_MAMBA2:
        return mamba2_step(S, k, v, alpha, beta)
    raise ValueError(f"unknown form {form}")


def readout(S, q):
    """o = S^T q."""
    return np.einsum("nij,ni->nj", S, q)


def f64(inp: dict) -> dict:
    """float32 synthetic inputs as float64 arrays."""
    return {key: np.asarray(val, dtype=np.float64) for key, val in inp.items()}


def dense_prefill(cfg, b, l, h, n_tokens: int | None = None):
    """Dense state after ``n_tokens`` prefill tokens from S_0 = 0, for units (b, l, h).

    b, l, h are 1-D arrays of equal length.  Inputs come from the shared seeded
    generator (phase 0).  Returns S (n, d_k, d_v) float64.
    """
    T = cfg.n_prefill if n_tokens is None else n_tokens
    b, l, h = (np.asarray(x, dtype=np.int64) for x in (b, l, h))
    S = np.zeros((b.size, cfg.d_k, cfg.d_v))
    chunk = 256
    for t0 in range(0, T, chunk):
        tt = np.arange(t0, min(T, t0 + chunk))
        inp = f64(philox.token_inputs(cfg, b[:, None], l[:, None], h[:, None], tt[None, :],
                                      philox.PHASE_PREFILL, need_q=False))
        for j in range(tt.size):
            S = dense_step(cfg.form, S, inp["k"][:, j], inp["v"][:, j],
                           inp["alpha"][:, j], inp["beta"][:, j])
    return S
