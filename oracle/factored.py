"""Sink-plus-low-rank state and its exact factored step, float64 (oracle).

State of one head (SEED summary (picx.dev), Methodology, "SEED Architecture",
decode "shallow in representation"):

    S = a v̄^T + U V^T,   v̄ in R^{d_v} fixed per head and shared by all requests,
                          a in R^{d_k}, U in R^{d_k x c}, V in R^{d_v x c}.

Value split (same page, Implications, Lemma 1):
    omega = v^T v̄ / ||v̄||^2,   eps = v - omega v̄,
and the sink coefficient follows the head's own recurrence
    a_t = Phi_t a_{t-1} + beta_t omega_t kappa_t.

Exact step (same page, "Exact Update (Lemma 2)"), Gated DeltaNet with decay g:
    a+ = g a + beta (omega - g kappa^T a) kappa
    U+ = [g U, kappa]
    V+ = [V, beta (eps - g V U^T kappa)]
Each step appends one column to each factor (SEED figures & tables
(thelatestinai.com), Figure 1(b): the step "updates the sink's coefficient a,
decays U and appends one column to each factor").

KDA replaces the scalar g by Diag(alpha) applied on the key side before the
erase, Phi = (I - beta kappa kappa^T) Diag(alpha):
    a+ = Diag(alpha) a + beta (omega - kappa^T Diag(alpha) a) kappa
    U+ = [Diag(alpha) U, kappa],  V+ = [V, beta (eps - V (Diag(alpha) U)^T kappa)]
Mamba-2 has no erase term and writes with Delta, Phi = alpha I:
    a+ = alpha a + Delta omega k,  U+ = [alpha U, k],  V+ = [V, Delta eps]
(these two readings of Lemma 2 for KDA and Mamba-2 are derived by substituting
each form's Phi into Lemma 1; the tests pin them against the dense recurrences).

Read-out after the step: o = S+^T q = v̄ (a+^T q) + V+ (U+^T q).

Batched layout: a (n, d_k), U (n, d_k, c), V (n, d_v, c), v̄ (n, d_v).
"""

from __future__ import annotations

import numpy as np

from workloads import FORM_GDN, FORM_KDA, FORM_MAMBA2


def split_value(v, vbar):
    """Lemma 1 split of v along v̄: returns (omega (n,), eps (n, d_v))."""
    omega = np.einsum("nj,nj->n", v, vbar) / np.einsum("nj,nj->n", vbar, vbar)
    eps = v - omega[:, None] * vbar
    return omega, eps


def reconstruct(a, U, V, vbar):
    """Dense state S = a v̄^T + U V^T, (n, d_k, d_v)."""
    return a[:, :, None] * vbar[:, None, :] + np.einsum("nir,njr->nij", U, V)


def sink_coefficient(S, vbar):
    """a = S v̄ / ||v̄||^2 (the projection of a dense state on v̄)."""
    return np.einsum("nij,nj->ni", S, vbar) / np.einsum("nj,nj->n", vbar, vbar)[:, None]


def step(form: int, a, U, V, vbar, q, k, v, alpha, beta):
    """One exact factored step followed by the read-out.

    alpha: GDN decay g (n,), KDA per-channel decay (n, d_k), Mamba-2 alpha (n,).
    beta:  GDN/KDA write strength (n,), Mamba-2 Delta (n,).
    Returns (a+, U+, V+, o) with c+1 columns in U+ and V+.
    """
    omega, eps = split_value(v, vbar)
    beta = np.asarray(beta, dtype=np.float64)
    if form == FORM_GDN:
        g = np.asarray(alpha, dtype=np.float64)
        ka = np.einsum("ni,ni->n", k, a)
        a_new = g[:, None] * a + (beta * (omega - g * ka))[:, None] * k
        U_dec = g[:, None, None] * U
        Utk = np.einsum("nir,ni->nr", U, k)
        v_col = beta[:, None] * (eps - g[:, None] * np.einsum("njr,nr->nj", V, Utk))
    elif form == FORM_KDA:
        Da = alpha * a
        kDa = np.einsum("ni,ni->n", k, Da)
        a_new = Da + (beta * (omega - kDa))[:, None] * k
        U_dec = alpha[:, :, None] * U
        DUtk = np.einsum("nir,ni->nr", U_dec, k)
        v_col = beta[:, None] * (eps - np.einsum("njr,nr->nj", V, DUtk))
    elif form == FORM_MAMBA2:
        al = np.asarray(alpha, dtype=np.float64)
        a_new = al[:, None] * a + (beta * omega)[:, None] * k
        U_dec = al[:, None, None] * U
        v_col = beta[:, None] * eps
    else:
        raise ValueError(f"unknown form {form}")
    U_new = np.concatenate([U_dec, k[:, :, None]], axis=2)
    V_new = np.concatenate([V, v_col[:, :, None]], axis=2)
    o = vbar * np.einsum("ni,ni->n", a_new, q)[:, None] + np.einsum(
        "njr,nr->nj", V_new, np.einsum("nir,ni->nr", U_new, q))
    return a_new, U_new, V_new, o


def step_general(a, U, V, vbar, q, k, v, g, beta_erase, beta_write):
    """Lemma 2 with separate erase and write coefficients (scalar decay g):

        S+ = g (I - beta_erase k k^T) S + beta_write k v^T
        a+ = g a + (beta_write omega - beta_erase g k^T a) k
        U+ = [g U, k],  V+ = [V, beta_write eps - beta_erase g V U^T k]

    Gated DeltaNet is beta_erase = beta_write = beta; Mamba-2 is beta_erase = 0,
    beta_write = Delta.  Used only to pin the Mamba-2 branch of ``step``.
    """
    omega, eps = split_value(v, vbar)
    g = np.asarray(g, dtype=np.float64)
    be = np.asarray(beta_erase, dtype=np.float64)
    bw = np.asarray(beta_write, dtype=np.float64)
    ka = np.einsum("ni,ni->n", k, a)
    a_new = g[:, None] * a + (bw * omega - be * g * ka)[:, None] * k
    Utk = np.einsum("nir,ni->nr", U, k)
    v_col = bw[:, None] * eps - (be * g)[:, None] * np.einsum("njr,nr->nj", V, Utk)
    U_new = np.concatenate([g[:, None, None] * U, k[:, :, None]], axis=2)
    V_new = np.concatenate([V, v_col[:, :, None]], axis=2)
    o = vbar * np.einsum("ni,ni->n", a_new, q)[:, None] + np.einsum(
        "njr,nr->nj", V_new, np.einsum("nir,ni->nr", U_new, q))
    return a_new, U_new, V_new, o
