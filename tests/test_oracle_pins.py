"""Pins of the fp64 oracle to facts fixed by the pages and by the mathematics.

Each test checks one oracle function against something other than itself: a
closed form, a special case that reduces to a textbook result, an invariant the
pages state (Lemma 1, Lemma 2, Corollary 4 of "Shallow Encoding Emits Deep
Memories"), brute force on tiny inputs, or the values printed in Table 2.
"""

import itertools
import os

import numpy as np
import pytest

from oracle import bytes_model, compress, convert, factored, recurrences, run
from workloads import FORM_GDN, FORM_KDA, FORM_MAMBA2, config, philox

RNG = np.random.default_rng(12345)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_state(n, dk, dv, c, rng=RNG):
    vb = rng.normal(size=(n, dv)) * rng.uniform(1, 4, size=(n, 1))
    a = rng.normal(size=(n, dk))
    U = rng.normal(size=(n, dk, c))
    V = rng.normal(size=(n, dv, c))
    V -= np.einsum("njr,nj->nr", V, vb)[:, None, :] * vb[:, :, None] / np.sum(vb * vb, 1)[:, None, None]
    return a, U, V, vb


def _rand_inputs(form, n, dk, dv, rng=RNG):
    q = _unit(rng.normal(size=(n, dk)))
    k = _unit(rng.normal(size=(n, dk)))
    v = rng.normal(size=(n, dv))
    beta = rng.uniform(0.05, 0.95, size=n)
    if form == FORM_KDA:
        alpha = rng.uniform(0.85, 1.0, size=(n, dk))
    else:
        alpha = rng.uniform(0.5, 1.0, size=n)
    return q, k, v, alpha, beta


# ----------------------------------------------------------------- dense steps

def test_gdn_step_closed_form_on_key_and_complement():
    """GDN: k^T S+ = g (1 - beta) k^T S + beta v^T, and x^T S+ = g x^T S for x _|_ k."""
    n, dk, dv = 6, 12, 9
    S = RNG.normal(size=(n, dk, dv))
    _, k, v, g, beta = _rand_inputs(FORM_GDN, n, dk, dv)
    Sp = recurrences.gdn_step(S, k, v, g, beta)
    lhs = np.einsum("ni,nij->nj", k, Sp)
    rhs = (g * (1 - beta))[:, None] * np.einsum("ni,nij->nj", k, S) + beta[:, None] * v
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)
    x = RNG.normal(size=(n, dk))
    x -= np.sum(x * k, 1)[:, None] * k
    np.testing.assert_allclose(np.einsum("ni,nij->nj", x, Sp),
                               g[:, None] * np.einsum("ni,nij->nj", x, S), atol=1e-12)


def test_gdn_delta_rule_writes_v_at_key():
    """g = 1, beta = 1, orthonormal keys: every key reads back exactly its value."""
    dk = dv = 8
    K = np.linalg.qr(RNG.normal(size=(dk, dk)))[0].T     # rows orthonormal
    vals = RNG.normal(size=(dk, dv))
    S = np.zeros((1, dk, dv))
    for t in range(dk):
        S = recurrences.gdn_step(S, K[t][None], vals[t][None], np.ones(1), np.ones(1))
    np.testing.assert_allclose(K @ S[0], vals, atol=1e-12)
    # rewriting one key replaces its value and leaves the others
    newv = RNG.normal(size=dv)
    S = recurrences.gdn_step(S, K[3][None], newv[None], np.ones(1), np.ones(1))
    expect = vals.copy()
    expect[3] = newv
    np.testing.assert_allclose(K @ S[0], expect, atol=1e-12)


def test_gdn_erase_is_a_contraction():
    """||g (I - beta k k^T) S||_2 <= g ||S||_2 for unit k and beta in (0, 1]."""
    n, dk, dv = 20, 10, 7
    S = RNG.normal(size=(n, dk, dv))
    _, k, _, g, beta = _rand_inputs(FORM_GDN, n, dk, dv)
    Sp = recurrences.gdn_step(S, k, np.zeros((n, dv)), g, beta)
    assert np.all(np.linalg.norm(Sp, 2, axis=(1, 2)) <= g * np.linalg.norm(S, 2, axis=(1, 2)) + 1e-12)


def test_kda_closed_form_and_gdn_special_case():
    """KDA: k^T S+ = (1-beta) k^T D S + beta v^T, x^T S+ = x^T D S (x _|_ k); alpha = g 1 gives GDN."""
    n, dk, dv = 5, 12, 10
    S = RNG.normal(size=(n, dk, dv))
    _, k, v, alpha, beta = _rand_inputs(FORM_KDA, n, dk, dv)
    Sp = recurrences.kda_step(S, k, v, alpha, beta)
    DS = alpha[:, :, None] * S
    np.testing.assert_allclose(np.einsum("ni,nij->nj", k, Sp),
                               (1 - beta)[:, None] * np.einsum("ni,nij->nj", k, DS) + beta[:, None] * v,
                               atol=1e-12)
    x = RNG.normal(size=(n, dk))
    x -= np.sum(x * k, 1)[:, None] * k
    np.testing.assert_allclose(np.einsum("ni,nij->nj", x, Sp), np.einsum("ni,nij->nj", x, DS), atol=1e-12)
    g = RNG.uniform(0.5, 1, size=n)
    np.testing.assert_allclose(recurrences.kda_step(S, k, v, np.repeat(g[:, None], dk, 1), beta),
                               recurrences.gdn_step(S, k, v, g, beta), atol=1e-12)


def test_mamba2_prefill_equals_unrolled_sum():
    """Mamba-2 from S_0 = 0: S_T = sum_t (prod_{s>t} alpha_s) Delta_t k_t v_t^T."""
    cfg = config(3, batch=1, layers=2, heads=2)
    T = 40
    b, l, h = np.array([0, 0]), np.array([1, 0]), np.array([0, 1])
    S = recurrences.dense_prefill(cfg, b, l, h, T)
    inp = recurrences.f64(philox.token_inputs(cfg, b[:, None], l[:, None], h[:, None],
                                              np.arange(T)[None, :], philox.PHASE_PREFILL))
    expect = np.zeros_like(S)
    for t in range(T):
        w = inp["beta"][:, t] * np.prod(inp["alpha"][:, t + 1:], axis=1)
        expect += w[:, None, None] * inp["k"][:, t, :, None] * inp["v"][:, t, None, :]
    np.testing.assert_allclose(S, expect, rtol=1e-12, atol=1e-14)


def test_readout_orientation():
    """o = S^T q: a state e_i e_j^T read with q = e_i gives e_j."""
    S = np.zeros((1, 5, 4))
    S[0, 2, 3] = 1.0
    q = np.zeros((1, 5))
    q[0, 2] = 1.0
    np.testing.assert_array_equal(recurrences.readout(S, q)[0], [0, 0, 0, 1.0])


# ------------------------------------------------------- Lemma 1 and Lemma 2

@pytest.mark.parametrize("form", [FORM_GDN, FORM_KDA, FORM_MAMBA2])
def test_lemma2_factored_step_is_exact(form):
    """Between compressions, a v̄^T + U V^T equals the dense recurrence, and so does o."""
    n, dk, dv, c = 4, 16, 12, 3
    a, U, V, vb = _rand_state(n, dk, dv, c)
    S = factored.reconstruct(a, U, V, vb)
    for _ in range(12):
        q, k, v, alpha, beta = _rand_inputs(form, n, dk, dv)
        a, U, V, o = factored.step(form, a, U, V, vb, q, k, v, alpha, beta)
        S = recurrences.dense_step(form, S, k, v, alpha, beta)
        Sf = factored.reconstruct(a, U, V, vb)
        assert np.max(np.abs(Sf - S)) <= 1e-12 * np.max(np.abs(S))
        np.testing.assert_allclose(o, recurrences.readout(S, q), rtol=0, atol=1e-12 * np.max(np.abs(S)))
    assert U.shape[2] == c + 12 and V.shape[2] == c + 12


@pytest.mark.parametrize("form", [FORM_GDN, FORM_KDA, FORM_MAMBA2])
def test_lemma1_sink_follows_its_own_recurrence(form):
    """a+ depends on v only through omega: changing eps at fixed omega leaves a+ bit-identical,
    and a+ equals the sink coefficient of the dense state."""
    n, dk, dv, c = 5, 10, 8, 2
    a, U, V, vb = _rand_state(n, dk, dv, c)
    q, k, v, alpha, beta = _rand_inputs(form, n, dk, dv)
    d = RNG.normal(size=(n, dv))
    d -= (np.sum(d * vb, 1) / np.sum(vb * vb, 1))[:, None] * vb     # d _|_ v̄
    a1, _, V1, _ = factored.step(form, a, U, V, vb, q, k, v, alpha, beta)
    U2 = RNG.normal(size=U.shape)                                  # other content too
    a2, _, _, _ = factored.step(form, a, U2, V, vb, q, k, v + d, alpha, beta)
    omega1, _ = factored.split_value(v, vb)
    omega2, _ = factored.split_value(v + d, vb)
    np.testing.assert_allclose(omega1, omega2, rtol=1e-14)
    np.testing.assert_allclose(a1, a2, rtol=1e-13, atol=1e-13)
    S = recurrences.dense_step(form, factored.reconstruct(a, U, V, vb), k, v, alpha, beta)
    np.testing.assert_allclose(a1, factored.sink_coefficient(S, vb), atol=1e-12)
    # content stays orthogonal to v̄
    assert np.max(np.abs(np.einsum("njr,nj->nr", V1, vb))) < 1e-12


def test_mamba2_is_the_general_update_with_erase_off():
    n, dk, dv, c = 4, 16, 8, 3
    a, U, V, vb = _rand_state(n, dk, dv, c)
    q, k, v, alpha, delta = _rand_inputs(FORM_MAMBA2, n, dk, dv)
    m2 = factored.step(FORM_MAMBA2, a, U, V, vb, q, k, v, alpha, delta)
    gen = factored.step_general(a, U, V, vb, q, k, v, alpha, np.zeros(n), delta)
    for x, y in zip(m2, gen):
        np.testing.assert_allclose(x, y, rtol=1e-14, atol=1e-14)
    # and Gated DeltaNet is the general update with erase = write = beta
    _, _, _, g, beta = _rand_inputs(FORM_GDN, n, dk, dv)
    gd = factored.step(FORM_GDN, a, U, V, vb, q, k, v, g, beta)
    gen = factored.step_general(a, U, V, vb, q, k, v, g, beta, beta)
    for x, y in zip(gd, gen):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------- compression

def test_truncation_of_a_known_spectrum():
    """U V^T = Q1 diag(s) Q2^T: rank-R truncation keeps exactly the top R terms."""
    d, c, R = 12, 8, 3
    Q1 = np.linalg.qr(RNG.normal(size=(d, c)))[0]
    Q2 = np.linalg.qr(RNG.normal(size=(d, c)))[0]
    s = np.array([9.0, 7.0, 5.0, 3.0, 2.0, 1.0, 0.5, 0.25])
    perm = RNG.permutation(c)
    U = (Q1[:, perm] * np.sqrt(s[perm]))[None]
    V = (Q2[:, perm] * np.sqrt(s[perm]))[None]
    expect = (Q1[:, :R] * s[:R]) @ Q2[:, :R].T
    for fn in (compress.truncate_product, compress.truncate_qr_core):
        Up, Vp, sv = fn(U, V, R)
        np.testing.assert_allclose(Up[0] @ Vp[0].T, expect, atol=1e-12)
        np.testing.assert_allclose(sv[0, :c], s, atol=1e-12)
        np.testing.assert_allclose(compress.tail_norm(sv, R), np.sqrt(np.sum(s[R:] ** 2)), atol=1e-12)


def test_eckart_young_by_brute_force_8x8():
    """On 8 x 8 products no rank-R candidate beats the truncation: not any R-subset of the
    SVD triplets, not random rank-R matrices, not local perturbations of the result."""
    R = 3
    for trial in range(5):
        rng = np.random.default_rng(100 + trial)
        U = rng.normal(size=(1, 8, 6))
        V = rng.normal(size=(1, 8, 6))
        A = U[0] @ V[0].T
        Up, Vp, s = compress.truncate_product(U, V, R)
        best = np.linalg.norm(A - Up[0] @ Vp[0].T)
        np.testing.assert_allclose(best, compress.tail_norm(s, R)[0], rtol=1e-12)
        X, sv, Yt = np.linalg.svd(A)
        for sub in itertools.combinations(range(8), R):
            sub = list(sub)
            cand = (X[:, sub] * sv[sub]) @ Yt[sub]
            assert np.linalg.norm(A - cand) >= best - 1e-12
        for _ in range(300):
            P = rng.normal(size=(8, R))
            Q = rng.normal(size=(8, R))
            # best rank-R matrix with column space P: least squares in Q
            Pq = np.linalg.qr(P)[0]
            cand = Pq @ (Pq.T @ A)
            assert np.linalg.norm(A - cand) >= best - 1e-12
            cand2 = (Up[0] + 1e-3 * P) @ (Vp[0] + 1e-3 * Q).T      # still rank R
            assert np.linalg.norm(A - cand2) >= best - 1e-12


def test_qr_core_route_equals_product_svd():
    R = 16
    for c, d in ((32, 128), (40, 64), (96, 128), (8, 16)):
        U = RNG.normal(size=(3, d, c)) * RNG.uniform(0.01, 3, size=(3, 1, c))
        V = RNG.normal(size=(3, d, c))
        Rr = min(R, c // 2)
        U1, V1, s1 = compress.truncate_product(U, V, Rr)
        U2, V2, s2 = compress.truncate_qr_core(U, V, Rr)
        A1 = np.einsum("nir,njr->nij", U1, V1)
        A2 = np.einsum("nir,njr->nij", U2, V2)
        assert np.max(np.abs(A1 - A2)) <= 1e-11 * np.max(np.abs(A1))
        np.testing.assert_allclose(s1[:, :c], s2[:, :c], rtol=1e-10, atol=1e-12)


def test_truncation_is_lossless_at_low_rank_and_pads_zero_columns():
    U = RNG.normal(size=(2, 10, 2))
    V = RNG.normal(size=(2, 7, 2))
    for fn in (compress.truncate_product, compress.truncate_qr_core):
        Up, Vp, _ = fn(U, V, 4)
        assert Up.shape == (2, 10, 4) and Vp.shape == (2, 7, 4)
        np.testing.assert_allclose(np.einsum("nir,njr->nij", Up, Vp),
                                   np.einsum("nir,njr->nij", U, V), atol=1e-12)


# -------------------------------------------------------------- conversion

def test_conversion_recovers_a_known_sink_and_content():
    """S = a0 v̄^T + C0 with C0 v̄ = 0 and rank(C0) <= R converts losslessly to (a0, C0)."""
    n, dk, dv, R = 3, 16, 12, 4
    vb = RNG.normal(size=(n, dv)) * 2.5
    a0 = RNG.normal(size=(n, dk))
    P = RNG.normal(size=(n, dk, R - 1))
    Q = RNG.normal(size=(n, dv, R - 1))
    Q -= np.einsum("njr,nj->nr", Q, vb)[:, None, :] * vb[:, :, None] / np.sum(vb * vb, 1)[:, None, None]
    C0 = np.einsum("nir,njr->nij", P, Q)
    S = a0[:, :, None] * vb[:, None, :] + C0
    a, U, V, s = convert.convert(S, vb, R)
    np.testing.assert_allclose(a, a0, atol=1e-12)
    np.testing.assert_allclose(np.einsum("nir,njr->nij", U, V), C0, atol=1e-11)
    assert np.max(np.abs(np.einsum("njr,nj->nr", V, vb))) < 1e-11
    assert np.all(s[:, R - 1:] < 1e-10)                 # rank(C0) = R - 1


def test_conversion_error_is_the_content_tail():
    n, dk, dv, R = 4, 16, 16, 4
    S = RNG.normal(size=(n, dk, dv))
    vb = RNG.normal(size=(n, dv))
    a, U, V, s = convert.convert(S, vb, R)
    err = np.linalg.norm(S - factored.reconstruct(a, U, V, vb), axis=(1, 2))
    np.testing.assert_allclose(err, compress.tail_norm(s, R), rtol=1e-10)
    # C v̄ = 0, so v̄ is a right null vector of the content and the last singular value is 0
    assert np.all(s[:, -1] < 1e-10 * s[:, 0])


# ------------------------------------------------ whole trajectories (tiny workload)

@pytest.fixture(scope="module")
def tiny_run():
    cfg = config(0)
    return cfg, run.run_units(cfg, [0, 0], [0, 0], [0, 1])


def test_compression_schedule_every_w_steps(tiny_run):
    cfg, r = tiny_run
    assert r["comp_steps"] == list(range(cfg.W, cfg.n_decode + 1, cfg.W))
    expect = [cfg.R + ((t + 1) % cfg.W) for t in range(cfg.n_decode)]
    np.testing.assert_array_equal(r["ncols"], expect)


@pytest.mark.parametrize("lead_in", [1, 3])
def test_ragged_schedule_lead_in(lead_in):
    """A request that joined j steps earlier holds R + j columns at step 0 and compresses
    after steps W - j, 2W - j, ...; Lemma 1 and Corollary 4 still hold over its whole run
    (the lead-in steps included), and its lead-in inputs differ from its decode inputs."""
    cfg = config(0)
    r = run.run_units(cfg, [0, 0], [0, 0], [0, 1], lead_in=lead_in)
    assert r["comp_steps"] == list(range(cfg.W - lead_in, cfg.n_decode + 1, cfg.W))
    expect = [cfg.R + ((t + 1 + lead_in) % cfg.W) for t in range(cfg.n_decode)]
    np.testing.assert_array_equal(r["ncols"], expect)
    assert np.max(r["sink_dev"]) < 1e-12 * max(1.0, np.max(np.abs(r["a_t"])))
    inp = philox.token_inputs(cfg, 0, 0, np.array([0, 1])[:, None], np.arange(cfg.n_decode)[None, :],
                              philox.PHASE_DECODE)
    lead = philox.token_inputs(cfg, 0, 0, np.array([0, 1])[:, None], np.arange(lead_in)[None, :],
                               philox.PHASE_LEADIN)
    g_bar = max(float(np.max(inp["alpha"])), float(np.max(lead["alpha"])))
    bound = np.max(r["tail"], axis=0) / (1.0 - g_bar ** cfg.W)
    assert np.all(np.max(r["err_open"], axis=0) <= bound)
    assert not np.allclose(lead["k"][:, 0], inp["k"][:, 0])
    # without lead-in the same call is the lockstep schedule
    r0 = run.run_units(cfg, [0, 0], [0, 0], [0, 1], lead_in=0)
    assert r0["comp_steps"] == list(range(cfg.W, cfg.n_decode + 1, cfg.W))


def test_lemma1_sink_is_exact_across_compressions(tiny_run):
    """a_t equals the sink coefficient of the never-compressed dense state at every step."""
    _, r = tiny_run
    assert np.max(r["sink_dev"]) < 1e-12 * max(1.0, np.max(np.abs(r["a_t"])))
    assert np.max(np.abs(np.einsum("njr,nj->nr", r["V"], r["vbar"]))) < 1e-12


def test_corollary4_open_loop_bound(tiny_run):
    """||S~_t - S_t||_F <= eps_bar / (1 - g_bar^W) with eps_bar the largest compression error
    (conversion included) and g_bar the largest decay."""
    cfg, r = tiny_run
    inp = philox.token_inputs(cfg, 0, 0, np.array([0, 1])[:, None], np.arange(cfg.n_decode)[None, :],
                              philox.PHASE_DECODE)
    g_bar = float(np.max(inp["alpha"]))
    eps_bar = np.max(r["tail"], axis=0)
    bound = eps_bar / (1.0 - g_bar ** cfg.W)
    worst = np.max(r["err_open"], axis=0)
    assert np.all(worst <= bound)
    assert np.all(worst > 0)


def test_tiny_workload_matches_the_plain_definition_route(tiny_run):
    """Re-running the tiny trajectory with the plain product SVD gives the same outputs."""
    cfg, r = tiny_run
    orig = compress.truncate_qr_core
    try:
        compress.truncate_qr_core = compress.truncate_product
        r2 = run.run_units(cfg, [0, 0], [0, 0], [0, 1], keep_shadow=False)
    finally:
        compress.truncate_qr_core = orig
    np.testing.assert_allclose(r2["o"], r["o"], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(r2["S"], r["S"], rtol=1e-9, atol=1e-10)


# ------------------------------------------------------------------- Table 2

def _read_table(path):
    rows = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows[parts[0]] = [float(x) for x in parts[1:]]
    return rows


def test_byte_account_reproduces_table2(golden_dir):
    vals = _read_table(os.path.join(golden_dir, "table2_state_bytes.txt"))
    shapes = _read_table(os.path.join(golden_dir, "table2_shapes.txt"))
    assert set(vals) == set(shapes) and len(vals) == 5
    for model, (orig, at_r, mean, peak, cache, res_o, res_s) in vals.items():
        heads, dk, dv, R, W = (int(x) for x in shapes[model])
        mb = lambda x: round(x / 1e6, 1)                  # noqa: E731
        assert mb(bytes_model.dense_state_bytes(heads, dk, dv)) == orig
        assert mb(bytes_model.shallow_state_bytes(heads, dk, dv, R, 0)) == at_r
        assert mb(bytes_model.shallow_state_bytes(heads, dk, dv, R, W // 2)) == mean
        assert mb(bytes_model.shallow_state_bytes(heads, dk, dv, R, W)) == peak
        T = 8192
        ro = bytes_model.resident_bytes(bytes_model.dense_state_bytes(heads, dk, dv), T, int(cache))
        rs = bytes_model.resident_bytes(bytes_model.shallow_state_bytes(heads, dk, dv, R, W // 2), T, int(cache))
        assert round(ro / 1e6) == res_o
        assert round(rs / 1e6) == res_s


# ------------------------------------------------------------------- small helpers

def test_rel_gap_and_numerical_rank_closed_forms():
    """The gap at the truncation point and the numerical-rank rule on spectra whose
    answers are written out: s = (4, 3, 3, 1) has gap (4-3)/4 at R = 1, none at R = 2
    (a tie) and no s_{R+1} at R = 4; singular values at or below max(d) eps s_1 count
    as zero, larger ones keep their square roots."""
    from oracle import compress as oc
    s = np.array([[4.0, 3.0, 3.0, 1.0]])
    assert oc.rel_gap(s, 1)[0] == 0.25
    assert oc.rel_gap(s, 2)[0] == 0.0
    assert oc.rel_gap(s, 3)[0] == 0.5
    assert oc.rel_gap(s, 4)[0] == 1.0
    assert oc.tail_norm(s, 2)[0] == np.sqrt(10.0)
    sq = oc.numerical_sqrt_sigma(np.array([[4.0, 1e-3, 1e-20, 0.0]]), (16, 16))
    np.testing.assert_array_equal(sq, [[2.0, np.sqrt(1e-3), 0.0, 0.0]])
