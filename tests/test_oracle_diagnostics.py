"""Pins of the energy diagnostics of the oracle (no GPU)."""

import numpy as np

from oracle import compress, diagnostics, factored


def _orth(rng, n, d, k):
    q, _ = np.linalg.qr(rng.normal(size=(n, d, k)))
    return q


def test_parts_add_up_to_the_energy_of_the_reconstructed_state():
    rng = np.random.default_rng(0)
    n, dk, dv, c = 5, 12, 9, 6
    a, vb = rng.normal(size=(n, dk)), rng.normal(size=(n, dv))
    U, V = rng.normal(size=(n, dk, c)), rng.normal(size=(n, dv, c))
    e = diagnostics.energies(a, U, V, vb)
    S = factored.reconstruct(a, U, V, vb)
    np.testing.assert_allclose(e[:, 3], np.sum(S ** 2, axis=(1, 2)), rtol=1e-12)
    np.testing.assert_allclose(e[:, 0] + e[:, 1] + e[:, 2], e[:, 3], rtol=1e-12)
    np.testing.assert_allclose(e[:, 0], np.sum(a ** 2, 1) * np.sum(vb ** 2, 1), rtol=1e-12)


def test_known_spectrum_and_orthogonal_sink():
    """Orthonormal factors with singular values s and V^T vbar = 0: content = sum s^2,
    cross = 0, and the content beyond rank R is the tail of s."""
    rng = np.random.default_rng(1)
    n, d, c, R = 4, 10, 5, 3
    s = np.sort(rng.uniform(0.1, 3.0, size=(n, c)), axis=1)[:, ::-1]
    Qu, QvB = _orth(rng, n, d, c), _orth(rng, n, d, c + 1)
    vb = QvB[:, :, c] * 2.0                           # orthogonal to the V columns
    U, V = Qu * s[:, None, :], QvB[:, :, :c]
    a = rng.normal(size=(n, d))
    e = diagnostics.energies(a, U, V, vb)
    np.testing.assert_allclose(e[:, 1], np.sum(s ** 2, axis=1), rtol=1e-12)
    np.testing.assert_allclose(e[:, 2], 0.0, atol=1e-12)
    beyond = diagnostics.content_beyond_rank(e, s[:, :R])
    np.testing.assert_allclose(beyond, np.sum(s[:, R:] ** 2, 1) / np.sum(s ** 2, 1), rtol=1e-10)
    np.testing.assert_allclose(np.sqrt(beyond * e[:, 1]), compress.tail_norm(s, R), rtol=1e-10)


def test_pure_sink_has_share_one_and_no_content():
    rng = np.random.default_rng(2)
    a, vb = rng.normal(size=(3, 8)), rng.normal(size=(3, 6))
    e = diagnostics.energies(a, np.zeros((3, 8, 2)), np.zeros((3, 6, 2)), vb)
    np.testing.assert_allclose(diagnostics.sink_share(e), 1.0)
    assert np.all(e[:, 1] == 0) and np.all(e[:, 2] == 0)


def test_spectra_of_known_factors_and_of_a_pure_sink():
    """Orthonormal factors with singular values s and V^T vbar = 0: the content's
    spectrum is s; with the sink a vbar^T orthogonal to both sides too, the state's
    spectrum is s together with ||a|| ||vbar||.  A pure sink has the single singular
    value ||a|| ||vbar||."""
    rng = np.random.default_rng(3)
    n, d, c = 4, 12, 5
    s = np.sort(rng.uniform(0.1, 3.0, size=(n, c)), axis=1)[:, ::-1]
    QuA, QvB = _orth(rng, n, d, c + 1), _orth(rng, n, d, c + 1)
    a = QuA[:, :, c] * 5.0                           # orthogonal to the U columns
    vb = QvB[:, :, c] * 2.0                          # orthogonal to the V columns
    U, V = QuA[:, :, :c] * s[:, None, :], QvB[:, :, :c]
    sS, sC = diagnostics.spectra(a, U, V, vb)
    np.testing.assert_allclose(sC[:, :c], s, rtol=1e-12)
    assert np.all(sC[:, c:] < 1e-12)
    want = np.sort(np.concatenate([s, np.full((n, 1), 10.0)], axis=1), axis=1)[:, ::-1]
    np.testing.assert_allclose(sS[:, :c + 1], want, rtol=1e-12)
    sS0, sC0 = diagnostics.spectra(a, np.zeros((n, d, 2)), np.zeros((n, d, 2)), vb)
    np.testing.assert_allclose(sS0[:, 0], 10.0, rtol=1e-12)
    assert np.all(sS0[:, 1:] < 1e-12) and np.all(sC0 < 1e-12)


def test_spectra_do_not_depend_on_the_factor_gauge():
    """U V^T = (U G)(V G^{-T})^T: the spectra are those of the products."""
    rng = np.random.default_rng(4)
    n, dk, dv, c = 3, 10, 8, 4
    a, vb = rng.normal(size=(n, dk)), rng.normal(size=(n, dv))
    U, V = rng.normal(size=(n, dk, c)), rng.normal(size=(n, dv, c))
    G = rng.normal(size=(n, c, c)) + 3 * np.eye(c)
    sS, sC = diagnostics.spectra(a, U, V, vb)
    sS2, sC2 = diagnostics.spectra(a, U @ G, V @ np.linalg.inv(np.swapaxes(G, 1, 2)), vb)
    np.testing.assert_allclose(sS2, sS, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(sC2, sC, rtol=1e-9, atol=1e-12)
    # the state's energy is the sum of its squared singular values
    e = diagnostics.energies(a, U, V, vb)
    np.testing.assert_allclose(np.sum(sS ** 2, axis=1), e[:, 3], rtol=1e-12)


def test_top_output_direction_cosine_closed_form():
    """S = 3 u1 w1^T + 1 u2 w2^T with w1 at a known angle theta to vbar: v* = +-w1 and
    |cos(v*, vbar)| = |cos theta|; the relative gap is (3 - 1) / 3."""
    rng = np.random.default_rng(5)
    n, dk, dv = 6, 9, 7
    Qu, Qw = _orth(rng, n, dk, 2), _orth(rng, n, dv, 3)
    theta = rng.uniform(0, np.pi, size=n)
    w1, w2, w3 = Qw[:, :, 0], Qw[:, :, 1], Qw[:, :, 2]
    # vbar in the plane of w1 and w3 (orthogonal to w2), at angle theta to w1, norm 2.5
    vb = 2.5 * (np.cos(theta)[:, None] * w1 + np.sin(theta)[:, None] * w3)
    U = np.stack([3.0 * Qu[:, :, 0], Qu[:, :, 1]], axis=2)
    V = np.stack([w1, w2], axis=2)
    cos, gap = diagnostics.top_output_cosine(np.zeros((n, dk)), U, V, vb)
    np.testing.assert_allclose(cos, np.abs(np.cos(theta)), atol=1e-12)
    np.testing.assert_allclose(gap, 2.0 / 3.0, rtol=1e-12)
    # a pure sink's top output direction is vbar itself
    cos0, _ = diagnostics.top_output_cosine(rng.normal(size=(n, dk)), np.zeros((n, dk, 1)),
                                            np.zeros((n, dv, 1)), vb)
    np.testing.assert_allclose(cos0, 1.0, rtol=1e-12)


def test_energy_rank_closed_forms():
    """Energies (9, 4, 1) of 14: 9/14 < 0.9 <= 13/14 gives rank 2 at 90 %, and 99 % needs
    all three; a rank-one spectrum holds everything in one direction; zero gives 0."""
    s = np.array([[3.0, 2.0, 1.0], [1.0, 2.0, 3.0], [5.0, 0.0, 0.0], [0.0, 0.0, 0.0]])
    np.testing.assert_array_equal(diagnostics.energy_rank(s, 0.9), [2, 2, 1, 0])
    np.testing.assert_array_equal(diagnostics.energy_rank(s, 0.99), [3, 3, 1, 0])
    # exactly at the threshold counts as holding it: energies (1, 1), 50 %
    np.testing.assert_array_equal(diagnostics.energy_rank(np.array([[1.0, 1.0]]), 0.5), [1])
