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
