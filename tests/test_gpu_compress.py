"""seed_compress on factor states built on the host, against the oracle's truncation.

The states are inputs (uploaded), so nothing the device computes reaches the
oracle.  Covers every form, the Cholesky-QR paths (R + W <= 32 with R <= 16, and
32 < R + W <= 64 with R <= 32, for d in {64, 128}), the Householder path (larger
windows, 16-wide heads), a key repeated inside one window (the Cholesky-QR paths
decline it), and exactly zero columns.
"""

import numpy as np
import pytest

from oracle import compress as ocomp
from workloads import FORM_GDN, FORM_KDA, FORM_MAMBA2

from parity_util import TOL, ensure_lib, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _host_state(form, n, dk, dv, R, W, rng, repeat=False, zero_cols=0):
    """Stored factors with m = R + W columns and their lazy scales, plus the true U."""
    m = R + W
    U = rng.normal(size=(n, dk, m)).astype(np.float32)
    if form != FORM_MAMBA2:
        U /= np.linalg.norm(U, axis=1, keepdims=True)
    V = (rng.normal(size=(n, dv, m)) * rng.uniform(0.2, 3, size=(n, 1, m))).astype(np.float32)
    if repeat:
        U[:, :, m - 1] = U[:, :, m - 3]
    if zero_cols:
        U[:, :, :zero_cols] = 0
        V[:, :, :zero_cols] = 0
    if form == FORM_KDA:
        scale = rng.uniform(0.3, 1.0, size=(n, dk)).astype(np.float32)
        Utrue = scale[:, :, None].astype(np.float64) * U
    else:
        slen = (m + 3) // 4 * 4
        scale = np.ones((n, slen), dtype=np.float32)
        scale[:, :m] = rng.uniform(0.05, 1.0, size=(n, m)).astype(np.float32)
        Utrue = U.astype(np.float64) * scale[:, None, :m].astype(np.float64)
    return U, V, scale, Utrue


def _run(form, dk, dv, R, W, repeat=False, zero_cols=0, n=24, seed=0):
    import torch
    from rank_recurrent_state_b200 import seed as S
    rng = np.random.default_rng(seed)
    m = R + W
    U, V, scale, Utrue = _host_state(form, n, dk, dv, R, W, rng, repeat, zero_cols)
    d = S.Dims(form, n, 1, 1, dk, dv, R, W)
    vbar = torch.ones(1, 1, dv, device="cuda")
    st = S.State.allocate(d, vbar)
    st.U.copy_(torch.from_numpy(np.ascontiguousarray(np.swapaxes(U, 1, 2))).view_as(st.U))
    st.V.copy_(torch.from_numpy(np.ascontiguousarray(np.swapaxes(V, 1, 2))).view_as(st.V))
    st.scale.copy_(torch.from_numpy(scale).view_as(st.scale))
    st.a.zero_()
    st.ncols.fill_(m)
    ws = S.Workspace(d)
    sig = torch.zeros(n, R, device="cuda")
    S.seed_compress(d, st, S.SEED_ALL_LAYERS, ws, sigma_out=sig)
    dense = torch.empty(n, dk, dv, device="cuda")
    S.seed_state_to_dense(d, st, S.SEED_ALL_LAYERS, dense, ws)
    flags = S.seed_get_status(ws)
    diag = S.seed_get_diagnostics(ws)
    assert flags == 0, hex(flags)
    assert np.all(st.ncols.cpu().numpy() == R)
    Up, Vp, s = ocomp.truncate_product(Utrue, V.astype(np.float64), R)
    ref = np.einsum("nir,njr->nij", Up, Vp)
    got = dense.cpu().numpy()
    for u in range(n):
        assert rel_fro(got[u], ref[u]) <= TOL, (u, rel_fro(got[u], ref[u]))
        assert rel_fro(sig.cpu().numpy()[u], s[u, :R]) <= TOL
    return diag


@pytest.mark.parametrize("form", [FORM_GDN, FORM_KDA, FORM_MAMBA2])
@pytest.mark.parametrize("dk,dv,R,W", [(128, 128, 16, 16), (128, 64, 8, 8), (64, 64, 4, 12),
                                       (128, 128, 8, 16), (64, 128, 12, 8), (128, 128, 32, 64),
                                       (16, 16, 4, 4), (128, 64, 8, 32),
                                       # the wide Cholesky-QR path, 32 < R + W <= 64
                                       (128, 128, 32, 32), (128, 128, 16, 32), (128, 128, 3, 30),
                                       (128, 128, 21, 12), (64, 128, 20, 20), (64, 64, 16, 24),
                                       (128, 64, 32, 17)])
def test_compress_matches_truncated_svd(form, dk, dv, R, W):
    _run(form, dk, dv, R, W, seed=dk + R + W + form)


@pytest.mark.parametrize("R,W", [(16, 16), (8, 32), (32, 32)], ids=["fast", "wide-40", "wide-64"])
def test_repeated_key_takes_the_householder_path(R, W):
    diag = _run(FORM_GDN, 128, 128, R, W, repeat=True, n=8, seed=7)
    assert diag["cholqr_declined"] == 8 and diag["householder_units"] == 8


@pytest.mark.parametrize("form,dk,dv,R,W", [(FORM_GDN, 128, 128, 16, 16), (FORM_MAMBA2, 128, 64, 8, 32),
                                            (FORM_KDA, 128, 128, 32, 32), (FORM_GDN, 128, 128, 16, 48)])
def test_well_conditioned_units_take_the_cholesky_qr_path(form, dk, dv, R, W):
    diag = _run(form, dk, dv, R, W, n=16, seed=11)
    assert diag["cholqr_units"] == 16 and diag["householder_units"] == 0, diag


@pytest.mark.parametrize("R,W", [(16, 16), (8, 32), (32, 32)], ids=["fast", "wide-40", "wide-64"])
def test_zero_columns_are_dropped_exactly(R, W):
    _run(FORM_GDN, 128, 128, R, W, zero_cols=5, n=8, seed=9)
    _run(FORM_KDA, 128, 128, R, W, zero_cols=min(16, R), n=8, seed=10)


def _graded_state(form, n, dk, dv, R, W, rng, lazy):
    """Columns whose magnitudes span 1 .. 1e-30, as a long-decayed window leaves them:
    either explicit in the stored U (scale 1) or carried by the lazy decay scales."""
    m = R + W
    mags = 10.0 ** (-rng.uniform(0, 30, size=(n, m)))
    mags[:, -4:] = rng.uniform(0.5, 1.0, size=(n, 4))          # the newest columns
    U = rng.normal(size=(n, dk, m))
    U /= np.linalg.norm(U, axis=1, keepdims=True)
    V = rng.normal(size=(n, dv, m)) * rng.uniform(0.2, 3, size=(n, 1, m))
    slen = (m + 3) // 4 * 4
    scale = np.ones((n, slen))
    if lazy:
        scale[:, :m] = mags
    else:
        U = U * mags[:, None, :]
    Utrue = U * scale[:, None, :m]
    return U.astype(np.float32), V.astype(np.float32), scale.astype(np.float32), Utrue


@pytest.mark.parametrize("lazy", [False, True])
@pytest.mark.parametrize("dk,dv,R,W", [(128, 128, 16, 16), (128, 64, 8, 32), (128, 128, 32, 32)])
def test_graded_spectrum_with_long_decayed_columns(lazy, dk, dv, R, W):
    import torch
    from rank_recurrent_state_b200 import seed as S
    rng = np.random.default_rng(21 + R + W + int(lazy))
    n, m = 12, R + W
    U, V, scale, Utrue = _graded_state(FORM_GDN, n, dk, dv, R, W, rng, lazy)
    d = S.Dims(FORM_GDN, n, 1, 1, dk, dv, R, W)
    st = S.State.allocate(d, torch.ones(1, 1, dv, device="cuda"))
    st.U.copy_(torch.from_numpy(np.ascontiguousarray(np.swapaxes(U, 1, 2))).view_as(st.U))
    st.V.copy_(torch.from_numpy(np.ascontiguousarray(np.swapaxes(V, 1, 2))).view_as(st.V))
    st.scale.copy_(torch.from_numpy(scale).view_as(st.scale))
    st.a.zero_()
    st.ncols.fill_(m)
    ws = S.Workspace(d)
    S.seed_compress(d, st, S.SEED_ALL_LAYERS, ws)
    dense = torch.empty(n, dk, dv, device="cuda")
    S.seed_state_to_dense(d, st, S.SEED_ALL_LAYERS, dense, ws)
    assert S.seed_get_status(ws) == 0
    Up, Vp, _ = ocomp.truncate_product(Utrue.astype(np.float64), V.astype(np.float64), R)
    ref = np.einsum("nir,njr->nij", Up, Vp)
    got = dense.cpu().numpy()
    for u in range(n):
        assert rel_fro(got[u], ref[u]) <= TOL, (u, rel_fro(got[u], ref[u]))
