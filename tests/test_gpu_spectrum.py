"""seed_state_spectrum against the oracle's spectra, top output direction and ranks.

States are built on the host (stored columns with lazy scales, KDA row products,
column counts below capacity) and uploaded, so nothing the device computes reaches
the oracle; a state produced by the device pipeline is checked through the dense
state the device returns (seed_state_to_dense), by a float64 SVD of that matrix.
"""

import numpy as np
import pytest

from oracle import diagnostics
from workloads import FORM_GDN, FORM_KDA, FORM_MAMBA2, configs

from parity_util import TOL, ensure_lib, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _host_state(form, n, dk, dv, R, W, c, rng, sink=3.0):
    m = R + W
    U = rng.normal(size=(n, m, dk)).astype(np.float32)
    # content columns with a graded spectrum, as a decayed window leaves them
    V = (rng.normal(size=(n, m, dv)) * (0.8 ** np.arange(m))[None, :, None]).astype(np.float32)
    U[:, c:] = 7.0   # beyond the column count: must be ignored
    V[:, c:] = 7.0
    a = (sink * rng.normal(size=(n, dk))).astype(np.float32)
    if form == FORM_KDA:
        scale = rng.uniform(0.3, 1.0, size=(n, dk)).astype(np.float32)
        Ut = scale[:, :, None].astype(np.float64) * np.swapaxes(U, 1, 2)[:, :, :c]
    else:
        slen = (m + 3) // 4 * 4
        scale = np.ones((n, slen), dtype=np.float32)
        scale[:, :m] = rng.uniform(0.05, 2.0, size=(n, m)).astype(np.float32)
        Ut = np.swapaxes(U, 1, 2)[:, :, :c].astype(np.float64) * scale[:, None, :c]
    Vt = np.swapaxes(V, 1, 2)[:, :, :c].astype(np.float64)
    return U, V, a, scale, Ut, Vt


def _upload(form, n, dk, dv, R, W, c, U, V, a, scale, vbar):
    import torch
    from rank_recurrent_state_b200 import seed as S
    d = S.Dims(form, n, 1, 1, dk, dv, R, W)
    st = S.State.allocate(d, torch.from_numpy(vbar).cuda())
    st.U.copy_(torch.from_numpy(U).view_as(st.U))
    st.V.copy_(torch.from_numpy(V).view_as(st.V))
    st.scale.copy_(torch.from_numpy(scale).view_as(st.scale))
    st.a.copy_(torch.from_numpy(a).view_as(st.a))
    st.ncols.fill_(c)
    return d, st, S.Workspace(d)


def _spectrum(d, st, ws, units=None):
    import torch
    from rank_recurrent_state_b200 import seed as S
    n = d.units if units is None else int(units.numel())
    sS = torch.full((n, d.m + 1), float("nan"), device="cuda")
    sC = torch.full((n, d.m + 1), float("nan"), device="cuda")
    cs = torch.full((n,), float("nan"), device="cuda")
    rk = torch.full((n, 2), -1, dtype=torch.int32, device="cuda")
    S.seed_state_spectrum(d, st, S.SEED_ALL_LAYERS, sS, sC, cs, rk, ws, units=units)
    return sS.cpu().numpy(), sC.cpu().numpy(), cs.cpu().numpy(), rk.cpu().numpy(), S.seed_get_status(ws)


def _rank_valid(k, sigma_ref, frac, slack=1e-5):
    """k is a correct energy rank of sigma_ref (float64) up to a threshold within slack:
    the k largest hold at least (frac - slack) of the energy, the k - 1 largest less than
    (frac + slack)."""
    s2 = np.sort(sigma_ref ** 2)[::-1]
    tot = s2.sum()
    if tot == 0:
        return k == 0
    cum = np.cumsum(s2)
    return k >= 1 and cum[k - 1] >= (frac - slack) * tot and (k == 1 or cum[k - 2] < (frac + slack) * tot)


@pytest.mark.parametrize("form", [FORM_GDN, FORM_KDA, FORM_MAMBA2])
@pytest.mark.parametrize("dk,dv,R,W,c", [(128, 128, 16, 16, 23), (128, 64, 8, 32, 40), (64, 128, 4, 12, 13),
                                         (64, 64, 4, 12, 4), (128, 128, 32, 64, 95), (16, 16, 4, 4, 0)])
def test_spectra_match_the_oracle(form, dk, dv, R, W, c):
    rng = np.random.default_rng(3 * dk + dv + R + W + c + form)
    n = 12
    U, V, a, scale, Ut, Vt = _host_state(form, n, dk, dv, R, W, c, rng)
    vbar = rng.normal(size=(1, 1, dv)).astype(np.float32)
    d, st, ws = _upload(form, n, dk, dv, R, W, c, U, V, a, scale, vbar)
    sS, sC, cs, rk, flags = _spectrum(d, st, ws)
    assert flags == 0, hex(flags)
    vb = np.repeat(vbar[0], n, axis=0).astype(np.float64)
    refS, refC = diagnostics.spectra(a, Ut, Vt, vb)
    cos_ref, gap = diagnostics.top_output_cosine(a, Ut, Vt, vb)
    k = d.m + 1
    for u in range(n):
        # the spectra up to rank R + W + 1 (the rest is zero): relative to the head's top
        # singular value, as the pages plot them
        assert np.max(np.abs(sS[u] - refS[u, :k])) <= TOL * refS[u, 0], (u, sS[u][:4], refS[u, :4])
        assert np.max(np.abs(sC[u] - refC[u, :k])) <= TOL * refS[u, 0], (u, sC[u][:4], refC[u, :4])
        if c:
            assert rel_fro(sC[u], refC[u, :k]) <= TOL
        # v* is defined to about rounding / gap
        if gap[u] > 1e-2:
            assert abs(cs[u] - cos_ref[u]) <= TOL, (u, cs[u], cos_ref[u], gap[u])
        assert _rank_valid(rk[u, 0], refC[u], 0.9) and _rank_valid(rk[u, 1], refC[u], 0.99), (u, rk[u])
    assert np.mean(gap > 1e-2) > 0.5
    # a unit list picks rows in its order
    import torch
    units = torch.tensor([5, 0, 11], dtype=torch.int32, device="cuda")
    sS2, sC2, cs2, rk2, _ = _spectrum(d, st, ws, units=units)
    np.testing.assert_array_equal(sS2, sS[[5, 0, 11]])
    np.testing.assert_array_equal(rk2, rk[[5, 0, 11]])


def test_pure_sink_has_one_direction_along_vbar():
    """c = 0: S = a vbar^T has the single singular value ||a|| ||vbar||, its top output
    direction is vbar itself, and the content is zero (ranks 0)."""
    rng = np.random.default_rng(17)
    n, dk, dv, R, W = 8, 128, 128, 16, 16
    U, V, a, scale, _, _ = _host_state(FORM_GDN, n, dk, dv, R, W, 0, rng)
    vbar = rng.normal(size=(1, 1, dv)).astype(np.float32)
    d, st, ws = _upload(FORM_GDN, n, dk, dv, R, W, 0, U, V, a, scale, vbar)
    sS, sC, cs, rk, flags = _spectrum(d, st, ws)
    assert flags == 0
    top = np.linalg.norm(a.astype(np.float64), axis=1) * np.linalg.norm(vbar.astype(np.float64))
    np.testing.assert_allclose(sS[:, 0], top, rtol=TOL)
    assert np.all(sS[:, 1:] <= TOL * top[:, None]) and np.all(sC == 0)
    np.testing.assert_allclose(cs, 1.0, atol=TOL)
    assert np.all(rk == 0)


def test_pipeline_states_spectra_and_sink_direction():
    """After a conversion and a few decode steps of the GDN layer workload: the spectra
    are those of the dense states the device reconstructs, and, the values sitting at
    3 vbar + noise, the top output direction lies along vbar and the content needs few
    directions."""
    import torch
    from rank_recurrent_state_b200 import seed as S
    from rank_recurrent_state_b200.pipeline import DeviceRun
    cfg = configs.config(1, batch=2)
    run = DeviceRun(cfg, n_prefill=256)
    run.prefill_and_convert()
    buf = S.alloc_step_inputs(run.dims)
    for _ in range(5):
        run.step(buf)
    d = run.dims
    sS, sC, cs, rk, flags = _spectrum(d, run.state, run.ws)
    assert flags == 0, hex(flags)
    dense = run.to_dense().double().cpu().numpy()
    ref = np.linalg.svd(dense, compute_uv=False)
    for u in range(d.units):
        assert np.max(np.abs(sS[u] - ref[u, :d.m + 1])) <= TOL * ref[u, 0]
    assert np.median(cs) > 0.9
    assert np.all(rk[:, 0] <= rk[:, 1]) and np.all(rk[:, 1] <= d.R + 5)
