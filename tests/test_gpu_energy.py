"""seed_state_energy against the oracle's energies.

States are built on the host (stored columns with lazy scales, KDA row products,
column counts below capacity) and uploaded, so nothing the device computes reaches
the oracle; a state produced by the device pipeline is checked through the state
the device returns (seed_state_to_dense) against the energy of that dense matrix.
"""

import numpy as np
import pytest

from oracle import diagnostics
from workloads import FORM_GDN, FORM_KDA, FORM_MAMBA2, configs

from parity_util import TOL, ensure_lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _host_state(form, n, dk, dv, R, W, c, rng):
    m = R + W
    U = rng.normal(size=(n, m, dk)).astype(np.float32)
    V = (rng.normal(size=(n, m, dv)) * rng.uniform(0.2, 3, size=(n, m, 1))).astype(np.float32)
    U[:, c:] = 7.0   # beyond the column count: must be ignored
    V[:, c:] = 7.0
    a = rng.normal(size=(n, dk)).astype(np.float32)
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


@pytest.mark.parametrize("form", [FORM_GDN, FORM_KDA, FORM_MAMBA2])
@pytest.mark.parametrize("dk,dv,R,W,c", [(128, 128, 16, 16, 23), (128, 64, 8, 32, 40), (64, 64, 4, 12, 4),
                                         (128, 128, 32, 64, 95), (16, 16, 4, 4, 0)])
def test_energies_match_the_oracle(form, dk, dv, R, W, c):
    import torch
    from rank_recurrent_state_b200 import seed as S
    rng = np.random.default_rng(dk + dv + R + W + c + form)
    n = 12
    U, V, a, scale, Ut, Vt = _host_state(form, n, dk, dv, R, W, c, rng)
    vbar = rng.normal(size=(1, 1, dv)).astype(np.float32)
    d = S.Dims(form, n, 1, 1, dk, dv, R, W)
    st = S.State.allocate(d, torch.from_numpy(vbar).cuda())
    st.U.copy_(torch.from_numpy(U).view_as(st.U))
    st.V.copy_(torch.from_numpy(V).view_as(st.V))
    st.scale.copy_(torch.from_numpy(scale).view_as(st.scale))
    st.a.copy_(torch.from_numpy(a).view_as(st.a))
    st.ncols.fill_(c)
    ws = S.Workspace(d)
    out = torch.full((n, 4), float("nan"), device="cuda")
    S.seed_state_energy(d, st, S.SEED_ALL_LAYERS, out, ws)
    assert S.seed_get_status(ws) == 0
    ref = diagnostics.energies(a, Ut, Vt, np.repeat(vbar[0], n, axis=0))
    got = out.cpu().numpy().astype(np.float64)
    scale_e = ref[:, 3:4]   # every part relative to the state's energy
    assert np.max(np.abs(got - ref) / scale_e) <= TOL, np.max(np.abs(got - ref) / scale_e)
    # a unit list picks rows in its order
    units = torch.tensor([5, 0, 11], dtype=torch.int32, device="cuda")
    out2 = torch.full((3, 4), float("nan"), device="cuda")
    S.seed_state_energy(d, st, S.SEED_ALL_LAYERS, out2, ws, units=units)
    np.testing.assert_array_equal(out2.cpu().numpy(), out.cpu().numpy()[[5, 0, 11]])


def test_pipeline_state_energy_and_sink_share():
    """After a conversion and a few decode steps of the GDN layer workload the sink
    holds most of the energy (the workload's values sit at 3 vbar + noise) and the
    energies equal those of the dense state the device reconstructs."""
    import torch
    from rank_recurrent_state_b200 import seed as S
    from rank_recurrent_state_b200.pipeline import DeviceRun
    cfg = configs.config(1, batch=4)
    run = DeviceRun(cfg, n_prefill=256)
    run.prefill_and_convert()
    buf = S.alloc_step_inputs(run.dims)
    for _ in range(5):
        run.step(buf)
    d = run.dims
    out = torch.empty(d.units, 4, device="cuda")
    S.seed_state_energy(d, run.state, S.SEED_ALL_LAYERS, out, run.ws)
    dense = run.to_dense().double()
    total = (dense ** 2).sum(dim=(1, 2)).cpu().numpy()
    e = out.double().cpu().numpy()
    assert run.status() == 0
    np.testing.assert_allclose(e[:, 3], total, rtol=TOL)
    assert np.all(np.abs(e[:, 2]) <= 1e-3 * e[:, 3])          # V^T vbar = 0 kept by the updates
    share = diagnostics.sink_share(e)
    assert np.median(share) > 0.5
