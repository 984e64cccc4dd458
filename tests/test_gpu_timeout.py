"""The bounded copy waits run out, on purpose, without a fault.

seed_debug_wait_fault makes every warp of the decode kernel (and every block of
the Cholesky-QR compression) withhold its first bulk copy and give up on it at
once.  Nothing is in flight when the wait fails, the second (draining) wait is
bounded too (1 s), and the kernel returns.  The tests check that the timeout is
reported in the status word, that the state is left as the documented behaviour
says, and that the same workspace and GPU run a clean step afterwards.
"""

import numpy as np
import pytest

from workloads import config

from parity_util import ensure_lib, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _run(cid=1, batch=2, n_prefill=64, factors=0):
    from rank_recurrent_state_b200.pipeline import DeviceRun
    run = DeviceRun(config(cid, batch=batch), n_prefill=n_prefill, factors=factors)
    run.prefill_and_convert()
    return run


# float32 factors: the ring kernel; 16-bit: the whole-unit stage kernel
@pytest.mark.parametrize("factors", [0, 1], ids=["f32-ring", "f16-whole-unit"])
def test_decode_wait_runs_out_and_leaves_the_state_unchanged(factors):
    import torch
    from rank_recurrent_state_b200 import seed as S
    run, twin = _run(factors=factors), _run(factors=factors)
    d = run.dims
    buf = S.alloc_step_inputs(d)
    run.gen_inputs(0, 0, buf)
    buf["o"].fill_(7.0)
    before = {k: v.clone() for k, v in run.state.state_dict().items()}
    S.seed_debug_wait_fault(run.ws, True)
    S.seed_decode_step(d, run.state, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                       buf["o"], run.ws)
    flags = run.status()
    assert flags & S.FLAG_TIMEOUT, hex(flags)
    assert flags & ~S.FLAG_TIMEOUT == 0, hex(flags)
    for k, v in run.state.state_dict().items():   # every warp failed on its first unit
        assert torch.equal(v, before[k]), k
    assert torch.all(buf["o"] == 7.0)
    # the same workspace, fault off: a clean step, bit-identical to a run that never faulted
    S.seed_debug_wait_fault(run.ws, False)
    S.seed_decode_step(d, run.state, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                       buf["o"], run.ws)
    o_run = buf["o"].clone()
    assert run.status() == 0
    S.seed_decode_step(d, twin.state, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                       buf["o"], twin.ws)
    assert twin.status() == 0
    assert torch.equal(o_run, buf["o"])
    for k, v in run.state.state_dict().items():
        assert torch.equal(v, getattr(twin.state, k)), k


def test_compress_wait_runs_out_and_the_householder_path_takes_over():
    import torch
    from rank_recurrent_state_b200 import seed as S
    run = _run()
    d = run.dims
    buf = S.alloc_step_inputs(d)
    for t in range(d.W):   # W steps without the compression: every unit at R + W columns
        for l in range(d.layers):
            run.gen_inputs(t, l, buf)
            S.seed_decode_step(d, run.state, l, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                               buf["o"], run.ws)
    assert run.status() == 0
    assert torch.all(run.state.ncols == d.m)
    saved = {k: v.clone() for k, v in run.state.state_dict().items()}
    S_pre = run.to_dense().cpu().numpy()
    sig_f = torch.zeros(d.units, d.R, device="cuda")
    sig_c = torch.zeros(d.units, d.R, device="cuda")
    S.seed_get_diagnostics(run.ws)   # clear the counters
    S.seed_debug_wait_fault(run.ws, True)
    S.seed_compress(d, run.state, S.SEED_ALL_LAYERS, run.ws, sigma_out=sig_f)
    flags = run.status()
    diag = S.seed_get_diagnostics(run.ws)
    S.seed_debug_wait_fault(run.ws, False)
    assert flags & S.FLAG_TIMEOUT, hex(flags)
    assert flags & ~S.FLAG_TIMEOUT == 0, hex(flags)
    assert diag["cholqr_units"] == 0 and diag["householder_units"] == d.units, diag
    assert torch.all(run.state.ncols == d.R)
    S_faulted = run.to_dense().cpu().numpy()
    # the same state compressed with the fault off (Cholesky QR): the same truncation
    run.state.load_state_dict(saved)
    S.seed_compress(d, run.state, S.SEED_ALL_LAYERS, run.ws, sigma_out=sig_c)
    assert run.status() == 0
    assert S.seed_get_diagnostics(run.ws)["cholqr_units"] == d.units
    S_clean = run.to_dense().cpu().numpy()
    sf, sc = sig_f.cpu().numpy(), sig_c.cpu().numpy()
    for u in range(d.units):
        # what is unique: the kept singular values and the truncation error (both
        # results are best rank-R truncations of the same state)
        assert rel_fro(sf[u], sc[u]) <= 1e-4
        nrm = np.linalg.norm(S_pre[u])
        dist_f = np.linalg.norm(S_faulted[u] - S_pre[u])
        dist_c = np.linalg.norm(S_clean[u] - S_pre[u])
        assert abs(dist_f - dist_c) <= 1e-4 * nrm, (u, dist_f, dist_c, nrm)
    # and, apart from near-ties at the truncation, the same state
    errs = np.array([rel_fro(S_faulted[u], S_clean[u]) for u in range(d.units)])
    assert np.mean(errs <= 1e-4) >= 0.75, np.sort(errs)[-10:]
