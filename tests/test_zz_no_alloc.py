"""seed_decode_step_noalloc against seed_decode_step.

Both run the same decode kernel; the no-allocation entry point only keeps its
status word in the library's own fixed device array instead of a caller
workspace.  So on identical states and inputs the outputs and the updated states
must agree bit for bit, on two calls in a row, and the flags a call raises must
reach status_out and not leak into the next call.  The file is named to be
collected last; it depends on nothing the other tests leave behind.
"""

import pytest

from workloads import configs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from parity_util import ensure_lib
    ensure_lib()


def _twin_runs(cid, batch, factors=0):
    """Two device runs on one seeded workload: prefill + conversion, then the second
    run's state is made a bit-identical copy of the first's."""
    from rank_recurrent_state_b200.pipeline import DeviceRun
    cfg = configs.config(cid)
    a = DeviceRun(cfg, batch=batch, n_prefill=24, factors=factors)
    a.prefill_and_convert()
    b = DeviceRun(cfg, batch=batch, n_prefill=24, factors=factors)
    b.prefill_and_convert()
    b.state.load_state_dict(a.state.state_dict())
    return a, b


def _assert_same_state(sa, sb):
    import torch
    for name in ("a", "U", "V", "scale", "ncols"):
        assert torch.equal(getattr(sa, name), getattr(sb, name)), name


@pytest.mark.parametrize("cid,factors", [(0, 0), (2, 0), (3, 0), (4, 0), (2, 1), (4, 2)])
def test_two_calls_in_a_row_match_the_workspace_entry_point(cid, factors):
    import torch
    from rank_recurrent_state_b200 import seed as S
    a, b = _twin_runs(cid, batch=4, factors=factors)
    d = a.dims
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for t in range(2):
        for layer in range(d.layers):
            buf = S.alloc_step_inputs(d)
            a.gen_inputs(t, layer, buf)
            o_ref = torch.full_like(buf["o"], float("nan"))
            o_new = torch.full_like(buf["o"], float("nan"))
            S.seed_decode_step(d, a.state, layer, buf["q"], buf["k"], buf["v"], buf["alpha"],
                               buf["beta"], o_ref, a.ws)
            S.seed_decode_step_noalloc(d, b.state, layer, buf["q"], buf["k"], buf["v"], buf["alpha"],
                                       buf["beta"], o_new, status_out=status)
            torch.cuda.synchronize()
            assert torch.equal(o_ref, o_new), (t, layer)
            assert int(status.item()) == 0
        _assert_same_state(a.state, b.state)
    assert a.status() == 0


def test_flags_reach_status_out_and_are_cleared_between_calls():
    import torch
    from rank_recurrent_state_b200 import seed as S
    a, b = _twin_runs(2, batch=2)
    d = a.dims
    buf = S.alloc_step_inputs(d)
    a.gen_inputs(0, 0, buf)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    full = S.State.allocate(d, b.vbar)
    full.load_state_dict(b.state.state_dict())
    full.ncols.fill_(d.m)                                  # every unit already holds R+W columns
    o = torch.empty_like(buf["o"])
    S.seed_decode_step_noalloc(d, full, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                               o, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == S.FLAG_FULL
    # the same call through a caller workspace raises the same flag
    S.seed_decode_step(d, full, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"], o, a.ws)
    assert a.status() == S.FLAG_FULL
    # the next call starts from a clear status word, with or without status_out
    S.seed_decode_step_noalloc(d, full, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"], o)
    S.seed_decode_step_noalloc(d, b.state, 0, buf["q"], buf["k"], buf["v"], buf["alpha"],
                               buf["beta"], o, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_rejected_arguments_enqueue_nothing():
    import torch
    from rank_recurrent_state_b200 import seed as S
    _, b = _twin_runs(0, batch=2)
    d = b.dims
    buf = S.alloc_step_inputs(d)
    b.gen_inputs(0, 0, buf)
    before = b.state.state_dict()
    before = {k: v.clone() for k, v in before.items()}
    status = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    with pytest.raises(S.SeedError):                       # layer out of range
        S.seed_decode_step_noalloc(d, b.state, d.layers, buf["q"], buf["k"], buf["v"], buf["alpha"],
                                   buf["beta"], buf["o"], status_out=status)
    with pytest.raises(S.SeedError):                       # status_out not 4-byte aligned
        S.seed_decode_step_noalloc(d, b.state, 0, buf["q"], buf["k"], buf["v"], buf["alpha"],
                                   buf["beta"], buf["o"],
                                   status_out=status.view(torch.uint8)[1:2])
    torch.cuda.synchronize()
    assert status.tolist() == [7, 7]
    _assert_same_state(b.state, S.State(**before, vbar=b.vbar))
    assert S.seed_noalloc_workspace_bytes() >= S.seed_workspace_bytes(d)
