"""Device path against the fp64 oracle, through the C ABI, on seeded synthetic inputs.

Tolerance: relative Frobenius error <= 1e-4 for states, outputs o and singular
values (fp32 device vs fp64 oracle); bookkeeping (column counts, compression
steps) bit-exact; generator outputs equal to the host generator's.
"""

import numpy as np
import pytest

from workloads import FORM_KDA, config, philox

from parity_util import TOL, compare, ensure_lib, record_set, rel_fro, run_device, run_oracle
from workloads import KDA_SWEEP_R, KDA_SWEEP_W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _torch():
    import torch
    return torch


# --------------------------------------------------------------- generator

@pytest.mark.parametrize("cid", [0, 1, 2, 3, 4])
def test_device_generator_matches_host_generator(cid):
    torch = _torch()
    from rank_recurrent_state_b200 import seed as S
    cfg = config(cid, batch=3)
    d = S.Dims.from_config(cfg)
    key = S.synth_key(cfg)
    vb = torch.empty(d.layers, d.heads, d.d_v, device="cuda")
    S.seed_synth_vbar(d, key, vb)
    host_vb = philox.vbar_table(cfg)
    assert np.mean(vb.cpu().numpy() == host_vb) > 0.999
    np.testing.assert_allclose(vb.cpu().numpy(), host_vb, rtol=3e-7, atol=1e-9)
    buf = S.alloc_step_inputs(d)
    for layer in sorted({0, d.layers - 1}):
        for t in (0, 7):
            S.seed_synth_token_inputs(d, key, S.SEED_PHASE_DECODE, t, layer, vb, buf["q"], buf["k"],
                                      buf["v"], buf["alpha"], buf["beta"])
            b = np.arange(d.batch)[:, None]
            h = np.arange(d.heads)[None, :]
            host = philox.token_inputs(cfg, b, layer, h, t, philox.PHASE_DECODE)
            for name in ("q", "k", "v", "alpha", "beta"):
                dev = buf[name].cpu().numpy()
                assert dev.shape == host[name].shape, name
                assert np.mean(dev == host[name]) > 0.999, name
                np.testing.assert_allclose(dev, host[name], rtol=3e-7, atol=1e-9, err_msg=name)


# --------------------------------------------------------------- prefill and conversion

@pytest.mark.parametrize("cid,batch,T", [(0, 1, 64), (1, 1, 200), (3, 1, 150), (4, 1, 120)])
def test_dense_prefill_matches_oracle(cid, batch, T):
    torch = _torch()
    from rank_recurrent_state_b200 import seed as S
    from oracle import recurrences
    cfg = config(cid, batch=batch)
    d = S.Dims.from_config(cfg)
    key = S.synth_key(cfg)
    vb = torch.empty(d.layers, d.heads, d.d_v, device="cuda")
    S.seed_synth_vbar(d, key, vb)
    Sd = torch.empty(d.units, d.d_k, d.d_v, device="cuda")
    S.seed_synth_dense_prefill(d, key, T, S.SEED_ALL_LAYERS, vb, Sd)
    rng = np.random.default_rng(cid)
    sample = rng.choice(d.units, size=min(12, d.units), replace=False)
    b, rem = np.divmod(sample, d.layers * d.heads)
    l, h = np.divmod(rem, d.heads)
    ref = recurrences.dense_prefill(cfg, b, l, h, T)
    dev = Sd.cpu().numpy()[sample]
    for u in range(sample.size):
        assert rel_fro(dev[u], ref[u]) <= TOL


# --------------------------------------------------------------- whole decode path

def _parity(cfg, sample, n_prefill, n_decode, batch=None, label=None):
    c = cfg if batch is None else cfg.replace(batch=batch)
    su = np.asarray(sample, dtype=np.int64)
    b, rem = np.divmod(su, c.layers * c.heads)
    l, h = np.divmod(rem, c.heads)
    ref = run_oracle(cfg, {"b": b, "l": l, "h": h}, n_prefill, n_decode)
    dev = run_device(cfg, sample, n_prefill, n_decode, batch=batch, record_units=record_set(cfg, ref))
    assert dev["flags"] == 0, hex(dev["flags"])
    return compare(cfg, dev, ref, label=label)


def test_tiny_gdn_workload_full():
    """Tiny GDN workload in full: 2 heads, 16x16, R=W=4, 64-token prefill, 32 steps."""
    cfg = config(0)
    out = _parity(cfg, [0, 1], cfg.n_prefill, cfg.n_decode)
    assert out["ties"] == 0


def test_gdn_layer_reduced():
    """One 48-head 128x128 GDN layer, R=W=16; 2 requests, 3 compressions."""
    cfg = config(1)
    _parity(cfg, np.arange(96), 256, 3 * cfg.W + 5, batch=2)


def test_mamba2_reduced():
    """Mamba-2 128x64, R=8, W=32 (all 40 layers x 64 heads of one request; 48 sampled)."""
    cfg = config(3)
    rng = np.random.default_rng(3)
    sample = np.sort(rng.choice(cfg.layers * cfg.heads, 48, replace=False))
    _parity(cfg, sample, 200, 2 * cfg.W + 3, batch=1)


@pytest.mark.parametrize("R,W", [(r, w) for r in KDA_SWEEP_R for w in KDA_SWEEP_W])
def test_kda_sweep_reduced(R, W):
    """KDA 128x128 with per-channel decay over the whole R x W sweep, R in {8, 16, 32},
    W in {8, 16, 32, 64} (one request, 24 sampled heads, two compressions)."""
    cfg = config(4, R=R, W=W)
    rng = np.random.default_rng(R * 100 + W)
    sample = np.sort(rng.choice(cfg.layers * cfg.heads, 24, replace=False))
    _parity(cfg, sample, 150, 2 * W + 2, batch=1, label=f"kda R{R} W{W} reduced")


@pytest.mark.parametrize("cid,over,batch", [(3, {}, 64), (4, {"R": 8, "W": 8}, 64), (0, {}, 2048),
                                             (1, {"R": 4, "W": 4}, 64)],
                         ids=["mamba2-b64", "kda-R8-W8-b64", "tiny-b2048", "gdn-R4-W4-b64"])
def test_several_units_per_warp(cid, over, batch):
    """Batches large enough that every warp of the persistent decode grid steps several
    units in turn, at column counts of one or two chunks per factor, so that the ring
    of each warp streams one unit's chunks while it still holds the previous one's
    (sampled units, two compressions)."""
    cfg = config(cid, **over)
    c = cfg.replace(batch=batch)
    rng = np.random.default_rng(cid * 7 + batch)
    n = c.units
    sample = np.unique(np.concatenate([rng.choice(n, 40, replace=False), np.arange(n - 8, n)]))
    _parity(cfg, sample, 64, 2 * cfg.W + 3, batch=batch, label=f"cfg{cid} batch {batch} (several units per warp)")


def test_odd_window_and_empty_prefill():
    """R + W odd (the core SVD pads a zero column) and a zero prefill state (rank 0)."""
    cfg = config(0, R=3, W=4)
    _parity(cfg, [0, 1], 0, 17)
    _parity(cfg, [0, 1], 40, 17)


# --------------------------------------------------------------- dense comparison kernel

@pytest.mark.parametrize("cid", [0, 1, 3, 4])
def test_dense_step_matches_oracle(cid):
    torch = _torch()
    from rank_recurrent_state_b200 import seed as S
    from oracle import recurrences
    cfg = config(cid, batch=1)
    d = S.Dims.from_config(cfg)
    key = S.synth_key(cfg)
    vb = torch.empty(d.layers, d.heads, d.d_v, device="cuda")
    S.seed_synth_vbar(d, key, vb)
    Sd = torch.empty(d.units, d.d_k, d.d_v, device="cuda")
    T, steps = 50, 6
    S.seed_synth_dense_prefill(d, key, T, S.SEED_ALL_LAYERS, vb, Sd)
    ws = S.Workspace(d)
    buf = S.alloc_step_inputs(d)
    layer = d.layers - 1
    sample = np.arange(d.heads)[: min(8, d.heads)]
    os_dev = []
    for t in range(steps):
        S.seed_synth_token_inputs(d, key, S.SEED_PHASE_DECODE, t, layer, vb, buf["q"], buf["k"],
                                  buf["v"], buf["alpha"], buf["beta"])
        S.seed_dense_step(d, Sd, layer, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                          buf["o"], ws)
        os_dev.append(buf["o"][0, sample].cpu().numpy())
    assert S.seed_get_status(ws) == 0
    b = np.zeros(sample.size, dtype=np.int64)
    l = np.full(sample.size, layer)
    St = recurrences.dense_prefill(cfg, b, l, sample, T)
    os_ref = []
    for t in range(steps):
        inp = recurrences.f64(philox.token_inputs(cfg, b, l, sample, t, philox.PHASE_DECODE))
        St = recurrences.dense_step(cfg.form, St, inp["k"], inp["v"], inp["alpha"], inp["beta"])
        os_ref.append(recurrences.readout(St, inp["q"]))
    units = layer * d.heads + sample
    dev_S = Sd.cpu().numpy()[units]
    for u in range(sample.size):
        assert rel_fro(dev_S[u], St[u]) <= TOL
        assert rel_fro(np.array(os_dev)[:, u], np.array(os_ref)[:, u]) <= TOL


# --------------------------------------------------------------- status flags and edge cases

def _small_run(cid=0, **kw):
    from rank_recurrent_state_b200.pipeline import DeviceRun
    run = DeviceRun(config(cid, **kw), n_prefill=16)
    run.prefill_and_convert()
    return run


def test_full_unit_is_skipped_and_flagged():
    torch = _torch()
    from rank_recurrent_state_b200 import seed as S
    run = _small_run()
    d = run.dims
    run.state.ncols.fill_(d.m)
    before = {k: v.clone() for k, v in run.state.state_dict().items()}
    buf = S.alloc_step_inputs(d)
    run.gen_inputs(0, 0, buf)
    S.seed_decode_step(d, run.state, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                       buf["o"], run.ws)
    assert run.status() & S.FLAG_FULL
    for k, v in run.state.state_dict().items():
        assert torch.equal(v, before[k]), k
    assert run.status() == 0   # reading clears the word


def test_nonfinite_input_is_flagged():
    from rank_recurrent_state_b200 import seed as S
    run = _small_run()
    d = run.dims
    buf = S.alloc_step_inputs(d)
    run.gen_inputs(0, 0, buf)
    buf["v"][0, 0, 3] = float("nan")
    S.seed_decode_step(d, run.state, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                       buf["o"], run.ws)
    assert run.status() & S.FLAG_NONFINITE


def test_zero_vbar_is_flagged_and_unit_left_unchanged():
    torch = _torch()
    from rank_recurrent_state_b200 import seed as S
    run = _small_run()
    d = run.dims
    run.vbar[0, 1].zero_()
    before = run.state.a.clone()
    buf = S.alloc_step_inputs(d)
    run.gen_inputs(0, 0, buf)
    S.seed_decode_step(d, run.state, 0, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"],
                       buf["o"], run.ws)
    assert run.status() & S.FLAG_ZERO_VBAR
    assert torch.equal(run.state.a[0, 0, 1], before[0, 0, 1])
    assert not torch.equal(run.state.a[0, 0, 0], before[0, 0, 0])


def test_compress_leaves_units_that_are_not_due():
    torch = _torch()
    from rank_recurrent_state_b200 import seed as S
    run = _small_run()
    before = {k: v.clone() for k, v in run.state.state_dict().items()}
    S.seed_compress(run.dims, run.state, S.SEED_ALL_LAYERS, run.ws)
    assert run.status() == 0
    for k, v in run.state.state_dict().items():
        assert torch.equal(v, before[k]), k


def test_to_dense_unit_list_matches_full_scope():
    torch = _torch()
    run = _small_run(1, batch=1)
    full = run.to_dense()
    idx = torch.tensor([5, 0, 47], dtype=torch.int32, device="cuda")
    part = run.to_dense(idx)
    assert torch.equal(part, full[idx.long()])


def test_checkpoint_resume_is_bit_identical():
    """Run t steps, save the state, reload into a fresh state, continue: bit-identical."""
    torch = _torch()
    import io
    from rank_recurrent_state_b200 import seed as S
    from rank_recurrent_state_b200.pipeline import DeviceRun
    cfg = config(1, batch=1)
    a = DeviceRun(cfg, n_prefill=64)
    a.prefill_and_convert()
    buf = S.alloc_step_inputs(a.dims)
    for _ in range(10):
        a.step(buf)
    blob = io.BytesIO()
    torch.save({k: v.cpu() for k, v in a.state.state_dict().items()} | {"c": a.c, "t": a.t}, blob)
    for _ in range(12):
        a.step(buf)
    b = DeviceRun(cfg, n_prefill=64)
    blob.seek(0)
    sd = torch.load(blob)
    b.state.load_state_dict({k: v.cuda() for k, v in sd.items() if k not in ("c", "t")})
    b.c, b.t = sd["c"], sd["t"]
    for _ in range(12):
        b.step(buf)
    for k, v in a.state.state_dict().items():
        assert torch.equal(v, getattr(b.state, k)), k
