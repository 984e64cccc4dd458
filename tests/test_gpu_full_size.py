"""Parity at the workloads' full sizes, in the launch configuration the benchmark
times: every (request, layer, head) unit of the workload resident on the device,
one decode launch per layer, one compression launch over all layers.

The single GDN layer (48 heads, batch 64, 2048-token prefill, 256 decode steps)
is compared in full: every one of its 3,072 units, every step.  The stacks are too
large for the oracle to follow every unit, so a seeded sample is compared: 64 units
at random plus every head of one (request, layer), through the workload's whole
decode run (1024, 512 and 1024 steps: 64, 16 and 64 compressions for the GDN,
Mamba-2 and KDA stacks; the KDA sweep's widest window, R + W = 96, over two
compressions), on bit-identical inputs regenerated on the host.  Every
compression of a recorded unit is also checked to be a best rank-R truncation of
the device's own state.
"""

import os

import numpy as np
import pytest

from workloads import configs

from parity_util import compare, ensure_lib, record_set, run_device, run_oracle_units

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _workers():
    return max(1, min(32, len(os.sched_getaffinity(0))))


def _sample(cfg, seed):
    rng = np.random.default_rng(seed)
    n_units = cfg.batch * cfg.layers * cfg.heads
    rand = rng.choice(n_units, size=64, replace=False)
    b, l = int(rng.integers(cfg.batch)), int(rng.integers(cfg.layers))
    heads = (b * cfg.layers + l) * cfg.heads + np.arange(cfg.heads)
    return np.unique(np.concatenate([rand, heads]))


def _check(cfg, units, label, chunk=8, n_decode=None):
    n_decode = cfg.n_decode if n_decode is None else n_decode
    b, rem = np.divmod(units, cfg.layers * cfg.heads)
    l, h = np.divmod(rem, cfg.heads)
    ref = run_oracle_units(cfg, b, l, h, cfg.n_prefill, n_decode, workers=_workers(), chunk=chunk)
    dev = run_device(cfg, units, cfg.n_prefill, n_decode, record_units=record_set(cfg, ref))
    assert dev["flags"] == 0, hex(dev["flags"])
    out = compare(cfg, dev, ref, label=label)
    assert out["o"].size == units.size
    assert len(ref["comp_steps"]) == n_decode // cfg.W
    return out


def test_gdn_layer_every_unit_at_full_size():
    """The single GDN layer as stated: 48 heads x batch 64, 2048-token prefill, 256
    decode steps (16 compressions), all 3,072 units."""
    cfg = configs.config(1)
    units = np.arange(cfg.batch * cfg.layers * cfg.heads)
    _check(cfg, units, "gdn-layer full size, every unit", chunk=32)


@pytest.mark.parametrize("cid,over", [(2, {}), (3, {}), (4, {})], ids=["gdn-stack", "mamba2-stack", "kda-stack"])
def test_full_size_sampled_units_whole_decode_run(cid, over):
    cfg = configs.config(cid, **over)
    units = _sample(cfg, 1000 + cid + cfg.R + cfg.W)
    _check(cfg, units, f"{cfg.name} R{cfg.R} W{cfg.W} full size, sampled, {cfg.n_decode} steps")


def test_full_size_kda_widest_window_sampled_units():
    """The KDA stack at the sweep's widest window, R = 32, W = 64 (R + W = 96, the
    Householder compression), full size, sampled units, 2W + 1 decode steps (two
    compressions of all 327,680 units)."""
    cfg = configs.config(4, R=32, W=64)
    units = _sample(cfg, 1000 + 4 + cfg.R + cfg.W)
    n_decode = 2 * cfg.W + 1
    _check(cfg, units, f"{cfg.name} R32 W64 full size, sampled, {n_decode} steps", n_decode=n_decode)
