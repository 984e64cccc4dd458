"""Ragged compression schedules: requests that joined the batch at different times.

Request b took phi_b = W - 1 - floor(b W / B) lead-in decode steps before the common
steps (inputs of the lead-in phase), so in one batched decode step different
requests hold different column counts and a compression launch after every step
compresses only the units that are due.  Each group of sampled units with the same
lead-in length is compared with the oracle run with that lead-in: outputs, states,
singular values, and bit-exact column counts and compression steps.
"""

import numpy as np
import pytest

from oracle import run as orun
from workloads import configs

from parity_util import compare, ensure_lib, ragged_group, run_device_ragged

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


@pytest.mark.parametrize("cid,over", [(1, dict(batch=16)), (3, dict(batch=8, layers=2)),
                                      (4, dict(batch=8, layers=2))],
                         ids=["gdn-layer", "mamba2", "kda"])
def test_ragged_schedules_match_the_oracle(cid, over):
    cfg = configs.config(cid, **over)
    rng = np.random.default_rng(500 + cid)
    n_prefill, n_decode = 128, cfg.W + 3
    units = []
    for b in range(cfg.batch):   # two units of every request (each request its own lead-in)
        for _ in range(2):
            l, h = rng.integers(cfg.layers), rng.integers(cfg.heads)
            units.append((b * cfg.layers + l) * cfg.heads + h)
    units = np.unique(units)
    dev = run_device_ragged(cfg, units, n_prefill, n_decode)
    assert dev["flags"] == 0, hex(dev["flags"])
    phases = np.unique(dev["phase"])
    assert phases.size == min(cfg.batch, cfg.W)   # the schedules really are ragged
    for phi in phases:
        idx = np.flatnonzero(dev["phase"] == phi)
        ref = orun.run_units(cfg, dev["b"][idx], dev["l"][idx], dev["h"][idx], n_prefill=n_prefill,
                             n_decode=n_decode, keep_shadow=True, lead_in=int(phi))
        assert ref["comp_steps"] == list(range(cfg.W - int(phi), n_decode + 1, cfg.W))
        compare(cfg, ragged_group(dev, idx), ref)
