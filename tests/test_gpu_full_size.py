"""Parity at the workloads' full sizes, in the launch configuration the benchmark
times: every (request, layer, head) unit of the workload resident on the device,
one decode launch per layer, one compression launch over all layers.

The oracle cannot run hundreds of thousands of units, so a seeded sample is
compared: 64 units at random plus every head of one (request, layer).  The oracle
runs only those units, on bit-identical inputs regenerated on the host, through
the prefill, the conversion and 2W + 1 decode steps (two compressions).
"""

import numpy as np
import pytest

from workloads import configs

from parity_util import compare, ensure_lib, run_device, run_oracle_units

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _sample(cfg, seed):
    rng = np.random.default_rng(seed)
    n_units = cfg.batch * cfg.layers * cfg.heads
    rand = rng.choice(n_units, size=64, replace=False)
    b, l = int(rng.integers(cfg.batch)), int(rng.integers(cfg.layers))
    heads = (b * cfg.layers + l) * cfg.heads + np.arange(cfg.heads)
    return np.unique(np.concatenate([rand, heads]))


@pytest.mark.parametrize("cid,over", [(2, {}), (3, {}), (4, {}), (4, {"R": 32, "W": 64})],
                         ids=["gdn-stack", "mamba2-stack", "kda-stack", "kda-stack-R32-W64"])
def test_full_size_sampled_units_match_the_oracle(cid, over):
    cfg = configs.config(cid, **over)
    units = _sample(cfg, 1000 + cid + cfg.R + cfg.W)
    n_decode = 2 * cfg.W + 1
    b, rem = np.divmod(units, cfg.layers * cfg.heads)
    l, h = np.divmod(rem, cfg.heads)
    ref = run_oracle_units(cfg, b, l, h, cfg.n_prefill, n_decode)
    dev = run_device(cfg, units, cfg.n_prefill, n_decode)
    assert dev["flags"] == 0, hex(dev["flags"])
    out = compare(cfg, dev, ref)
    assert out["o"].size == units.size
