"""seed_decode_step_overlapped: the decode step launched so that it may begin while the
previous layer's step finishes (programmatic dependent launch).

The overlapped launch runs the same arithmetic on the same data as seed_decode_step;
only when its first copies start differs.  Trajectories through it (every layer after
the first overlapped with the one before, compressions every W steps, the first layer
after a compression launched plainly) must equal those of the plain calls bit for bit,
and match the oracle.  With 16-bit factors the whole-unit kernel takes the same
launch and must equal its plain calls likewise.
"""

import numpy as np
import pytest

from workloads import configs

from parity_util import compare, ensure_lib, run_device, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


CASES = [
    ("gdn-stack-3layers", 2, dict(layers=3, batch=8), 256, 48, 0),    # 128x128, R = W = 16 (ring)
    ("gdn-stack-3layers-f16", 2, dict(layers=3, batch=8), 256, 48, 1),  # whole-unit 16-bit kernel
    ("kda-r8w32", 4, dict(R=8, W=32, layers=2, batch=8), 150, 24, 0),  # 41 columns
    ("mamba2-3layers", 3, dict(layers=3, batch=4), 200, 32, 0),        # 128x64, R + W = 40
]


@pytest.mark.parametrize("name,cid,over,n_prefill,n_sample,factors", CASES, ids=[c[0] for c in CASES])
def test_overlapped_steps_equal_plain_steps_and_the_oracle(name, cid, over, n_prefill, n_sample, factors):
    cfg = configs.config(cid, **over)
    units = cfg.layers * cfg.heads * cfg.batch
    rng = np.random.default_rng(cid + 11)
    sample = np.sort(rng.choice(units, min(n_sample, units), replace=False))
    n_decode = 2 * cfg.W + 3
    ov = run_device(cfg, sample, n_prefill, n_decode, factors=factors, overlap=True)
    pl = run_device(cfg, sample, n_prefill, n_decode, factors=factors)
    assert ov["flags"] == 0 and pl["flags"] == 0
    assert ov["comp_steps"] == pl["comp_steps"]
    for key in ("o", "ncols", "sigma", "S", "a"):
        np.testing.assert_array_equal(ov[key], pl[key], err_msg=key)
    if factors == 0:   # 16-bit trajectories against the oracle: tests/test_gpu_factors16.py
        compare(cfg, ov, run_oracle(cfg, ov, n_prefill, n_decode), label=f"overlap {name}")
