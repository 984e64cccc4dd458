"""seed_decode_step_compress: the decode step with the compression fused into it.

The fused launch runs the same step and the same compression as seed_decode_step
followed by seed_compress, only in one launch: trajectories through it must equal
those of the separate calls bit for bit, and match the oracle (prefill, conversion,
steps and compressions every W steps, or per request with ragged schedules) as
the separate path does.  A unit whose new key repeats an old one is declined by
the fused Cholesky-QR path and compressed by the Householder launch that follows.
"""

import numpy as np
import pytest

from oracle import compress as ocomp
from oracle import factored
from oracle import run as orun
from workloads import FORM_GDN, configs

from parity_util import (TOL, compare, ensure_lib, ragged_group, rel_fro, run_device, run_device_ragged,
                         run_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


CASES = [
    ("gdn-layer", 1, {}, 2, 256, None),                    # 128x128, R = W = 16 (tile 32)
    ("kda-r16w16", 4, dict(R=16, W=16), 1, 150, 24),       # per-channel decay
    ("kda-r8w8", 4, dict(R=8, W=8), 1, 150, 24),           # R + W = 16 (tile 16)
    ("mamba2-r8w16", 3, dict(R=8, W=16), 1, 200, 32),      # 128x64, no erase
    ("tiny-16x16", 0, {}, None, 64, None),                 # no fast path: decode + compress launches
]


@pytest.mark.parametrize("factors", [0, 1], ids=["f32", "f16"])
@pytest.mark.parametrize("name,cid,over,batch,n_prefill,n_sample", CASES, ids=[c[0] for c in CASES])
def test_fused_equals_separate_calls_and_the_oracle(factors, name, cid, over, batch, n_prefill, n_sample):
    cfg = configs.config(cid, **over)
    b = cfg.batch if batch is None else batch
    units = cfg.layers * cfg.heads * b
    rng = np.random.default_rng(cid + 7)
    sample = np.arange(units) if n_sample is None else np.sort(rng.choice(units, n_sample, replace=False))
    n_decode = 2 * cfg.W + 3
    fused = run_device(cfg, sample, n_prefill, n_decode, batch=batch, factors=factors, fused=True)
    sep = run_device(cfg, sample, n_prefill, n_decode, batch=batch, factors=factors)
    assert fused["flags"] == 0 and sep["flags"] == 0
    assert fused["comp_steps"] == sep["comp_steps"]
    for key in ("o", "ncols", "sigma", "S", "a"):
        np.testing.assert_array_equal(fused[key], sep[key], err_msg=key)
    if factors == 0:
        compare(cfg, fused, run_oracle(cfg, fused, n_prefill, n_decode))


def test_fused_ragged_schedules_match_the_oracle():
    cfg = configs.config(1, batch=16)
    rng = np.random.default_rng(77)
    n_prefill, n_decode = 128, cfg.W + 3
    units = np.unique([(bb * cfg.layers) * cfg.heads + rng.integers(cfg.heads)
                       for bb in range(cfg.batch) for _ in range(2)])
    dev = run_device_ragged(cfg, units, n_prefill, n_decode, fused=True)
    sep = run_device_ragged(cfg, units, n_prefill, n_decode)
    assert dev["flags"] == 0
    np.testing.assert_array_equal(dev["S"], sep["S"])
    np.testing.assert_array_equal(dev["o"], sep["o"])
    for phi in np.unique(dev["phase"]):
        idx = np.flatnonzero(dev["phase"] == phi)
        ref = orun.run_units(cfg, dev["b"][idx], dev["l"][idx], dev["h"][idx], n_prefill=n_prefill,
                             n_decode=n_decode, keep_shadow=True, lead_in=int(phi))
        compare(cfg, ragged_group(dev, idx), ref)


def test_repeated_key_is_declined_and_compressed_by_householder():
    """State with R + W - 1 columns whose next key equals a stored key: the fused
    launch's Cholesky-QR path declines every unit, the Householder launch compresses
    them; the result is the truncation of the exact step."""
    import torch
    from rank_recurrent_state_b200 import seed as S
    rng = np.random.default_rng(31)
    n, dk, dv, R, W = 16, 128, 128, 16, 16
    m, c = R + W, R + W - 1
    U = rng.normal(size=(n, m, dk)).astype(np.float32)
    U /= np.linalg.norm(U, axis=2, keepdims=True)
    V = (rng.normal(size=(n, m, dv)) * rng.uniform(0.2, 3, size=(n, m, 1))).astype(np.float32)
    slen = (m + 3) // 4 * 4
    scale = np.ones((n, slen), dtype=np.float32)
    scale[:, :c] = rng.uniform(0.3, 1.0, size=(n, c)).astype(np.float32)
    vbar = rng.normal(size=dv).astype(np.float32)
    a = (0.3 * rng.normal(size=(n, dk))).astype(np.float32)
    k = U[:, 5].copy()                                  # the key of slot 5 again
    q = rng.normal(size=(n, dk)).astype(np.float32)
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    v = (3 * vbar[None] + 0.3 * rng.normal(size=(n, dv))).astype(np.float32)
    g = rng.uniform(0.9, 1.0, size=n).astype(np.float32)
    beta = rng.uniform(0.2, 1.0, size=n).astype(np.float32)
    d = S.Dims(FORM_GDN, n, 1, 1, dk, dv, R, W)
    st = S.State.allocate(d, torch.from_numpy(vbar).reshape(1, 1, dv).cuda())
    st.U.copy_(torch.from_numpy(U).view_as(st.U))
    st.V.copy_(torch.from_numpy(V).view_as(st.V))
    st.scale.copy_(torch.from_numpy(scale).view_as(st.scale))
    st.a.copy_(torch.from_numpy(a).view_as(st.a))
    st.ncols.fill_(c)
    ws = S.Workspace(d)
    dev = {key: torch.from_numpy(x).cuda() for key, x in dict(q=q, k=k, v=v, g=g, beta=beta).items()}
    o = torch.empty(n, dv, device="cuda")
    sig = torch.zeros(n, R, device="cuda")
    S.seed_decode_step_compress(d, st, 0, dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], o, ws,
                                sigma_out=sig)
    assert S.seed_get_status(ws) == 0
    diag = S.seed_get_diagnostics(ws)
    assert diag["cholqr_declined"] == n and diag["householder_units"] == n
    np.testing.assert_array_equal(st.ncols.cpu().numpy().reshape(-1), R)
    Ut = np.swapaxes(U, 1, 2)[:, :, :c].astype(np.float64) * scale[:, None, :c]
    Vt = np.swapaxes(V, 1, 2)[:, :, :c].astype(np.float64)
    vb = np.repeat(vbar.astype(np.float64)[None], n, axis=0)
    a_n, U_n, V_n, o_ref = factored.step(FORM_GDN, a.astype(np.float64), Ut, Vt, vb, q.astype(np.float64),
                                         k.astype(np.float64), v.astype(np.float64), g.astype(np.float64),
                                         beta.astype(np.float64))
    Up, Vp, s = ocomp.truncate_product(U_n, V_n, R)
    dense = torch.empty(n, dk, dv, device="cuda")
    S.seed_state_to_dense(d, st, S.SEED_ALL_LAYERS, dense, ws)
    ref = factored.reconstruct(a_n, Up, Vp, vb)
    got = dense.cpu().numpy()
    for u in range(n):
        assert rel_fro(got[u], ref[u]) <= TOL
        assert rel_fro(sig.cpu().numpy()[u], s[u, :R]) <= TOL
    assert rel_fro(o.cpu().numpy(), o_ref) <= TOL
