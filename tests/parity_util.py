"""Helpers for the GPU parity tests: run the device path and the oracle on the same
seeded workload and compare what the method fixes.

The device side goes only through the C ABI (rank_recurrent_state_b200.seed and
.pipeline); the oracle side only through oracle/ with inputs from workloads/.
Nothing computed on the device is ever fed to the oracle.
"""

from __future__ import annotations

import numpy as np

TOL = 1e-4          # relative Frobenius error, fp32 device vs fp64 oracle
U32 = 2.0 ** -24    # float32 unit roundoff


def rel_fro(x, y) -> float:
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    den = np.linalg.norm(y)
    return float(np.linalg.norm(x - y) / (den if den > 0 else 1.0))


def ensure_lib():
    import torch
    from rank_recurrent_state_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need CUDA"


def run_device(cfg, sample_units, n_prefill, n_decode, batch=None, factors=0, fused=False,
               record_compress=True, record_units=None, overlap=False):
    """Run prefill, conversion and n_decode steps of every unit of (cfg, batch) on the
    device; return the trajectories of the sampled global units as numpy arrays.
    factors: storage format of U and V (seed_factors); fused: compress inside the
    decode launch of the step that fills R + W (seed_decode_step_compress); overlap:
    layers after the first step through seed_decode_step_overlapped.
    record_compress: also return, per compression, the sampled units' dense states
    right before and right after it (``S_pre``, ``S_post``; not with fused) and their
    sink a x vbar^T, for the optimality check of compare(); record_units: positions in
    the sample to record (default: all), returned as ``rec_idx``."""
    import torch
    from rank_recurrent_state_b200 import seed as S
    from rank_recurrent_state_b200.pipeline import DeviceRun

    run = DeviceRun(cfg, batch=batch, n_prefill=n_prefill, factors=factors, fused=fused, overlap=overlap)
    d = run.dims
    run.prefill_and_convert()
    su = np.asarray(sample_units, dtype=np.int64)
    b, rem = np.divmod(su, d.layers * d.heads)
    l, h = np.divmod(rem, d.heads)
    dev = run.device
    units_t = torch.as_tensor(su, dtype=torch.int32, device=dev)
    bl, ll, hl = (torch.as_tensor(x, dtype=torch.long, device=dev) for x in (b, l, h))
    buf = S.alloc_step_inputs(d, dev)
    outs = [None] * d.layers
    sig = torch.empty(d.units, d.R, dtype=torch.float32, device=dev)
    o_traj, ncols_traj, sig_traj, comp_steps = [], [], [], []
    pre, post, sink = [], [], []
    rec_idx = np.arange(su.size) if record_units is None else np.asarray(record_units, dtype=np.int64)
    rec_t = units_t[torch.as_tensor(rec_idx, dtype=torch.long, device=dev)]
    vb = run.vbar[ll, hl][torch.as_tensor(rec_idx, dtype=torch.long, device=dev)]   # [n_rec][d_v]

    def grab_pre():
        if record_compress and rec_idx.size:
            pre.append(run.to_dense(rec_t).cpu().numpy())
            a_now = run.state.a.reshape(-1, d.d_k)[rec_t.long()]
            sink.append((a_now[:, :, None] * vb[:, None, :]).cpu().numpy())

    conv = run.sigma_conv.reshape(-1, d.R)[units_t.long()].cpu().numpy()
    S0 = run.to_dense(units_t).cpu().numpy()
    for t in range(n_decode):
        fired = run.step(buf, outs=outs, sigma=sig, pre_compress=None if fused else grab_pre)
        o_all = torch.stack(outs)                       # [L][B][H][d_v]
        o_traj.append(o_all[ll, bl, hl].cpu().numpy())
        ncols_traj.append(run.state.ncols.reshape(-1)[units_t.long()].cpu().numpy())
        if fired:
            comp_steps.append(t + 1)
            sig_traj.append(sig[units_t.long()].cpu().numpy())
            if record_compress and not fused and rec_idx.size:
                post.append(run.to_dense(rec_t).cpu().numpy())
    torch.cuda.synchronize()
    S_fin = run.to_dense(units_t).cpu().numpy()
    a_fin = run.state.a.reshape(-1, d.d_k)[units_t.long()].cpu().numpy()
    flags = run.status()
    out = dict(o=np.array(o_traj), ncols=np.array(ncols_traj), sigma=np.array(sig_traj),
               comp_steps=comp_steps, S=S_fin, a=a_fin, S_conv=S0, conv_sigma=conv, flags=flags,
               b=b, l=l, h=h)
    if pre and len(pre) == len(post):
        out.update(S_pre=np.array(pre), S_post=np.array(post), sink=np.array(sink), rec_idx=rec_idx)
    return out


def run_device_ragged(cfg, sample_units, n_prefill, n_decode, batch=None, fused=False):
    """Like run_device, with ragged compression schedules: requests joined the batch at
    different times (DeviceRun's lead-in) and every step ends with a compression of the
    units that are due.  Returns the trajectories of the sampled units plus, per unit,
    its lead-in length ``phase``; ``comp_steps`` and ``sigma`` are per unit (lists)."""
    import torch
    from rank_recurrent_state_b200 import seed as S
    from rank_recurrent_state_b200.pipeline import DeviceRun

    run = DeviceRun(cfg, batch=batch, n_prefill=n_prefill, ragged=True, fused=fused)
    d = run.dims
    run.prefill_and_convert()
    su = np.asarray(sample_units, dtype=np.int64)
    b, rem = np.divmod(su, d.layers * d.heads)
    l, h = np.divmod(rem, d.heads)
    units_t = torch.as_tensor(su, dtype=torch.int32, device=run.device)
    conv = run.sigma_conv.reshape(-1, d.R)[units_t.long()].cpu().numpy()
    S0 = run.to_dense(units_t).cpu().numpy()
    buf = S.alloc_step_inputs(d, run.device)
    run.lead_in(buf)
    outs = [None] * d.layers
    sig = torch.zeros(d.units, d.R, dtype=torch.float32, device=run.device)
    o_traj, ncols_traj, sig_traj = [], [], []
    for t in range(n_decode):
        run.step(buf, outs=outs, sigma=sig)
        o_traj.append(np.stack([outs[li][bi, hi].cpu().numpy() for bi, li, hi in zip(b, l, h)]))
        ncols_traj.append(run.state.ncols.reshape(-1)[units_t.long()].cpu().numpy())
        sig_traj.append(sig[units_t.long()].cpu().numpy())
    torch.cuda.synchronize()
    ncols = np.array(ncols_traj)
    comp = [[t + 1 for t in range(n_decode) if ncols[t, u] == cfg.R] for u in range(su.size)]
    sigma = [np.array([sig_traj[t - 1][u] for t in comp[u]]) for u in range(su.size)]
    return dict(o=np.array(o_traj), ncols=ncols, comp_steps=comp, sigma=sigma,
                S=run.to_dense(units_t).cpu().numpy(),
                a=run.state.a.reshape(-1, d.d_k)[units_t.long()].cpu().numpy(), S_conv=S0,
                conv_sigma=conv, flags=run.status(), b=b, l=l, h=h,
                phase=run.phase[torch.as_tensor(b)].cpu().numpy())


def ragged_group(dev, idx):
    """The device trajectories of the sampled units idx (one lead-in length), in the
    layout compare() takes."""
    comp = dev["comp_steps"][idx[0]]
    assert all(dev["comp_steps"][u] == comp for u in idx)
    sig = np.stack([dev["sigma"][u] for u in idx], axis=1) if comp else np.zeros((0, len(idx), 0))
    return dict(o=dev["o"][:, idx], ncols=dev["ncols"][:, idx], comp_steps=comp, sigma=sig, S=dev["S"][idx],
                a=dev["a"][idx], S_conv=dev["S_conv"][idx], conv_sigma=dev["conv_sigma"][idx],
                flags=dev["flags"], b=dev["b"][idx], l=dev["l"][idx], h=dev["h"][idx])


def run_oracle(cfg, dev, n_prefill, n_decode):
    from oracle import run as orun
    return orun.run_units(cfg, dev["b"], dev["l"], dev["h"], n_prefill=n_prefill, n_decode=n_decode,
                          keep_shadow=True)


_UNIT_AXIS1 = ("o", "a_t", "sigma", "gap", "tail", "err_open", "sink_dev")
_SHARED = ("ncols", "comp_steps")


def _one_blas_thread():
    """Pool initializer: one BLAS thread per oracle worker (the workers already use
    every core)."""
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:   # pragma: no cover - speed only
        pass


def _oracle_chunk(args):
    from oracle import run as orun
    cfg, b, l, h, n_prefill, n_decode = args
    return orun.run_units(cfg, b, l, h, n_prefill=n_prefill, n_decode=n_decode, keep_shadow=True)


def run_oracle_units(cfg, b, l, h, n_prefill, n_decode, workers=8, chunk=8):
    """The oracle on the sampled units (b, l, h), split into chunks run by a pool of
    spawned processes (units are independent), merged along the unit axis."""
    import multiprocessing as mp
    b, l, h = (np.asarray(x, dtype=np.int64) for x in (b, l, h))
    parts = [(cfg, b[i:i + chunk], l[i:i + chunk], h[i:i + chunk], n_prefill, n_decode)
             for i in range(0, b.size, chunk)]
    with mp.get_context("spawn").Pool(min(workers, len(parts)), initializer=_one_blas_thread) as pool:
        outs = pool.map(_oracle_chunk, parts)
    merged = {}
    for key in outs[0]:
        if key in _SHARED:
            merged[key] = outs[0][key]
            for o in outs[1:]:
                assert np.array_equal(np.asarray(o[key]), np.asarray(outs[0][key])), key
        else:
            merged[key] = np.concatenate([o[key] for o in outs], axis=1 if key in _UNIT_AXIS1 else 0)
    return merged


def max_decay(cfg, dev, n_decode) -> np.ndarray:
    """Largest per-step contraction factor over the decode run, per sampled unit
    (g for GDN, alpha for Mamba-2, max_i alpha_i for KDA), from the host generator."""
    from workloads import philox
    inp = philox.token_inputs(cfg, dev["b"][:, None], dev["l"][:, None], dev["h"][:, None],
                              np.arange(n_decode)[None, :], philox.PHASE_DECODE, need_q=False)
    al = np.asarray(inp["alpha"], dtype=np.float64)
    return al.max(axis=(1, 2)) if al.ndim == 3 else al.max(axis=1)


# Per-test parity records, printed in pytest's terminal summary (tests/conftest.py).
SUMMARY: list[dict] = []


def first_near_tie(cfg, ref, tol=TOL):
    """Per sampled unit, the first truncation of the oracle's trajectory that is a
    near-tie (event 0 the conversion, i >= 1 compression i), -1 if none.

    A truncation to rank R is ill-conditioned when the singular values sigma_R and
    sigma_{R+1} nearly coincide: a perturbation of relative size u of the matrix turns
    the kept subspace by about u sigma_1 / (sigma_R - sigma_{R+1}) and moves the
    truncated matrix by about that times sigma_R.  Any float32 computation perturbs it
    by the unit roundoff u = 2^-24 at least, so where the predicted error
        u (sigma_R / sigma_1) / g,   g = (sigma_R - sigma_{R+1}) / sigma_1,
    exceeds 0.3 of the tolerance, float32 cannot be expected to reproduce the float64
    truncation to the tolerance, and several truncations are correct to working
    precision: a near-tie.  (On the GDN layer workload at full size -- 3,072 units, 17
    truncations each -- the one unit whose error exceeded the tolerance had a predicted
    error of 3.4e-4, at most twice below its measured 6.9e-4; every unit predicted below
    0.3 of the tolerance stayed within 0.6 of it.)"""
    gaps = [ref["conv_gap"]] + [ref["gap"][i] for i in range(ref["gap"].shape[0])]
    sigs = [ref["conv_sigma"]] + [ref["sigma"][i] for i in range(ref["sigma"].shape[0])]
    first = np.full(gaps[0].shape[0], -1)
    for ev_i, (g, sg) in enumerate(zip(gaps, sigs)):
        top = np.where(sg[:, 0] > 0, sg[:, 0], 1.0)
        ratio = sg[:, -1] / top
        predicted = U32 * ratio / np.maximum(g, 1e-300)
        hit = (predicted > 0.3 * tol) & (first < 0)
        first[hit] = ev_i
    return first


def record_set(cfg, ref, n_first=64):
    """Sample positions whose compressions run_device records: the first n_first units
    and every near-tie unit."""
    n = ref["conv_gap"].shape[0]
    ties = np.nonzero(first_near_tie(cfg, ref) >= 0)[0]
    return np.unique(np.concatenate([np.arange(min(n, n_first)), ties]))


def check_compressions(dev, R, tol=TOL):
    """Each device compression against what makes a truncation correct, on the device's
    own states (a property check, float64 SVD of the device's data): with C the content
    S - a vbar^T right before a compression and C' right after it (the sink is not
    touched), C' must have rank R (its (R+1)-th singular value below tol x its first),
    the kept singular values must be C's top R, and ||C' - C||_F must equal C's
    truncation error sqrt(sum_{i>R} sigma_i^2) -- a rank-R matrix at that distance is
    a best rank-R approximation (Eckart-Young).  Returns the largest errors, relative
    to ||S||_F (distance) and to ||sigma||."""
    if "S_pre" not in dev:
        return None
    n_comp, n = dev["S_pre"].shape[:2]
    idx = dev["rec_idx"]
    worst = {"sigma": 0.0, "distance": 0.0, "rank": 0.0, "checked": n_comp * n}
    for i in range(n_comp):
        C = dev["S_pre"][i].astype(np.float64) - dev["sink"][i]
        Cp = dev["S_post"][i].astype(np.float64) - dev["sink"][i]
        s = np.linalg.svd(C, compute_uv=False)
        sp = np.linalg.svd(Cp, compute_uv=False)
        for k in range(n):
            u = int(idx[k])
            tail = np.sqrt(np.sum(s[k, R:] ** 2))
            dist = np.linalg.norm(Cp[k] - C[k])
            nrm = max(float(np.linalg.norm(dev["S_pre"][i, k])), 1e-30)
            e_sig = rel_fro(dev["sigma"][i, u], s[k, :R])
            e_dist = abs(dist - tail) / nrm
            e_rank = (sp[k, R] / sp[k, 0]) if sp.shape[1] > R and sp[k, 0] > 0 else 0.0
            assert e_sig <= tol, ("kept sigma are not the top R of the state before", i, u, e_sig)
            assert e_dist <= tol, ("not at the optimal distance", i, u, dist, tail, nrm)
            assert e_rank <= tol, ("content after the compression has rank above R", i, u, e_rank)
            worst["sigma"] = max(worst["sigma"], e_sig)
            worst["distance"] = max(worst["distance"], e_dist)
            worst["rank"] = max(worst["rank"], e_rank)
    return worst


def compare(cfg, dev, ref, tol=TOL, max_tie_frac=0.1, label=None):
    """Device against oracle.

    Units with an ill-conditioned truncation (first_near_tie) at the conversion or at a
    compression are near-ties: several truncations are correct there.  For them, what is
    unique is compared: the sink coefficient a (no truncation touches it), and the
    trajectory up to the first ambiguous truncation -- the outputs o of every step up
    to it, and the kept singular values of every compression up to and including it.
    The states that follow are checked for validity: every device compression is a
    best rank-R truncation of the device's own state (check_compressions, for every
    unit), and the final state lies within Corollary 4's open-loop bound of the
    never-compressed dense state.  Every other unit is compared in full, per unit and
    pooled.  Bookkeeping is bit-exact.  The near-tie count is returned, recorded for
    the terminal summary, and bounded by max_tie_frac.
    """
    n = dev["o"].shape[1]
    first_tie = first_near_tie(cfg, ref, tol)   # event index: 0 conversion, i >= 1 compression i
    ties = first_tie >= 0
    ok = ~ties
    errs = {"o": [], "S": [], "sigma": [], "a": []}
    for u in range(n):
        errs["o"].append(rel_fro(dev["o"][:, u], ref["o"][:, u]))
        errs["S"].append(rel_fro(dev["S"][u], ref["S"][u]))
        errs["a"].append(rel_fro(dev["a"][u], ref["a"][u]))
        if dev["sigma"].size:
            errs["sigma"].append(rel_fro(dev["sigma"][:, u], ref["sigma"][:, u]))
    out = {k: np.array(v) for k, v in errs.items()}
    out["ties"] = int(ties.sum())
    out["conv_S"] = np.array([rel_fro(dev["S_conv"][u], ref["S_conv"][u]) for u in range(n)])
    out["conv_sigma"] = np.array([rel_fro(dev["conv_sigma"][u], ref["conv_sigma"][u]) for u in range(n)])
    # bookkeeping must be bit-exact
    assert dev["comp_steps"] == ref["comp_steps"], (dev["comp_steps"], ref["comp_steps"])
    np.testing.assert_array_equal(dev["ncols"], np.repeat(ref["ncols"][:, None], n, axis=1))
    # full comparison on units with a unique truncation
    for key in ("o", "S", "a", "sigma", "conv_S", "conv_sigma"):
        if out[key].size:
            assert np.all(out[key][ok] <= tol), (key, out[key])
    if ok.any():
        out["pooled_o"] = rel_fro(dev["o"][:, ok], ref["o"][:, ok])
        out["pooled_S"] = rel_fro(dev["S"][ok], ref["S"][ok])
        out["pooled_sigma"] = rel_fro(dev["sigma"][:, ok], ref["sigma"][:, ok]) if dev["sigma"].size else 0.0
        for key in ("pooled_o", "pooled_S", "pooled_sigma"):
            assert out[key] <= tol, (key, out[key])
    # every compression of every sampled unit is a best rank-R truncation of the
    # device's own state (covers the near-ties' later compressions too)
    out["compressions"] = check_compressions(dev, cfg.R, tol)
    # near-ties: what is unique, and validity of the state
    if ties.any():
        assert np.all(out["a"][ties] <= tol), ("a (near-tie units)", out["a"][ties])
        for u in np.nonzero(ties)[0]:
            j = int(first_tie[u])
            if j == 0:
                continue   # the conversion itself was ambiguous: only a and its sigma are unique
            assert out["conv_S"][u] <= tol, ("conversion before the first near-tie", u, out["conv_S"][u])
            t_end = ref["comp_steps"][j - 1]   # o up to the ambiguous compression's step is unique
            e_o = rel_fro(dev["o"][:t_end, u], ref["o"][:t_end, u])
            e_s = rel_fro(dev["sigma"][:j, u], ref["sigma"][:j, u])
            assert e_o <= tol and e_s <= tol, ("near-tie unit before its first near-tie", u, j, e_o, e_s)
        assert np.all(out["conv_sigma"][ties] <= tol), ("conv_sigma (near-tie units)", out["conv_sigma"][ties])
        g_bar = max_decay(cfg, dev, dev["o"].shape[0])
        eps_bar = np.max(ref["tail"], axis=0)
        bound = eps_bar / (1.0 - g_bar ** cfg.W)
        dist = np.array([np.linalg.norm(dev["S"][u] - ref["S_exact"][u]) for u in range(n)])
        assert np.all(dist[ties] <= bound[ties] * (1 + 1e-3) + 1e-4 * np.linalg.norm(ref["S_exact"][ties])), \
            ("near-tie state outside the Corollary 4 bound", dist[ties], bound[ties])
    rec = {"label": label or f"cfg{cfg.cid} R{cfg.R} W{cfg.W}", "units": n, "steps": int(dev["o"].shape[0]),
           "compressions": len(ref["comp_steps"]), "near_ties": out["ties"],
           "max_err_o": float(out["o"][ok].max()) if ok.any() else None,
           "max_err_S": float(out["S"][ok].max()) if ok.any() else None,
           "max_err_sigma": float(out["sigma"][ok].max()) if ok.any() and out["sigma"].size else None,
           "compressions_checked": out["compressions"]["checked"] if out["compressions"] else 0}
    SUMMARY.append(rec)
    assert out["ties"] <= max_tie_frac * n, ("too many near-ties", out["ties"], n)
    return out
