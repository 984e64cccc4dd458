"""16-bit factor storage (fp16, bf16) against the oracle, one operation at a time.

SEED figures & tables (thelatestinai.com), Table 9: the shallow state's factors can
be kept in 16 bits, rounded when written.  The device computes in float32 and rounds
every value it stores to nearest; the oracle computes in float64 and rounds the same
quantities (oracle/precision.py).  A rounding decision taken from a float32 value
can differ from the one taken from the float64 value when the value lies within
the float32 error of a midpoint, so a stored column passes when every stored value
is a correct rounding of a value within delta of the oracle's,
|stored - x| <= ulp(x) / 2 + delta, with delta the float32 error of the arithmetic
that produced it (zero where no arithmetic is involved).  Products of rounded
factors (a compression's or a conversion's U V^T) are compared with the oracle's
truncation within the bound that rounding the factors allows, plus the float32
tolerance: with |dU| <= u'|U| + eta elementwise (u' = u / (1 - u), eta half the
subnormal spacing),
    ||U V^T - U~ V~^T||_F <= ||dU||_F ||V||_2 + (||U||_2 + ||dU||_F) ||dV||_F.
Every operation starts from a state built on the host (16-bit values uploaded), so
nothing the device computed reaches the oracle.  A whole trajectory then checks
the pages' claim that the drift with 16-bit factors is that of float32 factors.
"""

import numpy as np
import pytest

from oracle import compress as ocomp
from oracle import convert as oconv
from oracle import diagnostics, factored
from oracle import precision as P
from workloads import FORM_GDN, FORM_KDA, FORM_MAMBA2, configs

from parity_util import TOL, ensure_lib, rel_fro, run_device, run_oracle_units

pytestmark = pytest.mark.gpu

F16, BF16 = 1, 2
FMT = {F16: "f16", BF16: "bf16"}
ETA = {"f16": 2.0 ** -25, "bf16": 2.0 ** -134}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _torch_dtype(factors):
    import torch
    return torch.float16 if factors == F16 else torch.bfloat16


def _to16(x, factors):
    """float32 host array -> 16-bit host tensor (the stored values) and their float64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(_torch_dtype(factors))
    return t, t.double().numpy()


def _stored_state(form, n, dk, dv, R, W, c, rng, factors, unit_cols=True):
    """Stored factors [n][m][d] (16-bit, slots >= c hold 7), lazy scales, a, and the
    true U (n, d_k, c) and V (n, d_v, c) in float64."""
    m = R + W
    U = rng.normal(size=(n, m, dk))
    if form != FORM_MAMBA2 and unit_cols:
        U /= np.linalg.norm(U, axis=2, keepdims=True)
    else:
        U /= np.sqrt(dk)
    V = rng.normal(size=(n, m, dv)) * rng.uniform(0.2, 3, size=(n, m, 1))
    U[:, c:] = 7.0
    V[:, c:] = 7.0
    U16, U64 = _to16(U, factors)
    V16, V64 = _to16(V, factors)
    a = (0.5 * rng.normal(size=(n, dk))).astype(np.float32)
    if form == FORM_KDA:
        scale = rng.uniform(0.3, 1.0, size=(n, dk)).astype(np.float32)
        Ut = scale[:, :, None].astype(np.float64) * np.swapaxes(U64, 1, 2)[:, :, :c]
    else:
        slen = (m + 3) // 4 * 4
        scale = np.ones((n, slen), dtype=np.float32)
        scale[:, :c] = rng.uniform(0.05, 2.0, size=(n, c)).astype(np.float32)
        Ut = np.swapaxes(U64, 1, 2)[:, :, :c] * scale[:, None, :c].astype(np.float64)
    Vt = np.swapaxes(V64, 1, 2)[:, :, :c]
    return dict(U16=U16, V16=V16, U64=U64, V64=V64, a=a, scale=scale, Ut=Ut, Vt=Vt)


def _upload(form, n, dk, dv, R, W, factors, host, c, vbar):
    import torch
    from rank_recurrent_state_b200 import seed as S
    d = S.Dims(form, n, 1, 1, dk, dv, R, W, factors)
    st = S.State.allocate(d, torch.from_numpy(vbar.astype(np.float32)).reshape(1, 1, dv).cuda())
    assert st.U.dtype == _torch_dtype(factors)
    st.U.copy_(host["U16"].view_as(st.U))
    st.V.copy_(host["V16"].view_as(st.V))
    st.scale.copy_(torch.from_numpy(host["scale"]).view_as(st.scale))
    st.a.copy_(torch.from_numpy(host["a"]).view_as(st.a))
    st.ncols.fill_(c)
    return d, st, S.Workspace(d)


def _assert_rounded(stored, x, fmt, delta):
    """stored (float64 of 16-bit values) is a correct rounding of a value within delta of x."""
    err = np.abs(stored - x)
    lim = 0.5 * np.maximum(P.ulp(x, fmt), P.ulp(stored, fmt)) + delta
    bad = err > lim
    assert not bad.any(), (int(bad.sum()), float(np.max(err - lim)))
    # and nearly always the same rounding as the oracle's
    flips = np.mean(stored != P.round_nearest(x, fmt))
    assert flips <= 0.01, flips


def _step_inputs(form, n, dk, dv, vbar, rng):
    def unit(x):
        return x / np.linalg.norm(x, axis=1, keepdims=True)
    if form == FORM_MAMBA2:
        k = rng.normal(size=(n, dk)) / np.sqrt(dk)
        q = rng.normal(size=(n, dk)) / np.sqrt(dk)
        v = vbar[None, :] + 0.5 * rng.normal(size=(n, dv))
        alpha = rng.uniform(0.5, 1.0, size=n)
        beta = rng.uniform(0.01, 0.5, size=n)
    else:
        k = unit(rng.normal(size=(n, dk)))
        q = unit(rng.normal(size=(n, dk)))
        v = 3 * vbar[None, :] + 0.3 * rng.normal(size=(n, dv))
        alpha = rng.uniform(0.85, 1.0, size=(n, dk)) if form == FORM_KDA else rng.uniform(0.9, 1.0, size=n)
        beta = rng.uniform(0.1, 1.0, size=n)
    return {key: np.ascontiguousarray(val, dtype=np.float32)
            for key, val in dict(q=q, k=k, v=v, alpha=alpha, beta=beta).items()}


@pytest.mark.parametrize("factors", [F16, BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("form", [FORM_GDN, FORM_KDA, FORM_MAMBA2])
@pytest.mark.parametrize("dk,dv,R,W,c", [(128, 128, 16, 16, 23), (128, 64, 8, 32, 37), (64, 64, 4, 12, 9),
                                         (16, 16, 4, 4, 3), (128, 128, 32, 64, 90)])
def test_decode_step_appends_rounded_columns(factors, form, dk, dv, R, W, c):
    import torch
    from rank_recurrent_state_b200 import seed as S
    fmt = FMT[factors]
    rng = np.random.default_rng(1000 * factors + 10 * form + dk + c)
    n, m = 64, R + W
    host = _stored_state(form, n, dk, dv, R, W, c, rng, factors)
    vbar = rng.normal(size=dv) * 2.0 / np.sqrt(dv)
    d, st, ws = _upload(form, n, dk, dv, R, W, factors, host, c, vbar)
    inp = _step_inputs(form, n, dk, dv, vbar, rng)
    dev = {key: torch.from_numpy(val).cuda() for key, val in inp.items()}
    o = torch.empty(n, dv, device="cuda")
    S.seed_decode_step(d, st, 0, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], o, ws)
    assert S.seed_get_status(ws) == 0
    x64 = {key: val.astype(np.float64) for key, val in inp.items()}
    a_n, U_n, V_n, o_ref = factored.step(form, host["a"].astype(np.float64), host["Ut"], host["Vt"],
                                         np.repeat(vbar[None, :], n, axis=0), x64["q"], x64["k"], x64["v"],
                                         x64["alpha"], x64["beta"])
    o_dev = o.cpu().numpy()
    for u in range(n):
        assert rel_fro(o_dev[u], o_ref[u]) <= TOL
    assert rel_fro(st.a.cpu().numpy().reshape(n, dk), a_n) <= TOL
    np.testing.assert_array_equal(st.ncols.cpu().numpy().reshape(-1), c + 1)
    Ug = st.U.reshape(n, m, dk).double().cpu().numpy()
    Vg = st.V.reshape(n, m, dv).double().cpu().numpy()
    # the slots other than c are untouched
    keep = [j for j in range(m) if j != c]
    np.testing.assert_array_equal(Ug[:, keep], host["U64"][:, keep])
    np.testing.assert_array_equal(Vg[:, keep], host["V64"][:, keep])
    # the scales are float32 products (exact roundings of the float64 products)
    sc = st.scale.cpu().numpy().reshape(n, -1)
    if form == FORM_KDA:
        pn = (host["scale"].astype(np.float64) * x64["alpha"]).astype(np.float32)
        np.testing.assert_array_equal(sc, pn)
        x_u = x64["k"] / pn.astype(np.float64)                      # stored as k / P+
        delta_u = 2.0 ** -22 * np.abs(x_u)                           # one float32 division
    else:
        g = inp["alpha"].astype(np.float64)
        expect = (host["scale"].astype(np.float64) * g[:, None]).astype(np.float32)
        expect[:, c] = 1.0
        expect[:, c + 1:] = host["scale"][:, c + 1:]
        np.testing.assert_array_equal(sc, expect)
        x_u, delta_u = x64["k"], 0.0                                 # k itself, rounded
    _assert_rounded(Ug[:, c], x_u, fmt, delta_u)
    # the new V column: float32 arithmetic over c columns
    x_v = V_n[:, :, c]
    delta_v = 1e-5 * np.max(np.abs(x_v), axis=1, keepdims=True)
    _assert_rounded(Vg[:, c], x_v, fmt, delta_v)


def _rounding_bound(Ut, Vt, fmt, s_col=None):
    """Bound on ||U V^T - U~ V~^T||_F from rounding the stored factors to fmt (true U
    = stored U times the column scales s_col, or the stored U)."""
    u = P.unit_roundoff(fmt)
    up = u / (1 - u)
    eta = ETA[fmt]
    dk, R = Ut.shape
    dv = Vt.shape[0]
    s_norm = np.linalg.norm(s_col) if s_col is not None else np.sqrt(R)
    dU = up * np.linalg.norm(Ut) + eta * np.sqrt(dk) * s_norm
    dV = up * np.linalg.norm(Vt) + eta * np.sqrt(dv * R)
    return dU * np.linalg.norm(Vt, 2) + (np.linalg.norm(Ut, 2) + dU) * dV


@pytest.mark.parametrize("factors", [F16, BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("form", [FORM_GDN, FORM_KDA, FORM_MAMBA2])
@pytest.mark.parametrize("dk,dv,R,W,repeat", [(128, 128, 16, 16, False), (128, 128, 16, 16, True),
                                              (128, 64, 8, 32, False), (64, 64, 4, 12, False),
                                              (16, 16, 4, 4, False), (128, 128, 32, 64, False)])
def test_compress_stores_the_rounded_truncation(factors, form, dk, dv, R, W, repeat):
    import torch
    from rank_recurrent_state_b200 import seed as S
    fmt = FMT[factors]
    rng = np.random.default_rng(2000 * factors + 10 * form + dk + R + int(repeat))
    n, m = 24, R + W
    host = _stored_state(form, n, dk, dv, R, W, m, rng, factors)
    if repeat:   # a key repeated inside the window: the Cholesky-QR path declines it
        U16 = host["U16"].clone()
        U16[:, m - 1] = U16[:, m - 3]
        host["U16"], host["U64"] = U16, U16.double().numpy()
        sc = host["scale"]
        if form == FORM_KDA:
            host["Ut"] = sc[:, :, None].astype(np.float64) * np.swapaxes(host["U64"], 1, 2)
        else:
            host["Ut"] = np.swapaxes(host["U64"], 1, 2) * sc[:, None, :m].astype(np.float64)
    vbar = np.ones(dv)
    d, st, ws = _upload(form, n, dk, dv, R, W, factors, host, m, vbar)
    sig = torch.zeros(n, R, device="cuda")
    S.seed_compress(d, st, S.SEED_ALL_LAYERS, ws, sigma_out=sig)
    assert S.seed_get_status(ws) == 0
    diag = S.seed_get_diagnostics(ws)
    if repeat and R + W <= 32:
        assert diag["cholqr_declined"] == n
    np.testing.assert_array_equal(st.ncols.cpu().numpy().reshape(-1), R)
    Ug = st.U.reshape(n, m, dk).double().cpu().numpy()
    Vg = st.V.reshape(n, m, dv).double().cpu().numpy()
    np.testing.assert_array_equal(Ug[:, R:], host["U64"][:, R:])     # slots R.. untouched
    np.testing.assert_array_equal(Vg[:, R:], host["V64"][:, R:])
    sc = st.scale.cpu().numpy().reshape(n, -1).astype(np.float64)
    Up, Vp, s = ocomp.truncate_product(host["Ut"], host["Vt"], R)
    sg = sig.cpu().numpy()
    for u in range(n):
        if form == FORM_KDA:
            Ut, s_col = sc[u][:, None] * Ug[u, :R].T, None
        else:
            Ut, s_col = Ug[u, :R].T * sc[u, None, :R], sc[u, :R]
        Vt = Vg[u, :R].T
        ref = Up[u] @ Vp[u].T
        err = np.linalg.norm(Ut @ Vt.T - ref)
        lim = _rounding_bound(Ut, Vt, fmt, s_col) + TOL * np.linalg.norm(ref)
        assert err <= lim, (u, err / np.linalg.norm(ref), lim / np.linalg.norm(ref))
        assert rel_fro(sg[u], s[u, :R]) <= TOL


@pytest.mark.parametrize("factors", [F16, BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("dk,dv,R", [(128, 128, 16), (128, 64, 8), (64, 128, 12), (16, 16, 4)])
def test_conversion_stores_the_rounded_truncation(factors, dk, dv, R):
    import torch
    from rank_recurrent_state_b200 import seed as S
    fmt = FMT[factors]
    rng = np.random.default_rng(3000 * factors + dk + dv + R)
    n = 16
    vbar = rng.normal(size=dv)
    a0 = rng.normal(size=(n, dk))
    r = min(dk, dv)
    X = np.linalg.qr(rng.normal(size=(n, dk, r)))[0]
    Y = np.linalg.qr(rng.normal(size=(n, dv, r)))[0]
    sv = 3.0 * 0.8 ** np.arange(r)
    Sd = (a0[:, :, None] * vbar[None, None, :] + np.einsum("nir,r,njr->nij", X, sv, Y)).astype(np.float32)
    W = 4
    d = S.Dims(FORM_GDN, n, 1, 1, dk, dv, R, W, factors)
    st = S.State.allocate(d, torch.from_numpy(vbar.astype(np.float32)).reshape(1, 1, dv).cuda())
    ws = S.Workspace(d)
    sig = torch.zeros(n, R, device="cuda")
    S.seed_state_init_from_dense(d, st, S.SEED_ALL_LAYERS, torch.from_numpy(Sd).cuda(), ws, sigma_out=sig)
    assert S.seed_get_status(ws) == 0
    vb32 = vbar.astype(np.float32).astype(np.float64)
    a_o, U_o, V_o, s = oconv.convert(Sd.astype(np.float64), np.repeat(vb32[None], n, axis=0), R)
    assert rel_fro(st.a.cpu().numpy().reshape(n, dk), a_o) <= TOL
    np.testing.assert_array_equal(st.ncols.cpu().numpy().reshape(-1), R)
    np.testing.assert_array_equal(st.scale.cpu().numpy(), 1.0)
    Ug = st.U.reshape(n, R + W, dk).double().cpu().numpy()
    Vg = st.V.reshape(n, R + W, dv).double().cpu().numpy()
    sg = sig.cpu().numpy()
    for u in range(n):
        Ut, Vt = Ug[u, :R].T, Vg[u, :R].T
        ref = U_o[u] @ V_o[u].T
        err = np.linalg.norm(Ut @ Vt.T - ref)
        lim = _rounding_bound(Ut, Vt, fmt) + TOL * np.linalg.norm(ref)
        assert err <= lim, (u, err / np.linalg.norm(ref), lim / np.linalg.norm(ref))
        assert rel_fro(sg[u], s[u, :R]) <= TOL


@pytest.mark.parametrize("factors", [F16, BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("form", [FORM_GDN, FORM_KDA, FORM_MAMBA2])
def test_to_dense_and_energy_read_16bit_factors(factors, form):
    import torch
    from rank_recurrent_state_b200 import seed as S
    rng = np.random.default_rng(4000 * factors + form)
    n, dk, dv, R, W, c = 16, 128, 64, 8, 32, 30
    host = _stored_state(form, n, dk, dv, R, W, c, rng, factors)
    vbar = rng.normal(size=dv)
    d, st, ws = _upload(form, n, dk, dv, R, W, factors, host, c, vbar)
    dense = torch.empty(n, dk, dv, device="cuda")
    S.seed_state_to_dense(d, st, S.SEED_ALL_LAYERS, dense, ws)
    en = torch.empty(n, 4, device="cuda")
    S.seed_state_energy(d, st, S.SEED_ALL_LAYERS, en, ws)
    assert S.seed_get_status(ws) == 0
    vb = np.repeat(vbar.astype(np.float32).astype(np.float64)[None], n, axis=0)
    a = host["a"].astype(np.float64)
    ref = factored.reconstruct(a, host["Ut"], host["Vt"], vb)
    got = dense.cpu().numpy()
    for u in range(n):
        assert rel_fro(got[u], ref[u]) <= TOL
    e_ref = diagnostics.energies(a, host["Ut"], host["Vt"], vb)
    e = en.double().cpu().numpy()
    assert np.max(np.abs(e - e_ref) / e_ref[:, 3:4]) <= TOL


@pytest.mark.parametrize("factors", [F16, BF16], ids=["f16", "bf16"])
def test_trajectory_drift_matches_float32_factors(factors):
    """The GDN layer workload (one layer, 48 heads, R = W = 16) through prefill,
    conversion and 2W + 3 decode steps with 16-bit and with float32 factors.  The
    bookkeeping is bit-exact; the open-loop error against the never-compressed dense
    state (Corollary 4's quantity) is that of the float32 run up to the rounding
    budget K u ||S|| with K = 2 sqrt(R) (1 + compressions) + 2 (decode steps): each
    conversion or compression perturbs the content by at most 2 u' ||U||_F ||V||_2
    <= 2 sqrt(R) u' ||C||_F, each appended pair by 2 u' ||k v^T||_F, and the GDN
    step is non-expansive."""
    fmt = FMT[factors]
    cfg = configs.config(1, batch=2)
    n_prefill, n_decode = 256, 2 * cfg.W + 3
    units = np.arange(cfg.batch * cfg.layers * cfg.heads)
    dev16 = run_device(cfg, units, n_prefill, n_decode, factors=factors)
    dev32 = run_device(cfg, units, n_prefill, n_decode)
    assert dev16["flags"] == 0 and dev32["flags"] == 0
    ref = run_oracle_units(cfg, dev32["b"], dev32["l"], dev32["h"], n_prefill, n_decode)
    assert dev16["comp_steps"] == ref["comp_steps"] == dev32["comp_steps"]
    np.testing.assert_array_equal(dev16["ncols"], dev32["ncols"])
    K = 2 * np.sqrt(cfg.R) * (1 + len(ref["comp_steps"])) + 2 * n_decode
    budget = K * P.unit_roundoff(fmt)
    n = units.size
    for u in range(n):
        nS = np.linalg.norm(ref["S_exact"][u])
        e16 = np.linalg.norm(dev16["S"][u] - ref["S_exact"][u])
        e32 = np.linalg.norm(dev32["S"][u] - ref["S_exact"][u])
        assert e16 <= e32 + budget * nS, (u, e16 / nS, e32 / nS, budget)
        assert rel_fro(dev16["S"][u], dev32["S"][u]) <= budget
        assert rel_fro(dev16["o"][:, u], dev32["o"][:, u]) <= budget
    # the sink a is never rounded: it follows its own float32 recurrence, and the
    # 16-bit content enters it only through omega, which does not involve U and V
    assert rel_fro(dev16["a"], dev32["a"]) <= TOL


@pytest.mark.parametrize("factors", [F16, BF16], ids=["f16", "bf16"])
def test_value_beyond_the_format_range_is_flagged(factors):
    """A new V column beyond fp16's largest finite value (65504) is stored as +-inf
    and raises SEED_FLAG_NONFINITE; bf16 has float32's range and stores it finite."""
    import torch
    from rank_recurrent_state_b200 import seed as S
    rng = np.random.default_rng(5000 + factors)
    n, dk, dv, R, W, c = 8, 128, 128, 16, 16, 20
    host = _stored_state(FORM_GDN, n, dk, dv, R, W, c, rng, factors)
    vbar = np.zeros(dv)
    vbar[0] = 1.0
    d, st, ws = _upload(FORM_GDN, n, dk, dv, R, W, factors, host, c, vbar)
    inp = _step_inputs(FORM_GDN, n, dk, dv, vbar, rng)
    inp["v"][:, 5] = 1e5          # orthogonal to vbar: lands in the new V column
    inp["beta"][:] = 1.0
    dev = {key: torch.from_numpy(val).cuda() for key, val in inp.items()}
    o = torch.empty(n, dv, device="cuda")
    S.seed_decode_step(d, st, 0, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], o, ws)
    flags = S.seed_get_status(ws)
    col = st.V.reshape(n, R + W, dv)[:, c, 5].double().cpu().numpy()
    if factors == F16:
        assert flags & S.FLAG_NONFINITE
        assert np.all(np.isinf(col))
    else:
        assert flags == 0
        assert np.all(np.isfinite(col)) and np.all(np.abs(col) > 5e4)
