"""Host emulations of the index logic inside the kernels (no GPU).

1. The register Jacobi of the fast compression (jacobi_regs): MP / 2 slots each
   hold a column pair (x, y); within a group of G slots the x columns shift by one
   slot per round for G rounds, then every group halves: the first half's slots
   take their partners' x as their y, the second half's take their partners' y as
   their x.  Every one of the MP (MP - 1) / 2 column pairs must meet exactly once
   per sweep, whatever the arrangement a sweep starts from.
2. The transposed warp reduction (warp_xreduce<NV>): after it, lane l holds the
   total of value (l >> (5 - log2 NV)) & (NV - 1).
3. The decode ring's chunk sequence (decode_ring_run): a warp's units u0, u0 +
   stride, ... pass through NSLOT slots as chunks (its U chunks, then its V chunks);
   lane 0 refills a slot with the next chunk of the sequence, which after the current
   unit's last chunk belongs to the next unit.  Every chunk the warp reads must be
   the one issued into that position for that unit, at most NSLOT may be in flight,
   none may be left in flight when the warp exits, and a unit's chunks must cover
   its stored columns exactly.
4. The compression's Cholesky in panels of four columns (cholesky_wide): every
   entry must receive the same multiply-adds in the same order as a column-by-column
   right-looking factorisation (emulated in float32 with the same operation for
   both, so the two agree bit for bit exactly when the orders agree), with the same
   dropped columns and the same rejection of small pivots.
"""

import itertools

import numpy as np
import pytest


def _jacobi_sweep(ix, iy):
    """One sweep of the slot schedule; returns the pairs met and the final layout."""
    ns = len(ix)
    ix, iy = list(ix), list(iy)
    met = []
    G = ns
    while G >= 1:
        for r in range(G):
            met.extend(frozenset((ix[s], iy[s])) for s in range(ns))
            if r + 1 < G:   # x moves one slot along its group: slot takes x of slot - 1
                new = list(ix)
                for s in range(ns):
                    gb = s & ~(G - 1)
                    new[s] = ix[gb + ((s - gb - 1) & (G - 1))]
                ix = new
        if G > 1:
            half = G >> 1
            nx, ny = list(ix), list(iy)
            for s in range(ns):
                p = s ^ half
                if (s & half) == 0:
                    ny[s] = ix[p]       # first half: y <- partner's x
                else:
                    nx[s] = iy[p]       # second half: x <- partner's y
            ix, iy = nx, ny
        G >>= 1
    return met, ix, iy


@pytest.mark.parametrize("mp", [16, 32])
def test_jacobi_schedule_meets_every_pair_once_per_sweep(mp):
    ns = mp // 2
    ix, iy = list(range(ns)), list(range(ns, mp))
    everything = {frozenset(p) for p in itertools.combinations(range(mp), 2)}
    for _ in range(3):   # consecutive sweeps start from the previous sweep's layout
        met, ix, iy = _jacobi_sweep(ix, iy)
        assert len(met) == len(everything) == mp * (mp - 1) // 2
        assert set(met) == everything
        assert sorted(ix + iy) == list(range(mp))   # a permutation of the columns
    # the rounds per sweep: MP - 1
    assert len(met) // ns == mp - 1


def _xreduce(vals):
    """vals (32 lanes, NV values): emulates warp_xreduce's recursive halving."""
    v = np.array(vals, dtype=np.float64)
    nv = v.shape[1]
    n = nv
    off = 16
    while off >= 1:
        lanes = np.arange(32)
        if n > 1:
            hi = (lanes & off) != 0
            new = v.copy()
            for i in range(n // 2):
                send = np.where(hi, v[:, i], v[:, i + n // 2])
                keep = np.where(hi, v[:, i + n // 2], v[:, i])
                new[:, i] = keep + send[lanes ^ off]
            v = new
            n >>= 1
        else:
            v[:, 0] = v[:, 0] + v[lanes ^ off, 0]
        off >>= 1
    return v[:, 0]


@pytest.mark.parametrize("nv", [1, 2, 8, 16, 32])
def test_transposed_warp_reduction_lane_mapping(nv):
    rng = np.random.default_rng(nv)
    vals = rng.integers(-100, 100, size=(32, nv)).astype(np.float64)
    out = _xreduce(vals)
    sh = 5 - int(np.log2(nv))
    totals = vals.sum(axis=0)
    for lane in range(32):
        assert out[lane] == totals[(lane >> sh) & (nv - 1)]


def _swz(j, e):
    """Offset of element e of column j in a swizzled float32 chunk (the kernels' swz)."""
    return j * 32 + ((((e >> 2) ^ (j & 7)) << 2) | (e & 3))


@pytest.mark.parametrize("mp,m", [(16, 9), (16, 16), (32, 24), (32, 32)])
def test_16bit_chunk_widening_lands_in_the_swizzled_layout(mp, m):
    """issue_chunk16 / widen_chunk16: lane l copies rows 8 (l & 3) .. of column
    8 pass + (l >> 2) and widens them into two float4 slots; together the lanes must
    write every (column, row) of the chunk exactly once, at swz(column, row), with
    zeros for the columns past m, and read only staging slots they filled."""
    chunk = np.full(mp * 32, np.nan)
    written = np.zeros(mp * 32, dtype=int)
    staged = set()
    for lane in range(32):
        q = lane & 3
        for p in range(mp // 8):
            j = p * 8 + (lane >> 2)
            if j < m:
                staged.add((lane, j))                      # the cp.async of this lane
            for half in range(2):                          # rows 8q .. 8q+3, 8q+4 .. 8q+7
                base = j * 32 + (((2 * q + half) ^ (j & 7)) << 2)
                for t in range(4):
                    e = 8 * q + 4 * half + t
                    assert base + t == _swz(j, e)
                    chunk[base + t] = (1000 * j + e) if j < m else 0.0
                    written[base + t] += 1
                if j < m:
                    assert (lane, j) in staged             # reads its own staging slot
    assert np.all(written == 1)
    for j in range(mp):
        for e in range(32):
            assert chunk[_swz(j, e)] == ((1000 * j + e) if j < m else 0.0)


RING_CHUNK = 8


def _ring_chunks(c, m):
    return 2 * ((c + RING_CHUNK - 1) // RING_CHUNK) if 0 < c < m else 0


def _ring_issue(c, kidx):
    """Columns of chunk kidx of a unit holding c columns: (is V, first column, count)."""
    n = (c + RING_CHUNK - 1) // RING_CHUNK
    is_v = kidx >= n
    col0 = (kidx - n if is_v else kidx) * RING_CHUNK
    return is_v, col0, min(c - col0, RING_CHUNK)


def _ring_warp(ncols, n_units, stride, u0, nslot, m):
    """The control flow of one warp of decode_ring_run: returns the chunks issued
    (sequence number -> (unit, kidx)) and read ((unit, kidx) in order), checking
    the in-flight bound as it goes."""
    issued_log, read = {}, []
    st = {"u": u0, "base": 0, "issued": 0, "consumed": 0}
    st["c_cur"] = ncols[u0] if u0 < n_units else 0
    st["c_nxt"] = ncols[u0 + stride] if u0 + stride < n_units else 0
    st["n_cur"] = _ring_chunks(st["c_cur"], m)
    st["n_nxt"] = _ring_chunks(st["c_nxt"], m) if u0 + stride < n_units else 0

    def fill():
        while st["issued"] < st["consumed"] + nslot:
            i, base = st["issued"], st["base"]
            if i < base + st["n_cur"]:
                uu, kk = st["u"], i - base
            elif i < base + st["n_cur"] + st["n_nxt"]:
                uu, kk = st["u"] + stride, i - base - st["n_cur"]
            else:
                break
            issued_log[i] = (uu, kk)
            st["issued"] += 1
            assert st["issued"] - st["consumed"] <= nslot

    def consume(unit, kidx):
        assert st["consumed"] < st["issued"], "a read with no chunk issued"
        assert issued_log[st["consumed"]] == (unit, kidx), (st["consumed"], issued_log[st["consumed"]], unit, kidx)
        read.append((unit, kidx))
        st["consumed"] += 1
        fill()

    fill()
    while st["u"] < n_units:
        u = st["u"]
        u_next = u + stride
        c_aft = ncols[u_next + stride] if u_next + stride < n_units else 0
        c = st["c_cur"]
        if 0 <= c < m:
            nch = st["n_cur"] // 2
            for ch in range(nch):        # U chunks
                consume(u, ch)
            for ch in range(nch):        # V chunks
                consume(u, nch + ch)
        st["base"] += st["n_cur"]
        st["n_cur"], st["c_cur"], st["c_nxt"] = st["n_nxt"], st["c_nxt"], c_aft
        st["n_nxt"] = _ring_chunks(c_aft, m) if u_next + stride < n_units else 0
        st["u"] = u_next
        fill()
    assert st["issued"] == st["consumed"], "copies left in flight at exit"
    return issued_log, read


@pytest.mark.parametrize("m,nslot", [(32, 4), (32, 3), (40, 4), (65, 8), (17, 5)])
@pytest.mark.parametrize("stride,n_units", [(1, 7), (3, 23), (7, 23), (30, 23)])
def test_decode_ring_reads_every_unit_chunk_in_order(m, nslot, stride, n_units):
    rng = np.random.default_rng(m * 1000 + nslot * 100 + stride * 10 + n_units)
    R = max(1, m // 2)
    ncols = list(rng.integers(R, m, size=n_units))      # R .. m - 1 columns held
    for i in rng.choice(n_units, size=min(3, n_units), replace=False):
        ncols[i] = int(rng.choice([0, m, -1]))          # empty, full and invalid units
    for u0 in range(min(stride, n_units)):
        _, read = _ring_warp(ncols, n_units, stride, u0, nslot, m)
        for u in range(u0, n_units, stride):
            c = ncols[u]
            got = [k for uu, k in read if uu == u]
            n = _ring_chunks(c, m)
            assert got == list(range(n)), (u, c, got)
            cols = {False: [], True: []}
            for k in got:
                is_v, col0, cnt = _ring_issue(c, k)
                assert 0 < cnt <= RING_CHUNK
                cols[is_v] += list(range(col0, col0 + cnt))
            if n:
                assert cols[False] == list(range(c)) and cols[True] == list(range(c)), (u, c)


PIVOT_MIN = np.float32(1e-2)   # kCholPivotMin


def _madd(a, b, c):
    # the same float32 operation for both orders (the device fuses it; only the order
    # of the updates is under test here)
    return np.float32(np.float32(a * b) + c)


def _equilibrate(G, m):
    G = G.astype(np.float32).copy()
    mp = G.shape[0]
    nrm = np.zeros(mp, np.float32)
    for i in range(m):
        nrm[i] = np.sqrt(max(G[i, i], np.float32(0)))
    ninv = np.array([np.float32(1) / n if n > 0 else np.float32(0) for n in nrm], np.float32)
    for i in range(mp):
        for j in range(mp):
            G[i, j] = np.float32(G[i, j] * np.float32(ninv[i] * ninv[j]))
    return G, nrm


def _pivot(d, n):
    zero = not (n > 0)
    drop = zero or not (d > 0)
    bad = False
    if not zero and d < PIVOT_MIN:
        drop, bad = True, True
    rs = np.float32(0) if drop else np.float32(1) / np.sqrt(d)
    return drop, bad, np.float32(rs)


def _chol_columns(G0, m):
    G, nrm = _equilibrate(G0, m)
    mp, bad = G.shape[0], False
    for j in range(m):
        d = G[j, j]
        drop, b, rs = _pivot(d, nrm[j])
        bad |= b
        col = np.zeros(mp, np.float32)
        for i in range(j + 1, mp):
            col[i] = np.float32(G[i, j] * rs)
            G[i, j] = col[i]
        G[j, j] = np.float32(0) if drop else np.float32(d * rs)
        for i in range(j + 1, m):
            if col[i] != 0:
                for c in range(j + 1, m):
                    G[i, c] = _madd(-col[i], col[c], G[i, c])
    return np.tril(G[:m, :m]), bad


def _chol_panels(G0, m):
    G, nrm = _equilibrate(G0, m)
    mp, bad = G.shape[0], False
    for jb in range(0, m, 4):
        p = G[:, jb:jb + 4].copy()                   # every row's panel entries
        for t in range(4):
            j = jb + t
            if j >= m:
                break
            d = p[j, t]
            drop, b, rs = _pivot(d, nrm[j])
            bad |= b
            l = np.zeros(mp, np.float32)
            for i in range(j + 1, mp):
                l[i] = np.float32(p[i, t] * rs)
                p[i, t] = l[i]
            p[j, t] = np.float32(0) if drop else np.float32(d * rs)
            for t2 in range(t + 1, 4):
                lc = l[jb + t2]
                for i in range(j + 1, m):
                    if l[i] != 0:
                        p[i, t2] = _madd(-l[i], lc, p[i, t2])
        G[:, jb:jb + 4] = p
        for i in range(jb + 4, m):                   # rank-4 update of the rows below
            for c4 in range(jb + 4, m, 4):
                for e in range(4):
                    c = c4 + e
                    g = G[i, c]
                    for t in range(4):
                        g = _madd(-p[i, t], G[c, jb + t], g)
                    G[i, c] = g
    return np.tril(G[:m, :m]), bad


@pytest.mark.parametrize("m,mp", [(7, 16), (16, 16), (23, 32), (32, 32), (40, 64), (61, 64)])
@pytest.mark.parametrize("kind", ["random", "zero-column", "near-parallel"])
def test_panel_cholesky_matches_the_column_order(m, mp, kind):
    rng = np.random.default_rng(m * 7 + mp)
    A = rng.standard_normal((3 * m, m))
    if kind == "zero-column":
        A[:, m // 2] = 0
    if kind == "near-parallel":
        A[:, m - 1] = A[:, 0] + 1e-3 * rng.standard_normal(3 * m)   # pivot below the minimum
    G = np.zeros((mp, mp))
    G[:m, :m] = A.T @ A
    L1, bad1 = _chol_columns(G, m)
    L2, bad2 = _chol_panels(G, m)
    assert bad1 == bad2 == (kind == "near-parallel")
    np.testing.assert_array_equal(L1, L2)
    if kind == "random":   # and it is the Cholesky factor of the equilibrated Gram
        d = np.sqrt(np.diag(G[:m, :m]))
        ref = np.linalg.cholesky(G[:m, :m] / np.outer(d, d))
        np.testing.assert_allclose(L1, ref, rtol=0, atol=1e-4)
