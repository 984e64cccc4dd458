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
