"""Host emulations of the index logic inside the kernels (no GPU).

1. The register Jacobi of the fast compression (jacobi_regs): MP / 2 slots each
   hold a column pair (x, y); within a group of G slots the x columns shift by one
   slot per round for G rounds, then every group halves: the first half's slots
   take their partners' x as their y, the second half's take their partners' y as
   their x.  Every one of the MP (MP - 1) / 2 column pairs must meet exactly once
   per sweep, whatever the arrangement a sweep starts from.
2. The transposed warp reduction (warp_xreduce<NV>): after it, lane l holds the
   total of value (l >> (5 - log2 NV)) & (NV - 1).
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
