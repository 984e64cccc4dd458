"""The host-side measurement model (no GPU): the byte accounts behind the bench's
roofline, the compression FLOP model, the scaling of the ncu traffic capture and
the bench's config object.

The float32 byte counts per head-step follow the accounting of Table 17 on the
SEED figures & tables page (GDN stack at the mean column count R + (W - 1) / 2:
26,304 B with lazy decay, 38,144 B with U rewritten; 50,176 B in the Table 2
convention, every state read and written at R + W / 2; 131,072 B dense; KDA
27,136 B; the Mamba-2 stack 20,032 B); the 16-bit counts follow from the same
terms with two bytes per stored U and V value.
"""

import pytest

from rank_recurrent_state_b200 import roofline as rf


def test_float32_byte_accounts():
    cbar = rf.mean_columns(16, 16)
    assert cbar == 23.5
    assert rf.lazy_bytes(0, 128, 128, cbar) == 26304
    assert rf.lazy_bytes(2, 128, 128, cbar) == 26304          # Mamba-2 moves what GDN moves
    assert rf.lazy_bytes(1, 128, 128, cbar) == 27136
    assert rf.explicit_bytes(128, 128, cbar) == 38144
    assert rf.table2_bytes(128, 128, 16, 16) == 50176
    assert rf.dense_bytes(128, 128) == 131072
    assert rf.lazy_bytes(2, 128, 64, rf.mean_columns(8, 32)) == 20032


def test_16bit_byte_accounts():
    cbar = rf.mean_columns(16, 16)
    # U, V values (read c, write one each) at 2 bytes; a, scales (or P) at 4
    gdn = 2 * ((128 + 128) * cbar + 128 + 128) + 4 * (2 * 128 + cbar + (cbar + 1))
    kda = 2 * ((128 + 128) * cbar + 128 + 128) + 4 * (2 * 128 + 2 * 128)
    assert rf.lazy_bytes(0, 128, 128, cbar, 2) == gdn == 13760
    assert rf.lazy_bytes(1, 128, 128, cbar, 2) == kda == 14592
    # halving the factor bytes leaves the per-unit float32 terms
    assert rf.lazy_bytes(0, 128, 128, 19, 4) - rf.lazy_bytes(0, 128, 128, 19, 2) == 2 * (256 * 19 + 256)


def test_compress_flop_model():
    # m = 32, R = 16, d = 128: Grams 2 (256) 32^2, Cholesky + core 4 32^3 / 3,
    # J sweeps of 496 pairs x 6 x 32, 6 32^2 16, 2 (256) 32 16
    m, R = 32, 16
    expect = lambda J: (2 * 256 * m * m + 4 * m ** 3 / 3 + J * (m * (m - 1) / 2) * 6 * m  # noqa: E731
                        + 6 * m * m * R + 2 * 256 * m * R)
    assert rf.compress_flops(128, 128, 16, 16, 0) == pytest.approx(expect(0))
    assert rf.compress_flops(128, 128, 16, 16, 7) == pytest.approx(expect(7))
    assert rf.fp32_peak_tflops(1965.0) == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)


def test_traffic_capture_scales_by_the_byte_model(monkeypatch):
    import bench
    from rank_recurrent_state_b200.seed import Dims
    d = Dims(0, 256, 36, 48, 128, 128, 16, 16)
    cap = {"kernel": bench.decode_kernel_name(d), "form": 0, "d_k": 128, "d_v": 128, "R": 16, "W": 16,
           "factors": 0, "units": 12288, "c": 19, "bytes": 2.9e8}
    monkeypatch.setattr(bench, "NCU_DECODE_TRAFFIC", [cap])
    t = bench.decode_traffic(d, 12288, 19)
    assert t == pytest.approx(cap["bytes"])                       # same units, same column count
    assert bench.decode_traffic(d, 2 * 12288, 19) == pytest.approx(2 * cap["bytes"])
    assert bench.decode_traffic(d, 12288, 23.5) > t                # more columns, more bytes
    other = Dims(2, 256, 40, 64, 128, 64, 8, 32)                  # no capture for this shape
    assert bench.decode_traffic(other, 16384, 23.5) is None


def test_config_object_names_the_workload():
    import bench
    from workloads import config
    cfg = config(2)
    c = bench.config_obj(cfg, cfg.batch, 1, cfg.n_prefill, ragged=False, factors="f16", fused=True)
    assert c["workload"].startswith("gdn-stack") and c["layers"] == 36 and c["heads"] == 48
    assert c["global_batch"] == 256 and c["factors"].startswith("f16") and "fused" in c["compression"]
    assert "L2" in c["l2"]


def test_kernel_launch_counts():
    import bench
    from rank_recurrent_state_b200.seed import Dims
    gdn = Dims(0, 256, 36, 48, 128, 128, 16, 16)
    m2 = Dims(2, 256, 40, 64, 128, 64, 8, 32)          # R + W = 40: wide Cholesky QR + Householder
    kda96 = Dims(1, 512, 20, 32, 128, 128, 32, 64)      # R + W = 96: Householder only
    tiny = Dims(0, 1, 1, 2, 16, 16, 4, 4)               # d = 16: Householder only
    assert bench.compress_kernel_launches(gdn) == 2 and bench.compress_kernel_launches(m2) == 2
    assert bench.compress_kernel_launches(kda96) == 1 and bench.compress_kernel_launches(tiny) == 1
    assert bench.fused_kernel_launches(gdn) == 2
    assert bench.fused_kernel_launches(m2) == 3 and bench.fused_kernel_launches(tiny) == 2


def test_bench_steady_state_is_independent_of_the_timed_window():
    """The headline step time is that of one compression window whatever K steps the
    window held: t_step = (sum_c layers x t_dec(c) + t_cmp) / W, column counts the
    window missed filled by the line through the measured ones."""
    import bench
    R, W, L = 16, 16, 36
    t_dec = lambda c: 0.040 + 0.001 * c   # noqa: E731  (ms, linear in the columns)
    t_cmp = 40.0
    exact = (L * sum(t_dec(c) for c in range(R, R + W)) + t_cmp) / W
    for warmup, steps in ((5, 20), (16, 320), (3, 7), (0, 16)):
        dec = []
        c = R + warmup % W
        for s in range(steps):
            dec += [(t_dec(c), c)] * L
            c = R if c + 1 == R + W else c + 1
        st = bench.steady_state(dec, [t_cmp], R, W, L)
        assert abs(st["ms_per_step"] - exact) <= 1e-9 * exact, (warmup, steps, st)


def test_step_wide_decode_timing_gives_the_same_steady_state():
    """With overlapped layer launches the bench times each step's L decode launches
    with one event pair; per_launch_times spreads it over the L launches, so the
    steady state equals that of per-launch events with the same total per step."""
    import bench

    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    R, W, L = 16, 16, 36
    per_launch, per_step = [], []
    clock, c = 0.0, R
    for s in range(2 * W):
        t0 = clock
        for _ in range(L):
            per_launch.append((Ev(clock), Ev(clock + 0.04 + 0.001 * c), c, 1))
            clock += 0.04 + 0.001 * c
        per_step.append((Ev(t0), Ev(clock), c, L))
        c = R if c + 1 == R + W else c + 1
    a = bench.per_launch_times(per_launch)
    b = bench.per_launch_times(per_step)
    assert len(a) == len(b) == 2 * W * L
    sa = bench.steady_state(a, [40.0], R, W, L)
    sb = bench.steady_state(b, [40.0], R, W, L)
    assert abs(sa["ms_per_step"] - sb["ms_per_step"]) <= 1e-9 * sa["ms_per_step"]
