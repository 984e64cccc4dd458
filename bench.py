#!/usr/bin/env python
"""Throughput of the SEED decode hot path on B200: head-steps/s and HBM GB/s.

A step is one pass of the whole hot path over one batch: the decode step of
every layer (one launch per layer; layers after the first through
seed_decode_step_overlapped, so that each starts during the previous one's tail),
and seed_compress over all layers after the step that fills R + W columns.
Default workload: 36 GDN layers x 48 heads of 128 x 128, R = W = 16, batch 256
requests per GPU (the full recurrent stack).

Timing: W untimed warm-up steps, then K steps between barriers and device
synchronisations, CUDA events on the launching stream (max over ranks).  The
headline is the steady state of a compression window, from the events of each
step's decode launches and of each compression.  Inputs (q, k, v, alpha, beta of
a pool of distinct steps) are generated on the device before the timed region
and are larger than L2, as is the 15 GB state.  The end-to-end figure copies a
step's inputs from pinned host memory and its o back inside its own timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun), every rank runs its own requests (weak scaling, no
collective on the data path).  Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode head-steps/s and achieved HBM GB/s (% of B200 peak) at R=16,W=16"
UNIT = "head-steps/s"
NOMINAL_HBM_GBS = 8000.0
# DRAM bytes (read + write) of one decode launch, measured by ncu (dram__bytes_read.sum +
# dram__bytes_write.sum, one captured launch on one B200) for a full
# per-layer launch of the GDN stack shape (256 requests x 48 heads) at c stored columns,
# per factor format.  Remove an entry whenever that kernel changes, until it is measured
# again (no entry: the line's roofline.traffic is null).
NCU_DECODE_TRAFFIC = [
    # decode_ring_kernel, float32 factors, layer 0 of step 3 after the conversion (c = 19):
    # dram__bytes_read.sum 266.10 MB + dram__bytes_write.sum 18.97 MB
    {"kernel": "decode_ring_kernel", "form": 0, "d_k": 128, "d_v": 128, "R": 16, "W": 16, "factors": 0,
     "units": 12288, "c": 19, "bytes": 285.08e6},
    # decode_warp_kernel, float16 factors, the same launch: 146.50 MB + 10.29 MB
    {"kernel": "decode_warp_kernel", "form": 0, "d_k": 128, "d_v": 128, "R": 16, "W": 16, "factors": 1,
     "units": 12288, "c": 19, "bytes": 156.79e6},
]
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=320)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=2, help="workload id (2: the full GDN stack)")
    ap.add_argument("--batch", type=int, default=None, help="requests per GPU (default: the workload's)")
    ap.add_argument("--prefill", type=int, default=None, help="prefill tokens (default: the workload's)")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers (default: the workload's; fewer only for a small profiling case)")
    ap.add_argument("--input-steps", type=int, default=48,
                    help="distinct pre-generated input steps, cycled (>= 3 W so that a key comes "
                         "back only after its old copy has decayed)")
    ap.add_argument("--factors", default="f32", choices=["f32", "f16", "bf16"],
                    help="storage format of the factors U and V (arithmetic stays f32)")
    ap.add_argument("--fused", action="store_true",
                    help="compress inside the decode launch of the step that fills R + W "
                         "(seed_decode_step_compress) instead of a separate compression launch")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch every layer's decode step plainly (seed_decode_step) instead of "
                         "letting it begin during the previous layer's (seed_decode_step_overlapped); "
                         "also times every launch with its own CUDA events")
    ap.add_argument("--ragged", action="store_true",
                    help="ragged compression schedules: requests joined at different times, a "
                         "compression launch after every step compresses the units that are due")
    ap.add_argument("--dense-steps", type=int, default=8)
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="end-to-end steps (default: one compression window, W)")
    ap.add_argument("--e2e-copy", default="step", choices=["step", "layer"],
                    help="end-to-end copy granularity: one copy per input tensor per step (all "
                         "layers, into a ring of device slots) and o out once per step, or five "
                         "copies in and one out per layer")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-units", type=int, default=384,
                    help="units of the workload the reference arm (the fp64 oracle) steps")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = os.environ.get("SEED_BENCH_BACKEND", "nccl")
        kw = {"timeout": datetime.timedelta(seconds=180)}
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, **kw)
    return world, rank, local


def shard(batch_per_rank: int, rank: int) -> int:
    """First global request index of this rank's shard (requests are independent)."""
    return rank * batch_per_rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None) -> None:
    if world > 1:
        import torch.distributed as dist
        if device is not None and device != "cpu":
            dist.barrier(device_ids=[device.index if hasattr(device, "index") else int(device)])
        else:
            dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.proc = None
        self.gpu_index = gpu_index
        self.enabled = enabled

    def __enter__(self):
        if self.enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (OSError, ValueError):
                self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self) -> dict | None:
        rows = []
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        load = [r[0] for r in rows]
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ peaks

def measured_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ CPU (oracle) arm

def cpu_oracle_rate(cfg, seconds: float, rank_seed: int = 0) -> dict:
    """Time the fp64 oracle's decode step + compression on a sample of units."""
    import numpy as np

    from oracle import compress as ocomp
    from oracle import convert as oconv
    from oracle import factored, recurrences
    from workloads import philox
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:   # pragma: no cover - reporting only
        threads = 1
    rng = np.random.default_rng(1234 + rank_seed)
    n = min(96, cfg.units)   # the sample, or every unit of a small workload
    u = rng.choice(cfg.units, size=n, replace=False)
    b, rem = np.divmod(u, cfg.layers * cfg.heads)
    l, h = np.divmod(rem, cfg.heads)
    n_pre = 256
    S0 = recurrences.dense_prefill(cfg, b, l, h, n_pre)
    vb = philox.vbar(cfg, l, h).astype(np.float64)
    a, U, V, _ = oconv.convert(S0, vb, cfg.R)
    inputs = [recurrences.f64(philox.token_inputs(cfg, b, l, h, t, philox.PHASE_DECODE))
              for t in range(cfg.W)]
    steps = 0
    c = cfg.R
    t0 = time.perf_counter()
    while True:
        for t in range(cfg.W):
            inp = inputs[t]
            a, U, V, _o = factored.step(cfg.form, a, U, V, vb, inp["q"], inp["k"], inp["v"],
                                        inp["alpha"], inp["beta"])
            c += 1
            if c == cfg.R + cfg.W:
                U, V, _s = ocomp.truncate_qr_core(U, V, cfg.R)
                c = cfg.R
            steps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": steps * n / dt, "unit": UNIT, "cores": int(threads), "kind": "oracle",
            "sample": (f"{n} sampled units of the workload, {steps} decode steps each "
                       f"({steps // cfg.W} compressions), fp64 NumPy, {dt:.1f} s; "
                       f"state from a {n_pre}-token oracle prefill (untimed)"),
            "affinity_cores": len(os.sched_getaffinity(0))}


def config_obj(cfg, batch, world, prefill, ragged=False, factors="f32", fused=False):
    schedule = ("ragged: request b joined W-1-floor(bW/B) steps before the others; a compression "
                "launch after every step compresses the units that are due" if ragged else
                "lockstep: every unit compresses after steps W, 2W, ...")
    return {"workload": f"{cfg.name}: {cfg.layers} GDN layers x {cfg.heads} heads, "
                        f"d_k=d_v={cfg.d_k}, R={cfg.R}, W={cfg.W}" if cfg.form == 0 else cfg.name,
            "form": {0: "gdn", 1: "kda", 2: "mamba2"}[cfg.form], "layers": cfg.layers,
            "heads": cfg.heads, "d_k": cfg.d_k, "d_v": cfg.d_v, "R": cfg.R, "W": cfg.W,
            "batch_per_gpu": batch, "global_batch": batch * world, "prefill_tokens": prefill,
            "parallelism": f"dp{world} (requests sharded, no collective)",
            "schedule": schedule,
            "compression": ("fused into the decode launch of the step that fills R + W" if fused
                            else "a separate launch over all units after the step that fills R + W"),
            "factors": factors + (" (U and V stored in 16 bits, rounded to nearest when written)"
                                  if factors != "f32" else ""),
            "l2": "inputs and state larger than L2 (no flush needed)"}


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle, as it stands, on the host cores.  Each of
    the W warm-up and K timed steps is one decode step (and the compression when it
    is due) of a fixed seeded sample of the workload's units; value = K x sample /
    the timed seconds.  Rank 0 alone runs it."""
    import numpy as np

    from oracle import compress as ocomp
    from oracle import convert as oconv
    from oracle import factored, recurrences
    from workloads import config, philox
    cfg = config(args.config)
    if args.batch:
        cfg = cfg.replace(batch=args.batch)
    if args.layers:
        cfg = cfg.replace(layers=args.layers)
    if rank != 0:
        return 0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:   # pragma: no cover - reporting only
        threads = 1
    n = min(args.reference_units, cfg.units)
    rng = np.random.default_rng(1234)
    u = rng.choice(cfg.units, size=n, replace=False)
    b, rem = np.divmod(u, cfg.layers * cfg.heads)
    l, h = np.divmod(rem, cfg.heads)
    n_pre = 256
    S0 = recurrences.dense_prefill(cfg, b, l, h, n_pre)
    vb = philox.vbar(cfg, l, h).astype(np.float64)
    a, U, V, _ = oconv.convert(S0, vb, cfg.R)
    c = cfg.R
    P = max(args.input_steps, 1)
    inputs = {}

    def step(t):
        nonlocal a, U, V, c
        if t % P not in inputs:
            inputs[t % P] = recurrences.f64(philox.token_inputs(cfg, b, l, h, t % P, philox.PHASE_DECODE))
        inp = inputs[t % P]
        a, U, V, _o = factored.step(cfg.form, a, U, V, vb, inp["q"], inp["k"], inp["v"],
                                    inp["alpha"], inp["beta"])
        c += 1
        if c == cfg.R + cfg.W:
            U, V, _s = ocomp.truncate_qr_core(U, V, cfg.R)
            c = cfg.R

    for t in range(min(P, args.warmup + args.steps)):   # input generation, outside the timing
        if t not in inputs:
            inputs[t] = recurrences.f64(philox.token_inputs(cfg, b, l, h, t, philox.PHASE_DECODE))
    for t in range(args.warmup):
        step(t)
    t0 = time.perf_counter()
    for t in range(args.steps):
        step(args.warmup + t)
    dt = time.perf_counter() - t0
    value = args.steps * n / dt
    prefill = cfg.n_prefill if args.prefill is None else args.prefill
    sample = (f"{n} seeded units of the workload (of {cfg.units}), each step one fp64 NumPy decode step of "
              f"all of them plus the compression when due; {args.steps} timed steps after {args.warmup} "
              f"warm-up steps, {dt:.2f} s; the sample's state comes from a {n_pre}-token oracle prefill "
              f"and conversion (untimed), inputs pre-generated")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Philox4x32-10 inputs)", "impl": "reference",
            "config": config_obj(cfg, cfg.batch, world, prefill),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(threads), "kind": "oracle",
                             "sample": sample, "affinity_cores": len(os.sched_getaffinity(0))},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "note": "ms_per_step is the measured time of one step of the sample, not of the whole workload"}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def decode_kernel_name(d):
    if d.R + d.W - 1 > 64:
        return "decode_step_kernel"
    return "decode_ring_kernel" if d.factors == 0 else "decode_warp_kernel"


def decode_traffic(d, units, cbar):
    """DRAM bytes per decode launch from the ncu capture, scaled from its units and
    column count to this launch's by the state + input/output bytes; None when the
    capture does not match this kernel and shape."""
    from rank_recurrent_state_b200 import roofline
    key = (decode_kernel_name(d), d.form, d.d_k, d.d_v, d.R, d.W, d.factors)
    match = [t for t in (NCU_DECODE_TRAFFIC or [])
             if (t["kernel"], t["form"], t["d_k"], t["d_v"], t["R"], t["W"], t["factors"]) == key]
    if not match:
        return None
    t = match[0]
    fb = 4 if d.factors == 0 else 2
    per = lambda c: roofline.lazy_bytes(d.form, d.d_k, d.d_v, c, fb) + roofline.io_bytes(d.form, d.d_k, d.d_v)  # noqa: E731
    return t["bytes"] / t["units"] * units * per(cbar) / per(t["c"])


def compress_kernel_launches(d) -> int:
    """Kernels one seed_compress call launches: a Cholesky-QR kernel where the shape
    allows one (R + W <= 32 with R <= 16, or 32 < R + W <= 64 with R <= 32; d_k, d_v in
    {64, 128}), then the Householder scan over the units still due."""
    dims_ok = d.d_k in (64, 128) and d.d_v in (64, 128)
    fast = d.R + d.W <= 32 and d.R <= 16
    wide = 32 < d.R + d.W <= 64 and d.R <= 32
    return 2 if dims_ok and (fast or wide) else 1


def fused_kernel_launches(d) -> int:
    """Kernels one seed_decode_step_compress call launches: the fused kernel and the
    Householder scan, or a decode launch and a compression."""
    if d.R + d.W - 1 <= 32 and compress_kernel_launches(d) == 2:
        return 2
    return 1 + compress_kernel_launches(d)


def compress_rate(d, diag, cmp_ms, clk):
    """FP32 rate of the compression launches (the FLOP model of roofline.compress_flops,
    with the measured mean Jacobi sweeps) and its fraction of the CUDA-core FP32 peak
    at the median SM clock sampled during the timed region."""
    from rank_recurrent_state_b200 import roofline
    if not cmp_ms or not diag["compress_units"]:
        return {}
    sweeps = diag["compress_sweeps"] / diag["compress_units"]
    flops = roofline.compress_flops(d.d_k, d.d_v, d.R, d.W, sweeps) * d.units
    tflops = flops / (sum(cmp_ms) / len(cmp_ms) / 1e3) / 1e12
    mhz = (clk or {}).get("sm_mhz") or 1965.0
    peak = roofline.fp32_peak_tflops(mhz)
    return {"flops_per_unit": flops / d.units, "tflops": tflops, "fp32_peak_tflops": peak,
            "frac_fp32_peak": tflops / peak}


def per_launch_times(records):
    """Decode timings per launch, (ms, column count), from the timed region's event
    records (start, end, c, n): n = 1 for a launch timed alone; n = L for one event
    pair around a step's L overlapped launches (an event between two launches would
    serialise them), which gives each of the L launches an equal share."""
    out = []
    for a, b, c, n in records:
        out += [(a.elapsed_time(b) / n, c)] * n
    return out


def steady_state(dec, cmp_ms, R, W, layers):
    """Steady-state step time from the run's own per-launch CUDA-event times.

    In lockstep every unit holds c = R, R + 1, ..., R + W - 1 columns before the
    W steps of one compression window, and one compression closes the window, so
    a step costs on average

        t_step = ( sum_c layers * t_dec(c) + t_cmp ) / W

    with t_dec(c) the mean decode-launch time at column count c and t_cmp the mean
    compression time.  Column counts the timed window did not reach take the
    least-squares line through the measured ones (the launch moves bytes linear
    in c).  dec: list of (ms, c).  Returns a dict (ms per step, the per-c means)."""
    import numpy as np
    by_c = {}
    for ms, c in dec:
        by_c.setdefault(int(round(c)), []).append(ms)
    cs = np.array(sorted(by_c), dtype=np.float64)
    means = np.array([sum(by_c[int(c)]) / len(by_c[int(c)]) for c in cs])
    if cs.size >= 2:
        slope, icpt = np.polyfit(cs, means, 1)
    else:
        slope, icpt = 0.0, float(means[0])
    window_cs = range(R, R + W)
    t_dec = {c: (sum(by_c[c]) / len(by_c[c]) if c in by_c else icpt + slope * c) for c in window_cs}
    t_cmp = sum(cmp_ms) / len(cmp_ms) if cmp_ms else 0.0
    dec_window = layers * sum(t_dec.values())
    return {"ms_per_step": (dec_window + t_cmp) / W, "decode_ms_per_launch_mean": sum(t_dec.values()) / W,
            "compress_ms": t_cmp, "decode_share": dec_window / (dec_window + t_cmp),
            "column_counts_measured": int(cs.size), "column_counts_in_window": W}


def gpu_numa_affinity(local: int):
    """CPUs local to this rank's GPU (NVML), or None when NVML cannot tell."""
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
            idx = int(visible[local]) if len(visible) > local and visible[local].isdigit() else local
            h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            n = (os.cpu_count() + 63) // 64
            masks = pynvml.nvmlDeviceGetCpuAffinity(h, n)
        finally:
            pynvml.nvmlShutdown()
    except Exception:   # pragma: no cover - reporting only
        return None
    cpus = {64 * i + b for i, m in enumerate(masks) for b in range(64) if (int(m) >> b) & 1}
    cpus &= os.sched_getaffinity(0)
    return cpus or None


def run_e2e(args, run, d, L, BH, q, k, v, alpha, beta, o, kda, stream, dev, world, local, units, step_ms, s_next):
    """The same metric through the public API with host buffers: every step copies its
    inputs from pinned host memory to the device and its o back, inside the timed
    region.  Timed over W steps (one compression) from the middle of a compression
    window; also measures the host link alone in the same run."""
    import torch

    from rank_recurrent_state_b200 import seed as S
    # pinned buffers on the GPU's NUMA node: allocate them from a thread bound to the
    # CPUs local to the GPU (pages are placed on the allocating thread's node)
    aff = gpu_numa_affinity(local)
    old_aff = os.sched_getaffinity(0)
    if aff:
        os.sched_setaffinity(0, aff)
    # the host pool cycles as many distinct steps as the device pool (3 W by default),
    # so that the W columns a window appends are distinct keys as in the timed loop; a
    # pool of a few steps repeats keys inside a window, and the compression then meets
    # rank-deficient factors (the Householder fallback) that the workload never has
    step_bytes = (q[0].numel() + k[0].numel() + v[0].numel() + alpha[0].numel() + beta[0].numel()) * 4
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except ImportError:
        avail = 64 << 30
    # a quarter of the host memory, shared by the ranks on this node
    ranks_here = max(1, int(os.environ.get("LOCAL_WORLD_SIZE", world)))
    Ph = max(2, min(q.shape[0], int(0.25 * avail / ranks_here) // step_bytes))
    try:
        hq = torch.empty(Ph, L, BH, d.d_k, dtype=torch.float32, pin_memory=True)
        hk = torch.empty_like(hq, pin_memory=True)
        hv = torch.empty(Ph, L, BH, d.d_v, dtype=torch.float32, pin_memory=True)
        ha = torch.empty(Ph, *alpha.shape[1:], dtype=torch.float32, pin_memory=True)
        hb = torch.empty(Ph, *beta.shape[1:], dtype=torch.float32, pin_memory=True)
        ho = torch.empty(L, BH, d.d_v, dtype=torch.float32, pin_memory=True)
    finally:
        if aff:
            os.sched_setaffinity(0, old_aff)
    for t in range(Ph):
        hq[t].copy_(q[t]); hk[t].copy_(k[t]); hv[t].copy_(v[t]); ha[t].copy_(alpha[t]); hb[t].copy_(beta[t])
    # inputs copied in on their own stream into a ring of device slots, outputs copied
    # out on a third, so that the transfers (host memory and PCIe bound) overlap the
    # decode launches.  "step": one slot holds a whole step (all layers); "layer": one
    # layer's inputs, with each layer's o copied out as soon as it is written
    per_step = args.e2e_copy == "step"
    nb = 3 if per_step else 2
    overlap = per_step and not (args.no_overlap or args.fused or args.ragged)   # as in the timed loop
    if per_step:
        bufs = [(torch.empty_like(q[0]), torch.empty_like(k[0]), torch.empty_like(v[0]),
                 torch.empty_like(alpha[0]), torch.empty_like(beta[0]), torch.empty_like(o)) for _ in range(nb)]
    else:
        bufs = [(torch.empty_like(q[0, 0]), torch.empty_like(k[0, 0]), torch.empty_like(v[0, 0]),
                 torch.empty_like(alpha[0, 0]), torch.empty_like(beta[0, 0])) for _ in range(nb)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nb)]
    ev_free = [torch.cuda.Event() for _ in range(nb)]
    ev_dec = [torch.cuda.Event() for _ in range(L)]
    ev_out = [torch.cuda.Event() for _ in range(max(L, nb))]
    h2d = (1 if per_step else L) * sum(x.numel() for x in bufs[0][:5]) * 4   # as copied
    d2h = o.numel() * 4

    # the host link alone: one step's inputs in (all layers, one copy per tensor), the
    # outputs out, then both at once (PCIe is full duplex)
    def timed(fn, reps=3):
        best = None
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        return best

    def h2d_all():
        q[1].copy_(hq[0], non_blocking=True); k[1].copy_(hk[0], non_blocking=True)
        v[1].copy_(hv[0], non_blocking=True); alpha[1].copy_(ha[0], non_blocking=True)
        beta[1].copy_(hb[0], non_blocking=True)

    def d2h_all():
        ho.copy_(o, non_blocking=True)

    def both():
        s_in.wait_stream(stream)
        with torch.cuda.stream(s_in):
            h2d_all()
        d2h_all()
        stream.wait_stream(s_in)

    h2d_bytes_all = (hq[0].numel() + hk[0].numel() + hv[0].numel() + ha[0].numel() + hb[0].numel()) * 4
    t_h2d, t_d2h, t_both = timed(h2d_all), timed(d2h_all), timed(both)
    link = {"h2d_GBps": h2d_bytes_all / (t_h2d / 1e3) / 1e9, "d2h_GBps": d2h / (t_d2h / 1e3) / 1e9,
            "duplex_ms_per_step": t_both, "pinned_on_gpu_numa_node": bool(aff),
            "gpu_local_cpus": len(aff) if aff else None}
    # restore the pool's step-1 inputs overwritten by the link test
    for l in range(L):
        al = alpha[1, l] if kda else alpha[1, l, :BH]
        S.seed_synth_token_inputs(d, run.key, S.SEED_PHASE_DECODE, 1, l, run.vbar, q[1, l], k[1, l],
                                  v[1, l], al, beta[1, l, :BH])
    bound_ms = max(t_both, step_ms)   # copies overlapped with the device work at best

    # align, untimed, to the middle of a compression window (c = R + W/2), cycling the
    # device pool's steps: the W timed steps then hold one compression, in their middle,
    # where the next steps' input copies overlap it as they do in a long run (a window
    # that ends with its compression leaves nothing to overlap it)
    P = q.shape[0]
    c_start = d.R + d.W // 2
    while run.c != c_start and not args.ragged:
        t = s_next % P
        for l in range(L):
            S.seed_decode_step(d, run.state, l, q[t, l], k[t, l], v[t, l],
                               alpha[t, l] if kda else alpha[t, l, :BH], beta[t, l, :BH], o[l], run.ws, stream)
        s_next += 1
        run.c += 1
        if run.c == d.m:
            S.seed_compress(d, run.state, S.SEED_ALL_LAYERS, run.ws, stream=stream)
            run.c = d.R
    n_steps = args.e2e_steps if args.e2e_steps else d.W
    torch.cuda.synchronize()
    diag0 = S.seed_get_diagnostics(run.ws)
    cmp_ev = []
    barrier(world, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    n = 0
    t_host = time.perf_counter()
    for s in range(n_steps):
        t = (s_next + s) % Ph   # the pool's steps in the order the timed loop left them
        fuse = args.fused and (args.ragged or run.c + 1 == d.m)
        step_fn = S.seed_decode_step_compress if fuse else S.seed_decode_step
        if per_step:
            j = s % nb
            bq, bk, bv, ba, bb, bo = bufs[j]
            with torch.cuda.stream(s_in):
                if s >= nb:
                    s_in.wait_event(ev_free[j])   # step s - nb's launches have read the slot
                bq.copy_(hq[t], non_blocking=True); bk.copy_(hk[t], non_blocking=True)
                bv.copy_(hv[t], non_blocking=True); ba.copy_(ha[t], non_blocking=True)
                bb.copy_(hb[t], non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if s >= nb:
                stream.wait_event(ev_out[j])   # step s - nb's o has left the slot
            for l in range(L):
                fn = S.seed_decode_step_overlapped if (overlap and not fuse and l > 0) else step_fn
                fn(d, run.state, l, bq[l], bk[l], bv[l], ba[l] if kda else ba[l, :BH], bb[l, :BH], bo[l],
                   run.ws, stream=stream)
            ev_free[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_free[j])
                ho.copy_(bo, non_blocking=True)
                ev_out[j].record(s_out)
            n += L
        else:
            for l in range(L):
                bi = n % nb
                bq, bk, bv, ba, bb = bufs[bi]
                with torch.cuda.stream(s_in):
                    if n >= nb:
                        s_in.wait_event(ev_free[bi])
                    bq.copy_(hq[t, l], non_blocking=True); bk.copy_(hk[t, l], non_blocking=True)
                    bv.copy_(hv[t, l], non_blocking=True); ba.copy_(ha[t, l], non_blocking=True)
                    bb.copy_(hb[t, l], non_blocking=True)
                    ev_in[bi].record(s_in)
                stream.wait_event(ev_in[bi])
                if s > 0:
                    stream.wait_event(ev_out[l])   # last step's o of this layer is out
                step_fn(d, run.state, l, bq, bk, bv, ba if kda else ba[:BH], bb[:BH], o[l], run.ws, stream=stream)
                ev_free[bi].record(stream)
                ev_dec[l].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_dec[l])
                    ho[l].copy_(o[l], non_blocking=True)
                    ev_out[l].record(s_out)
                n += 1
        run.c += 1
        if run.c == d.m or args.ragged:   # ragged: some request is due after every step
            if not fuse:
                cmp_ev.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
                cmp_ev[-1][0].record(stream)
                S.seed_compress(d, run.state, S.SEED_ALL_LAYERS, run.ws, stream=stream)
                cmp_ev[-1][1].record(stream)
            run.c = d.R
    host_ms = (time.perf_counter() - t_host) * 1e3
    stream.wait_stream(s_out)
    stream.wait_stream(s_in)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world, dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    step_e2e = e2e_ms / n_steps
    diag1 = S.seed_get_diagnostics(run.ws)
    e2e_cmp = {"launches": len(cmp_ev),
               "ms_per_launch": (sum(a.elapsed_time(b) for a, b in cmp_ev) / len(cmp_ev)) if cmp_ev else None,
               "cholqr_units": diag1["cholqr_units"] - diag0["cholqr_units"],
               "householder_units": diag1["householder_units"] - diag0["householder_units"]}
    return {"value": n_steps * units * world / (e2e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_steps,
            "ms_per_step": step_e2e,
            "h2d_GBps_achieved": h2d / (step_e2e / 1e3) / 1e9, "d2h_GBps_achieved": d2h / (step_e2e / 1e3) / 1e9,
            "copies": args.e2e_copy, "host_enqueue_ms_per_step": host_ms / n_steps,
            "host_pool_steps": Ph, "compress": e2e_cmp,
            "host_link": link,
            "host_link_bound_value": units * world / (bound_ms / 1e3),
            "frac_of_host_link_bound": bound_ms / step_e2e,
            "note": "pinned host buffers; every step copies its inputs in and its o out (copies on their own "
                    "streams, overlapping the decode launches; 'copies' = step: one copy per tensor for all "
                    "layers into a ring of three device slots, layer: per layer into two); timed over W steps "
                    "(default) from the middle of a compression window, so that they hold one compression "
                    "with copies around it; host_link_bound_value = units / max(device "
                    "step, one step's input and output copies run alone and together)"}


def run_ours(args, world, rank, local):
    import torch

    from rank_recurrent_state_b200 import build as build_mod
    from rank_recurrent_state_b200 import roofline
    from rank_recurrent_state_b200 import seed as S
    from rank_recurrent_state_b200.pipeline import DeviceRun
    from workloads import config

    if rank == 0 or not os.path.exists(build_mod.LIB):
        build_mod.build()
    if world > 1:
        barrier(world, None)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = config(args.config)
    if args.batch:
        cfg = cfg.replace(batch=args.batch)
    if args.layers:
        cfg = cfg.replace(layers=args.layers)
    B = cfg.batch
    prefill = cfg.n_prefill if args.prefill is None else args.prefill
    run = DeviceRun(cfg, b0=shard(B, rank), device=str(dev), n_prefill=prefill,
                    keep_dense=not args.no_dense and not args.ragged, ragged=args.ragged,
                    factors=S.FACTOR_NAMES[args.factors])
    d = run.dims
    fb = 4 if args.factors == "f32" else 2   # bytes per stored U / V value
    t_setup = time.perf_counter()
    run.prefill_and_convert()
    if args.ragged:
        run.lead_in(S.alloc_step_inputs(d, dev))
    torch.cuda.synchronize()
    t_setup = time.perf_counter() - t_setup

    # ---- input pool: P distinct steps x L layers, generated on the device
    P, L, BH = args.input_steps, d.layers, d.batch * d.heads
    BHp = (BH + 3) // 4 * 4
    f32 = dict(dtype=torch.float32, device=dev)
    q = torch.empty(P, L, BH, d.d_k, **f32)
    k = torch.empty(P, L, BH, d.d_k, **f32)
    v = torch.empty(P, L, BH, d.d_v, **f32)
    kda = d.form == S.SEED_KDA
    alpha = torch.empty(P, L, BH, d.d_k, **f32) if kda else torch.empty(P, L, BHp, **f32)
    beta = torch.empty(P, L, BHp, **f32)
    for t in range(P):
        for l in range(L):
            al = alpha[t, l] if kda else alpha[t, l, :BH]
            S.seed_synth_token_inputs(d, run.key, S.SEED_PHASE_DECODE, t, l, run.vbar, q[t, l], k[t, l],
                                      v[t, l], al, beta[t, l, :BH])
    o = torch.empty(L, BH, d.d_v, **f32)
    stream = torch.cuda.current_stream(dev)

    def inputs(t, l):
        return (q[t, l], k[t, l], v[t, l], alpha[t, l] if kda else alpha[t, l, :BH], beta[t, l, :BH])

    # layers after the first step through seed_decode_step_overlapped: the launch before
    # each is the previous layer's step, which writes none of its state
    overlap = not (args.no_overlap or args.fused or args.ragged)

    def one_step(s, ev=None):
        t = s % P
        fuse = args.fused and (args.ragged or run.c + 1 == d.m)
        for l in range(L):
            qq, kk, vv, aa, bb = inputs(t, l)
            if fuse:
                if ev is not None:
                    ev["fus"].append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
                    ev["fus"][-1][0].record(stream)
                S.seed_decode_step_compress(d, run.state, l, qq, kk, vv, aa, bb, o[l], run.ws, stream=stream)
                if ev is not None:
                    ev["fus"][-1][1].record(stream)
                continue
            # overlapped launches: an event between two launches would serialise them,
            # so one event pair spans the step's L launches (n = L in the record)
            timed_here = ev is not None and (not overlap or l == 0)
            if timed_here:
                ev["dec"].append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                                  roofline.mean_columns(d.R, d.W) if args.ragged else run.c, L if overlap else 1))
                ev["dec"][-1][0].record(stream)
            step_fn = S.seed_decode_step_overlapped if (overlap and l > 0) else S.seed_decode_step
            step_fn(d, run.state, l, qq, kk, vv, aa, bb, o[l], run.ws, stream)
            if ev is not None and (not overlap or l == L - 1):
                ev["dec"][-1][1].record(stream)
        run.c += 1
        if fuse:
            run.c = d.R if run.c == d.m else run.c
        elif run.c == d.m or args.ragged:
            if ev is not None:
                ev["cmp"].append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
                ev["cmp"][-1][0].record(stream)
            S.seed_compress(d, run.state, S.SEED_ALL_LAYERS, run.ws, stream=stream)
            if ev is not None:
                ev["cmp"][-1][1].record(stream)
            run.c = d.R

    for s in range(args.warmup):
        one_step(s)
    torch.cuda.synchronize()
    flags_warm = S.seed_get_status(run.ws)

    ev = {"dec": [], "cmp": [], "fus": []}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    gpu_index = int(visible[local]) if len(visible) > local and visible[local].isdigit() else local
    barrier(world, dev)
    torch.cuda.synchronize()
    with ClockSampler(gpu_index, enabled=not args.no_clocks) as clk:
        start.record(stream)
        for s in range(args.steps):
            one_step(args.warmup + s, ev)
        end.record(stream)
        torch.cuda.synchronize()
    barrier(world, dev)
    elapsed_ms = max_over_ranks(start.elapsed_time(end), world, dev)
    flags = S.seed_get_status(run.ws)
    diag = S.seed_get_diagnostics(run.ws)
    s_next = args.warmup + args.steps

    units = d.units
    dec_pairs = per_launch_times(ev["dec"])
    cmp_ms = [a.elapsed_time(b) for a, b in ev["cmp"]]
    fus_ms = [a.elapsed_time(b) for a, b in ev["fus"]]
    extra_cmp = False
    if not args.ragged and not cmp_ms and not fus_ms and d.m - d.R > 0:
        # the timed window held no compression (fewer steps than W): time the next
        # one, after the timed region, so that the steady state below has its cost
        while True:
            due = run.c + 1 == d.m
            ev2 = {"dec": [], "cmp": [], "fus": []}
            one_step(s_next, ev2)
            s_next += 1
            if due:
                break
        torch.cuda.synchronize()
        cmp_ms = [a.elapsed_time(b) for a, b in ev2["cmp"]]
        fus_ms = [a.elapsed_time(b) for a, b in ev2["fus"]]
        extra_cmp = True
        diag2 = S.seed_get_diagnostics(run.ws)
        for key in diag:
            diag[key] += diag2[key]
        flags |= S.seed_get_status(run.ws)
    raw_value = args.steps * units * world / (elapsed_ms / 1e3)
    # steady state of one compression window (lockstep), from the per-launch times
    if args.ragged:
        steady = None   # every step holds every column count and compresses 1/W of the units
        step_ms = elapsed_ms / args.steps
    elif args.fused:
        # the fused launches replace the decode launches of the window's last step and
        # the compression: window = decode at c = R .. R + W - 2, then the fused launches
        steady = steady_state(dec_pairs, [], d.R, d.W - 1, L)
        t_fus = sum(fus_ms) / len(fus_ms) if fus_ms else 0.0
        step_ms = (steady["ms_per_step"] * (d.W - 1) + L * t_fus) / d.W
        steady["ms_per_step"] = step_ms
        steady["fused_ms_per_launch"] = t_fus
    else:
        steady = steady_state(dec_pairs, cmp_ms, d.R, d.W, L)
        step_ms = steady["ms_per_step"]
    value = units * world / (step_ms / 1e3)
    step_ms = max_over_ranks(step_ms, world, dev)
    value = units * world / (step_ms / 1e3)
    dec_ms = [ms for ms, _ in dec_pairs]
    if steady is not None and dec_ms:
        dec_launch_ms = steady["decode_ms_per_launch_mean"]
    else:
        dec_launch_ms = sum(dec_ms) / len(dec_ms) if dec_ms else None
    peak, peak_kind = measured_peak_hbm()
    cbar = roofline.mean_columns(d.R, d.W)
    if steady is not None and args.fused:
        cbar = roofline.mean_columns(d.R, d.W - 1)
    # algorithmic bytes of the mean launch of a window (the byte model is linear in c)
    dec_bytes = BH * roofline.lazy_bytes(d.form, d.d_k, d.d_v, cbar, fb)
    dec_gbs = dec_bytes / (dec_launch_ms / 1e3) / 1e9 if dec_launch_ms else None
    t_cmp = sum(cmp_ms) / len(cmp_ms) if cmp_ms else None

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded Philox4x32-10 inputs and prefill, generated on the device)",
        "config": config_obj(cfg, B, world, prefill, args.ragged, args.factors, args.fused),
        "steady_state": (None if steady is None else dict(
            steady, how="value = units / t_step with t_step = (sum over the window's column counts "
                        "c = R .. R+W-1 of layers x t_decode(c) + t_compress) / W, every t the mean "
                        "CUDA-event time of those launches in the timed region"
                        + ("; the compression was timed right after the timed region (fewer timed "
                           "steps than W)" if extra_cmp else ""))),
        "window": {"ms_per_step": elapsed_ms / args.steps, "value": raw_value,
                   "compressions": len(cmp_ms) + len(fus_ms) // max(L, 1) if not extra_cmp else 0,
                   "note": "the K timed steps as they fell, K x units / (max over ranks of the "
                           "event time between the barriers)"},
        "roofline": {"bound": "hbm", "kernel": decode_kernel_name(d), "achieved": dec_gbs, "peak": peak,
                     "unit": "GB/s", "frac": dec_gbs / peak if dec_gbs else None,
                     "peak_source": f"{peak_kind} copy bandwidth",
                     "frac_of_nominal_8TBs": dec_gbs / NOMINAL_HBM_GBS if dec_gbs else None,
                     "traffic": decode_traffic(d, BH, cbar),
                     "algorithmic_bytes_per_head_step_mean": roofline.lazy_bytes(d.form, d.d_k, d.d_v, cbar, fb),
                     "algorithmic_bytes_per_launch": dec_bytes,
                     "avg_launch_us": 1e3 * dec_launch_ms if dec_launch_ms else None,
                     "launches": len(dec_ms),
                     "timing": ("CUDA events around each step's L overlapped launches, divided by L"
                                if overlap else "CUDA events around each launch"),
                     "layer_launches": ("layers after the first begin during the previous layer's launch "
                                        "(seed_decode_step_overlapped, programmatic dependent launch)"
                                        if overlap else "one after another (seed_decode_step)")},
        "decode_only": {"head_steps_per_s": BH * world / (dec_launch_ms / 1e3) if dec_launch_ms else None,
                        "GBps": dec_gbs},
        "compress": {"launches": len(cmp_ms), "ms_per_launch": t_cmp,
                     "ns_per_head_step_amortized": (1e6 * t_cmp / (d.W * units) if t_cmp and not args.ragged
                                                    else 1e6 * sum(cmp_ms) / (args.steps * units)),
                     "share_of_step": ((t_cmp / d.W) / step_ms if t_cmp and not args.ragged
                                       else sum(cmp_ms) / elapsed_ms),
                     "jacobi_sweeps_mean": (diag["compress_sweeps"] / diag["compress_units"]
                                            if diag["compress_units"] else None),
                     "cholqr_units": diag["cholqr_units"], "householder_units": diag["householder_units"],
                     **compress_rate(d, diag, cmp_ms, clk.summary())},
        "gpu_launches": (len(dec_ms) + (len(cmp_ms) if not extra_cmp else 0) * compress_kernel_launches(d)
                         + (len(fus_ms) if not extra_cmp else 0) * fused_kernel_launches(d)),
        "status_flags": flags | flags_warm,
        "setup_s": t_setup,
    }
    if fus_ms:
        line["fused"] = {"launches": len(fus_ms), "ms_per_launch": sum(fus_ms) / len(fus_ms),
                         "note": "decode step of one layer with the compression of its due units "
                                 "(seed_decode_step_compress); the Householder launch for declined "
                                 "units is included"}
    clocks = clk.summary()
    line["clocks"] = clocks

    # ---- dense comparison on the same inputs
    if not args.no_dense and run.dense is not None:
        dev_ms = []
        od = torch.empty(BH, d.d_v, **f32)
        for s in range(2):
            for l in range(L):
                S.seed_dense_step(d, run.dense, l, *inputs(s % P, l), od, run.ws, stream)
        torch.cuda.synchronize()
        for s in range(args.dense_steps):
            for l in range(L):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                S.seed_dense_step(d, run.dense, l, *inputs(s % P, l), od, run.ws, stream)
                e1.record(stream)
                dev_ms.append((e0, e1))
        torch.cuda.synchronize()
        dms = [a.elapsed_time(b) for a, b in dev_ms]
        dense_hs = len(dms) * BH / (sum(dms) / 1e3)
        dense_gbs = len(dms) * BH * roofline.dense_bytes(d.d_k, d.d_v) / (sum(dms) / 1e3) / 1e9
        line["dense"] = {"head_steps_per_s": dense_hs * world, "GBps": dense_gbs, "frac": dense_gbs / peak,
                         "bytes_per_head_step": roofline.dense_bytes(d.d_k, d.d_v)}
        line["speedup_vs_dense"] = {
            "decode_only": line["decode_only"]["head_steps_per_s"] / line["dense"]["head_steps_per_s"],
            "with_compress": value / line["dense"]["head_steps_per_s"],
            "byte_ratio_lazy": roofline.dense_bytes(d.d_k, d.d_v) / roofline.lazy_bytes(d.form, d.d_k, d.d_v, cbar, fb),
            "byte_ratio_explicit": roofline.dense_bytes(d.d_k, d.d_v) / roofline.explicit_bytes(d.d_k, d.d_v, cbar,
                                                                                                 fb)}
        del run.dense
        run.dense = None
        torch.cuda.empty_cache()

    # ---- end to end: host inputs in pinned memory, copies inside the timed region
    if not args.no_e2e:
        line["e2e"] = run_e2e(args, run, d, L, BH, q, k, v, alpha, beta, o, kda, stream, dev, world, local,
                              units, step_ms, s_next)
        line["status_flags"] |= S.seed_get_status(run.ws)

    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_oracle_rate(cfg, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None) -> int:
    args = parse_args(argv)
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
