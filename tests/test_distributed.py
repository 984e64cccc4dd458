"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The decode path shards by request with no data-path collective: each rank owns
requests [rank * B, (rank + 1) * B).  The only collectives are the timing ones
(barrier, max over ranks).  These run here as two gloo processes.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from workloads import config, philox


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank), SEED_BENCH_BACKEND="gloo")
    import bench
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank)
    B = 3
    b0 = bench.shard(B, rank)
    # the rank's slice of requests, and its share of the synthetic inputs
    cfg = config(1, batch=B)
    mine = philox.token_inputs(cfg, b0 + np.arange(B)[:, None], 0, np.arange(4)[None, :], 5,
                               philox.PHASE_DECODE)
    bench.barrier(world, None)
    t = bench.max_over_ranks(float(10 + rank), world, "cpu")
    out[rank] = (b0, t, mine["k"].copy())
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_sharding_and_max_timing():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    b0s = sorted(out[r][0] for r in range(world))
    assert b0s == [0, 3]                              # disjoint shards covering 0..5
    assert all(out[r][1] == 11.0 for r in range(world))   # max over ranks on every rank
    cfg = config(1, batch=6)
    full = philox.token_inputs(cfg, np.arange(6)[:, None], 0, np.arange(4)[None, :], 5,
                               philox.PHASE_DECODE)["k"]
    got = np.concatenate([out[0][2], out[1][2]])
    np.testing.assert_array_equal(got, full)


def test_reference_arm_prints_only_on_rank0(capsys):
    import bench
    args = bench.parse_args(["--impl", "reference", "--cpu-seconds", "0.01", "--config", "0"])
    assert bench.run_reference(args, world=2, rank=1) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_carries_the_contract_keys(capsys):
    """Rank 0 of the reference arm prints one JSON line with the keys of the bench
    contract (the oracle timed on the host cores, a bounded sample)."""
    import json

    import bench
    args = bench.parse_args(["--impl", "reference", "--cpu-seconds", "0.2", "--config", "0"])
    assert bench.run_reference(args, world=1, rank=0) == 0
    lines = [x for x in capsys.readouterr().out.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
