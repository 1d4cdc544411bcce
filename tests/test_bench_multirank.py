"""The host side of `bench.py --gpus N` with two ranks on the CPU (gloo).

Every rank runs its own batch (weak scaling); the job's time is the slowest
rank's, taken with one all-reduce (max) per timed quantity; the reported value
is all ranks' tokens over that time; the reference arm runs on rank 0 alone.
No GPU and no CUDA kernel is involved: these are the collective and
bookkeeping steps the GPU run takes around its kernels.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # per-rank timings of 10 steps: rank 1 is the slow one
        local_ms = [100.0, 130.0][rank]
        total = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value, ms_per_step = bench.aggregate(total, 10, 32768, world)
        e2e = bench.max_over_ranks([55.0, 41.0][rank], world, torch.device("cpu"))

        class A:
            steps, warmup = 2, 1

        ref = bench.run_reference(A, rank, world) if rank != 0 else "rank-0 arm not run here"
        out.put((rank, total, value, ms_per_step, e2e, bench.replica_seed(rank), ref))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_aggregation():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(world))
    for rank, total, value, ms_per_step, e2e, seed, ref in res:
        assert total == 130.0 and e2e == 55.0            # every rank sees the slowest rank's time
        assert ms_per_step == pytest.approx(13.0)
        assert value == pytest.approx(2 * 32768 / 0.013)   # all ranks' tokens over the slowest time
    assert res[0][5] != res[1][5]                          # independent batches per rank
    assert res[1][6] is None                               # the reference arm runs on rank 0 only


def test_launch_plan():
    import bench
    assert bench.launch_plan(None, {}) == ("run", 1)
    assert bench.launch_plan(1, {}) == ("run", 1)
    assert bench.launch_plan(4, {}) == ("relaunch", 4)
    assert bench.launch_plan(None, {"WORLD_SIZE": "2"}) == ("run", 2)
    assert bench.launch_plan(2, {"WORLD_SIZE": "2"}) == ("run", 2)
    assert bench.launch_plan(8, {"WORLD_SIZE": "2"})[0] == "error"
    assert bench.launch_plan(0, {})[0] == "error"


def test_gpus_flag_runs_that_many_ranks():
    """`bench.py --gpus 2` outside a launcher starts two ranks under
    torch.distributed.run; the reference arm (CPU, rank 0 alone) then reports
    n_gpus 2.  (The other arm needs CUDA devices.)"""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0", "--sample-tokens", "16"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
