"""The benchmark's multi-GPU path on the CPU: two gloo ranks.

Each rank runs its own batch (weak scaling, no collective on the data path);
the only collectives are the barrier and the max over ranks of the timings.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from io_aware_tiled_b200.inputs import attention_inputs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # a different "time" per rank: the reduction must hand everyone the max
        local_ms = 10.0 + 5.0 * rank
        got = bench.max_over_ranks(local_ms, world)
        # the per-rank batches differ
        q = attention_inputs(1, 1, 8, 64, seed=bench.rank_seed(0, rank), with_do=False)[0]
        gathered = [torch.zeros_like(q.float()) for _ in range(world)]
        dist.all_gather(gathered, q.float())
        distinct = not torch.equal(gathered[0], gathered[1])
        out[rank] = (got, distinct)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_distinct_batches():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] and res[1][1]


def test_whole_job_throughput_counts_every_rank():
    # 2 ranks x 1e12 flop per step x 10 steps in 10 ms (the slowest rank) = 2000 TFLOP/s
    assert bench.whole_job_tflops(2, 1e12, 10, 10.0) == pytest.approx(2000.0)
    assert bench.whole_job_tflops(1, 1e12, 10, 10.0) == pytest.approx(1000.0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def _run_bench(args, env_extra=None, timeout=600):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=root, env=env, capture_output=True, text=True,
                       timeout=timeout)
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.strip().startswith("{")]
    return r, lines


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` with no launcher starts two ranks through
    torch.distributed.run (rendezvous on 127.0.0.1).  The reference arm runs
    on the host cores, so the launcher is exercised here without a GPU: rank 0
    prints the one line, with n_gpus = 2; rank 1 exits without work."""
    r, lines = _run_bench(["--gpus", "2", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-3000:]
    assert len(lines) == 1, r.stdout
    assert lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_gpus_flag_and_world_size_must_agree():
    """A rank whose WORLD_SIZE differs from --gpus refuses to time anything."""
    r, lines = _run_bench(["--gpus", "2", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                          env_extra={"WORLD_SIZE": "1", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode == 2 and not lines
    assert "WORLD_SIZE=1" in r.stderr


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the refusal when GPUs are missing")
def test_gpu_arm_refuses_more_ranks_than_devices():
    r, lines = _run_bench(["--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 2 and not lines
    assert "visible CUDA devices" in r.stderr
