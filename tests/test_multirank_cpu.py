"""Multi-rank host logic of the benchmark on CPU with the gloo backend
(world size 2): max-over-ranks timing, weak-scaling value, per-rank batches,
and the reference arm running on rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    from exact_io_aware_67_b200 import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank])
        w = workloads.custom("t", 1, 2, 1, 8, 64, True)
        wr = bench.rank_workload(w, rank)
        inp = workloads.generate(wr)
        first = float(inp.q.float().view(-1)[0])
        firsts = [None] * world
        dist.all_gather_object(firsts, first)
        q.put((rank, got, firsts, wr.seed))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, firsts, seed in res:
        assert got == [2.0, 10.0]          # max over both ranks, on every rank
        assert seed == rank
        assert firsts[0] != firsts[1]      # ranks hold different batches


def test_weak_scaling_value():
    import bench
    # 2 ranks x 3 steps x 1e12 FLOP in 1.5 s (the slower rank) -> 4 TFLOP/s
    assert abs(bench.weak_scaling_value(2, 1e12, 3, 1500.0) - 4.0) < 1e-12


def test_reference_arm_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "single_head_n128_d64", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env["RANK"], env["WORLD_SIZE"] = "0", "1"
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "single_head_n128_d64", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert "cpu_model" in line["cpu_baseline"] and line["cpu_baseline"]["per_core_value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
