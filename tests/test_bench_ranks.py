"""Multi-rank logic of bench.py, on CPU with the gloo backend.

The decode path has no exchange step, so `bench.py --gpus N` runs N
independent replicas; what needs testing is the rank plumbing: max of the
timed region over ranks, sum of the bytes every rank processed, the same
collective sequence on every rank (errors included), and the reference arm
printing from rank 0 only.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench
        ms, bits = bench.reduce_ranks([10.0 + rank, float(rank == 1) * 4.0], "max", "cpu", world)
        total, = bench.reduce_ranks([100.0 * (rank + 1)], "sum", "cpu", world)
        q.put((rank, ms, bits, total))
    finally:
        dist.destroy_process_group()


def test_reduce_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 2000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, bits, total in res:
        assert ms == 11.0          # max over ranks
        assert bits == 4.0         # an error on one rank is seen by all
        assert total == 300.0      # whole-job bytes


def test_reduce_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_ranks([3.0, 5.0], "max", "cpu", 1) == [3.0, 5.0]


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
        assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []
