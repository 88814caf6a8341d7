"""The benchmark's multi-rank host logic, on CPU with the gloo backend (world size 2):
per-rank seeds and inputs differ, the job time is the max over ranks, the rate counts
every rank's units, and the reference arm prints on rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        mx = bench.reduce_max(ms, "cpu")
        rate = bench.job_rate(world, 256, 32, 48, 100, mx)
        out.put((rank, mx, rate, bench.rank_seed(5000, rank), bench.rank_input_step(rank, 1)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, mx0, rate0, s0, i0), (r1, mx1, rate1, s1, i1) = res
    assert mx0 == mx1 == 15.0                       # both ranks see the slowest time
    assert rate0 == rate1 == 2 * 256 * 32 * 48 * 100 / 0.015
    assert s0 != s1 and i0 != i1                    # ranks decode different sequences


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank0_only(rank):
    env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 0:
        d = json.loads(lines[-1])
        assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
        assert d["e2e"]["h2d_bytes_per_step"] == 0
    else:
        assert not lines
