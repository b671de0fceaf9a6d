"""Host-side logic of the benchmark's multi-process (torchrun) path, on CPU with
the gloo backend and two ranks: the max-over-ranks reduction of the timings,
the whole-job throughput, and the reference arm's behaviour on ranks other
than 0 (no work, no output, exit status 0)."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = [1.0 + rank, 5.0 - rank, 2.5, 10.0 * rank]
        got = bench.max_over_ranks(mine, "cpu")
        out.put((rank, got, bench._dist()))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict()
    for _ in procs:
        rank, got, d = q.get(timeout=120)
        res[rank] = (got, d)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        got, (ws, r, _) = res[rank]
        assert got == [2.0, 5.0, 2.5, 10.0]          # element-wise max of both ranks' values
        assert ws == 2 and r == rank


def test_max_over_ranks_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 1.5], "cpu") == [3.0, 1.5]


def test_job_throughput_sums_ranks_over_the_slowest_time():
    import bench
    # two ranks, 1 GB each, slowest rank 0.5 s: 4 GB/s for the job
    assert bench.job_gbs(2, 1e9, 500.0) == pytest.approx(4.0)
    assert bench.job_gbs(1, 536870912, 0.4287) == pytest.approx(536870912 / 0.4287e-3 / 1e9)


def test_reference_arm_on_other_ranks_does_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
