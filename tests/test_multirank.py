"""The multi-rank (N > 1) host paths of bench.py, on CPU.

The path has no exchange step: `bench.py --gpus N` under torchrun runs N
independent replicas, so the only cross-rank logic is the timing reduction
(the job's time is its slowest rank's) and the rank-0-only report.  Both are
exercised here with world size 2: the reduction over a gloo process group, the
reference arm as two ranks.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _reduce_worker(rank, world, port, queue):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        slowest = bench.max_over_ranks(10.0 + rank, world, dist, "cpu")  # rank r took 10 + r ms
        queue.put((rank, slowest, bench.job_throughput(1e12, 4, world, slowest)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_reduce_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(2):
        rank, slowest, tops = queue.get(timeout=120)
        got[rank] = (slowest, tops)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slowest rank's time; the job did 2 ranks x 4 steps x 1e12 ops in 11 ms
    for rank in (0, 1):
        assert got[rank][0] == 11.0
        assert got[rank][1] == pytest.approx(2 * 4 * 1e12 / 11e-3 / 1e12)


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, None, None) == 3.5
    assert bench.job_throughput(2e12, 10, 1, 1000.0) == pytest.approx(20.0)


def test_nearest_rank_percentiles():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.nearest_rank([3.0], (0.1, 0.5, 0.9)) == [3.0, 3.0, 3.0]
    xs = [float(x) for x in range(11, 0, -1)]          # 11 .. 1, unsorted input
    assert bench.nearest_rank(xs, (0.0, 0.1, 0.5, 0.9, 1.0)) == [1.0, 2.0, 6.0, 10.0, 11.0]


def test_reference_arm_reports_on_rank_zero_only():
    """Under torchrun every rank runs bench.py; the reference arm (the CPU oracle) runs and
    prints on rank 0 alone and the other ranks exit 0 without work."""
    outs = {}
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                            "--workload", "C1", "--steps", "1", "--warmup", "0", "--cpu-rows", "4"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        outs[rank] = [l for l in r.stdout.splitlines() if l.strip()]
    assert outs[1] == []
    assert len(outs[0]) == 1
    line = json.loads(outs[0][0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
