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
    # the ceil(p * n)-th smallest value (1-based): for n = 4 the median is the 2nd value, for
    # n = 20 the 10th percentile is the 2nd and the 90th the 18th
    assert bench.nearest_rank([4.0, 1.0, 3.0, 2.0], (0.5,)) == [2.0]
    ys = [float(x) for x in range(1, 21)]
    assert bench.nearest_rank(ys, (0.1, 0.9)) == [2.0, 18.0]


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


# ------------------------------------------------------------------ column-parallel split
def _column_worker(rank, world, port, queue):
    """One rank of the column split, on CPU: the oracle stands in for the rank's local
    forward (the CUDA forward of the same rows is checked against it on the GPU); the
    partitioning and the all-gather are the package's own."""
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from int8_mixed_precision_vectorwise_b200 import column_parallel as cp
    from int8_mixed_precision_vectorwise_b200 import workloads as wl

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        M, K, N = 9, 64, 40
        X, _ = wl.activation(wl.BASE_SEED + 5, M, K, 2, (20.0, 40.0))
        CB, SCB = oracle.quantize_weight_rowwise(wl.weight(6, N, K))
        bias = wl.bias(7, N)
        n0, n1 = cp.shard_range(N, world, rank)
        local = oracle.linear8bit_forward(X, CB[n0:n1], SCB[n0:n1], bias[n0:n1], 6.0)
        G = cp.gather_column_blocks(torch.from_numpy(local), world)
        queue.put((rank, (n0, n1), G.numpy()))
    finally:
        dist.destroy_process_group()


def test_column_split_two_gloo_ranks():
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from int8_mixed_precision_vectorwise_b200 import workloads as wl
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_column_worker, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, rng, G = queue.get(timeout=120)
        got[rank] = (rng, G)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the shards tile the output columns in rank order
    assert [got[r][0] for r in range(world)] == [(0, 20), (20, 40)]
    # every rank holds the same gather: rank-major blocks; laid out as out[m, p*Np + j] = G[p, m, j]
    # it is the whole layer's output, bit for bit (the oracle treats each output column alone)
    assert np.array_equal(got[0][1].view(np.uint16), got[1][1].view(np.uint16))
    G = got[0][1]
    P, M, Np = G.shape
    out = np.transpose(G, (1, 0, 2)).reshape(M, P * Np)
    X, _ = wl.activation(wl.BASE_SEED + 5, 9, 64, 2, (20.0, 40.0))
    CB, SCB = oracle.quantize_weight_rowwise(wl.weight(6, 40, 64))
    ref = oracle.linear8bit_forward(X, CB, SCB, wl.bias(7, 40), 6.0)
    assert np.array_equal(out.view(np.uint16), ref.view(np.uint16))


def test_shard_range_rules():
    sys.path.insert(0, ROOT)
    from int8_mixed_precision_vectorwise_b200 import column_parallel as cp
    assert [cp.shard_range(28672, 8, r) for r in (0, 7)] == [(0, 3584), (25088, 28672)]
    assert cp.shard_range(5, 1, 0) == (0, 5)
    with pytest.raises(ValueError):
        cp.shard_range(10, 3, 0)
    with pytest.raises(ValueError):
        cp.shard_range(10, 2, 2)
