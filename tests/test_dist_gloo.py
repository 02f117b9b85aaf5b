"""Multi-rank host logic of bench.py on CPU: two gloo ranks (the data path has no collective)."""
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank reports its own step times; the job uses the slowest rank's
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * (rank + 1)])
        val = bench.job_throughput(2.0e12, world, got[0])
        q.put((rank, got, val))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, val in out:
        assert got == [2.0, 10.0, 1.0]
        # 2 ranks x 2 TFLOP each over 2 ms = 2 PFLOP/s = 2000 TFLOP/s
        assert abs(val - 2000.0) < 1e-9


def _shard_worker(rank, world, port, q):
    # Strong scaling: one batch split into row blocks; every rank computes its block of a row-wise
    # function and the blocks, gathered, must reassemble the whole batch's result in order.
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        M = 37
        X = torch.arange(M * 3, dtype=torch.float64).reshape(M, 3)
        lo, hi = bench.row_block(M, rank, world)
        Y = (X[lo:hi] * 2.0 + 1.0).contiguous()
        # blocks differ in size by at most one row: gather them padded to the largest, then trim
        cap = max(b - a for a, b in (bench.row_block(M, r, world) for r in range(world)))
        pad = torch.zeros((cap, 3), dtype=torch.float64)
        pad[:hi - lo] = Y
        parts = [torch.zeros((cap, 3), dtype=torch.float64) for _ in range(world)]
        dist.all_gather(parts, pad)
        full = torch.cat([p[:b - a] for p, (a, b) in zip(parts, (bench.row_block(M, r, world)
                                                                 for r in range(world)))])
        q.put((rank, bool(torch.equal(full, X * 2.0 + 1.0)), (lo, hi)))
    finally:
        dist.destroy_process_group()


def test_row_sharded_replicas_reassemble_the_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok, _ in out)
    assert out[0][2] == (0, 18) and out[1][2] == (18, 37)


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]


def test_reference_arm_non_zero_rank_does_no_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert res.returncode == 0
    assert res.stdout.strip() == ""
