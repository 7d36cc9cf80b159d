"""Multi-rank host logic of bench.py on CPU: two gloo ranks, no GPU.

Each rank reports a different timed-region length; both must see the slowest one, the job
throughput must count every rank's tokens over that time, and only rank 0 prints the JSON line
of the reference arm (the other ranks exit without work).
"""

import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 135.5][rank]
        bench.barrier(world)
        slowest = bench.max_over_ranks(local_ms, world)
        value = bench.job_value(world, 1000, slowest / 5)
        q.put((rank, slowest, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in results] == [135.5, 135.5]  # both ranks see the slowest time
    # 2 ranks x 1000 tokens per step, 27.1 ms per step
    for _, _, v in results:
        assert abs(v - 2000 / 0.0271) < 1e-6 * v


def test_reference_arm_nonzero_rank_does_no_work():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        warmup, steps, ref_rows = 3, 1, 1

    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(Args, world=2, rank=1) is None
    assert buf.getvalue() == ""


def test_job_value_single_rank():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert abs(bench.job_value(1, 131072, 343.8) - 131072 / 0.3438) < 1e-6
    json.dumps({"v": bench.job_value(1, 1, 1.0)})


def test_balanced_row_blocks_cover_and_balance():
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench

    L, k = 131072, 2048
    t = np.arange(L, dtype=np.float64) + 1
    cost = 137.0 * t / t.sum() + 145.0 * np.minimum(t, k) / np.minimum(t, k).sum()
    for world in (1, 2, 3, 4, 8):
        b = bench.balanced_row_blocks(L, k, world)
        assert b[0] == 0 and b[-1] == L and len(b) == world + 1
        assert all(b[i] < b[i + 1] for i in range(world))
        per = [cost[b[i]:b[i + 1]].sum() for i in range(world)]
        assert max(per) - min(per) <= 1e-3 * sum(per)   # balanced to a row
    tiny = bench.balanced_row_blocks(5, 2048, 8)   # more ranks than rows: some blocks empty
    assert tiny[0] == 0 and tiny[-1] == 5 and all(tiny[i] <= tiny[i + 1] for i in range(8))
    assert bench.even_row_blocks(10, 3) == [0, 3, 6, 10]


def _gather_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = 12
        full_ref = torch.arange(L * 3, dtype=torch.float32).reshape(L, 3)
        kb = bench.even_row_blocks(L, world)
        local = full_ref[kb[rank]:kb[rank + 1]].clone()
        full = torch.zeros_like(full_ref)
        bench.gather_rows(local, full, world)
        q.put((rank, bool(torch.equal(full, full_ref))))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_gather_rows_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == [(0, True), (1, True)]
