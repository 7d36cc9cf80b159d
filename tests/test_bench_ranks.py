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


def test_row_partition_covers_and_balances():
    """The library's row partition (dsa_row_partition through the binding, host only): blocks
    cover [0, L), are non-empty and carry equal estimated cost to within one row's cost; the
    cost model is the two kernels' measured times spread over the rows."""
    sys.path.insert(0, ROOT)
    import numpy as np

    from sparse_attention_09_b200 import sharding

    L, k = 131072, 2048
    t = np.arange(L, dtype=np.float64) + 1
    for idx_ms, mla_ms in ((142.0, 93.0), (137.0, 145.0), (1.0, 0.0), (0.0, 1.0)):
        cost = idx_ms * t / t.sum() + mla_ms * np.minimum(t, k) / np.minimum(t, k).sum()
        for world in (1, 2, 3, 4, 8):
            b = sharding.row_blocks(L, k, world, idx_ms, mla_ms)
            assert b[0] == 0 and b[-1] == L and len(b) == world + 1
            assert all(b[i] < b[i + 1] for i in range(world))
            per = [cost[b[i]:b[i + 1]].sum() for i in range(world)]
            assert max(per) - min(per) <= 2 * cost.max() + 1e-9 * sum(per), (idx_ms, mla_ms, world, per)
    # the indexer alone: the 2-way split sits at L / sqrt(2) (half of the causal pairs)
    b = sharding.row_blocks(L, k, 2, 1.0, 0.0)
    assert abs(b[1] - L / np.sqrt(2)) < 2
    assert sharding.row_blocks(8, 2048, 8, 1.0, 1.0) == list(range(9))   # as many ranks as rows
    assert sharding.even_blocks(10, 3) == [0, 3, 6, 10]


def test_row_partition_rejects_bad_arguments():
    sys.path.insert(0, ROOT)
    import pytest

    import sparse_attention_09_b200 as dsa

    for args in ((0, 2048, 1, 1.0, 1.0), (5, 2048, 6, 1.0, 1.0), (10, 0, 2, 1.0, 1.0), (10, 64, 2, 0.0, 0.0),
                 (10, 64, 2, -1.0, 2.0), (10, 64, 0, 1.0, 1.0)):
        with pytest.raises(RuntimeError):
            dsa.dsa_row_partition(*args)


def _gather_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    from sparse_attention_09_b200 import sharding

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ok = True
        for L in (12, 13):   # even and uneven row blocks
            full_ref = torch.arange(L * 3, dtype=torch.float32).reshape(L, 3)
            kb = sharding.even_blocks(L, world)
            local = full_ref[kb[rank]:kb[rank + 1]].clone()
            full = torch.zeros_like(full_ref)
            sharding.gather_sequence(local, full, world, rank)
            ok = ok and bool(torch.equal(full, full_ref))
        q.put((rank, ok))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_gather_sequence_two_gloo_ranks():
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
