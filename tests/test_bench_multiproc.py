"""Multi-rank plumbing of bench.py on CPU: world size 2 over gloo.

Each rank owns an independent batch (weak scaling, no data-path collective);
the only collective is the max-reduction of the measured time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import bench
    from causal_kernelized_linear_la_b200 import inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_env()
        local_ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
        mx = bench.max_over_ranks(local_ms, world, device="cpu")
        spec = inputs.WORKLOADS["plain_bf16"]
        p = inputs.make_workload("plain_bf16", N=64, seed=bench.rank_seed(spec["seed"], rank))
        q.put((r, w, mx, bench.aggregate_throughput(1000.0, w, mx / 1e3), p.q_bits[0, 0, 0, :4].tolist()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, m0, v0, x0), (r1, w1, m1, v1, x1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert m0 == m1 == 15.0                      # every rank sees the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 1000.0 / 0.015)  # units of all ranks / max time
    assert x0 != x1                              # ranks draw independent batches


def test_single_rank_defaults():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.aggregate_throughput(100.0, 1, 0.5) == 200.0
    assert bench.rank_seed(44, 0) == 44 and bench.rank_seed(44, 3) == 3044
