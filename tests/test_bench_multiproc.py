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


def _probe_rank(tag):
    """One rank started by bench.spawn_ranks: the benchmark's own process
    group set-up (gloo without a GPU), per-rank seed, max-over-ranks time and
    rank-0 printing."""
    import torch.distributed as dist
    import bench
    from causal_kernelized_linear_la_b200 import inputs
    world, rank, local = bench.dist_env()
    backend = bench.init_dist(world, local)
    spec = inputs.WORKLOADS["plain_bf16"]
    seed = bench.rank_seed(spec["seed"], rank)
    p = inputs.make_workload("plain_bf16", N=64, seed=seed)
    first = [None] * world
    dist.all_gather_object(first, (rank, seed, p.q_bits[0, 0, 0, :4].tolist()))
    local_ms = 10.0 + 5.0 * rank                 # the last rank is the slow one
    total = bench.max_over_ranks(local_ms, world, device="cpu")
    bench.finish_line({"tag": tag, "n_gpus": world, "backend": backend, "ms": total,
                       "value": bench.aggregate_throughput(1000.0, world, total / 1e3), "ranks": first}, world)


def test_spawned_ranks_through_the_benchmark_launcher():
    """bench.spawn_ranks (what `bench.py --gpus N` uses without torchrun)
    starts N ranks with the torchrun environment; only rank 0 prints."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys; sys.path.insert(0, %r); import bench; from tests import test_bench_multiproc as t; "
            "bench.spawn_ranks(3, t._probe_rank, ('x',))" % root)
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1                       # rank 0 alone prints
    line = lines[0]
    assert line["n_gpus"] == 3 and line["backend"] == "gloo" and line["ms"] == 20.0
    assert line["value"] == pytest.approx(3 * 1000.0 / 0.020)
    ranks = sorted(tuple(x[:2]) for x in line["ranks"])
    assert [r_ for r_, _ in ranks] == [0, 1, 2]
    assert len({s for _, s in ranks}) == 3       # a seed of its own per rank
    assert len({tuple(x[2]) for x in line["ranks"]}) == 3


def test_gpus_flag_starts_ranks_or_checks_the_launcher(monkeypatch):
    import bench
    calls = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench, "spawn_ranks", lambda n, fn, a=(): calls.append((n, fn, a)))
    bench.main(["--gpus", "4", "--steps", "2"])
    assert calls == [(4, bench.run_rank, (["--gpus", "4", "--steps", "2"],))]
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "4"])


def test_single_rank_defaults():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.aggregate_throughput(100.0, 1, 0.5) == 200.0
    assert bench.rank_seed(44, 0) == 44 and bench.rank_seed(44, 3) == 3044
