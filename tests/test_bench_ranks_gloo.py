"""bench.py's multi-rank logic on two CPU ranks (gloo): the timed duration
is the maximum over ranks, replicas draw different inputs, and the
whole-job value counts every replica's work."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads
        w = workloads.CONFIGS[2]
        mx = bench.max_over_ranks(10.0 + 3.0 * rank, "cpu")
        seed = bench.rank_seed(w, rank)
        q, _, _ = workloads.make_qkv(workloads.small(N_q=16, d=64), seed=seed)
        out[rank] = (mx, seed, float(q.float().sum()))
    finally:
        dist.destroy_process_group()


def test_bench_rank_helpers_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    res = ctx.Manager().dict()
    port = _port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, res)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == 13.0          # max over ranks, on every rank
    assert res[0][1] != res[1][1]                   # replicas use different seeds
    assert res[0][2] != res[1][2]                   # ... and so different inputs


def test_aggregate_counts_every_replica():
    import bench
    assert abs(bench.aggregate_tflops(8.0e12, 1, 10.0) - 800.0) < 1e-9
    assert abs(bench.aggregate_tflops(8.0e12, 4, 10.0) - 3200.0) < 1e-9
    # A single process without a process group: the value passes through.
    assert bench.max_over_ranks(7.5, "cpu") == 7.5
