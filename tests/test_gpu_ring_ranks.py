"""The ring across real ranks with the library's CUDA kernels as the compute.

2 and 3 gloo ranks (separate processes) share one GPU.  Each rank's visits
run the library's kernels (ring_attn_block_step, ring_attn_finalize,
ring_attn_bwd_block_step, ring_attn_add_and_clear) on device copies of its
chunks, while the KV chunks and the travelling dK / dV accumulators move
between the ranks as CPU tensors over gloo.  The kernels of different ranks
never wait on one another.  Every rank's forward (out, lse) and backward
(dq, dk, dv) must match the float64 oracle on its rows, for the contiguous
and the zigzag chunk layouts, the one-way and the bidirectional ring, causal
and not.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

CASES = [  # (B, Hq, Hkv, L per rank, d, causal)
    (1, 4, 2, 256, 128, True),
    (2, 2, 2, 192, 64, False),
]
# (chunk layout, bidirectional)
MODES = [("contiguous", False), ("zigzag", False), ("contiguous", True), ("zigzag", True)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _cuda_compute(dev):
    """Block-step callables that run the library on `dev` for CPU-resident state."""
    import long_context_exact_blockwise_b200.ringattn as R

    def block_step(q, k, v, q_off, k_off, acc, m, l, *, causal, scale):
        xs = [t.to(dev) for t in (q, k, v, acc, m, l)]
        R.ring_attn_block_step(*xs[:3], q_off, k_off, *xs[3:], causal=causal, scale=scale)
        for host, d_ in zip((acc, m, l), xs[3:]):
            host.copy_(d_.cpu())

    def finalize(acc, m, l, out_dtype):
        o, ls = R.ring_attn_finalize(acc.to(dev), m.to(dev), l.to(dev), out_dtype=out_dtype)
        return o.cpu(), ls.cpu()

    def init_state(B, Hq, Lq, d, device):
        return (torch.zeros((B, Hq, Lq, d)), torch.full((B, Hq, Lq), float("-inf")), torch.zeros((B, Hq, Lq)))

    def block_step_bwd(q, k, v, out, dout, lse, q_off, k_off, dq, dk, dv, *, causal, scale):
        xs = [t.to(dev) for t in (q, k, v, out, dout, lse, dq, dk, dv)]
        R.ring_attn_bwd_block_step(*xs[:6], q_off, k_off, *xs[6:], causal=causal, scale=scale)
        for host, d_ in zip((dq, dk, dv), xs[6:]):
            host.copy_(d_.cpu())

    def add_and_clear(acc, part):
        a, p = acc.to(dev), part.to(dev)
        R.ring_attn_add_and_clear(a, p)
        acc.copy_(a.cpu())
        part.copy_(p.cpu())

    return block_step, finalize, init_state, block_step_bwd, add_and_clear


def _worker(rank, world, port, results):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        import workloads
        from long_context_exact_blockwise_b200.ring import ring_attention, ring_attention_bwd, shard

        dev = torch.device("cuda", 0)
        bs, fin, init, bs_bwd, add_clear = _cuda_compute(dev)
        for ci, (B, Hq, Hkv, L, d, causal) in enumerate(CASES):
            for layout, bi in MODES:
                w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=world * L, d=d, causal=causal, P=world,
                                    seed=70 + 10 * world + ci)
                q, k, v = workloads.make_qkv(w)  # bf16 on the CPU, the same on every rank
                dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(71 + ci)).to(torch.bfloat16)
                qc, kc, vc, dc = (shard(x, rank, world, layout) for x in (q, k, v, dout))
                out, lse = ring_attention(qc, kc, vc, causal=causal, scale=w.scale, layout=layout, bidirectional=bi,
                                          block_step=bs, finalize=fin, init_state=init)
                dq, dk, dv = ring_attention_bwd(qc, kc, vc, out, dc, lse, causal=causal, scale=w.scale,
                                                layout=layout, bidirectional=bi, block_step_bwd=bs_bwd,
                                                add_and_clear=add_clear)
                ro, rl = oracle.attention_ref(q, k, v, causal=causal, scale=w.scale)
                ro = shard(torch.from_numpy(ro), rank, world, layout).numpy()
                rl = shard(torch.from_numpy(rl), rank, world, layout, dim=2).numpy()
                grads = oracle.attention_bwd_ref(q, k, v, dout, causal=causal, scale=w.scale)
                # Gradient error relative to the 2e-2 + 2e-2 |ref| bound (<= 1 passes).
                g_ratio = max(float(np.max(np.abs(g.float().numpy() - r_) / (2e-2 + 2e-2 * np.abs(r_))))
                              for g, r_ in zip((dq, dk, dv),
                                               (shard(torch.from_numpy(x), rank, world, layout).numpy()
                                                for x in grads)))
                results[(rank, ci, layout, bi)] = (float(np.max(np.abs(out.float().numpy() - ro))),
                                               float(np.max(np.abs(lse.numpy() - rl))), g_ratio)
        torch.cuda.synchronize(dev)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_ranks_with_cuda_kernels_match_oracle(world):
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = dict(results)
    assert sorted(got) == sorted((r, ci, lay, bi) for r in range(world) for ci in range(len(CASES)) for lay, bi in MODES)
    for key, (eo, el, gr) in got.items():
        assert eo <= 2e-2 and el <= 1e-3 and gr <= 1.0, (key, eo, el, gr)
