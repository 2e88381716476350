"""The sequence-parallel ring protocol across ranks, on CPU (gloo).

Each rank holds one chunk of Q, K, V; ring_attention passes KV chunks around
the ring and folds them into the running state.  For the CPU test the
per-visit compute is the oracle's block step (float64), so what is checked
here is the protocol: visit order, message routing, buffer swaps, causal
skipping and the final normalisation.  The result on every rank must equal
direct attention over the whole sequence for that rank's rows.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_compute():
    import oracle

    def block_step(q, k, v, q_off, k_off, acc, m, l, *, causal, scale):
        a, mm, ll = oracle.block_step_ref(q, k, v, q_off, k_off, acc, m, l, causal=causal, scale=scale)
        acc.copy_(torch.from_numpy(a))
        m.copy_(torch.from_numpy(mm))
        l.copy_(torch.from_numpy(ll))

    def finalize(acc, m, l, out_dtype):
        o, ls = oracle.finalize_ref(acc, m, l)
        return torch.from_numpy(o), torch.from_numpy(ls)

    def init_state(B, Hq, L, d, device):
        a, mm, ll = oracle.init_state(B, Hq, L, d)
        return torch.from_numpy(a), torch.from_numpy(mm), torch.from_numpy(ll)

    return block_step, finalize, init_state


def _worker(rank, world, port, case, results):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        from long_context_exact_blockwise_b200.ring import ring_attention

        B, Hq, Hkv, L, d, causal = case
        w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=world * L, d=d, dtype="f32", causal=causal, P=world,
                            seed=11 + world)
        q, k, v = workloads.make_qkv(w)
        q, k, v = q.double(), k.double(), v.double()
        sl = slice(rank * L, (rank + 1) * L)
        bs, fin, init = _oracle_compute()
        qc, kc, vc = q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous()
        before = [x.clone() for x in (qc, kc, vc)]
        out, lse = ring_attention(qc, kc, vc, causal=causal, scale=w.scale, block_step=bs, finalize=fin,
                                  init_state=init)
        # The ring only reads the caller's chunks.
        assert all(torch.equal(a, b) for a, b in zip(before, (qc, kc, vc)))
        ro, rl = oracle.attention_ref(q, k, v, causal=causal, scale=w.scale)
        err_o = float(np.max(np.abs(out.numpy() - ro[:, sl])))
        err_l = float(np.max(np.abs(lse.numpy() - rl[:, :, sl])))
        results[rank] = (err_o, err_l)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("case", [(1, 2, 2, 16, 8, True), (2, 4, 2, 12, 8, False), (1, 4, 1, 9, 4, True)])
def test_ring_protocol_matches_full_attention(world, case):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    assert sorted(results.keys()) == list(range(world))
    for r, (eo, el) in results.items():
        assert eo <= 1e-10 and el <= 1e-10, (r, eo, el)


def _oracle_bwd_step():
    import oracle

    def block_step_bwd(q, k, v, out, dout, lse, q_off, k_off, dq, dk, dv, *, causal, scale):
        delta = torch.einsum("bthe,bthe->bht", dout, out)
        a, b, c = oracle.block_step_bwd_ref(q, k, v, dout, lse, delta, q_off, k_off, dq, dk, dv, causal=causal,
                                            scale=scale)
        dq.copy_(torch.from_numpy(a))
        dk.copy_(torch.from_numpy(b))
        dv.copy_(torch.from_numpy(c))

    return block_step_bwd


def _bwd_worker(rank, world, port, case, results):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        from long_context_exact_blockwise_b200.ring import ring_attention_bwd

        B, Hq, Hkv, L, d, causal = case
        w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=world * L, d=d, dtype="f32", causal=causal, P=world,
                            seed=31 + world)
        q, k, v = (x.double() for x in workloads.make_qkv(w))
        dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(5), dtype=torch.float64)
        out, lse = (torch.from_numpy(x) for x in oracle.attention_ref(q, k, v, causal=causal, scale=w.scale))
        sl = slice(rank * L, (rank + 1) * L)
        chunks = [x[:, sl].contiguous() for x in (q, k, v, out, dout)]
        before = [x.clone() for x in chunks]
        dq, dk, dv = ring_attention_bwd(*chunks, lse[:, :, sl].contiguous(), causal=causal, scale=w.scale,
                                        block_step_bwd=_oracle_bwd_step())
        assert all(torch.equal(a, b) for a, b in zip(before, chunks))
        rq, rk, rv = oracle.attention_bwd_ref(q, k, v, dout, causal=causal, scale=w.scale)
        results[rank] = tuple(float(np.max(np.abs(g.numpy() - r[:, sl]))) for g, r in ((dq, rq), (dk, rk), (dv, rv)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("case", [(1, 2, 2, 16, 8, True), (2, 4, 2, 12, 8, False), (1, 4, 1, 9, 4, True)])
def test_ring_backward_protocol_matches_full_gradient(world, case):
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, case, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    assert sorted(results.keys()) == list(range(world))
    for r, errs in results.items():
        assert max(errs) <= 1e-10, (r, errs)


def test_ring_visit_order_matches_schedule_figure():
    from long_context_exact_blockwise_b200.ring import ring_visit_order
    # 4 ranks: GPU0 holds K0, K1, K2, K3 at steps 0..3; GPU1 holds K1, K2, K3, K0.
    assert ring_visit_order(0, 4) == [0, 1, 2, 3]
    assert ring_visit_order(1, 4) == [1, 2, 3, 0]
    assert ring_visit_order(3, 4) == [3, 0, 1, 2]


def _dying_worker(rank, world, port, results):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        # This rank leaves before the ring exchange starts (between steps).
        os._exit(0)
    from long_context_exact_blockwise_b200.ring import ring_attention
    bs, fin, init = _oracle_compute()
    q = torch.randn(1, 8, 2, 4, dtype=torch.float64)
    try:
        ring_attention(q, q.clone(), q.clone(), causal=False, scale=0.5, block_step=bs, finalize=fin,
                       init_state=init)
        results[rank] = "finished"
    except Exception as e:  # the dead peer surfaces as an error, not a hang
        results[rank] = "error: " + type(e).__name__


def test_ring_peer_loss_surfaces_as_error():
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode is not None for p in procs), "a rank hung"
    assert results.get(0, "").startswith("error"), dict(results)
