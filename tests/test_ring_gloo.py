"""The sequence-parallel ring protocol across ranks, on CPU (gloo).

Each rank holds one chunk of Q, K, V; ring_attention passes KV chunks around
the ring (one-way, or both ways in the bidirectional ring) and folds them into
the running state.  For the CPU test the
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


CASES = [(1, 2, 2, 16, 8, True), (2, 4, 2, 12, 8, False), (1, 4, 1, 10, 4, True)]
# (chunk layout, bidirectional)
MODES = [("contiguous", False), ("zigzag", False), ("contiguous", True), ("zigzag", True)]


def _setup(rank, world, port):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _worker(rank, world, port, results):
    _setup(rank, world, port)
    try:
        import oracle
        import workloads
        from long_context_exact_blockwise_b200.ring import ring_attention, shard

        # Every case and layout in one process group (every rank takes the
        # same steps in the same order).
        for ci, case in enumerate(CASES):
            for layout, bi in MODES:
                B, Hq, Hkv, L, d, causal = case
                w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=world * L, d=d, dtype="f32", causal=causal, P=world,
                                    seed=11 + world + ci)
                q, k, v = (x.double() for x in workloads.make_qkv(w))
                bs, fin, init = _oracle_compute()
                qc, kc, vc = (shard(x, rank, world, layout) for x in (q, k, v))
                before = [x.clone() for x in (qc, kc, vc)]
                out, lse = ring_attention(qc, kc, vc, causal=causal, scale=w.scale, layout=layout, bidirectional=bi,
                                          block_step=bs, finalize=fin, init_state=init)
                # The ring only reads the caller's chunks.
                assert all(torch.equal(a, b) for a, b in zip(before, (qc, kc, vc)))
                ro, rl = oracle.attention_ref(q, k, v, causal=causal, scale=w.scale)
                ro = shard(torch.from_numpy(ro), rank, world, layout).numpy()
                rl = shard(torch.from_numpy(rl), rank, world, layout, dim=2).numpy()
                results[(rank, ci, layout, bi)] = (float(np.max(np.abs(out.numpy() - ro))),
                                                   float(np.max(np.abs(lse.numpy() - rl))))
    finally:
        dist.destroy_process_group()


def _run_ranks(target, world):
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    got = dict(results)
    assert sorted(got) == sorted((r, ci, lay, bi) for r in range(world) for ci in range(len(CASES)) for lay, bi in MODES)
    return got


@pytest.mark.parametrize("world", [2, 3, 4])
def test_ring_protocol_matches_full_attention(world):
    for key, (eo, el) in _run_ranks(_worker, world).items():
        assert eo <= 1e-10 and el <= 1e-10, (key, eo, el)


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

def _add_and_clear_cpu(acc, part):
    acc += part
    part.zero_()


def _bwd_worker(rank, world, port, results):
    _setup(rank, world, port)
    try:
        import oracle
        import workloads
        from long_context_exact_blockwise_b200.ring import ring_attention_bwd, shard

        for ci, case in enumerate(CASES):
            for layout, bi in MODES:
                B, Hq, Hkv, L, d, causal = case
                w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=world * L, d=d, dtype="f32", causal=causal, P=world,
                                    seed=31 + world + ci)
                q, k, v = (x.double() for x in workloads.make_qkv(w))
                dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(5), dtype=torch.float64)
                out, lse = (torch.from_numpy(x) for x in oracle.attention_ref(q, k, v, causal=causal, scale=w.scale))
                chunks = [shard(x, rank, world, layout) for x in (q, k, v, out, dout)]
                before = [x.clone() for x in chunks]
                dq, dk, dv = ring_attention_bwd(*chunks, shard(lse, rank, world, layout, dim=2), causal=causal,
                                                scale=w.scale, layout=layout, bidirectional=bi,
                                                block_step_bwd=_oracle_bwd_step(), add_and_clear=_add_and_clear_cpu)
                assert all(torch.equal(a, b) for a, b in zip(before, chunks))
                rq, rk, rv = oracle.attention_bwd_ref(q, k, v, dout, causal=causal, scale=w.scale)
                results[(rank, ci, layout, bi)] = tuple(
                    float(np.max(np.abs(g.numpy() - shard(torch.from_numpy(r), rank, world, layout).numpy())))
                    for g, r in ((dq, rq), (dk, rk), (dv, rv)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
def test_ring_backward_protocol_matches_full_gradient(world):
    for key, errs in _run_ranks(_bwd_worker, world).items():
        assert max(errs) <= 1e-10, (key, errs)


def test_bidirectional_visit_order_and_pieces():
    from long_context_exact_blockwise_b200.ring import _kv_plan, ring_visit_order_bidirectional
    # 4 ranks: rank 1 holds the first piece of ranks 1, 2, 3, 0 (from its
    # right-hand neighbour) and the second piece of ranks 1, 0, 3, 2 (from
    # its left-hand neighbour).
    assert ring_visit_order_bidirectional(1, 4) == [(1, 1), (2, 0), (3, 3), (0, 2)]
    # Over the P steps every rank sees both pieces of every rank exactly once.
    for world in (1, 2, 3, 5):
        for rank in range(world):
            order = ring_visit_order_bidirectional(rank, world)
            assert sorted(a for a, _ in order) == list(range(world))
            assert sorted(b for _, b in order) == list(range(world))
    # Key offsets: contiguous halves of a 16-key chunk; zigzag chunks of 8 keys
    # (rank 1 of 4 holds chunks 1 and 6).
    n_k, offs = _kv_plan(1, 4, "contiguous", 16, True)
    assert n_k == 2 and offs(0) == [16, 24] and offs(1) == [32, 8] and offs(3) == [0, 40]
    n_k, offs = _kv_plan(1, 4, "zigzag", 16, True)
    assert n_k == 2 and offs(0) == [8, 48] and offs(1) == [16, 56] and offs(2) == [24, 32]
    # Every key offset appears exactly once over the ring.
    for layout in ("contiguous", "zigzag"):
        n_k, offs = _kv_plan(2, 4, layout, 16, True)
        assert sorted(o for s in range(4) for o in offs(s)) == list(range(0, 64, 8))


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


def test_zigzag_layout_balances_causal_work():
    # Causal visits that are not skipped, per rank: the contiguous layout
    # gives rank i (i + 1) of them; the zigzag layout gives every rank the same
    # number of (query piece, key piece) pairs with work in them.
    from long_context_exact_blockwise_b200.ring import chunk_ids, ring_visit_order

    def work(rank, world, layout):
        n = len(chunk_ids(rank, world, layout))
        pairs = 0
        for owner in ring_visit_order(rank, world):
            for kc in chunk_ids(owner, world, layout):
                for qc in chunk_ids(rank, world, layout):
                    pairs += 2 if kc < qc else (1 if kc == qc else 0)  # full tile = 2 halves, diagonal = 1
        return pairs / n ** 2

    for world in (2, 3, 4, 8):
        contiguous = [work(r, world, "contiguous") for r in range(world)]
        zigzag = [work(r, world, "zigzag") for r in range(world)]
        assert contiguous == [2 * r + 1 for r in range(world)]
        assert len(set(zigzag)) == 1, zigzag
        assert sum(zigzag) == sum(contiguous)


def test_shard_layouts_partition_the_sequence():
    from long_context_exact_blockwise_b200.ring import shard
    x = torch.arange(24).reshape(1, 24, 1, 1)
    for layout in ("contiguous", "zigzag"):
        got = torch.cat([shard(x, r, 3, layout) for r in range(3)], dim=1).flatten().tolist()
        assert sorted(got) == list(range(24))
    assert shard(x, 0, 3, "zigzag").flatten().tolist() == [0, 1, 2, 3, 20, 21, 22, 23]
    assert shard(x, 1, 3, "zigzag").flatten().tolist() == [4, 5, 6, 7, 16, 17, 18, 19]
