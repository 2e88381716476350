"""Sequence-parallel ring attention across ranks (one process per GPU).

The pages' ring ("Ring Attention: the secret of million-token context", §2.1
chunking, §2.2 ring schedule figure, §3.1 two-level loop, §3.2 overlap of
the next KV transfer with the current block's compute): the sequence is cut
into chunks spread over the P = world-size ranks; rank i holds its chunks of
Q, K, V and owns their output rows.  At step s rank i folds the KV chunks of
rank (i + s) mod P into its running (acc, m, l) state with
``ring_attn_block_step``, while the KV it will need at step s + 1 is
received from rank i + 1 and the KV it holds is sent to rank i - 1
(double-buffered point-to-point messages).  After P steps
``ring_attn_finalize`` normalises the state once over all keys.  There is no
output collective.

Chunk layouts:
  - "contiguous": P chunks; rank i holds chunk i.  Under causal masking
    rank i then does i + 1 non-empty visits, so the last rank does P times
    the work of the first.
  - "zigzag": 2P chunks; rank i holds chunks i and 2P - 1 - i (its q, k and
    v are those two chunks concatenated along the sequence).  Every rank's
    causal work is then the same (the pages ask for load balancing across
    the ring: "RingAttention vs RAG", §2.1, dynamic load balancing).
Causal visits whose keys all lie in the future of a query chunk change
nothing and are skipped on the host.

Directions ("From hundreds of milliseconds to a million tokens", key design
decisions, communication topology: a bidirectional ring sends to both
neighbours and halves the communication time):
  - one-way (default): all of a rank's KV travels to rank - 1, so at step s
    rank i holds the KV of rank (i + s) mod P;
  - ``bidirectional=True``: a rank's KV is cut into two pieces of half its
    length (the zigzag layout's two chunks, or the two halves of a contiguous
    chunk).  The first piece travels to rank - 1 and the second to rank + 1,
    so at step s rank i holds the first piece of rank (i + s) mod P and the
    second piece of rank (i - s) mod P.  Each step still folds a whole
    chunk's worth of keys, but each directed link carries half the bytes,
    and both directions of every link are busy.

The backward (``ring_attention_bwd``) runs the same ring: rank i adds each
visit's share of dq into its own accumulator with
``ring_attn_bwd_block_step``, while the float32 dK / dV accumulators of the
KV it holds travel with that KV, one hop per step.  The hop overlaps the
next visit: that visit's dK / dV share is computed into a zeroed scratch
buffer while the accumulators are in flight, then folded into them on
arrival (``ring_attn_add_and_clear``) and sent on.  Every hop is one batch
of a send and a receive on every rank, so no rank's receive waits behind its
own send.  After P hops every chunk's accumulators have visited every rank
and the last hop hands them to the chunk's owner; in the bidirectional ring
each piece's accumulators follow that piece, in its own direction.

The per-visit compute and the final normalisation are injectable so the
communication protocol can be exercised on CPU ranks (gloo) with any
implementation of the same block-step semantics; by default they are the
library's CUDA kernels.
"""
from __future__ import annotations

import math
from typing import Callable, List, Optional, Tuple

import torch
import torch.distributed as dist

LAYOUTS = ("contiguous", "zigzag")


def _default_block_step(q, k, v, q_off, k_off, acc, m, l, *, causal, scale):
    from . import ringattn
    ringattn.ring_attn_block_step(q, k, v, q_off, k_off, acc, m, l, causal=causal, scale=scale)


def _default_block_step_bwd(q, k, v, out, dout, lse, q_off, k_off, dq, dk, dv, *, causal, scale):
    from . import ringattn
    ringattn.ring_attn_bwd_block_step(q, k, v, out, dout, lse, q_off, k_off, dq, dk, dv, causal=causal, scale=scale)


def _default_add_and_clear(acc, part):
    from . import ringattn
    ringattn.ring_attn_add_and_clear(acc, part)


def _default_finalize(acc, m, l, out_dtype):
    from . import ringattn
    return ringattn.ring_attn_finalize(acc, m, l, out_dtype=out_dtype)


def _default_init_state(B, Hq, Lq, d, device):
    acc = torch.zeros((B, Hq, Lq, d), device=device, dtype=torch.float32)
    m = torch.full((B, Hq, Lq), float("-inf"), device=device, dtype=torch.float32)
    l = torch.zeros((B, Hq, Lq), device=device, dtype=torch.float32)
    return acc, m, l


def ring_visit_order(rank: int, world: int) -> list:
    """Rank whose KV `rank` holds at each step s: (rank + s) mod world."""
    return [(rank + s) % world for s in range(world)]


def ring_visit_order_bidirectional(rank: int, world: int) -> list:
    """Per step s of the bidirectional ring: the ranks whose first and second
    KV pieces `rank` holds, ((rank + s) mod world, (rank - s) mod world)."""
    return [((rank + s) % world, (rank - s) % world) for s in range(world)]


def chunk_ids(rank: int, world: int, layout: str = "contiguous") -> List[int]:
    """Global chunk indices held by `rank`, in the order they are concatenated:
    [rank] of `world` chunks ("contiguous"), or [rank, 2 world - 1 - rank] of
    2 world chunks ("zigzag")."""
    if layout == "contiguous":
        return [rank]
    if layout == "zigzag":
        return [rank, 2 * world - 1 - rank]
    raise ValueError(f"layout must be one of {LAYOUTS}")


def shard(x: torch.Tensor, rank: int, world: int, layout: str = "contiguous", dim: int = 1) -> torch.Tensor:
    """This rank's part of a full-sequence tensor (sequence along `dim`) under `layout`."""
    n = world * (1 if layout == "contiguous" else 2)
    if x.shape[dim] % n != 0:
        raise ValueError(f"sequence length {x.shape[dim]} is not a multiple of {n} chunks")
    L = x.shape[dim] // n
    return torch.cat([x.narrow(dim, c * L, L) for c in chunk_ids(rank, world, layout)], dim=dim).contiguous()


def _pieces(x: torch.Tensor, n: int, dim: int = 1) -> List[torch.Tensor]:
    L = x.shape[dim] // n
    return [x.narrow(dim, i * L, L).contiguous() for i in range(n)]


def _peers(group, world, rank):
    """Global ranks of (rank - 1, rank + 1) in the ring."""
    prev, nxt = (rank - 1) % world, (rank + 1) % world
    if group is not None:
        return dist.get_global_rank(group, prev), dist.get_global_rank(group, nxt)
    return prev, nxt


class _Routes:
    """Where each held KV tensor goes next.  The held list is [k pieces, v
    pieces] (n_k each); tensor j belongs to piece j % n_k.  One-way: every
    piece goes to rank - 1 and its successor comes from rank + 1.
    Bidirectional: piece 0 as one-way, piece 1 to rank + 1 and from rank - 1."""

    def __init__(self, prev: int, nxt: int, n_k: int, bidirectional: bool):
        self.prev, self.nxt, self.n_k, self.bi = prev, nxt, n_k, bidirectional

    def __call__(self, j: int) -> Tuple[int, int]:
        if self.bi and j % self.n_k == 1:
            return self.nxt, self.prev
        return self.prev, self.nxt


def _exchange(send: List[torch.Tensor], recv: List[torch.Tensor], routes: _Routes, group, tag: int):
    """One batch of every send and receive of a hop (tensor j under tag + j)."""
    ops = [dist.P2POp(dist.isend, t, routes(j)[0], group, tag + j) for j, t in enumerate(send)]
    ops += [dist.P2POp(dist.irecv, t, routes(j)[1], group, tag + j) for j, t in enumerate(recv)]
    return dist.batch_isend_irecv(ops) if ops else []


def _kv_plan(rank: int, world: int, layout: str, L: int, bidirectional: bool):
    """(n_k, key offsets per step): the held KV is n_k pieces of L / n_k keys,
    and offsets(s) gives each held piece's global key offset at step s."""
    if not bidirectional:
        n = len(chunk_ids(rank, world, layout))
        Lp = L // n
        return n, lambda s: [c * Lp for c in chunk_ids((rank + s) % world, world, layout)]
    if L % 2 != 0:
        raise ValueError("the bidirectional ring needs an even chunk length per rank")
    Lh = L // 2

    def piece_offset(owner: int, h: int) -> int:
        if layout == "zigzag":
            return chunk_ids(owner, world, layout)[h] * Lh
        return owner * L + h * Lh

    return 2, lambda s: [piece_offset((rank + s) % world, 0), piece_offset((rank - s) % world, 1)]


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool,
                   scale: Optional[float] = None, group=None, layout: str = "contiguous",
                   bidirectional: bool = False,
                   block_step: Optional[Callable] = None,
                   finalize: Optional[Callable] = None,
                   init_state: Optional[Callable] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact attention for this rank's query chunks over the whole sequence.

    q: [B, L, Hq, d]; k, v: [B, L, Hkv, d]: this rank's chunks under
    `layout` (``shard`` cuts them from full tensors).  Every rank holds the
    same L.  Returns (out [B, L, Hq, d], lse [B, Hq, L]) for this rank's rows,
    in the same chunk order.  Every rank must call this with the same shapes,
    layout and direction; the group defaults to the world.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, L, Hq, d = q.shape
    if k.shape[1] != L or v.shape != k.shape:
        raise ValueError("every rank must hold equal-length q, k, v chunks")
    n = len(chunk_ids(rank, world, layout))
    if L % n != 0:
        raise ValueError(f"the {layout} layout needs a chunk length divisible by {n}")
    Lp = L // n
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    block_step = block_step or _default_block_step
    finalize = finalize or _default_finalize
    init_state = init_state or _default_init_state
    n_k, key_offsets = _kv_plan(rank, world, layout, L, bidirectional)
    routes = _Routes(*_peers(group, world, rank), n_k, bidirectional)

    q_p = _pieces(q, n)
    q_ids = chunk_ids(rank, world, layout)
    states = [init_state(B, Hq, Lp, d, q.device) for _ in range(n)]
    # The held KV as n_k pieces; received KV goes to two buffer sets owned here.
    cur = _pieces(k, n_k) + _pieces(v, n_k)
    bufs = [[torch.empty_like(t) for t in cur] for _ in range(min(2, world - 1))]
    for s in range(world):
        reqs = _exchange(cur, bufs[s % 2], routes, group, 0) if s + 1 < world else []
        for ki, k_off in enumerate(key_offsets(s)):
            for qi, qc in enumerate(q_ids):
                q_off = qc * Lp
                # A causal visit whose first key is past every query of the
                # chunk leaves its state unchanged: skip it.
                if causal and k_off > q_off + Lp - 1:
                    continue
                block_step(q_p[qi], cur[ki], cur[n_k + ki], q_off, k_off, *states[qi], causal=causal, scale=scale)
        for r in reqs:
            r.wait()
        if s + 1 < world:
            cur = bufs[s % 2]
    outs = [finalize(*st, q.dtype) for st in states]
    if n == 1:
        return outs[0]
    return torch.cat([o for o, _ in outs], dim=1), torch.cat([ls for _, ls in outs], dim=2)


def ring_attention_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                       lse: torch.Tensor, *, causal: bool, scale: Optional[float] = None, group=None,
                       layout: str = "contiguous", bidirectional: bool = False,
                       block_step_bwd: Optional[Callable] = None,
                       add_and_clear: Optional[Callable] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients of ``ring_attention`` for this rank's chunks.

    q, out, dout: [B, L, Hq, d] and lse [B, Hq, L] (this rank's query chunks
    and the forward's results for them); k, v: [B, L, Hkv, d] (this rank's KV
    chunks), all under `layout`.  Returns (dq, dk, dv) for this rank's chunks,
    in the input dtypes.  Every rank must call this with the same shapes.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, L, Hq, d = q.shape
    if k.shape[1] != L or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("every rank must hold equal-length q, k, v, out, dout chunks")
    n = len(chunk_ids(rank, world, layout))
    if L % n != 0:
        raise ValueError(f"the {layout} layout needs a chunk length divisible by {n}")
    Lp = L // n
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    block_step_bwd = block_step_bwd or _default_block_step_bwd
    add_and_clear = add_and_clear or _default_add_and_clear
    acc_dtype = torch.float64 if q.dtype == torch.float64 else torch.float32
    n_k, key_offsets = _kv_plan(rank, world, layout, L, bidirectional)
    routes = _Routes(*_peers(group, world, rank), n_k, bidirectional)

    q_ids = chunk_ids(rank, world, layout)
    q_p, o_p, do_p = _pieces(q, n), _pieces(out, n), _pieces(dout, n)
    lse_p = _pieces(lse, n, dim=2)
    dq_p = [torch.zeros(x.shape, device=x.device, dtype=acc_dtype) for x in q_p]
    cur = _pieces(k, n_k) + _pieces(v, n_k)
    bufs = [[torch.empty_like(t) for t in cur] for _ in range(min(2, world - 1))]
    # dK / dV accumulators of the held KV (n_k pieces each).  With more than
    # one rank two sets alternate: each hop sends one and receives into the
    # other, and is waited for (once) before the next hop is posted.  From
    # step 1 on a visit's share goes to `scratch` (zero) while the
    # accumulators it adds into are in flight, and is folded into them once
    # they have arrived.
    accs = [[torch.zeros(t.shape, device=t.device, dtype=acc_dtype) for t in cur]]
    if world > 1:
        accs.append([torch.empty_like(t) for t in accs[0]])
        scratch = [torch.zeros_like(t) for t in accs[0]]
    hop = []  # the previous step's accumulator hop (send + receive)
    a = 0
    for s in range(world):
        reqs = _exchange(cur, bufs[s % 2], routes, group, 0) if s + 1 < world else []
        target = accs[a] if s == 0 else scratch
        for ki, k_off in enumerate(key_offsets(s)):
            for qi, qc in enumerate(q_ids):
                q_off = qc * Lp
                if causal and k_off > q_off + Lp - 1:
                    continue
                block_step_bwd(q_p[qi], cur[ki], cur[n_k + ki], o_p[qi], do_p[qi], lse_p[qi], q_off, k_off,
                               dq_p[qi], target[ki], target[n_k + ki], causal=causal, scale=scale)
        if world > 1:
            if s > 0:
                for r in hop:
                    r.wait()
                for acc_t, part in zip(accs[a], scratch):
                    add_and_clear(acc_t, part)
            # The accumulators follow their KV (the last hop brings this
            # rank's own pieces home) and the next ones arrive, in one batch
            # on every rank; the next visit runs while it is in flight.
            hop = _exchange(accs[a], accs[1 - a], routes, group, 2 * n_k)
            a = 1 - a
        for r in reqs:
            r.wait()
        if s + 1 < world:
            cur = bufs[s % 2]
    for r in hop:
        r.wait()
    dk = torch.cat(accs[a][:n_k], dim=1) if n_k > 1 else accs[a][0]
    dv = torch.cat(accs[a][n_k:], dim=1) if n_k > 1 else accs[a][n_k]
    dq = torch.cat(dq_p, dim=1) if n > 1 else dq_p[0]
    return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype)
