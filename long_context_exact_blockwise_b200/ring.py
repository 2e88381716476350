"""Sequence-parallel ring attention across ranks (one process per GPU).

The pages' ring ("Ring Attention: the secret of million-token context", §2.1
chunking, §2.2 ring schedule figure, §3.1 two-level loop, §3.2 overlap of
the next KV transfer with the current block's compute): the sequence is cut
into P = world-size chunks; rank i holds Q_i, K_i, V_i and owns output
rows i.  At step s rank i folds KV chunk (i + s) mod P into its running
(acc, m, l) state with ``ring_attn_block_step``, while the chunk it will
need at step s + 1 is received from rank i + 1 and the chunk it holds is
sent to rank i - 1 (double-buffered point-to-point messages).  After P
steps ``ring_attn_finalize`` normalises the state once over all keys.

Causal visits whose keys all lie in the future of the rank's queries change
nothing and are skipped on the host.  There is no output collective.

The backward (``ring_attention_bwd``) runs the same ring: rank i adds each
visit's share of dq into its own accumulator with
``ring_attn_bwd_block_step``, while the float32 dK / dV accumulators of the
KV chunk it holds travel with that chunk, one hop per step, after the
visit's compute.  After P steps every chunk's accumulators have visited
every rank and the last hop hands them to the chunk's owner.

The per-visit compute and the final normalisation are injectable so the
communication protocol can be exercised on CPU ranks (gloo) with any
implementation of the same block-step semantics; by default they are the
library's CUDA kernels.
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist


def _default_block_step(q, k, v, q_off, k_off, acc, m, l, *, causal, scale):
    from . import ringattn
    ringattn.ring_attn_block_step(q, k, v, q_off, k_off, acc, m, l, causal=causal, scale=scale)


def _default_block_step_bwd(q, k, v, out, dout, lse, q_off, k_off, dq, dk, dv, *, causal, scale):
    from . import ringattn
    ringattn.ring_attn_bwd_block_step(q, k, v, out, dout, lse, q_off, k_off, dq, dk, dv, causal=causal, scale=scale)


def _default_finalize(acc, m, l, out_dtype):
    from . import ringattn
    return ringattn.ring_attn_finalize(acc, m, l, out_dtype=out_dtype)


def _default_init_state(B, Hq, Lq, d, device):
    acc = torch.zeros((B, Hq, Lq, d), device=device, dtype=torch.float32)
    m = torch.full((B, Hq, Lq), float("-inf"), device=device, dtype=torch.float32)
    l = torch.zeros((B, Hq, Lq), device=device, dtype=torch.float32)
    return acc, m, l


def ring_visit_order(rank: int, world: int) -> list:
    """KV chunk held by `rank` at each step s: (rank + s) mod world."""
    return [(rank + s) % world for s in range(world)]


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool,
                   scale: Optional[float] = None, group=None,
                   block_step: Optional[Callable] = None,
                   finalize: Optional[Callable] = None,
                   init_state: Optional[Callable] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact attention for this rank's query chunk over the whole sequence.

    q: [B, L, Hq, d] (chunk ``rank`` of the query sequence); k, v:
    [B, L, Hkv, d] (chunk ``rank`` of the KV sequence).  All ranks hold
    chunks of the same length L.  Returns (out [B, L, Hq, d], lse
    [B, Hq, L]) for this rank's rows.  Every rank must call this with the
    same shapes; the group defaults to the world.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, L, Hq, d = q.shape
    if k.shape[1] != L or v.shape != k.shape:
        raise ValueError("every rank must hold equal-length q, k, v chunks")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    block_step = block_step or _default_block_step
    finalize = finalize or _default_finalize
    init_state = init_state or _default_init_state

    send_to = (rank - 1) % world      # the rank that needs our chunk next
    recv_from = (rank + 1) % world    # the rank holding the chunk we need next
    g_send = dist.get_global_rank(group, send_to) if group is not None else send_to
    g_recv = dist.get_global_rank(group, recv_from) if group is not None else recv_from

    acc, m, l = init_state(B, Hq, L, d, q.device)
    # The caller's chunks are only read (sent at step 0); received chunks go
    # to two buffers owned here, used alternately.
    cur_k, cur_v = k.contiguous(), v.contiguous()
    bufs = [(torch.empty_like(cur_k), torch.empty_like(cur_v)) for _ in range(min(2, world - 1))]
    q_off = rank * L
    for s, j in enumerate(ring_visit_order(rank, world)):
        reqs = []
        if s + 1 < world:
            nxt_k, nxt_v = bufs[s % 2]
            ops = [dist.P2POp(dist.isend, cur_k, g_send, group),
                   dist.P2POp(dist.isend, cur_v, g_send, group),
                   dist.P2POp(dist.irecv, nxt_k, g_recv, group),
                   dist.P2POp(dist.irecv, nxt_v, g_recv, group)]
            reqs = dist.batch_isend_irecv(ops)
        k_off = j * L
        # A causal visit whose first key is past every query of this chunk
        # leaves the state unchanged: skip it.
        if not (causal and k_off > q_off + L - 1):
            block_step(q, cur_k, cur_v, q_off, k_off, acc, m, l, causal=causal, scale=scale)
        for r in reqs:
            r.wait()
        if s + 1 < world:
            cur_k, cur_v = bufs[s % 2]
    return finalize(acc, m, l, q.dtype)


def ring_attention_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                       lse: torch.Tensor, *, causal: bool, scale: Optional[float] = None, group=None,
                       block_step_bwd: Optional[Callable] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients of ``ring_attention`` for this rank's chunks.

    q, out, dout: [B, L, Hq, d] and lse [B, Hq, L] (this rank's query chunk
    and the forward's results for it); k, v: [B, L, Hkv, d] (this rank's KV
    chunk).  Returns (dq, dk, dv) for this rank's chunks, in the input dtypes.
    Every rank must call this with the same shapes.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, L, Hq, d = q.shape
    if k.shape[1] != L or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("every rank must hold equal-length q, k, v, out, dout chunks")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    block_step_bwd = block_step_bwd or _default_block_step_bwd
    acc_dtype = torch.float64 if q.dtype == torch.float64 else torch.float32

    send_to = (rank - 1) % world
    recv_from = (rank + 1) % world
    g_send = dist.get_global_rank(group, send_to) if group is not None else send_to
    g_recv = dist.get_global_rank(group, recv_from) if group is not None else recv_from

    dq = torch.zeros(q.shape, device=q.device, dtype=acc_dtype)
    # Accumulators of the KV chunk held now, and a buffer for the next ones.
    acc = [torch.zeros(k.shape, device=k.device, dtype=acc_dtype) for _ in range(2)]
    acc_next = [torch.empty_like(a) for a in acc] if world > 1 else None
    cur_k, cur_v = k.contiguous(), v.contiguous()
    bufs = [(torch.empty_like(cur_k), torch.empty_like(cur_v)) for _ in range(min(2, world - 1))]
    q_off = rank * L
    for s, j in enumerate(ring_visit_order(rank, world)):
        reqs = []
        if s + 1 < world:
            nxt_k, nxt_v = bufs[s % 2]
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, cur_k, g_send, group),
                                           dist.P2POp(dist.isend, cur_v, g_send, group),
                                           dist.P2POp(dist.irecv, nxt_k, g_recv, group),
                                           dist.P2POp(dist.irecv, nxt_v, g_recv, group)])
        k_off = j * L
        if not (causal and k_off > q_off + L - 1):
            block_step_bwd(q, cur_k, cur_v, out, dout, lse, q_off, k_off, dq, acc[0], acc[1], causal=causal,
                           scale=scale)
        for r in reqs:
            r.wait()
        if world > 1:
            # The accumulators follow their chunk to rank - 1; the last hop
            # brings this rank's own chunk home.
            for r in dist.batch_isend_irecv([dist.P2POp(dist.isend, acc[0], g_send, group),
                                             dist.P2POp(dist.isend, acc[1], g_send, group),
                                             dist.P2POp(dist.irecv, acc_next[0], g_recv, group),
                                             dist.P2POp(dist.irecv, acc_next[1], g_recv, group)]):
                r.wait()
            acc, acc_next = acc_next, acc
        if s + 1 < world:
            cur_k, cur_v = bufs[s % 2]
    return dq.to(q.dtype), acc[0].to(k.dtype), acc[1].to(v.dtype)
