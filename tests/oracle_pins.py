"""Pins that tie the CPU oracle to things other than itself.

Each ``pin_*`` takes the oracle module ``O`` (the real ``oracle.attention`` or
a deliberately broken copy) and raises AssertionError on a mismatch.  The
pins use: torch's float64 scaled_dot_product_attention and logsumexp (library
routines independent of the oracle's NumPy code), brute force in pure-Python
scalar loops, closed forms, invariants of the method, and the ring schedule
printed in the pages' figure (``tests/golden/ring_schedule.json``).
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-11


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale)


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin), f"{what}: finiteness differs"
    assert np.array_equal(a[~fin], b[~fin]), f"{what}: infinities differ"
    err = np.max(np.abs(a[fin] - b[fin])) if fin.any() else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def _sdpa_case(q, k, v, causal, scale, cache_idx):
    """torch SDPA in float64 with an explicit boolean mask; GQA by repeating KV heads."""
    B, N_q, Hq, d = q.shape
    N_kv, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kr = k.repeat_interleave(G, dim=2)
    vr = v.repeat_interleave(G, dim=2)
    qpos = torch.arange(N_q) + (0 if cache_idx < 0 else cache_idx)
    kpos = torch.arange(N_kv)
    mask = (kpos[None, :] <= qpos[:, None]) if causal else torch.ones(N_q, N_kv, dtype=torch.bool)
    out = F.scaled_dot_product_attention(q.transpose(1, 2), kr.transpose(1, 2), vr.transpose(1, 2),
                                         attn_mask=mask, scale=scale).transpose(1, 2)
    s = torch.einsum("bqhd,bkhd->bhqk", q, kr) * scale
    s = s.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return out.numpy(), lse.numpy()


SDPA_CASES = [
    # (B, N_q, N_kv, Hq, Hkv, d, causal, scale, cache_idx)
    (2, 37, 37, 3, 3, 16, False, 0.25, -1),
    (1, 50, 50, 2, 2, 8, True, 1 / math.sqrt(8), -1),
    (2, 7, 27, 4, 4, 16, True, 0.3, 20),
    (1, 33, 33, 6, 2, 8, True, 0.35, -1),
    (1, 5, 40, 4, 1, 8, False, 0.2, 35),
]


def pin_sdpa(O):
    for i, (B, N_q, N_kv, Hq, Hkv, d, causal, scale, ci) in enumerate(SDPA_CASES):
        q = _rand((B, N_q, Hq, d), 10 + i)
        k = _rand((B, N_kv, Hkv, d), 20 + i)
        v = _rand((B, N_kv, Hkv, d), 30 + i)
        ref_o, ref_l = _sdpa_case(q, k, v, causal, scale, ci)
        o, l = O.attention_ref(q, k, v, causal=causal, scale=scale, cache_idx=ci)
        _close(o, ref_o, 1e-10, f"sdpa out case {i}")
        _close(l, ref_l, 1e-10, f"sdpa lse case {i}")


def _brute(q, k, v, causal, scale, cache_idx):
    """Scalar loops straight from the definition (tiny sizes only)."""
    q, k, v = q.tolist(), k.tolist(), v.tolist()
    B, N_q, Hq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    N_kv, Hkv = len(k[0]), len(k[0][0])
    G = Hq // Hkv
    out = [[[[0.0] * d for _ in range(Hq)] for _ in range(N_q)] for _ in range(B)]
    lse = [[[0.0] * N_q for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for t in range(N_q):
                pos = t if cache_idx < 0 else cache_idx + t
                keys = [j for j in range(N_kv) if (not causal or j <= pos)]
                sc = [scale * sum(q[b][t][h][e] * k[b][j][hk][e] for e in range(d)) for j in keys]
                mx = max(sc)
                ws = [math.exp(x - mx) for x in sc]
                tot = sum(ws)
                for e in range(d):
                    out[b][t][h][e] = sum(w * v[b][j][hk][e] for w, j in zip(ws, keys)) / tot
                lse[b][h][t] = mx + math.log(tot)
    return np.array(out), np.array(lse)


def pin_bruteforce(O):
    cases = [(1, 6, 6, 2, 1, 3, True, 0.7, -1), (2, 5, 5, 2, 2, 4, False, 0.5, -1),
             (1, 3, 9, 3, 1, 2, True, 1.1, 6)]
    for i, (B, N_q, N_kv, Hq, Hkv, d, causal, scale, ci) in enumerate(cases):
        q = _rand((B, N_q, Hq, d), 40 + i)
        k = _rand((B, N_kv, Hkv, d), 50 + i)
        v = _rand((B, N_kv, Hkv, d), 60 + i)
        bo, bl = _brute(q, k, v, causal, scale, ci)
        o, l = O.attention_ref(q, k, v, causal=causal, scale=scale, cache_idx=ci)
        _close(o, bo, 1e-12, f"brute out {i}")
        _close(l, bl, 1e-12, f"brute lse {i}")


def pin_closed_forms(O):
    N, d, scale = 24, 8, 0.4
    v = _rand((1, N, 1, d), 70)
    # Identical keys: every visible key has the same score s, so the output is
    # the plain mean of the visible values and lse = s + ln(#visible).
    q = _rand((1, N, 1, d), 71)
    k1 = _rand((1, 1, 1, d), 72)
    k = k1.expand(1, N, 1, d).contiguous()
    o, l = O.attention_ref(q, k, v, causal=True, scale=scale)
    vv = v[0, :, 0].numpy()
    cnt = np.arange(1, N + 1)
    prefix_mean = np.cumsum(vv, axis=0) / cnt[:, None]
    s = scale * (q[0, :, 0] @ k1[0, 0, 0]).numpy()
    _close(o[0, :, 0], prefix_mean, 1e-12, "identical keys out")
    _close(l[0, 0], s + np.log(cnt), 1e-12, "identical keys lse")
    # Non-causal identical keys: mean over all values.
    o, l = O.attention_ref(q, k, v, causal=False, scale=scale)
    _close(o[0, :, 0], np.broadcast_to(vv.mean(axis=0), (N, d)), 1e-12, "identical keys mean")
    _close(l[0, 0], s + np.log(N), 1e-12, "identical keys lse all")
    # A single key returns its value; lse is its score.
    o, l = O.attention_ref(q[:, :5], k1, v[:, :1], causal=False, scale=scale)
    _close(o[0, :, 0], np.broadcast_to(vv[0], (5, d)), 1e-14, "single key out")
    _close(l[0, 0], scale * (q[0, :5, 0] @ k1[0, 0, 0]).numpy(), 1e-12, "single key lse")
    # Causal row 0 sees only key 0.
    kk = _rand((1, N, 1, d), 73)
    o, l = O.attention_ref(q, kk, v, causal=True, scale=scale)
    _close(o[0, 0, 0], vv[0], 1e-14, "causal row 0")
    _close(l[0, 0, 0], scale * float(q[0, 0, 0] @ kk[0, 0, 0]), 1e-12, "causal row 0 lse")
    # scale = 0: uniform weights -> prefix mean, lse = ln(t + 1).
    o, l = O.attention_ref(q, kk, v, causal=True, scale=0.0)
    _close(o[0, :, 0], prefix_mean, 1e-12, "scale 0 out")
    _close(l[0, 0], np.log(cnt), 1e-12, "scale 0 lse")
    # A dominant key: orthonormal keys and q = 60 e_j pick v_j.
    kd = torch.eye(d, dtype=torch.float64).reshape(1, d, 1, d)
    vd = _rand((1, d, 1, d), 74)
    j = 5
    qd = torch.zeros(1, 1, 1, d, dtype=torch.float64)
    qd[0, 0, 0, j] = 60.0
    o, l = O.attention_ref(qd, kd, vd, causal=False, scale=1.0)
    _close(o[0, 0, 0], vd[0, j, 0].numpy(), 1e-12, "dominant key")
    _close(l[0, 0, 0], 60.0 + np.log1p((d - 1) * np.exp(-60.0)), 1e-12, "dominant key lse")


def pin_ring_equals_full(O):
    rng = np.random.default_rng(3)
    N, d = 64, 8
    for causal in (True, False):
        for Hq, Hkv in ((2, 2), (4, 2)):
            q = _rand((2, N, Hq, d), 80)
            k = _rand((2, N, Hkv, d), 81)
            v = _rand((2, N, Hkv, d), 82)
            fo, fl = O.attention_ref(q, k, v, causal=causal, scale=0.3)
            for P in (1, 2, 4, 8, 16):
                orders = ["forward", "backward", list(rng.permutation(P))]
                for order in orders:
                    ro, rl = O.ring_ref(q, k, v, causal=causal, scale=0.3, P=P, chunk=N // P,
                                        order=order)
                    _close(ro, fo, 1e-12, f"ring P={P} {order} causal={causal}")
                    _close(rl, fl, 1e-12, f"ring lse P={P} {order}")
    # Incremental queries through the ring.
    N_kv, N_q, ci = 64, 10, 50
    q = _rand((1, N_q, 2, d), 83)
    k = _rand((1, N_kv, 1, d), 84)
    v = _rand((1, N_kv, 1, d), 85)
    fo, fl = O.attention_ref(q, k, v, causal=True, scale=0.3, cache_idx=ci)
    for P in (1, 4, 8):
        for order in ("forward", "backward", list(rng.permutation(P))):
            ro, rl = O.ring_ref(q, k, v, causal=True, scale=0.3, P=P, chunk=N_kv // P,
                                cache_idx=ci, order=order)
            _close(ro, fo, 1e-12, f"ring cache_idx P={P} {order}")
            _close(rl, fl, 1e-12, f"ring cache_idx lse P={P} {order}")


def pin_invariants(O):
    N, d = 40, 8
    q = _rand((3, N, 4, d), 90)
    k = _rand((3, N, 2, d), 91)
    v = _rand((3, N, 2, d), 92)
    fo, fl = O.attention_ref(q, k, v, causal=True, scale=0.3)
    # cache_idx rows equal the matching rows of full causal prefill.
    for c in (0, 1, 17, 39):
        co, cl = O.attention_ref(q[:, c:], k, v, causal=True, scale=0.3, cache_idx=c)
        _close(co, fo[:, c:], 1e-12, f"cache_idx {c} out")
        _close(cl, fl[:, :, c:], 1e-12, f"cache_idx {c} lse")
    # GQA with KV heads replicated into MHA gives the same result.
    mo, ml = O.attention_ref(q, k.repeat_interleave(2, dim=2), v.repeat_interleave(2, dim=2),
                             causal=True, scale=0.3)
    _close(mo, fo, 1e-12, "gqa vs mha")
    _close(ml, fl, 1e-12, "gqa vs mha lse")
    # Batches are independent.
    bo, bl = O.attention_ref(q[1:2], k[1:2], v[1:2], causal=True, scale=0.3)
    _close(bo, fo[1:2], 1e-12, "batch independence")
    # Non-causal: permuting (K, V) jointly leaves the result unchanged.
    no, nl = O.attention_ref(q, k, v, causal=False, scale=0.3)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(5))
    po, pl = O.attention_ref(q, k[:, perm], v[:, perm], causal=False, scale=0.3)
    _close(po, no, 1e-12, "kv permutation")
    _close(pl, nl, 1e-12, "kv permutation lse")
    # Causal differs from non-causal except on the last row.
    assert np.max(np.abs(no[:, :-1] - fo[:, :-1])) > 1e-3, "causal mask has no effect"
    _close(no[:, -1], fo[:, -1], 1e-12, "last row sees every key")


def pin_block_step(O):
    # One visit then finalize equals attention over that chunk; an all-masked
    # visit leaves the state unchanged.
    B, Lq, Lk, Hq, Hkv, d = 2, 6, 9, 4, 2, 8
    q = _rand((B, Lq, Hq, d), 100)
    k = _rand((B, Lk, Hkv, d), 101)
    v = _rand((B, Lk, Hkv, d), 102)
    acc, m, l = O.init_state(B, Hq, Lq, d)
    acc, m, l = O.block_step_ref(q, k, v, 0, 0, acc, m, l, causal=False, scale=0.5)
    o, ls = O.finalize_ref(acc, m, l)
    ro, rl = O.attention_ref(q, k, v, causal=False, scale=0.5)
    _close(o, ro, 1e-12, "single visit")
    _close(ls, rl, 1e-12, "single visit lse")
    a2, m2, l2 = O.block_step_ref(q, k, v, 0, 100, acc, m, l, causal=True, scale=0.5)
    _close(a2, acc, 0.0, "masked visit acc")
    _close(m2, m, 0.0, "masked visit m")
    _close(l2, l, 0.0, "masked visit l")
    # From the empty state an all-masked visit stays empty: out 0, lse -inf.
    e = O.init_state(B, Hq, Lq, d)
    a3, m3, l3 = O.block_step_ref(q, k, v, 0, 100, *e, causal=True, scale=0.5)
    o3, ls3 = O.finalize_ref(a3, m3, l3)
    assert np.all(o3 == 0) and np.all(np.isneginf(ls3)), "empty row"
    # Causal diagonal visit equals causal attention of the chunk with itself.
    k2 = _rand((B, Lq, Hkv, d), 103)
    v2 = _rand((B, Lq, Hkv, d), 104)
    acc, m, l = O.block_step_ref(q, k2, v2, 7, 7, *O.init_state(B, Hq, Lq, d), causal=True,
                                 scale=0.5)
    o, ls = O.finalize_ref(acc, m, l)
    ro, rl = O.attention_ref(q, k2, v2, causal=True, scale=0.5)
    _close(o, ro, 1e-12, "diagonal visit")
    _close(ls, rl, 1e-12, "diagonal visit lse")


def pin_lse_merge(O):
    # Split the keys of a non-causal problem into disjoint sets; attention over
    # each set gives normalised partials whose merge is attention over all keys.
    B, N_q, N_kv, Hq, d = 2, 7, 30, 3, 8
    q = _rand((B, N_q, Hq, d), 110)
    k = _rand((B, N_kv, Hq, d), 111)
    v = _rand((B, N_kv, Hq, d), 112)
    full_o, full_l = O.attention_ref(q, k, v, causal=False, scale=0.4)
    cuts = [0, 4, 13, 22, 30]
    parts = [O.attention_ref(q, k[:, a:b], v[:, a:b], causal=False, scale=0.4)
             for a, b in zip(cuts[:-1], cuts[1:])]
    po = np.stack([p[0] for p in parts])
    pl = np.stack([p[1] for p in parts])
    mo, ml = O.lse_merge_ref(po, pl)
    _close(mo, full_o, 1e-12, "merge = full")
    _close(ml, full_l, 1e-12, "merge lse = full")
    # Commutative: any order of partials.
    for perm in itertools.permutations(range(4)):
        co, cl = O.lse_merge_ref(po[list(perm)], pl[list(perm)])
        _close(co, mo, 1e-12, "merge commutative")
        _close(cl, ml, 1e-12, "merge commutative lse")
    # Associative: merging merged groups gives the same answer.
    ao, al = O.lse_merge_ref(po[:2], pl[:2])
    bo, bl = O.lse_merge_ref(po[2:], pl[2:])
    to, tl = O.lse_merge_ref(np.stack([ao, bo]), np.stack([al, bl]))
    _close(to, mo, 1e-12, "merge associative")
    _close(tl, ml, 1e-12, "merge associative lse")
    # Identity: a partial with lse = -inf (no keys) changes nothing.
    io, il = O.lse_merge_ref(np.stack([po[0], np.full_like(po[0], 123.0)]),
                             np.stack([pl[0], np.full_like(pl[0], -np.inf)]))
    _close(io, po[0], 1e-14, "merge identity")
    _close(il, pl[0], 1e-14, "merge identity lse")
    # All partials empty: out 0, lse -inf.
    eo, el = O.lse_merge_ref(np.ones((2, 1, 2, 1, 4)), np.full((2, 1, 1, 2), -np.inf))
    assert np.all(eo == 0) and np.all(np.isneginf(el)), "merge of empties"


def pin_schedule(O):
    g = json.load(open(os.path.join(GOLDEN, "ring_schedule.json")))
    fig = g["figure_4gpu"]
    for e in fig["entries"]:
        got = O.ring_visit_chunk(e["gpu"], e["step"], fig["P"], 1)
        assert got == e["chunk"], f"figure: step {e['step']} gpu {e['gpu']} -> {got}"
    for e in fig["inconsistent_entries"]:
        # Garbled entry: neither direction reproduces it at the printed step.
        assert O.ring_visit_chunk(e["gpu"], e["step"], fig["P"], 1) != e["chunk"]
        assert O.ring_visit_chunk(e["gpu"], e["step"], fig["P"], -1) != e["chunk"]
    # ppermute ring: simulate the sends and compare with direction -1.
    pr = g["ppermute_ring"]
    n = pr["n"]
    holding = list(range(n))
    for s in range(1, n):
        new = [None] * n
        for src, dst in pr["perm"]:
            new[dst] = holding[src]
        holding = new
        for i in range(n):
            assert O.ring_visit_chunk(i, s, n, -1) == holding[i], "ppermute direction"
    # Home chunk of an incremental query block, and the page's chunk-start rule.
    qcs = g["cache_idx_chunk_start"]["query_chunk_size"]
    for ci in (0, 511, 512, 4095, 4096, 261632):
        assert O.query_home_chunk(ci, 4096) * 4096 <= ci < (O.query_home_chunk(ci, 4096) + 1) * 4096
        if ci % qcs == 0:
            assert (ci // qcs) * qcs == ci


def pin_backward_autograd(O):
    # Gradients against torch autograd through float64 SDPA (explicit mask,
    # GQA by repeating KV heads so autograd sums the group's gradients).
    cases = [(2, 13, 13, 4, 2, 8, True, 0.3, -1), (1, 9, 9, 2, 2, 4, False, 0.7, -1),
             (1, 5, 20, 4, 1, 8, True, 0.25, 15)]
    for i, (B, N_q, N_kv, Hq, Hkv, d, causal, scale, ci) in enumerate(cases):
        q = _rand((B, N_q, Hq, d), 130 + i).requires_grad_(True)
        k = _rand((B, N_kv, Hkv, d), 140 + i).requires_grad_(True)
        v = _rand((B, N_kv, Hkv, d), 150 + i).requires_grad_(True)
        do = _rand((B, N_q, Hq, d), 160 + i)
        G = Hq // Hkv
        qpos = torch.arange(N_q) + (0 if ci < 0 else ci)
        kpos = torch.arange(N_kv)
        mask = (kpos[None, :] <= qpos[:, None]) if causal else torch.ones(N_q, N_kv, dtype=torch.bool)
        out = F.scaled_dot_product_attention(q.transpose(1, 2), k.repeat_interleave(G, dim=2).transpose(1, 2),
                                             v.repeat_interleave(G, dim=2).transpose(1, 2), attn_mask=mask,
                                             scale=scale).transpose(1, 2)
        out.backward(do)
        dq, dk, dv = O.attention_bwd_ref(q.detach(), k.detach(), v.detach(), do, causal=causal, scale=scale,
                                         cache_idx=ci)
        _close(dq, q.grad.numpy(), 1e-10, f"bwd dq {i}")
        _close(dk, k.grad.numpy(), 1e-10, f"bwd dk {i}")
        _close(dv, v.grad.numpy(), 1e-10, f"bwd dv {i}")


def pin_backward_finite_difference(O):
    # Central differences of L = sum(out * g) against the analytic gradient
    # on a few coordinates of q, k and v (second-order accurate).
    B, N, Hq, Hkv, d, scale = 1, 6, 2, 1, 3, 0.6
    q = _rand((B, N, Hq, d), 170).numpy()
    k = _rand((B, N, Hkv, d), 171).numpy()
    v = _rand((B, N, Hkv, d), 172).numpy()
    g = _rand((B, N, Hq, d), 173).numpy()
    dq, dk, dv = O.attention_bwd_ref(q, k, v, g, causal=True, scale=scale)

    def loss(qq, kk, vv):
        o, _ = O.attention_ref(qq, kk, vv, causal=True, scale=scale)
        return float(np.sum(o * g))

    eps = 1e-5
    for arr, grad, name in ((q, dq, "q"), (k, dk, "k"), (v, dv, "v")):
        for idx in [(0, 1, 0, 0), (0, 3, 0, 2), (0, 5, 0, 1)]:
            idx = idx if arr.shape[2] > idx[2] else (idx[0], idx[1], 0, idx[3])
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += eps
            a2[idx] -= eps
            args1 = {"q": (a1, k, v), "k": (q, a1, v), "v": (q, k, a1)}[name]
            args2 = {"q": (a2, k, v), "k": (q, a2, v), "v": (q, k, a2)}[name]
            fd = (loss(*args1) - loss(*args2)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7, f"finite difference d{name}{idx}: {fd} vs {grad[idx]}"


def _autograd_grads(q, k, v, do, causal, scale):
    """Gradients by torch autograd through float64 SDPA (GQA by repeated heads)."""
    q, k, v = (x.clone().requires_grad_(True) for x in (q, k, v))
    G = q.shape[2] // k.shape[2]
    N_q, N_kv = q.shape[1], k.shape[1]
    mask = (torch.arange(N_kv)[None, :] <= torch.arange(N_q)[:, None]) if causal else \
        torch.ones(N_q, N_kv, dtype=torch.bool)
    out = F.scaled_dot_product_attention(q.transpose(1, 2), k.repeat_interleave(G, dim=2).transpose(1, 2),
                                         v.repeat_interleave(G, dim=2).transpose(1, 2), attn_mask=mask,
                                         scale=scale).transpose(1, 2)
    out.backward(do)
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


def pin_backward_ring(O):
    # The ring backward (block_step_bwd_ref over every (query chunk, KV
    # chunk) visit, in ring order, forward, backward or a random order per
    # query chunk) against torch autograd of the whole-sequence attention.
    rng = np.random.default_rng(7)
    cases = [(2, 12, 4, 2, 8, True, 0.3), (1, 12, 2, 2, 4, False, 0.7), (1, 10, 4, 1, 8, True, 0.45)]
    for i, (B, N, Hq, Hkv, d, causal, scale) in enumerate(cases):
        q = _rand((B, N, Hq, d), 180 + i)
        k = _rand((B, N, Hkv, d), 190 + i)
        v = _rand((B, N, Hkv, d), 200 + i)
        do = _rand((B, N, Hq, d), 210 + i)
        ref = _autograd_grads(q, k, v, do, causal, scale)
        for P in [x for x in (1, 2, 3, 4, 5) if N % x == 0]:
            perm = [list(rng.permutation(P)) for _ in range(P)]
            for order in ("forward", "backward", perm):
                got = O.ring_bwd_ref(q, k, v, do, causal=causal, scale=scale, P=P, order=order)
                for g, r, name in zip(got, ref, ("dq", "dk", "dv")):
                    _close(g, r, 1e-10, f"ring bwd {name} case {i} P={P} order={order}")
    # A visit whose keys all lie in the future of every query adds nothing.
    q, k, v, do = (_rand((1, 4, 2, 4), 220 + j) for j in range(4))
    lse = np.zeros((1, 2, 4))
    z = np.zeros((1, 4, 2, 4))
    dq, dk, dv = O.block_step_bwd_ref(q, k, v, do, lse, lse, 0, 4, z, z, z, causal=True, scale=0.5)
    assert not (dq.any() or dk.any() or dv.any()), "a fully masked backward visit changed the gradients"


def pin_fp8_decode(O):
    # Every E4M3 code against torch's float8_e4m3fn (a library decoder), and
    # values fixed by the format: 1.0, the largest finite 448, the smallest
    # subnormal 2^-9, the smallest normal 2^-6, signed zero, NaN.
    codes = np.arange(256, dtype=np.uint8)
    got = O.decode_e4m3(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(lib)), "E4M3 NaN codes differ from the library"
    fin = ~np.isnan(lib)
    assert np.array_equal(got[fin], lib[fin]), "E4M3 decode differs from the library"
    assert np.array_equal(np.signbit(got[fin]), np.signbit(lib[fin])), "E4M3 sign of zero differs"
    fixed = {0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0xB8: -1.0, 0x3C: 1.5, 0x00: 0.0}
    for c, v in fixed.items():
        assert O.decode_e4m3(np.array([c], dtype=np.uint8))[0] == v, hex(c)
    assert np.isnan(O.decode_e4m3(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def pin_fp8kv_attention(O):
    # Attention over an FP8 cache against torch float64 SDPA on keys and values
    # dequantised through torch's own float8 type (GQA by repeated heads,
    # cache_idx by an explicit mask), plus the scale identities.
    B, N_q, N_kv, Hq, Hkv, d, ci, scale = 2, 5, 40, 4, 2, 8, 35, 0.4
    rng = np.random.default_rng(3)
    q = torch.from_numpy(rng.standard_normal((B, N_q, Hq, d)))
    k8 = torch.from_numpy(rng.integers(0, 256, (B, N_kv, Hkv, d), dtype=np.uint8))
    v8 = torch.from_numpy(rng.integers(0, 256, (B, N_kv, Hkv, d), dtype=np.uint8))
    # Keep the codes finite (0x7f / 0xff are NaN) and the logits moderate.
    k8 = torch.where((k8 & 0x7F) >= 0x70, k8 & 0xB7, k8)
    v8 = torch.where((v8 & 0x7F) == 0x7F, v8 & 0xF7, v8)
    ks = torch.tensor([[0.003, 0.005], [0.004, 0.002]], dtype=torch.float64)
    vs = torch.tensor([[0.02, 0.01], [0.03, 0.015]], dtype=torch.float64)
    out, lse = O.attention_fp8kv_ref(q, k8, v8, ks, vs, causal=True, scale=scale, cache_idx=ci)
    kd = k8.view(torch.float8_e4m3fn).to(torch.float64) * ks[:, None, :, None]
    vd = v8.view(torch.float8_e4m3fn).to(torch.float64) * vs[:, None, :, None]
    ro, rl = _sdpa_case(q, kd, vd, True, scale, ci)
    _close(out, ro, TOL, "fp8kv out vs sdpa")
    _close(lse, rl, TOL, "fp8kv lse vs sdpa")
    o2, l2 = O.attention_fp8kv_ref(q / 2, k8, v8, ks * 2, vs, causal=True, scale=scale, cache_idx=ci)
    _close(o2, out, 1e-12, "k_scale x2 with q / 2")
    _close(l2, lse, 1e-12, "k_scale x2 with q / 2 (lse)")
    o3, l3 = O.attention_fp8kv_ref(q, k8, v8, ks, vs * 2, causal=True, scale=scale, cache_idx=ci)
    _close(o3, 2 * out, 1e-12, "v_scale x2 doubles out")
    _close(l3, lse, 1e-12, "v_scale leaves lse")


def _torch_window_anchor_mask(n, window, period):
    """The window-and-anchor mask built with torch band and scatter ops."""
    ones = torch.ones(n, n, dtype=torch.bool)
    band = torch.tril(ones) & torch.triu(ones, diagonal=-window)   # i - window <= j <= i
    rows = torch.arange(n)
    a = rows - rows % period
    m = band.clone()
    m[rows, a] = True
    lo = a > 0
    m[rows[lo], a[lo] - 1] = True
    hi = a + period < n
    m[rows[hi], a[hi] + period] = True
    return m


def pin_window_anchor(O):
    # The sparse mask against an independent torch construction, attention
    # under it against float64 SDPA with that mask, and the reductions that
    # must hold: window and period covering the sequence give causal
    # attention; window 0 leaves each row its own key plus the anchors.
    for n, W, A in [(12, 2, 4), (40, 7, 8), (33, 0, 16), (64, 100, 64), (50, 5, 10)]:
        got = O.window_anchor_visible(np.arange(n), np.arange(n), n, W, A)
        ref = _torch_window_anchor_mask(n, W, A).numpy()
        assert np.array_equal(got, ref), f"window/anchor mask n={n} W={W} A={A}"
    B, N, Hq, Hkv, d, W, A, scale = 2, 48, 4, 2, 8, 5, 16, 0.35
    q, k, v = _rand((B, N, Hq, d), 230), _rand((B, N, Hkv, d), 231), _rand((B, N, Hkv, d), 232)
    out, lse = O.attention_window_anchor_ref(q, k, v, window=W, anchor_period=A, scale=scale)
    mask = _torch_window_anchor_mask(N, W, A)
    G = Hq // Hkv
    kr, vr = k.repeat_interleave(G, dim=2), v.repeat_interleave(G, dim=2)
    ro = F.scaled_dot_product_attention(q.transpose(1, 2), kr.transpose(1, 2), vr.transpose(1, 2), attn_mask=mask,
                                        scale=scale).transpose(1, 2)
    sc = (torch.einsum("bqhd,bkhd->bhqk", q, kr) * scale).masked_fill(~mask, float("-inf"))
    _close(out, ro.numpy(), 1e-10, "window/anchor out vs sdpa")
    _close(lse, torch.logsumexp(sc, dim=-1).numpy(), 1e-10, "window/anchor lse vs sdpa")
    rows = np.array([0, 5, 17, 47])
    o_s, l_s = O.attention_window_anchor_ref(q, k, v, window=W, anchor_period=A, scale=scale, rows=rows,
                                             heads=[3, 0])
    _close(o_s, out[:, rows][:, :, [3, 0]], 1e-13, "window/anchor sampled rows")
    _close(l_s, lse[:, [3, 0]][:, :, rows], 1e-13, "window/anchor sampled lse")
    oc, lc = O.attention_window_anchor_ref(q, k, v, window=N, anchor_period=N, scale=scale)
    rc, rlc = O.attention_ref(q, k, v, causal=True, scale=scale)
    _close(oc, rc, 1e-12, "full window = causal")
    _close(lc, rlc, 1e-12, "full window = causal (lse)")


def _sdpa_rows(q, k, v, causal, scale, cache_idx, rows, heads, chunk=64):
    """torch float64 SDPA on selected query rows and heads, a few rows per call
    (rows are independent, so calling the library per group of rows changes
    nothing but the memory it needs)."""
    rows = np.asarray(rows, dtype=np.int64)
    Hq, Hkv = q.shape[2], k.shape[2]
    G = Hq // Hkv
    kpos = torch.arange(k.shape[1])
    outs, lses = [], []
    for c0 in range(0, rows.shape[0], chunk):
        r = torch.from_numpy(rows[c0:c0 + chunk])
        qs = q[:, r][:, :, heads]
        hk = [h // G for h in heads]
        ks, vs = k[:, :, hk], v[:, :, hk]
        qpos = r + (0 if cache_idx < 0 else cache_idx)
        mask = (kpos[None, :] <= qpos[:, None]) if causal else torch.ones(r.shape[0], k.shape[1], dtype=torch.bool)
        o = F.scaled_dot_product_attention(qs.transpose(1, 2), ks.transpose(1, 2), vs.transpose(1, 2),
                                           attn_mask=mask, scale=scale).transpose(1, 2)
        sc = (torch.einsum("bqhd,bkhd->bhqk", qs, ks) * scale).masked_fill(~mask, float("-inf"))
        outs.append(o.numpy())
        lses.append(torch.logsumexp(sc, dim=-1).numpy())
    return np.concatenate(outs, axis=1), np.concatenate(lses, axis=2)


def pin_row_blocks(O):
    # attention_ref walks the query rows in blocks of 256 (fewer when a key
    # row is long).  Cases with several blocks, so that blocks after the
    # first (r0 > 0) and a ragged last block are written, against float64
    # SDPA; and the rows= / heads= sample against SDPA's full result sliced.
    cases = [(1, 600, 600, 4, 2, 4, True, 0.4, -1), (2, 600, 600, 1, 1, 4, False, 0.3, -1),
             (1, 300, 633, 2, 2, 4, True, 0.5, 333)]
    for i, (B, N_q, N_kv, Hq, Hkv, d, causal, scale, ci) in enumerate(cases):
        q = _rand((B, N_q, Hq, d), 240 + i)
        k = _rand((B, N_kv, Hkv, d), 250 + i)
        v = _rand((B, N_kv, Hkv, d), 260 + i)
        ref_o, ref_l = _sdpa_case(q, k, v, causal, scale, ci)
        o, l = O.attention_ref(q, k, v, causal=causal, scale=scale, cache_idx=ci)
        _close(o, ref_o, 1e-10, f"row blocks out case {i}")
        _close(l, ref_l, 1e-10, f"row blocks lse case {i}")
        rows = np.random.default_rng(i).permutation(N_q)[:290]   # unsorted, two blocks
        heads = list(range(Hq))[::-1]
        so, sl = O.attention_ref(q, k, v, causal=causal, scale=scale, cache_idx=ci, rows=rows, heads=heads)
        _close(so, ref_o[:, rows][:, :, heads], 1e-10, f"sampled rows out case {i}")
        _close(sl, ref_l[:, heads][:, :, rows], 1e-10, f"sampled rows lse case {i}")


def pin_long_key_rows(O):
    # Key rows longer than 131072 shrink the row block below 256 rows (255
    # at 131200 keys).  A causal prefill of 131200 tokens on an unsorted
    # sample of rows spanning two blocks (the second ragged), in reversed
    # head order, against float64 SDPA per group of rows; then identical
    # keys, whose result is closed-form: the prefix mean of V and
    # lse = s + ln(position + 1).
    B, N, Hq, Hkv, d, scale = 1, 131200, 2, 1, 4, 0.5
    q = _rand((B, N, Hq, d), 270)
    k = _rand((B, N, Hkv, d), 271)
    v = _rand((B, N, Hkv, d), 272)
    rng = np.random.default_rng(11)
    rows = np.concatenate([rng.integers(0, N, 296), [0, N - 1, 131071, 131072]])
    heads = [1, 0]
    o, l = O.attention_ref(q, k, v, causal=True, scale=scale, rows=rows, heads=heads)
    ro, rl = _sdpa_rows(q, k, v, True, scale, -1, rows, heads)
    _close(o, ro, 1e-10, "long key rows out")
    _close(l, rl, 1e-10, "long key rows lse")
    k1 = _rand((1, 1, 1, d), 273)
    kk = k1.expand(B, N, Hkv, d).contiguous()
    o, l = O.attention_ref(q, kk, v, causal=True, scale=scale, rows=rows, heads=heads[:1])
    prefix_mean = (np.cumsum(v[0, :, 0].numpy(), axis=0) / np.arange(1, N + 1)[:, None])[rows]
    for hi, h in enumerate(heads[:1]):
        s = scale * (q[0, rows, h] @ k1[0, 0, 0]).numpy()
        _close(o[0, :, hi], prefix_mean, 1e-12, f"long identical keys out head {h}")
        _close(l[0, hi], s + np.log(rows + 1.0), 1e-12, f"long identical keys lse head {h}")


ALL_PINS = [pin_sdpa, pin_bruteforce, pin_closed_forms, pin_ring_equals_full, pin_invariants,
            pin_block_step, pin_lse_merge, pin_schedule, pin_backward_autograd, pin_backward_finite_difference,
            pin_backward_ring, pin_fp8_decode, pin_fp8kv_attention, pin_window_anchor, pin_row_blocks,
            pin_long_key_rows]
