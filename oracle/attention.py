"""Plain float64 CPU definition of exact (ring) attention -- test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may use this module.  It is deliberately slow and literal:

* ``attention_ref`` is the textbook definition, one full score row per query
  (the attention definition on the pages [BT] "core challenge", [LC] "the
  mathematical essence of attention", [RA] §2.3), with the readings below.
* ``ring_ref`` / ``block_step_ref`` / ``finalize_ref`` follow the ring
  algorithm step by step: cut the sequence into P chunks ([RA] §2.1), let
  query chunk i visit KV chunk (i+s) mod P at step s ([RA] §2.2 figure), fold
  each visit into running (acc, m, l) statistics ([RA] §3.1 inner loop,
  "softmax in SRAM"), then normalise once over all keys ([LC] fusion layer:
  global softmax normalisation of the local outputs).
* ``lse_merge_ref`` combines independently normalised partials by their
  log-sum-exp weights (the same global normalisation, [LC] fusion layer).

Readings where the pages are silent or wrong (each listed in the design notes):
  - [RA] §2.3 writes the sum of independently normalised per-chunk softmaxes;
    taken literally that is not attention.  The sentence after it says the
    accumulated result *is* full attention, and [LC] normalises globally, so
    the merge here is the global softmax over all keys.
  - causal masking is per token (causal_block_size=1 in [CI]): key position
    k_pos is visible to query position q_pos iff k_pos <= q_pos.
  - cache_idx = -1 means "None": query t sits at global position t.
    cache_idx >= 0: query t sits at cache_idx + t (the exact offset; [CI]
    floors it to a query-chunk multiple, identical whenever cache_idx is a
    multiple of the query chunk).
  - GQA (not on the pages): query head h reads KV head h // (Hq // Hkv).
  - a masked logit is -inf; a row with no visible key has out = 0, lse = -inf;
    an all-masked visit leaves the running state unchanged.
  - lse is the natural log of sum_j exp(scale * q.k_j) over visible keys.

Array layouts (token-major): q/out [B, N_q, Hq, d]; k/v [B, N_kv, Hkv, d];
lse [B, Hq, N_q]; running state acc [B, Hq, Lq, d], m and l [B, Hq, Lq];
split partials o_parts [S, B, N_q, Hq, d], lse_parts [S, B, Hq, N_q].
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf

# Rows of queries per dense score block in attention_ref.  Rows are
# independent, so this only bounds memory; each row still sees its whole
# score row at once.
_ROW_BLOCK = 256


def _f64(x) -> np.ndarray:
    """Upcast a torch tensor (any float dtype, any device) or array to float64."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().cpu().to(dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _kv_head(h_q: int, Hq: int, Hkv: int) -> int:
    """Query head h_q reads KV head h_q // G with G = Hq / Hkv (contiguous groups)."""
    return h_q // (Hq // Hkv)


def _query_positions(N_q: int, cache_idx: int) -> np.ndarray:
    """Global token position of each query row ([CI] "how cache_idx works")."""
    base = 0 if cache_idx < 0 else int(cache_idx)
    return base + np.arange(N_q, dtype=np.int64)


def _visible(q_pos: np.ndarray, k_pos: np.ndarray, causal: bool) -> np.ndarray:
    """[len(q_pos), len(k_pos)] boolean: may query q_pos attend to key k_pos?"""
    if not causal:
        return np.ones((q_pos.shape[0], k_pos.shape[0]), dtype=bool)
    return k_pos[None, :] <= q_pos[:, None]


def _softmax_rows(s: np.ndarray):
    """Stable softmax statistics of score rows that may hold -inf entries.

    Returns (w, m, l): w = exp(s - m) with m the row max (0 used as the
    subtraction base for rows that are entirely -inf), l = row sum of w.
    """
    m = s.max(axis=1)
    base = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(s - base[:, None])
    l = w.sum(axis=1)
    return w, m, l


def attention_ref(q, k, v, *, causal: bool, scale: float, cache_idx: int = -1,
                  rows=None, heads=None):
    """Exact attention by definition, in float64.

    out[b, t, h, :] = sum_j softmax_j(scale * q[b,t,h,:] . k[b,j,hk,:]) v[b,j,hk,:]
    over the keys j visible to row t, and lse[b, h, t] = log sum_j exp(...).

    ``rows`` (query indices) and ``heads`` (query heads) restrict the
    computation to a sample; the returned arrays then have len(rows) rows
    and len(heads) heads in the order given.
    Returns (out [B, R, Hh, d], lse [B, Hh, R]) as float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N_q, Hq, d = q.shape
    N_kv, Hkv = k.shape[1], k.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    rows = np.arange(N_q) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(Hq)) if heads is None else list(heads)
    pos_all = _query_positions(N_q, cache_idx)
    out = np.zeros((B, rows.shape[0], len(heads), d), dtype=np.float64)
    lse = np.full((B, len(heads), rows.shape[0]), NEG_INF, dtype=np.float64)
    k_pos_all = np.arange(N_kv, dtype=np.int64)
    for b in range(B):
        for hi, h in enumerate(heads):
            hk = _kv_head(h, Hq, Hkv)
            # Bound the dense score block to about 2^25 entries (256 MB).
            blk = max(1, min(_ROW_BLOCK, (1 << 25) // max(1, N_kv)))
            for r0 in range(0, rows.shape[0], blk):
                r = rows[r0:r0 + blk]
                qp = pos_all[r]
                # Keys past the last query position carry zero weight under
                # causal masking; leave them out of the product.
                n_keys = N_kv if not causal else int(min(N_kv, qp.max() + 1))
                if n_keys <= 0:
                    continue
                s = scale * (q[b, r, h, :] @ k[b, :n_keys, hk, :].T)
                s = np.where(_visible(qp, k_pos_all[:n_keys], causal), s, NEG_INF)
                w, m, l = _softmax_rows(s)
                has = l > 0
                o = np.zeros((r.shape[0], d))
                o[has] = (w[has] @ v[b, :n_keys, hk, :]) / l[has, None]
                out[b, r0:r0 + r.shape[0], hi, :] = o
                lse[b, hi, r0:r0 + r.shape[0]] = np.where(
                    has, m + np.log(np.where(has, l, 1.0)), NEG_INF)
    return out, lse


# ---------------------------------------------------------------------------
# The ring algorithm, step by step.
# ---------------------------------------------------------------------------

def ring_visit_chunk(i: int, s: int, P: int, direction: int = 1) -> int:
    """KV chunk held by query chunk i at ring step s.

    direction=+1: (i + s) mod P, the schedule of the [RA] §2.2 figure
    (GPU0 receives K1, K2, K3 at steps 1, 2, 3).  direction=-1: (i - s) mod P,
    what a ring that sends to (i+1) mod n delivers ([CI] ppermute, [BT]).
    """
    return (i + direction * s) % P


def query_home_chunk(q_pos0: int, chunk: int) -> int:
    """Ring rank whose chunk holds global position q_pos0 (the block's first query)."""
    return int(q_pos0) // int(chunk)


def init_state(B: int, Hq: int, Lq: int, d: int):
    """Empty running statistics: acc = 0, m = -inf, l = 0."""
    return (np.zeros((B, Hq, Lq, d)), np.full((B, Hq, Lq), NEG_INF), np.zeros((B, Hq, Lq)))


def block_step_ref(q_chunk, k_chunk, v_chunk, q_off: int, k_off: int, acc, m, l, *,
                   causal: bool, scale: float):
    """Fold one ring visit (a query chunk against one KV chunk) into (acc, m, l).

    q_chunk [B, Lq, Hq, d] at global positions q_off + t; k/v_chunk
    [B, Lk, Hkv, d] at k_off + j.  m is in natural-log units of
    scale * q.k.  Per row: m' = max(m, max_j s_j), alpha = exp(m - m'),
    l' = alpha l + sum_j exp(s_j - m'), acc' = alpha acc + sum_j exp(s_j - m') v_j.
    Returns new (acc, m, l); the inputs are not modified.
    """
    q, kc, vc = _f64(q_chunk), _f64(k_chunk), _f64(v_chunk)
    acc, m, l = (np.array(_f64(x), copy=True) for x in (acc, m, l))
    B, Lq, Hq, d = q.shape
    Lk, Hkv = kc.shape[1], kc.shape[2]
    vis = _visible(q_off + np.arange(Lq, dtype=np.int64),
                   k_off + np.arange(Lk, dtype=np.int64), causal)
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            s = scale * (q[b, :, h, :] @ kc[b, :, hk, :].T)
            s = np.where(vis, s, NEG_INF)
            m_new = np.maximum(m[b, h], s.max(axis=1) if Lk > 0 else NEG_INF)
            base = np.where(np.isfinite(m_new), m_new, 0.0)
            alpha = np.exp(m[b, h] - base)
            p = np.exp(s - base[:, None])
            l[b, h] = alpha * l[b, h] + p.sum(axis=1)
            acc[b, h] = alpha[:, None] * acc[b, h] + p @ vc[b, :, hk, :]
            m[b, h] = m_new
    return acc, m, l


def finalize_ref(acc, m, l):
    """out = acc / l, lse = m + log l; rows with l == 0 give out 0 and lse -inf.

    Returns (out [B, Lq, Hq, d], lse [B, Hq, Lq]).
    """
    acc, m, l = _f64(acc), _f64(m), _f64(l)
    has = l > 0
    safe = np.where(has, l, 1.0)
    out = np.where(has[..., None], acc / safe[..., None], 0.0)
    lse = np.where(has, m + np.log(safe), NEG_INF)
    return np.transpose(out, (0, 2, 1, 3)), lse


def ring_ref(q, k, v, *, causal: bool, scale: float, P: int, chunk: int, cache_idx: int = -1,
             order="forward"):
    """Ring attention emulated on the CPU: every query block visits all P KV chunks.

    Prefill (cache_idx = -1): query chunk i holds rows [i*chunk, (i+1)*chunk)
    and starts from KV chunk i.  Incremental (cache_idx >= 0): all N_q new
    queries form one block homed at the chunk holding position cache_idx.
    ``order`` picks the visit sequence: "forward" (i+s) mod P, "backward"
    (i-s) mod P, or an explicit permutation of range(P) (same for every block).
    Returns (out [B, N_q, Hq, d], lse [B, Hq, N_q]) in float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N_q, Hq, d = q.shape
    N_kv = k.shape[1]
    if P * chunk != N_kv:
        raise ValueError("N_kv must equal P * chunk")
    if cache_idx < 0:
        if N_q != N_kv:
            raise ValueError("prefill needs N_q == N_kv")
        blocks = [(i, i * chunk, slice(i * chunk, (i + 1) * chunk)) for i in range(P)]
    else:
        blocks = [(query_home_chunk(cache_idx, chunk), int(cache_idx), slice(0, N_q))]

    def visits(i):
        if isinstance(order, str):
            direction = {"forward": 1, "backward": -1}[order]
            return [ring_visit_chunk(i, s, P, direction) for s in range(P)]
        seq = [int(x) for x in order]
        if sorted(seq) != list(range(P)):
            raise ValueError("order must be a permutation of range(P)")
        return seq

    out = np.zeros((B, N_q, Hq, d))
    lse = np.zeros((B, Hq, N_q))
    for i, q_off, rs in blocks:
        qb = q[:, rs]
        acc, m, l = init_state(B, Hq, qb.shape[1], d)
        for j in visits(i):
            ks = slice(j * chunk, (j + 1) * chunk)
            acc, m, l = block_step_ref(qb, k[:, ks], v[:, ks], q_off, j * chunk, acc, m, l,
                                       causal=causal, scale=scale)
        ob, lb = finalize_ref(acc, m, l)
        out[:, rs] = ob
        lse[:, :, rs] = lb
    return out, lse


def lse_merge_ref(o_parts, lse_parts):
    """Merge S normalised partial results by their log-sum-exp weights.

    o_parts [S, B, N_q, Hq, d], lse_parts [S, B, Hq, N_q].  Per row:
    M = max_s lse_s, w_s = exp(lse_s - M), lse = M + log sum_s w_s,
    out = sum_s w_s O_s / sum_s w_s.  A partial with lse = -inf has weight 0;
    a row whose partials are all -inf gives out 0 and lse -inf.
    Returns (out [B, N_q, Hq, d], lse [B, Hq, N_q]).
    """
    o, L = _f64(o_parts), _f64(lse_parts)
    M = L.max(axis=0)
    base = np.where(np.isfinite(M), M, 0.0)
    w = np.exp(L - base[None])                    # [S, B, Hq, N_q]
    W = w.sum(axis=0)
    has = W > 0
    safe = np.where(has, W, 1.0)
    w_t = np.transpose(w, (0, 1, 3, 2))[..., None]  # [S, B, N_q, Hq, 1]
    out = (w_t * o).sum(axis=0) / np.transpose(safe, (0, 2, 1))[..., None]
    out = np.where(np.transpose(has, (0, 2, 1))[..., None], out, 0.0)
    lse = np.where(has, base + np.log(safe), NEG_INF)
    return out, lse


# ---------------------------------------------------------------------------
# Backward pass (gradients of the exact attention), by definition.
# ---------------------------------------------------------------------------

def attention_bwd_ref(q, k, v, dout, *, causal: bool, scale: float, cache_idx: int = -1):
    """Gradients of out = attention(q, k, v) for an upstream gradient dout.

    The pages define only the forward; they use it for training ([BT]
    production parameters: Ring Attention with FSDP for 7B-13B models; [CI]
    blockwise configuration with a gradient-checkpoint policy), so the
    backward is the mathematical gradient of the forward definition above.

    Per (b, query head h, row t) with visible keys J(t), writing
    s_j = scale * q_t . k_j, p_j = softmax_j(s), o_t = sum_j p_j v_j:
        dv_j  += p_tj * dout_t                      (summed over t and the
        dp_tj  = dout_t . v_j                         query heads of the group)
        D_t    = dout_t . o_t   ( = sum_j p_tj dp_tj )
        ds_tj  = p_tj (dp_tj - D_t)
        dq_t   = scale * sum_j ds_tj k_j
        dk_j  += scale * ds_tj q_t
    The softmax is recomputed here from the definition (full score rows).
    Returns (dq [B, N_q, Hq, d], dk [B, N_kv, Hkv, d], dv [B, N_kv, Hkv, d]).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N_q, Hq, d = q.shape
    N_kv, Hkv = k.shape[1], k.shape[2]
    pos = _query_positions(N_q, cache_idx)
    vis = _visible(pos, np.arange(N_kv, dtype=np.int64), causal)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            s = scale * (q[b, :, h, :] @ k[b, :, hk, :].T)
            s = np.where(vis, s, NEG_INF)
            w, m, l = _softmax_rows(s)
            has = l > 0
            p = np.zeros_like(w)
            p[has] = w[has] / l[has, None]
            o = p @ v[b, :, hk, :]
            dp = do[b, :, h, :] @ v[b, :, hk, :].T
            D = np.sum(do[b, :, h, :] * o, axis=1)
            ds = p * (dp - D[:, None])
            dv[b, :, hk, :] += p.T @ do[b, :, h, :]
            dq[b, :, h, :] = scale * (ds @ k[b, :, hk, :])
            dk[b, :, hk, :] += scale * (ds.T @ q[b, :, h, :])
    return dq, dk, dv


def block_step_bwd_ref(q_chunk, k_chunk, v_chunk, dout_chunk, lse_chunk, delta_chunk, q_off: int, k_off: int,
                       dq, dk, dv, *, causal: bool, scale: float):
    """Fold one ring visit's share of the gradients into (dq, dk, dv).

    The backward of a ring visit: a query chunk (q, dout, its final lse and
    delta = rowsum(dout * out), all for the whole sequence's softmax)
    against one KV chunk.  With p_tj = exp(s_tj - lse_t) on the visible pairs
    of this visit (s_tj = scale * q_t . k_j, positions q_off + t and k_off + j)
    and zero elsewhere, every term of attention_bwd_ref that involves only
    this visit's keys is added:
        dv_j += sum_t p_tj dout_t
        ds_tj = p_tj (dout_t . v_j - delta_t)
        dq_t += scale * sum_j ds_tj k_j
        dk_j += scale * sum_t ds_tj q_t
    (dk, dv summed over the query heads of a GQA group).  Summed over all
    visits this is the full gradient, because p_tj and ds_tj depend on the
    other chunks only through lse_t and delta_t.

    q_chunk, dout_chunk, dq: [B, Lq, Hq, d]; k_chunk, v_chunk, dk, dv:
    [B, Lk, Hkv, d]; lse_chunk, delta_chunk: [B, Hq, Lq].  Rows with
    lse = -inf (no visible key anywhere) contribute nothing.  Returns new
    (dq, dk, dv); the inputs are not modified.
    """
    q, kc, vc, do = _f64(q_chunk), _f64(k_chunk), _f64(v_chunk), _f64(dout_chunk)
    lse, delta = _f64(lse_chunk), _f64(delta_chunk)
    dq, dk, dv = (np.array(_f64(x), copy=True) for x in (dq, dk, dv))
    B, Lq, Hq, d = q.shape
    Lk, Hkv = kc.shape[1], kc.shape[2]
    vis = _visible(q_off + np.arange(Lq, dtype=np.int64),
                   k_off + np.arange(Lk, dtype=np.int64), causal)
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            s = scale * (q[b, :, h, :] @ kc[b, :, hk, :].T)
            live = vis & np.isfinite(lse[b, h])[:, None]
            base = np.where(np.isfinite(lse[b, h]), lse[b, h], 0.0)
            p = np.where(live, np.exp(np.where(live, s, 0.0) - base[:, None]), 0.0)
            dp = do[b, :, h, :] @ vc[b, :, hk, :].T
            ds = p * (dp - delta[b, h][:, None])
            dv[b, :, hk, :] += p.T @ do[b, :, h, :]
            dq[b, :, h, :] += scale * (ds @ kc[b, :, hk, :])
            dk[b, :, hk, :] += scale * (ds.T @ q[b, :, h, :])
    return dq, dk, dv


def ring_bwd_ref(q, k, v, dout, *, causal: bool, scale: float, P: int, order="forward"):
    """The backward emulated as a ring: query chunk i visits every KV chunk.

    The forward (out, lse) comes from attention_ref; delta = rowsum(dout *
    out).  Query chunk i visits KV chunks in ring order; its dq accumulates
    locally, while the (dk, dv) accumulators of each KV chunk gather one
    visit's share from every query chunk (in the ring they travel with the
    chunk).  Square causal prefill or non-causal, N divisible by P.  Returns
    (dq, dk, dv) in the layouts of attention_bwd_ref.
    """
    q64, k64, v64, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, Hq, d = q64.shape
    if k64.shape[1] != N or N % P != 0:
        raise ValueError("ring_bwd_ref needs N_q == N_kv divisible by P")
    L = N // P
    out, lse = attention_ref(q64, k64, v64, causal=causal, scale=scale)
    delta = np.einsum("bthe,bthe->bht", do, out)
    dq = np.zeros_like(q64)
    dk = np.zeros_like(k64)
    dv = np.zeros_like(v64)
    for i in range(P):
        qs = slice(i * L, (i + 1) * L)
        for s in range(P):
            if order == "forward":
                j = ring_visit_chunk(i, s, P, 1)
            elif order == "backward":
                j = ring_visit_chunk(i, s, P, -1)
            else:
                j = int(order[i][s])
            ks = slice(j * L, (j + 1) * L)
            dq[:, qs], dk[:, ks], dv[:, ks] = block_step_bwd_ref(
                q64[:, qs], k64[:, ks], v64[:, ks], do[:, qs], lse[:, :, qs], delta[:, :, qs], i * L, j * L,
                dq[:, qs], dk[:, ks], dv[:, ks], causal=causal, scale=scale)
    return dq, dk, dv


def decode_e4m3(codes) -> np.ndarray:
    """FP8 E4M3 codes (uint8) to float64, from the format's definition.

    Bit 7 is the sign, bits 6..3 the exponent field e (bias 7), bits 2..0 the
    mantissa m.  e = 0: subnormal, (-1)^s * 2^-6 * m/8.  e = 15 with m = 7:
    NaN (the format has no infinities).  Otherwise (-1)^s * 2^(e-7) * (1 + m/8).
    The largest finite magnitude is 448.
    """
    # The definition is applied to the 256 codes once; arrays of codes then
    # index that table.
    c = np.arange(256, dtype=np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return (sign * mag)[np.asarray(codes, dtype=np.uint8)]


def attention_fp8kv_ref(q, k8, v8, k_scale, v_scale, *, causal: bool, scale: float, cache_idx: int = -1):
    """Attention over an FP8 (E4M3) KV cache with per-(batch, KV head) scales.

    The pages ask for a quantised KV cache in serving ("Billion-token context
    window engineering", production parameters: 4-/8-bit KV quantisation;
    "RingAttention vs RAG" §2.3: FP8 deployment; "From hundreds of
    milliseconds to a million tokens", KV-cache compression by quantisation).
    The cache holds codes k8, v8 [B, N_kv, Hkv, d] (uint8) and float32 scales
    k_scale, v_scale [B, Hkv]; the keys and values it stands for are
        k[b, j, h, :] = decode_e4m3(k8[b, j, h, :]) * k_scale[b, h]
    (likewise v), and the result is exact attention (attention_ref) over
    those dequantised keys and values.  Returns (out, lse) as attention_ref.
    """
    ks = np.asarray(_f64(k_scale))
    vs = np.asarray(_f64(v_scale))
    k = decode_e4m3(_u8(k8)) * ks[:, None, :, None]
    v = decode_e4m3(_u8(v8)) * vs[:, None, :, None]
    return attention_ref(q, k, v, causal=causal, scale=scale, cache_idx=cache_idx)


def _u8(x) -> np.ndarray:
    """uint8 codes from a torch tensor (any device) or array."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.asarray(x, dtype=np.uint8)


def window_anchor_visible(q_pos, k_pos, n: int, window: int, anchor_period: int) -> np.ndarray:
    """[len(q_pos), len(k_pos)] boolean: the sparse mask of "Ring Attention:
    the secret of million-token context" §4.3 (sparse attention mask), for a
    sequence of n tokens attending to itself.

    Query i sees the local window j in [max(0, i - window), i], and the
    anchors of its period: a = (i // anchor_period) * anchor_period, the key
    a, the key a - 1 when a > 0, and the key a + anchor_period when
    a < n - anchor_period (that last anchor lies after i).
    """
    qp = np.asarray(q_pos, dtype=np.int64)[:, None]
    kp = np.asarray(k_pos, dtype=np.int64)[None, :]
    vis = (kp <= qp) & (kp >= np.maximum(0, qp - window))
    a = (qp // anchor_period) * anchor_period
    vis |= kp == a
    vis |= (a > 0) & (kp == a - 1)
    vis |= (a < n - anchor_period) & (kp == a + anchor_period)
    return vis


def attention_window_anchor_ref(q, k, v, *, window: int, anchor_period: int, scale: float, rows=None, heads=None):
    """Exact attention restricted to the window-and-anchor mask
    (window_anchor_visible) of a square prefill: N_q == N_kv == n, query t at
    position t.  Every row keeps its full (masked) score row; rows and heads
    restrict the computation to a sample as in attention_ref.
    Returns (out [B, R, Hh, d], lse [B, Hh, R]) as float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape[1] != N:
        raise ValueError("the window-and-anchor mask is defined for N_q == N_kv")
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(Hq)) if heads is None else list(heads)
    out = np.zeros((B, rows.shape[0], len(heads), d), dtype=np.float64)
    lse = np.full((B, len(heads), rows.shape[0]), NEG_INF, dtype=np.float64)
    k_pos = np.arange(N, dtype=np.int64)
    for b in range(B):
        for hi, h in enumerate(heads):
            hk = _kv_head(h, Hq, Hkv)
            blk = max(1, min(_ROW_BLOCK, (1 << 25) // max(1, N)))
            for r0 in range(0, rows.shape[0], blk):
                r = rows[r0:r0 + blk]
                s = scale * (q[b, r, h, :] @ k[b, :, hk, :].T)
                s = np.where(window_anchor_visible(r, k_pos, N, window, anchor_period), s, NEG_INF)
                w, m, l = _softmax_rows(s)
                has = l > 0
                o = np.zeros((r.shape[0], d))
                o[has] = (w[has] @ v[b, :, hk, :]) / l[has, None]
                out[b, r0:r0 + r.shape[0], hi, :] = o
                lse[b, hi, r0:r0 + r.shape[0]] = np.where(has, m + np.log(np.where(has, l, 1.0)), NEG_INF)
    return out, lse
