"""Shared helpers for the GPU parity tests: run the library and the CPU
oracle on the same seeded inputs and compare element by element.

Tolerances (max absolute error against the float64 oracle):
  bf16 inputs, float32 accumulation : out <= 2e-2, lse <= 1e-3
  float32 path                      : out <= 1e-4, lse <= 1e-3
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

TOL_OUT = {"bf16": 2e-2, "f32": 1e-4}
TOL_LSE = 1e-3


def ra():
    import long_context_exact_blockwise_b200.ringattn as m
    return m


def run_fwd(w: workloads.Workload, device="cuda", host=False):
    """Run the library's forward on workload w; returns (q, k, v, out, lse).
    host=True goes through ring_attn_fwd_host (pinned host buffers, default
    groups, as the benchmark's end-to-end line); out and lse are then on the
    host."""
    q, k, v = workloads.make_qkv(w, device=device)
    R = ra()
    ci = None if w.cache_idx < 0 else w.cache_idx
    if host:
        assert w.dtype == "bf16"
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        out = torch.full(q.shape, float("nan"), dtype=q.dtype).pin_memory()
        lse = torch.full((w.B, w.Hq, w.N_q), float("nan"), dtype=torch.float32).pin_memory()
        R.ring_attn_fwd_host(hq, hk, hv, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci, scale=w.scale, out=out,
                             lse=lse)
        torch.cuda.synchronize()
        assert R.ring_attn_sync_status() == 0, "device status word set"
        return q, k, v, out, lse
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.Hq, w.N_q), float("nan"), device=device, dtype=torch.float32)
    fn = R.ring_attn_fwd_f32 if w.dtype == "f32" else R.ring_attn_fwd
    fn(q, k, v, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci, scale=w.scale, out=out, lse=lse)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0, "device status word set"
    return q, k, v, out, lse


def compare(got_out, got_lse, ref_out, ref_lse, dtype: str, what: str):
    go = got_out.detach().float().cpu().numpy().astype(np.float64)
    gl = got_lse.detach().float().cpu().numpy().astype(np.float64)
    assert go.shape == ref_out.shape, f"{what}: out shape {go.shape} vs {ref_out.shape}"
    assert gl.shape == ref_lse.shape, f"{what}: lse shape {gl.shape} vs {ref_lse.shape}"
    assert np.isfinite(go).all(), f"{what}: non-finite output"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(gl), fin), f"{what}: lse finiteness differs"
    e_out = float(np.max(np.abs(go - ref_out))) if go.size else 0.0
    e_lse = float(np.max(np.abs(gl[fin] - ref_lse[fin]))) if fin.any() else 0.0
    assert e_out <= TOL_OUT[dtype], f"{what}: max |out err| {e_out:.3e} > {TOL_OUT[dtype]}"
    assert e_lse <= TOL_LSE, f"{what}: max |lse err| {e_lse:.3e} > {TOL_LSE}"
    return e_out, e_lse


def check_workload(w: workloads.Workload, rows=None, heads=None, host=False):
    """Full-tensor parity when rows/heads are None, else on the sampled rows/heads
    (host=True: through the host-buffer forward)."""
    q, k, v, out, lse = run_fwd(w, host=host)
    if rows is None and heads is None:
        ro, rl = oracle.attention_ref(q, k, v, causal=w.causal, scale=w.scale, cache_idx=w.cache_idx)
        return compare(out, lse, ro, rl, w.dtype, w.name)
    rows_t = torch.as_tensor(rows if rows is not None else np.arange(w.N_q), dtype=torch.long)
    heads_l = list(heads) if heads is not None else list(range(w.Hq))
    G = w.Hq // w.Hkv
    kv_heads = sorted({h // G for h in heads_l})
    # Copy only what the sampled rows need: their q rows and the KV heads read.
    q_s = q[:, rows_t.to(q.device)][:, :, heads_l].cpu().double().numpy()
    k_s = k[:, :, kv_heads].cpu().double().numpy()
    v_s = v[:, :, kv_heads].cpu().double().numpy()
    # Remap heads so that sampled head i reads kv head index kv_heads.index(h // G).
    ro = np.zeros((w.B, len(rows_t), len(heads_l), w.d))
    rl = np.zeros((w.B, len(heads_l), len(rows_t)))
    for hi, h in enumerate(heads_l):
        kh = kv_heads.index(h // G)
        # cache_idx positions: row r sits at cache_idx + r; pass the rows as
        # a one-head problem whose queries are exactly the sampled rows.
        o1, l1 = _sampled_rows_oracle(q_s[:, :, hi:hi + 1], k_s[:, :, kh:kh + 1], v_s[:, :, kh:kh + 1], rows_t,
                                      w)
        ro[:, :, hi] = o1[:, :, 0]
        rl[:, hi] = l1[:, 0]
    got_o = out[:, rows_t.to(out.device)][:, :, heads_l]
    got_l = lse[:, heads_l][:, :, rows_t.to(lse.device)]
    assert torch.isfinite(out.float()).all(), f"{w.name}: non-finite output somewhere"
    return compare(got_o, got_l, ro, rl, w.dtype, w.name + " (sampled)")


def _sampled_rows_oracle(q_rows, k, v, rows, w):
    """Oracle for arbitrary query rows: each row is its own one-row problem at
    its global position (cache_idx form), so causal masking stays exact."""
    B = q_rows.shape[0]
    outs = np.zeros((B, len(rows), 1, w.d))
    lses = np.zeros((B, 1, len(rows)))
    base = 0 if w.cache_idx < 0 else w.cache_idx
    # Group consecutive rows to reduce calls: a run of rows r0..r1 is a
    # cache_idx problem at position base + r0.
    rows_np = rows.numpy()
    i = 0
    while i < len(rows_np):
        j = i
        while j + 1 < len(rows_np) and rows_np[j + 1] == rows_np[j] + 1:
            j += 1
        pos0 = base + int(rows_np[i])
        o, l = oracle.attention_ref(q_rows[:, i:j + 1], k, v, causal=w.causal, scale=w.scale, cache_idx=pos0)
        outs[:, i:j + 1] = o
        lses[:, :, i:j + 1] = l
        i = j + 1
    return outs, lses


def sample_rows(w: workloads.Workload, n_random=256, seed=0):
    """Rows 0..127, first/last row of every chunk, +-1 around 128-row tile
    edges of the first chunks, the last 128 rows, and random rows."""
    N = w.N_q
    s = set(range(min(128, N)))
    s.update(range(max(0, N - 128), N))
    if w.cache_idx < 0:
        for c in range(w.P):
            a, b = c * w.chunk, (c + 1) * w.chunk - 1
            s.update(x for x in (a, b) if 0 <= x < N)
        for t in range(128, min(N, 4 * w.chunk), 128):
            s.update(x for x in (t - 1, t, t + 1) if 0 <= x < N)
    rng = np.random.default_rng(seed)
    s.update(rng.integers(0, N, size=min(n_random, N)).tolist())
    return np.array(sorted(s), dtype=np.int64)
