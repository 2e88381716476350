"""GPU parity of the host-buffer forward and backward (ring_attn_fwd_host,
ring_attn_bwd_host).

Inputs and results live in host memory; the library streams KV-head groups
through device staging slots with the copies overlapped with the compute.
Prefill groups are computed exactly as ring_attn_fwd computes those heads, so
out and lse must be bit-identical to the device-buffer call.  Incremental
queries choose their split-KV count per group, so those are checked against
the float64 oracle (bf16 tolerances: out 2e-2, lse 1e-3).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import compare, ra

pytestmark = pytest.mark.gpu

W = workloads.small


def _host(x, pinned=True):
    h = x.cpu().contiguous()
    return h.pin_memory() if pinned else h


def _run_host(w, q, k, v, kvg, pinned=True):
    R = ra()
    ci = None if w.cache_idx < 0 else w.cache_idx
    hq, hk, hv = (_host(x, pinned) for x in (q, k, v))
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16)
    lse = torch.full((w.B, w.Hq, w.N_q), float("nan"), dtype=torch.float32)
    if pinned:
        out, lse = out.pin_memory(), lse.pin_memory()
    R.ring_attn_fwd_host(hq, hk, hv, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci, scale=w.scale, out=out,
                         lse=lse, kv_heads_per_group=kvg)
    assert R.ring_attn_sync_status() == 0
    return out, lse


def _run_device(w, q, k, v):
    R = ra()
    ci = None if w.cache_idx < 0 else w.cache_idx
    out, lse = R.ring_attn_fwd(q, k, v, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci, scale=w.scale)
    assert R.ring_attn_sync_status() == 0
    return out.cpu(), lse.cpu()


PREFILL = [
    # (B, Hq, Hkv, N, d, causal, P, kv heads per group)
    (1, 8, 8, 1000, 128, True, 4, 0),    # default: 8 groups of one KV head
    (1, 8, 8, 1000, 128, True, 4, 2),    # 4 groups
    (1, 8, 8, 1000, 128, True, 4, 8),    # one group: no overlap, same result
    (2, 8, 2, 640, 64, False, 5, 1),     # GQA 4, two groups, B = 2
    (1, 12, 4, 384, 128, True, 3, 0),    # GQA 3, default 4 groups
    (1, 4, 4, 77, 128, True, 1, 1),      # single ragged tile per group
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,P,kvg", PREFILL)
def test_host_prefill_is_bit_identical_to_device(B, Hq, Hkv, N, d, causal, P, kvg):
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N, d=d, causal=causal, P=P, seed=900 + N + kvg)
    q, k, v = workloads.make_qkv(w, device="cuda")
    ho, hl = _run_host(w, q, k, v, kvg)
    do, dl = _run_device(w, q, k, v)
    assert torch.equal(ho.view(torch.int16), do.view(torch.int16))
    assert torch.equal(hl, dl)


def test_host_prefill_matches_oracle_with_pageable_buffers():
    # Pageable host memory: the copies do not overlap, the result is the same.
    w = W(B=1, Hq=4, Hkv=2, N_q=512, d=128, causal=True, P=4, seed=951)
    q, k, v = workloads.make_qkv(w, device="cuda")
    ho, hl = _run_host(w, q, k, v, 1, pinned=False)
    ro, rl = oracle.attention_ref(q, k, v, causal=True, scale=w.scale)
    compare(ho, hl, ro, rl, "bf16", "host prefill, pageable")


INCREMENTAL = [
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, d, P, causal, kvg)
    (1, 8, 2, 300, 4096, 3796, 128, 8, True, 0),   # split-KV per group
    (2, 16, 4, 1, 2048, 2047, 128, 16, True, 1),   # decode, 4 groups
    (1, 8, 8, 8, 1024, 1016, 64, 4, True, 4),      # decode, d = 64, 2 groups
    (1, 4, 2, 33, 512, 400, 128, 4, False, 1),     # non-causal incremental
]


@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,d,P,causal,kvg", INCREMENTAL)
def test_host_incremental_matches_oracle(B, Hq, Hkv, N_q, N_kv, ci, d, P, causal, kvg):
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=causal, P=P, seed=960 + N_q + kvg)
    q, k, v = workloads.make_qkv(w, device="cuda")
    ho, hl = _run_host(w, q, k, v, kvg)
    ro, rl = oracle.attention_ref(q, k, v, causal=causal, scale=w.scale, cache_idx=ci)
    compare(ho, hl, ro, rl, "bf16", w.name)


def test_host_calls_in_a_row_and_on_a_side_stream():
    # Two calls back to back on a non-default stream: each result complete
    # once that stream is synchronised, and neither disturbs the other.
    R = ra()
    w1 = W(B=1, Hq=8, Hkv=4, N_q=256, d=128, causal=True, P=2, seed=971)
    w2 = W(B=1, Hq=4, Hkv=4, N_q=384, d=64, causal=False, P=3, seed=972)
    side = torch.cuda.Stream()
    results, keep = [], []
    for w in (w1, w2):
        q, k, v = workloads.make_qkv(w, device="cuda")
        hq, hk, hv = (_host(x) for x in (q, k, v))
        keep.append((hq, hk, hv))  # host inputs must outlive the queued copies
        results.append((w, q, k, v, R.ring_attn_fwd_host(hq, hk, hv, causal=w.causal, P=w.P, scale=w.scale,
                                                        stream=side)))
    side.synchronize()
    assert R.ring_attn_sync_status(side) == 0
    for w, q, k, v, (ho, hl) in results:
        ro, rl = oracle.attention_ref(q, k, v, causal=w.causal, scale=w.scale)
        compare(ho, hl, ro, rl, "bf16", w.name)


def test_host_rejects_device_tensors_and_bad_groups():
    R = ra()
    w = W(B=1, Hq=4, Hkv=2, N_q=128, d=128, causal=True, P=1, seed=981)
    q, k, v = workloads.make_qkv(w, device="cuda")
    with pytest.raises(ValueError):
        R.ring_attn_fwd_host(q, k, v, causal=True, P=1)
    hq, hk, hv = (_host(x) for x in (q, k, v))
    with pytest.raises(R.RingAttnError):
        R.ring_attn_fwd_host(hq, hk, hv, causal=True, P=1, kv_heads_per_group=3)


BWD = [
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, d, causal, kv heads per group)
    (1, 8, 8, 640, 640, -1, 128, True, 0),     # default: 8 groups
    (1, 8, 2, 384, 384, -1, 64, False, 1),     # GQA 4, two groups
    (2, 4, 4, 200, 200, -1, 128, True, 2),     # ragged, B = 2
]


def _bwd_inputs(w):
    R = ra()
    q, k, v = workloads.make_qkv(w, device="cuda")
    ci = None if w.cache_idx < 0 else w.cache_idx
    out, lse = R.ring_attn_fwd(q, k, v, causal=w.causal, P=1, cache_idx=ci, scale=w.scale)
    g = torch.Generator(device="cuda").manual_seed(w.N_q + 17)
    dout = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    return q, k, v, out, dout, lse


@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,d,causal,kvg", BWD)
def test_host_backward_is_bit_identical_to_device(B, Hq, Hkv, N_q, N_kv, ci, d, causal, kvg):
    R = ra()
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=causal, P=1, seed=990 + N_q + kvg)
    xs = _bwd_inputs(w)
    cci = None if ci < 0 else ci
    dq, dk, dv = R.ring_attn_bwd(*xs, causal=causal, cache_idx=cci, scale=w.scale)
    hs = [_host(x) for x in xs]
    hq, hk, hv = R.ring_attn_bwd_host(*hs, causal=causal, cache_idx=cci, scale=w.scale, kv_heads_per_group=kvg)
    assert R.ring_attn_sync_status() == 0
    for got, ref in ((hq, dq), (hk, dk), (hv, dv)):
        assert torch.equal(got.view(torch.int16), ref.cpu().view(torch.int16))


def test_host_backward_incremental_matches_oracle():
    R = ra()
    w = W(B=1, Hq=4, Hkv=2, N_q=96, N_kv=512, cache_idx=416, d=128, causal=True, P=1, seed=997)
    xs = _bwd_inputs(w)
    hs = [_host(x) for x in xs]
    dq, dk, dv = R.ring_attn_bwd_host(*hs, causal=True, cache_idx=416, scale=w.scale, kv_heads_per_group=1)
    assert R.ring_attn_sync_status() == 0
    q, k, v, out, dout, lse = xs
    rq, rk, rv = oracle.attention_bwd_ref(q, k, v, dout, causal=True, scale=w.scale, cache_idx=416)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        err = np.abs(got.float().numpy() - ref) / (2e-2 + 2e-2 * np.abs(ref))
        assert float(err.max()) <= 1.0


WA = [
    # (B, Hq, Hkv, N, d, window, anchor period, P, kv heads per group)
    (1, 8, 4, 1024, 128, 300, 256, 4, 0),
    (2, 4, 2, 768, 64, 100, 512, 3, 1),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,W,A,P,kvg", WA)
def test_host_window_anchor_is_bit_identical_to_device(B, Hq, Hkv, N, d, W, A, P, kvg):
    R = ra()
    w = W_(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, W=W, A=A, P=P)
    q, k, v = workloads.make_qkv(w, device="cuda")
    do, dl = R.ring_attn_fwd_window_anchor(q, k, v, window=W, anchor_period=A, P=P, chunk=w.chunk, scale=w.scale)
    hq, hk, hv = (_host(x) for x in (q, k, v))
    ho, hl = R.ring_attn_fwd_window_anchor_host(hq, hk, hv, window=W, anchor_period=A, P=P, chunk=w.chunk,
                                                scale=w.scale, kv_heads_per_group=kvg)
    assert R.ring_attn_sync_status() == 0
    assert torch.equal(ho.view(torch.int16), do.cpu().view(torch.int16))
    assert torch.equal(hl, dl.cpu())


def W_(B, Hq, Hkv, N, d, W, A, P):
    return workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N, d=d, causal=False, P=P, seed=1000 + N + W, window=W,
                           anchor_period=A)
