"""ring_attn_fwd_noalloc: the incremental-query forward for callers that
cannot let the library allocate device memory (their own pool owns the
budget, or an allocation on a latency-critical path is not acceptable).

It must give the same result as ring_attn_fwd, and as the float64 oracle,
within the parity tolerance, on consecutive calls that share its fixed
scratch array; the second call uses other inputs and another shape, so stale
scratch contents from the first call would show up.  It must also succeed
while the allocating path is made to fail (RINGATTN_FAULT=alloc), which shows
that it never reaches the library's workspace allocation.  This file is
collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import TOL_LSE, TOL_OUT

pytestmark = pytest.mark.gpu


def _ra():
    import long_context_exact_blockwise_b200.ringattn as m
    return m


def _case(w):
    q, k, v = workloads.make_qkv(w, device="cuda")
    return q, k, v


def _call_noalloc_c_abi(R, w, q, k, v):
    """Call the entry point through the C ABI with caller-owned outputs."""
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.Hq, w.N_q), float("nan"), device="cuda", dtype=torch.float32)
    st = R.lib.ring_attn_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), w.B, w.Hq, w.Hkv, w.N_q, w.N_kv, w.d,
        int(w.causal), w.chunk, w.P, w.cache_idx, w.scale,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out, lse


def _check_same(got_out, got_lse, ref_out, ref_lse):
    assert torch.isfinite(got_out.float()).all()
    assert (got_out.float() - ref_out.float()).abs().max().item() <= TOL_OUT["bf16"]
    assert (got_lse - ref_lse).abs().max().item() <= TOL_LSE


def _check_oracle(w, q, k, v, got_out, got_lse):
    ro, rl = oracle.attention_ref(q, k, v, causal=w.causal, scale=w.scale, cache_idx=w.cache_idx)
    assert np.max(np.abs(got_out.float().cpu().numpy() - ro)) <= TOL_OUT["bf16"]
    assert np.max(np.abs(got_lse.cpu().numpy() - rl)) <= TOL_LSE


def test_noalloc_matches_fwd_on_two_calls_in_a_row():
    R = _ra()
    w1 = workloads.small(B=2, Hq=8, Hkv=2, N_q=4, N_kv=4096, cache_idx=4092, d=128, causal=True, P=16, seed=41)
    w2 = workloads.small(B=1, Hq=4, Hkv=1, N_q=40, N_kv=2048, cache_idx=1000, d=64, causal=True, P=8, seed=42)
    results = []
    for w in (w1, w2):
        q, k, v = _case(w)
        ref_out, ref_lse = R.ring_attn_fwd(q, k, v, causal=w.causal, P=w.P, cache_idx=w.cache_idx, scale=w.scale)
        st, out, lse = _call_noalloc_c_abi(R, w, q, k, v)
        assert st == R.RA_OK, R.lib.ring_attn_last_error().decode()
        torch.cuda.synchronize()
        assert R.ring_attn_sync_status() == 0
        results.append((w, q, k, v, out, lse, ref_out, ref_lse))
    for w, q, k, v, out, lse, ref_out, ref_lse in results:
        _check_same(out, lse, ref_out, ref_lse)
        _check_oracle(w, q, k, v, out, lse)


def test_noalloc_never_takes_the_allocating_path(monkeypatch):
    # With RINGATTN_FAULT=alloc every workspace allocation of the library
    # fails.  A split-KV call of ring_attn_fwd therefore fails with
    # RA_ERR_OOM, while the allocation-free call, on the same inputs and
    # split count, succeeds and matches the oracle.
    R = _ra()
    w = workloads.small(B=1, Hq=8, Hkv=2, N_q=3, N_kv=4096, cache_idx=4093, d=128, causal=True, P=8, seed=45)
    q, k, v = _case(w)
    monkeypatch.setenv("RINGATTN_SPLITS", "4")
    monkeypatch.setenv("RINGATTN_FAULT", "alloc")
    with pytest.raises(RuntimeError):
        R.ring_attn_fwd(q, k, v, causal=w.causal, P=w.P, cache_idx=w.cache_idx, scale=w.scale)
    st, out, lse = _call_noalloc_c_abi(R, w, q, k, v)
    assert st == R.RA_OK, R.lib.ring_attn_last_error().decode()
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    _check_oracle(w, q, k, v, out, lse)


def test_noalloc_rejects_oversize_and_prefill():
    R = _ra()
    # Config-5-sized incremental query: its split partials exceed the 16 MiB scratch.
    w = workloads.small(B=4, Hq=32, Hkv=8, N_q=512, N_kv=8192, cache_idx=8192 - 512, d=128, causal=True, P=8,
                        seed=43)
    q, k, v = _case(w)
    import os
    old = os.environ.get("RINGATTN_SPLITS")
    os.environ["RINGATTN_SPLITS"] = "4"
    try:
        st, _, _ = _call_noalloc_c_abi(R, w, q, k, v)
    finally:
        if old is None:
            del os.environ["RINGATTN_SPLITS"]
        else:
            os.environ["RINGATTN_SPLITS"] = old
    assert st == R.RA_ERR_INVALID_ARG
    assert "scratch" in R.lib.ring_attn_last_error().decode()
    wp = workloads.small(B=1, Hq=2, Hkv=2, N_q=256, d=128, causal=True, P=2, seed=44)
    q, k, v = _case(wp)
    st, _, _ = _call_noalloc_c_abi(R, wp, q, k, v)
    assert st == R.RA_ERR_INVALID_ARG
