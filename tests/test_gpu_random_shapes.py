"""Seeded random shapes against the float64 oracle: forward (every kernel the
routing can pick: general tiles, packed GQA rows, the keys-on-M decode kernel,
split-KV partials), FP8-cache forward and the backward.  The shapes are drawn
once from a fixed seed, so every run checks the same cases; they mix ragged
lengths, unaligned cache offsets, GQA factors, head sizes and ring splits."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import compare, ra

pytestmark = pytest.mark.gpu


def _draw(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        Hkv = int(rng.choice([1, 2, 4]))
        G = int(rng.choice([1, 2, 4, 8]))
        d = int(rng.choice([64, 128]))
        B = int(rng.integers(1, 3))
        causal = bool(rng.integers(0, 2))
        if rng.random() < 0.5:  # prefill
            N_q = int(rng.integers(1, 700))
            N_kv, ci = N_q, -1
        else:                   # incremental queries at the end of (or inside) a cache
            N_q = int(rng.choice([1, 2, 3, 8, int(rng.integers(1, 200))]))
            N_kv = int(rng.integers(N_q, 3000))
            ci = int(rng.integers(0, N_kv - N_q + 1)) if not causal or rng.random() < 0.3 else N_kv - N_q
        divisors = [p for p in range(1, 9) if N_kv % p == 0]
        P = int(rng.choice(divisors))
        cases.append((i, B, Hkv * G, Hkv, N_q, N_kv, ci, d, causal, P))
    return cases


FWD_CASES = _draw(120, 2026)


@pytest.mark.parametrize("i,B,Hq,Hkv,N_q,N_kv,ci,d,causal,P", FWD_CASES, ids=[f"c{c[0]}" for c in FWD_CASES])
def test_random_forward(i, B, Hq, Hkv, N_q, N_kv, ci, d, causal, P):
    R = ra()
    w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=causal, P=P,
                        seed=9000 + i)
    q, k, v = workloads.make_qkv(w, device="cuda")
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, N_q), float("nan"), device="cuda")
    R.ring_attn_fwd(q, k, v, causal=causal, P=P, cache_idx=None if ci < 0 else ci, scale=w.scale, out=out, lse=lse)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    ro, rl = oracle.attention_ref(q, k, v, causal=causal, scale=w.scale, cache_idx=ci)
    compare(out, lse, ro, rl, "bf16", f"case {i}")


FP8_CASES = [c for c in FWD_CASES if c[6] >= 0][:30]


@pytest.mark.parametrize("i,B,Hq,Hkv,N_q,N_kv,ci,d,causal,P", FP8_CASES, ids=[f"c{c[0]}" for c in FP8_CASES])
def test_random_fp8kv(i, B, Hq, Hkv, N_q, N_kv, ci, d, causal, P):
    R = ra()
    w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=causal, P=P,
                        seed=9100 + i, kv_dtype="fp8")
    q, k8, v8, ks, vs = workloads.make_fp8_kv(w, device="cuda")
    out, lse = R.ring_attn_fwd_fp8kv(q, k8, v8, ks, vs, causal=causal, P=P, cache_idx=ci, scale=w.scale)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    ro, rl = oracle.attention_fp8kv_ref(q, k8, v8, ks, vs, causal=causal, scale=w.scale, cache_idx=ci)
    compare(out, lse, ro, rl, "bf16", f"fp8 case {i}")


BWD_CASES = [c for c in FWD_CASES if c[4] * c[2] * c[5] <= 4e6][:30]


@pytest.mark.parametrize("i,B,Hq,Hkv,N_q,N_kv,ci,d,causal,P", BWD_CASES, ids=[f"c{c[0]}" for c in BWD_CASES])
def test_random_backward(i, B, Hq, Hkv, N_q, N_kv, ci, d, causal, P):
    R = ra()
    w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=causal, P=1,
                        seed=9200 + i)
    q, k, v = workloads.make_qkv(w, device="cuda")
    dout = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(9300 + i),
                       device="cuda").to(torch.bfloat16)
    cache = None if ci < 0 else ci
    out, lse = R.ring_attn_fwd(q, k, v, causal=causal, P=1, cache_idx=cache, scale=w.scale)
    dq, dk, dv = R.ring_attn_bwd(q, k, v, out, dout, lse, causal=causal, cache_idx=cache, scale=w.scale)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    for got, ref, name in zip((dq, dk, dv), oracle.attention_bwd_ref(q, k, v, dout, causal=causal, scale=w.scale,
                                                                      cache_idx=ci), ("dq", "dk", "dv")):
        g = got.float().cpu().numpy()
        bad = np.abs(g - ref) > 2e-2 + 2e-2 * np.abs(ref)
        assert np.isfinite(g).all() and not bad.any(), f"case {i} {name}: {bad.sum()} out of tolerance"
