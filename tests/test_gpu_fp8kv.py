"""Forward over an FP8 (E4M3) KV cache on the GPU against the float64 oracle.

The oracle attends over the dequantised cache (codes decoded by the format's
definition, times the per-(batch, KV head) scales).  Decode-shaped blocks
(d = 128, at most 32 packed rows per KV head) run on the 8-bit MMA path with
the codes as operands; other shapes decode the codes to bf16 (exact) in
shared memory.  Both fold the scales into the score scale and the final
normalisation.  Tolerances are the bf16 path's.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import TOL_LSE, TOL_OUT, compare, ra

pytestmark = pytest.mark.gpu

CASES = [
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, d, causal, P)
    (2, 8, 2, 1, 1024, 1023, 128, True, 4),     # decode, 4 query heads packed per tile
    (1, 32, 8, 8, 2048, 2040, 128, True, 8),    # 8 new tokens x 4 heads = 32 packed rows
    (1, 4, 4, 1, 700, 699, 128, True, 1),       # ragged cache length
    (2, 4, 1, 3, 520, 517, 64, True, 4),        # d = 64, 12 packed rows
    (1, 2, 2, 200, 200, -1, 128, True, 2),      # prefill over an FP8 cache
    (1, 4, 2, 130, 384, 254, 128, False, 3),    # incremental queries, non-causal
    (1, 16, 2, 64, 4096, 4032, 128, True, 8),   # 512 rows per KV head: several query tiles
]


def _run(w):
    R = ra()
    q, k8, v8, ks, vs = workloads.make_fp8_kv(w, device="cuda")
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.Hq, w.N_q), float("nan"), device="cuda")
    ci = None if w.cache_idx < 0 else w.cache_idx
    R.ring_attn_fwd_fp8kv(q, k8, v8, ks, vs, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci, scale=w.scale,
                          out=out, lse=lse)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    return q, k8, v8, ks, vs, out, lse


@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,d,causal,P", CASES)
def test_fp8kv_matches_oracle(B, Hq, Hkv, N_q, N_kv, ci, d, causal, P):
    w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=causal, P=P,
                        seed=600 + N_kv + d, kv_dtype="fp8")
    q, k8, v8, ks, vs, out, lse = _run(w)
    ro, rl = oracle.attention_fp8kv_ref(q, k8, v8, ks, vs, causal=causal, scale=w.scale, cache_idx=ci)
    compare(out, lse, ro, rl, "bf16", w.name)


def test_fp8kv_equals_bf16_path_on_the_decoded_cache():
    # With power-of-two scales the converter kernel (FP8 codes decoded to bf16
    # in shared memory) and the bf16 kernel on the decoded cache do the same
    # float operations in the same order: the results must agree bit for bit
    # (this checks the decode and its layout).  16 tokens x 4 heads = 64
    # packed rows: more than the 8-bit decode kernel takes.
    R = ra()
    w = workloads.small(B=2, Hq=8, Hkv=2, N_q=16, N_kv=2048, cache_idx=2032, d=128, causal=True, P=4, seed=650,
                        kv_dtype="fp8")
    q, k8, v8, _, _ = workloads.make_fp8_kv(w, device="cuda")
    sc = torch.full((w.B, w.Hkv), 2.0 ** -6, device="cuda")
    o8, l8 = R.ring_attn_fwd_fp8kv(q, k8, v8, sc, sc, causal=True, P=w.P, cache_idx=w.cache_idx, scale=w.scale)
    kd = (k8.view(torch.float8_e4m3fn).to(torch.float32) * 2.0 ** -6).to(torch.bfloat16)
    vd = (v8.view(torch.float8_e4m3fn).to(torch.float32) * 2.0 ** -6).to(torch.bfloat16)
    ob, lb = R.ring_attn_fwd(q, kd, vd, causal=True, P=w.P, cache_idx=w.cache_idx, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o8, ob)
    assert torch.equal(l8, lb)


def test_fp8kv_full_size_decode():
    # The full-length decode (N_kv = 262144) on every batch row and the first
    # and last KV-head group.
    w = workloads.CONFIGS["5d1f8"]
    q, k8, v8, ks, vs, out, lse = _run(w)
    assert torch.isfinite(out.float()).all()
    G = w.Hq // w.Hkv
    for b in range(w.B):
        for hk in (0, w.Hkv - 1):
            hs = slice(hk * G, (hk + 1) * G)
            ro, rl = oracle.attention_fp8kv_ref(q[b:b + 1, :, hs], k8[b:b + 1, :, hk:hk + 1],
                                                v8[b:b + 1, :, hk:hk + 1], ks[b:b + 1, hk:hk + 1],
                                                vs[b:b + 1, hk:hk + 1], causal=True, scale=w.scale,
                                                cache_idx=w.cache_idx)
            compare(out[b:b + 1, :, hs], lse[b:b + 1, hs], ro, rl, "bf16", f"{w.name} b={b} hk={hk}")


def test_fp8kv_rejects_a_state_free_misuse():
    R = ra()
    q = torch.zeros((1, 1, 2, 128), device="cuda", dtype=torch.bfloat16)
    k8 = torch.zeros((1, 256, 2, 128), device="cuda", dtype=torch.uint8)
    sc = torch.ones((1, 2), device="cuda")
    with pytest.raises(ValueError):
        R.ring_attn_fwd_fp8kv(q, k8, k8, sc[:, :1], sc, causal=True, P=2, cache_idx=255)
