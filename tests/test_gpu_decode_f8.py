"""The FP8-cache decode on the 8-bit MMA path (E4M3 codes as tcgen05
operands; bf16 queries and the probabilities each split into two E4M3
planes, x = hi + lo / 16) against the float64 oracle over the dequantised
cache.

The split is exact for bf16 queries within 2^14 of their row's largest
entry (a per-row power-of-two scale puts that entry in [224, 448]), so rows
of very different magnitudes, all-zero rows and padding rows are the cases
that exercise it; peaky scores exercise the running base and the rescale of
both planes of O.  Tolerances are the bf16 path's.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import compare, ra

pytestmark = pytest.mark.gpu

W = workloads.small

CASES = [
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, causal, P)
    (1, 8, 1, 2, 700, 698, True, 7),        # G = 8, 16 rows; chunks of 100 keys (ragged tiles)
    (2, 2, 2, 16, 1000, 984, True, 4),      # G = 1, 16 tokens per block
    (1, 16, 8, 9, 3000, 2991, True, 3),     # G = 2, 18 rows in a 32-row block
    (1, 32, 1, 1, 4096, 4095, True, 8),     # G = 32, one token
    (1, 4, 1, 3, 2048, 1000, False, 8),     # not causal
    (1, 4, 2, 6, 512, 5, True, 4),          # queries near the start: most keys masked
    (3, 12, 3, 5, 900, 895, True, 9),       # G = 4, 20 rows, B = 3
    (4, 32, 8, 1, 16384, 16383, True, 16),  # decode, 4 heads per KV head, 32 batch x head blocks
]


def _fp8_case(w, q_row_exp=None, k_mult=1.0):
    q, k8, v8, ks, vs = workloads.make_fp8_kv(w, device="cuda")
    if q_row_exp is not None:
        # Scale each (token, head) row of q by 2^e (exact in bf16).
        q = (q.float() * torch.exp2(q_row_exp.to(q.device).float())[None, :, :, None]).to(torch.bfloat16)
    if k_mult != 1.0:
        ks = ks * k_mult
    return q, k8, v8, ks, vs


def _run_and_compare(w, q, k8, v8, ks, vs, what):
    R = ra()
    ci = None if w.cache_idx < 0 else w.cache_idx
    out, lse = R.ring_attn_fwd_fp8kv(q, k8, v8, ks, vs, causal=w.causal, P=w.P, cache_idx=ci, scale=w.scale)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    ro, rl = oracle.attention_fp8kv_ref(q, k8, v8, ks, vs, causal=w.causal, scale=w.scale, cache_idx=w.cache_idx)
    return compare(out, lse, ro, rl, "bf16", what)


@pytest.mark.parametrize("route", ["", "all"])
@pytest.mark.parametrize("splits", ["", "1", "3"])
@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,causal,P", CASES)
def test_decode_f8_matches_oracle(monkeypatch, route, splits, B, Hq, Hkv, N_q, N_kv, ci, causal, P):
    # route "all": blocks of 17-32 packed rows also take the 8-bit kernel
    # (32-row configuration); by default they take the converter kernel.
    monkeypatch.setenv("RINGATTN_DECODE", route)
    monkeypatch.setenv("RINGATTN_SPLITS", splits)
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=128, causal=causal, P=P, seed=N_kv + 31,
          kv_dtype="fp8")
    _run_and_compare(w, *_fp8_case(w), w.name)


@pytest.mark.parametrize("N_q,Hq,Hkv", [(1, 16, 1), (4, 32, 8)])
def test_decode_f8_query_rows_of_any_magnitude(N_q, Hq, Hkv):
    # Rows scaled by 2^e for e from -40 to +2, and all-zero rows: each row
    # gets its own power-of-two scale before the split into E4M3 planes.
    # (Larger rows would make logits too large for any float32 lse to stay
    # within an absolute 1e-3.)
    w = W(B=2, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=1536, cache_idx=1536 - N_q, d=128, causal=True, P=3, seed=777,
          kv_dtype="fp8")
    g = torch.Generator().manual_seed(5)
    e = torch.randint(-40, 3, (N_q, Hq), generator=g)
    q, k8, v8, ks, vs = _fp8_case(w, q_row_exp=e)
    q[:, 0, 0] = 0  # an all-zero query row: uniform weights over its keys
    _run_and_compare(w, q, k8, v8, ks, vs, "rows of any magnitude")


def test_decode_f8_peaky_scores_rescale_both_planes():
    # Large k_scale makes scores spread over tens of log2 units, so the
    # running base moves often and both E4M3 planes of O are rescaled.
    w = W(B=1, Hq=8, Hkv=2, N_q=2, N_kv=4096, cache_idx=4094, d=128, causal=True, P=4, seed=778, kv_dtype="fp8")
    q, k8, v8, ks, vs = _fp8_case(w, k_mult=8.0)
    _run_and_compare(w, q, k8, v8, ks, vs, "peaky scores")


def test_decode_f8_agrees_with_the_converter_kernel(monkeypatch):
    # The same FP8 decode on the 8-bit MMA path and, with the decode kernels
    # switched off, on the general kernel that converts the codes to bf16.
    R = ra()
    w = W(B=2, Hq=32, Hkv=8, N_q=1, N_kv=8192, cache_idx=8191, d=128, causal=True, P=8, seed=92, kv_dtype="fp8")
    q, k8, v8, ks, vs = workloads.make_fp8_kv(w, device="cuda")
    o1, l1 = R.ring_attn_fwd_fp8kv(q, k8, v8, ks, vs, causal=True, P=8, cache_idx=8191, scale=w.scale)
    monkeypatch.setenv("RINGATTN_DECODE", "0")
    o2, l2 = R.ring_attn_fwd_fp8kv(q, k8, v8, ks, vs, causal=True, P=8, cache_idx=8191, scale=w.scale)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


@pytest.mark.parametrize("route", ["", "all"])
def test_decode_f8_full_length_8_tokens(monkeypatch, route):
    # 8 new tokens x 4 heads = 32 packed rows against the 262144-token FP8
    # cache: sampled batch rows and KV-head groups against the oracle.
    monkeypatch.setenv("RINGATTN_DECODE", route)
    R = ra()
    w = workloads.CONFIGS["5d8f8"]
    q, k8, v8, ks, vs = workloads.make_fp8_kv(w, device="cuda")
    out, lse = R.ring_attn_fwd_fp8kv(q, k8, v8, ks, vs, causal=True, P=w.P, cache_idx=w.cache_idx, scale=w.scale)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    assert torch.isfinite(out.float()).all()
    G = w.Hq // w.Hkv
    for b, hk in ((0, 0), (w.B - 1, w.Hkv - 1)):
        hs = slice(hk * G, (hk + 1) * G)
        ro, rl = oracle.attention_fp8kv_ref(q[b:b + 1, :, hs], k8[b:b + 1, :, hk:hk + 1], v8[b:b + 1, :, hk:hk + 1],
                                            ks[b:b + 1, hk:hk + 1], vs[b:b + 1, hk:hk + 1], causal=True,
                                            scale=w.scale, cache_idx=w.cache_idx)
        compare(out[b:b + 1, :, hs], lse[b:b + 1, hs], ro, rl, "bf16", f"5d8f8 b={b} hk={hk}")
