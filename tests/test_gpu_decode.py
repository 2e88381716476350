"""The keys-on-M decode kernel (d = 128, incremental queries with at most 32
packed rows per KV head) against the float64 oracle, for both KV-cache
types, over the row-packing shapes it takes (G from 1 to 32, padding rows,
16- and 32-row blocks) and several split counts."""
import pytest
import torch

import oracle
import workloads
from parity_util import check_workload, compare, ra

pytestmark = pytest.mark.gpu

W = workloads.small

DECODE_CASES = [
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, causal, P)
    (1, 8, 1, 2, 700, 698, True, 7),        # G = 8, 16 rows; chunks of 100 keys
    (2, 2, 2, 16, 1000, 984, True, 4),      # G = 1, 16 tokens per block
    (1, 16, 8, 9, 3000, 2991, True, 3),     # G = 2, 18 rows in a 32-row block
    (1, 32, 1, 1, 4096, 4095, True, 8),     # G = 32, one token
    (1, 32, 2, 2, 2048, 2046, True, 8),     # G = 16, 32 rows
    (1, 4, 1, 3, 2048, 1000, False, 8),     # not causal: keys after the queries count
    (1, 2, 2, 30, 1280, 1250, True, 5),     # G = 1, 30 tokens in a 32-row block
    (1, 4, 2, 6, 512, 5, True, 4),          # queries near the start: most keys masked
    (3, 12, 3, 5, 900, 895, True, 9),       # G = 4, 20 rows, B = 3
]


@pytest.mark.parametrize("route", ["", "all"])
@pytest.mark.parametrize("splits", ["", "1", "7", "64"])
@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,causal,P", DECODE_CASES)
def test_decode_bf16(monkeypatch, route, splits, B, Hq, Hkv, N_q, N_kv, ci, causal, P):
    # route "all": 17-32-row blocks also go to the decode kernel.
    monkeypatch.setenv("RINGATTN_DECODE", route)
    monkeypatch.setenv("RINGATTN_SPLITS", splits)
    check_workload(W(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=128, causal=causal, P=P,
                     seed=N_kv + Hq + N_q))


@pytest.mark.parametrize("route", ["", "all"])
@pytest.mark.parametrize("splits", ["", "1", "5"])
@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,causal,P", DECODE_CASES[:6])
def test_decode_fp8kv(monkeypatch, route, splits, B, Hq, Hkv, N_q, N_kv, ci, causal, P):
    monkeypatch.setenv("RINGATTN_DECODE", route)
    monkeypatch.setenv("RINGATTN_SPLITS", splits)
    R = ra()
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=128, causal=causal, P=P, seed=N_kv + 17,
          kv_dtype="fp8")
    q, k8, v8, ks, vs = workloads.make_fp8_kv(w, device="cuda")
    out, lse = R.ring_attn_fwd_fp8kv(q, k8, v8, ks, vs, causal=causal, P=P, cache_idx=ci, scale=w.scale)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    ro, rl = oracle.attention_fp8kv_ref(q, k8, v8, ks, vs, causal=causal, scale=w.scale, cache_idx=ci)
    compare(out, lse, ro, rl, "bf16", w.name)


def test_decode_kernel_agrees_with_the_general_kernel(monkeypatch):
    # The same decode step through the keys-on-M kernel and, with it switched
    # off, through the general kernel: both within tolerance of each other.
    R = ra()
    w = W(B=2, Hq=32, Hkv=8, N_q=1, N_kv=8192, cache_idx=8191, d=128, causal=True, P=8, seed=91)
    q, k, v = workloads.make_qkv(w, device="cuda")
    o1, l1 = R.ring_attn_fwd(q, k, v, causal=True, P=8, cache_idx=8191, scale=w.scale)
    monkeypatch.setenv("RINGATTN_DECODE", "0")
    o2, l2 = R.ring_attn_fwd(q, k, v, causal=True, P=8, cache_idx=8191, scale=w.scale)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-4
