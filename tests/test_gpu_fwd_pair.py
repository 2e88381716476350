"""The CTA-pair forward (cta_group::2 MMAs over 256-row pair tiles; each CTA
holds half of every K and V tile; P through shared memory) against the
float64 oracle, and against the single-CTA kernel.

It takes bf16 problems with d = 128 and more than 128 query rows, for the
final output and for split-KV partials, when RINGATTN_PAIR=1 (it is off by
default; these tests turn it on).  The cases cover pair query blocks
cut by the end of the sequence (N not a multiple of 512, so the second CTA
or the second pair tile has few or no valid rows), GQA, causal and not,
ring chunks that are not multiples of 128, incremental queries (cache_idx)
with split counts, and peaky scores that move the running base so the O
accumulators are rescaled.
"""
import pytest
import torch

import workloads
from parity_util import check_workload, ra

pytestmark = pytest.mark.gpu

W = workloads.small

CASES = [
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, causal, P, k_scale)
    (1, 2, 2, 512, None, -1, True, 2, 1.0),
    (1, 2, 1, 257, None, -1, True, 1, 1.0),       # second pair tile: one valid row
    (1, 4, 2, 300, None, -1, True, 3, 1.0),       # the second CTA of the pair tile 0 has 44 valid rows
    (2, 2, 2, 600, None, -1, False, 4, 1.0),
    (1, 4, 4, 1000, None, -1, True, 8, 1.0),      # chunks of 125 keys
    (1, 8, 2, 1536, None, -1, True, 3, 2.0),      # peaky scores
    (1, 2, 2, 777, None, -1, True, 7, 4.0),       # very peaky, ragged
    (2, 4, 1, 384, 2048, 1664, True, 8, 1.0),     # incremental queries
    (1, 8, 8, 200, 1000, 800, False, 5, 1.0),     # incremental, not causal
]


@pytest.mark.parametrize("splits", ["", "1", "3"])
@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,causal,P,ks", CASES)
def test_pair_forward_matches_oracle(monkeypatch, splits, B, Hq, Hkv, N_q, N_kv, ci, causal, P, ks):
    monkeypatch.setenv("RINGATTN_PAIR", "1")
    monkeypatch.setenv("RINGATTN_SPLITS", splits)
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=128, causal=causal, P=P, k_scale=ks,
          seed=N_q + 7 * Hq + P)
    check_workload(w)


def test_pair_kernel_agrees_with_single_cta_kernel(monkeypatch):
    R = ra()
    w = W(B=1, Hq=4, Hkv=2, N_q=4096, d=128, causal=True, P=4, seed=811)
    q, k, v = workloads.make_qkv(w, device="cuda")
    monkeypatch.setenv("RINGATTN_PAIR", "1")
    o1, l1 = R.ring_attn_fwd(q, k, v, causal=True, P=w.P, scale=w.scale)
    monkeypatch.setenv("RINGATTN_PAIR", "0")
    o2, l2 = R.ring_attn_fwd(q, k, v, causal=True, P=w.P, scale=w.scale)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-4
