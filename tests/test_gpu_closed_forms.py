"""GPU results against closed forms that need no oracle.  Exact softmax
attention ("Ring Attention: the secret of million-token context", §2.3,
with the blockwise inner loop of §3.1) gives:

- a query that sees exactly one key gets that key's value (its softmax
  weight is 1) and lse = scale * q.k;
- when all keys are equal, every visible key gets the same weight, so a
  query gets the mean of the values it sees and lse = scale * q.k + ln n.

These hold for any ring size P, chunking and visit order, so they check
the blockwise merge as well as the tile arithmetic.  Tolerances: the weight
of a single key is exp2 of a rounding error, so out is within one bf16 ulp
(2^-7 of the value at most) of the value; means are compared at the bf16
bound 2e-2, lse at 1e-3."""
import numpy as np
import pytest
import torch

import workloads
from parity_util import ra

pytestmark = pytest.mark.gpu

BF16_ULP = 2.0 ** -7  # one bf16 ulp relative to a value at the bottom of its binade


def _f64(t):
    return t.detach().double().cpu().numpy()


def _run(q, k, v, causal, P, cache_idx, scale):
    R = ra()
    out, lse = R.ring_attn_fwd(q, k, v, causal=causal, P=P, cache_idx=cache_idx, scale=scale)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    return out, lse


@pytest.mark.parametrize("B,Hq,Hkv,N,d,P", [
    (2, 4, 2, 300, 128, 3),    # two query tiles per CTA, chunk 100
    (1, 8, 1, 1000, 128, 8),   # GQA 8, chunk 125
    (1, 2, 2, 256, 64, 2),
])
def test_first_causal_row_is_first_value(B, Hq, Hkv, N, d, P):
    w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N, d=d, causal=True, P=P, seed=500 + N + d)
    q, k, v = workloads.make_qkv(w, device="cuda")
    out, lse = _run(q, k, v, True, P, None, w.scale)
    G = Hq // Hkv
    o0, v0 = _f64(out[:, 0]), _f64(v[:, 0])
    q0, k0 = _f64(q[:, 0]), _f64(k[:, 0])
    for h in range(Hq):
        err = np.abs(o0[:, h] - v0[:, h // G])
        assert (err <= BF16_ULP * np.abs(v0[:, h // G])).all(), f"head {h}: {err.max():.3e}"
        ref_lse = w.scale * np.sum(q0[:, h] * k0[:, h // G], axis=-1)
        assert np.abs(_f64(lse[:, h, 0]) - ref_lse).max() <= 1e-3


@pytest.mark.parametrize("splits", ["", "1", "4"])
def test_lone_query_at_cache_start_sees_one_key(monkeypatch, splits):
    # The query sits at position 0 of a 4096-key cache: one key is visible,
    # so every split but one is empty and must carry no weight in the merge.
    monkeypatch.setenv("RINGATTN_SPLITS", splits)
    w = workloads.small(B=2, Hq=8, Hkv=2, N_q=1, N_kv=4096, cache_idx=0, d=128, causal=True, P=4, seed=611)
    q, k, v = workloads.make_qkv(w, device="cuda")
    out, lse = _run(q, k, v, True, 4, 0, w.scale)
    o, v0 = _f64(out[:, 0]), _f64(v[:, 0])
    q0, k0 = _f64(q[:, 0]), _f64(k[:, 0])
    for h in range(8):
        assert (np.abs(o[:, h] - v0[:, h // 4]) <= BF16_ULP * np.abs(v0[:, h // 4])).all(), h
        ref_lse = w.scale * np.sum(q0[:, h] * k0[:, h // 4], axis=-1)
        assert np.abs(_f64(lse[:, h, 0]) - ref_lse).max() <= 1e-3


@pytest.mark.parametrize("causal,N,d,P", [
    (False, 500, 128, 5),
    (True, 300, 128, 3),
    (True, 384, 64, 4),
])
def test_equal_keys_give_mean_of_visible_values(causal, N, d, P):
    B, Hq, Hkv = 1, 4, 2
    w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N, d=d, causal=causal, P=P, seed=700 + N)
    q, k, v = workloads.make_qkv(w, device="cuda")
    k = k[:, :1].expand(-1, N, -1, -1).contiguous()  # every key equals key 0
    out, lse = _run(q, k, v, causal, P, None, w.scale)
    vv, qq, k0 = _f64(v), _f64(q), _f64(k[:, 0])
    n_vis = np.arange(1, N + 1) if causal else np.full(N, N)
    # Mean of the visible values per row: cumulative for causal rows.
    csum = np.cumsum(vv, axis=1)
    mean = (csum / n_vis[None, :, None, None]) if causal else np.broadcast_to(vv.mean(axis=1, keepdims=True), vv.shape)
    o = _f64(out)
    for h in range(Hq):
        hk = h // (Hq // Hkv)
        assert np.abs(o[:, :, h] - mean[:, :, hk]).max() <= 2e-2, h
        s = w.scale * np.sum(qq[:, :, h] * k0[:, None, hk], axis=-1)
        ref_lse = s + np.log(n_vis)[None, :]
        assert np.abs(_f64(lse[:, h]) - ref_lse).max() <= 1e-3, h
