"""Forward under the window-and-anchor sparse mask on the GPU against the
float64 oracle (exact attention under the same mask).  Tolerances are the
bf16 path's."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import compare, ra, sample_rows

pytestmark = pytest.mark.gpu

CASES = [
    # (B, Hq, Hkv, N, d, window, period, P)
    (2, 4, 2, 1024, 128, 100, 256, 1),
    (1, 2, 2, 1024, 128, 300, 512, 4),     # ring chunks of 256 keys
    (1, 4, 1, 1000, 128, 130, 256, 5),     # ragged length, chunks of 200 keys
    (1, 2, 1, 2048, 64, 0, 512, 2),        # window 0: each row's own key plus its anchors
    (1, 2, 2, 768, 128, 768, 256, 3),      # window covering the sequence
    (2, 8, 2, 64, 128, 16, 256, 1),        # short: packed GQA rows, one anchor period
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,W,A,P", CASES)
def test_window_anchor_matches_oracle(B, Hq, Hkv, N, d, W, A, P):
    R = ra()
    w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N, d=d, causal=False, P=P, seed=700 + N + W, window=W,
                        anchor_period=A)
    q, k, v = workloads.make_qkv(w, device="cuda")
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, N), float("nan"), device="cuda")
    R.ring_attn_fwd_window_anchor(q, k, v, window=W, anchor_period=A, P=P, chunk=w.chunk, scale=w.scale, out=out,
                                  lse=lse)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    ro, rl = oracle.attention_window_anchor_ref(q, k, v, window=W, anchor_period=A, scale=w.scale)
    compare(out, lse, ro, rl, "bf16", f"window/anchor N={N} W={W} A={A} P={P}")


def test_window_anchor_full_size_sampled():
    R = ra()
    w = workloads.CONFIGS["wa3"]
    q, k, v = workloads.make_qkv(w, device="cuda")
    out, lse = R.ring_attn_fwd_window_anchor(q, k, v, window=w.window, anchor_period=w.anchor_period, P=w.P,
                                             chunk=w.chunk, scale=w.scale)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    assert torch.isfinite(out.float()).all()
    rows = sample_rows(w, n_random=96, seed=5)
    rows = rows[np.linspace(0, len(rows) - 1, 192).astype(int)]
    heads = [0, 13, 31]
    ro, rl = oracle.attention_window_anchor_ref(q, k, v, window=w.window, anchor_period=w.anchor_period,
                                                scale=w.scale, rows=rows, heads=heads)
    rt = torch.as_tensor(rows, device="cuda")
    compare(out[:, rt][:, :, heads], lse[:, heads][:, :, rt], ro, rl, "bf16", w.name + " (sampled)")


def test_window_anchor_rejects_bad_period():
    R = ra()
    q = torch.zeros((1, 512, 2, 128), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(R.RingAttnError) as ei:
        R.ring_attn_fwd_window_anchor(q, q, q, window=16, anchor_period=100)
    assert ei.value.status == R.RA_ERR_INVALID_ARG
