"""Backward pass on the GPU against the float64 gradient oracle.

Tolerance (no bound is given for gradients; derived from the arithmetic):
every element within 2e-2 + 2e-2 * |ref|.  The gradients are written as
bf16 (relative rounding 2^-9) and the GEMMs take bf16 P and dS (relative
2^-9 each, accumulated in float32), so errors stay a small fraction of
that bound; the forward's own out (bf16) and lse feed D and P here, as
they would in training.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import ra

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 2e-2


def _check(got, ref, what):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite"
    err = np.abs(g - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, max err {err.max():.3e}"
    return float(err.max())


CASES = [
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, d, causal)
    (1, 2, 2, 128, 128, -1, 128, True),
    (1, 2, 2, 256, 256, -1, 128, False),
    (2, 4, 2, 384, 384, -1, 128, True),
    (1, 4, 1, 200, 200, -1, 128, True),     # ragged, GQA 4
    (1, 2, 2, 300, 300, -1, 64, True),
    (1, 2, 1, 130, 130, -1, 64, False),
    (1, 4, 2, 96, 512, 416, 128, True),     # incremental queries at the end of the cache
    (1, 2, 2, 64, 640, 100, 128, True),     # unaligned cache_idx: keys past the queries get zero grads
]


@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,d,causal", CASES)
def test_backward_matches_oracle(B, Hq, Hkv, N_q, N_kv, ci, d, causal):
    R = ra()
    w = workloads.small(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=causal, P=1,
                        seed=N_q + 3 * d)
    q, k, v = workloads.make_qkv(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(w.seed + 9)
    dout = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    cache = None if ci < 0 else ci
    out, lse = R.ring_attn_fwd(q, k, v, causal=causal, P=1, cache_idx=cache, scale=w.scale)
    poison = [torch.full_like(x, float("nan")) for x in (q, k, v)]
    dq, dk, dv = R.ring_attn_bwd(q, k, v, out, dout, lse, causal=causal, cache_idx=cache, scale=w.scale,
                                 dq=poison[0], dk=poison[1], dv=poison[2])
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    rq, rk, rv = oracle.attention_bwd_ref(q, k, v, dout, causal=causal, scale=w.scale, cache_idx=ci)
    _check(dv, rv, "dv")
    _check(dk, rk, "dk")
    _check(dq, rq, "dq")


def test_backward_rejects_bad_arguments():
    R = ra()
    q = torch.zeros((1, 128, 2, 96), device="cuda", dtype=torch.bfloat16)  # d = 96 unsupported
    lse = torch.zeros((1, 2, 128), device="cuda")
    with pytest.raises(R.RingAttnError) as ei:
        R.ring_attn_bwd(q, q, q, q, q, lse, causal=True)
    assert ei.value.status == R.RA_ERR_INVALID_ARG


def test_backward_medium_size():
    # 16 query tiles x 16 key tiles per head, causal, GQA 2.
    R = ra()
    w = workloads.small(B=1, Hq=4, Hkv=2, N_q=2048, d=128, causal=True, P=1, seed=77)
    q, k, v = workloads.make_qkv(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(78)
    dout = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    out, lse = R.ring_attn_fwd(q, k, v, causal=True, P=1, scale=w.scale)
    dq, dk, dv = R.ring_attn_bwd(q, k, v, out, dout, lse, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd_ref(q, k, v, dout, causal=True, scale=w.scale)
    _check(dv, rv, "dv")
    _check(dk, rk, "dk")
    _check(dq, rq, "dq")
