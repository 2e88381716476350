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


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("P,L,d,Hq,Hkv", [(3, 256, 128, 4, 2), (4, 200, 64, 2, 1), (2, 130, 128, 2, 2)])
def test_backward_block_steps_sum_to_full_gradient(causal, P, L, d, Hq, Hkv):
    # Every (query chunk, KV chunk) visit through ring_attn_bwd_block_step
    # into float32 accumulators, in ring order; fully future causal visits
    # are skipped as the ring driver skips them.  The sum is the gradient.
    R = ra()
    N = P * L
    w = workloads.small(B=1, Hq=Hq, Hkv=Hkv, N_q=N, d=d, causal=causal, P=P, seed=300 + L + d)
    q, k, v = workloads.make_qkv(w, device="cuda")
    dout = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(w.seed + 1),
                       device="cuda").to(torch.bfloat16)
    out, lse = R.ring_attn_fwd(q, k, v, causal=causal, P=1, scale=w.scale)
    dq = torch.zeros(q.shape, device="cuda")
    dk = torch.zeros(k.shape, device="cuda")
    dv = torch.zeros(v.shape, device="cuda")
    for i in range(P):
        qs = slice(i * L, (i + 1) * L)
        q_i, o_i, do_i = (x[:, qs].contiguous() for x in (q, out, dout))
        lse_i = lse[:, :, qs].contiguous()
        dq_i = torch.zeros(q_i.shape, device="cuda")
        for s in range(P):
            j = (i + s) % P
            if causal and j > i:
                continue
            ks = slice(j * L, (j + 1) * L)
            k_j, v_j = k[:, ks].contiguous(), v[:, ks].contiguous()
            dk_j, dv_j = dk[:, ks].contiguous(), dv[:, ks].contiguous()
            R.ring_attn_bwd_block_step(q_i, k_j, v_j, o_i, do_i, lse_i, i * L, j * L, dq_i, dk_j, dv_j,
                                       causal=causal, scale=w.scale)
            dk[:, ks] = dk_j
            dv[:, ks] = dv_j
        dq[:, qs] = dq_i
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    rq, rk, rv = oracle.attention_bwd_ref(q, k, v, dout, causal=causal, scale=w.scale)
    _check(dv, rv, "dv")
    _check(dk, rk, "dk")
    _check(dq, rq, "dq")


def test_backward_block_step_adds_to_accumulators():
    # One diagonal causal visit at nonzero offsets against the oracle's visit,
    # starting from nonzero accumulators (the call adds, it does not overwrite).
    R = ra()
    w = workloads.small(B=2, Hq=4, Hkv=2, N_q=384, d=128, causal=True, P=1, seed=410)
    q, k, v = workloads.make_qkv(w, device="cuda")
    dout = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(411),
                       device="cuda").to(torch.bfloat16)
    out, lse = R.ring_attn_fwd(q, k, v, causal=True, P=1, scale=w.scale)
    qs, ks = slice(256, 384), slice(128, 384)   # queries 256..383 against keys 128..383
    q_c, o_c, do_c = (x[:, qs].contiguous() for x in (q, out, dout))
    lse_c = lse[:, :, qs].contiguous()
    k_c, v_c = k[:, ks].contiguous(), v[:, ks].contiguous()
    g = torch.Generator(device="cuda").manual_seed(412)
    dq0 = torch.randn(q_c.shape, generator=g, device="cuda")
    dk0 = torch.randn(k_c.shape, generator=g, device="cuda")
    dv0 = torch.randn(v_c.shape, generator=g, device="cuda")
    dq, dk, dv = dq0.clone(), dk0.clone(), dv0.clone()
    R.ring_attn_bwd_block_step(q_c, k_c, v_c, o_c, do_c, lse_c, 256, 128, dq, dk, dv, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    delta = torch.einsum("bthe,bthe->bht", do_c.double(), o_c.double()).cpu()
    rq, rk, rv = oracle.block_step_bwd_ref(q_c, k_c, v_c, do_c, lse_c, delta, 256, 128, dq0, dk0, dv0, causal=True,
                                           scale=w.scale)
    _check(dv, rv, "dv")
    _check(dk, rk, "dk")
    _check(dq, rq, "dq")
