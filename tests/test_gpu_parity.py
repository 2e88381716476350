"""GPU parity: the CUDA path through the C ABI against the float64 oracle,
element by element, on seeded inputs.  Sizes span several 128-row/128-key
tiles and ragged tails; tolerances are in parity_util (bf16: out 2e-2,
lse 1e-3; float32: out 1e-4, lse 1e-3)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import TOL_LSE, TOL_OUT, check_workload, compare, ra

pytestmark = pytest.mark.gpu

W = workloads.small

PREFILL_CASES = [
    # (B, Hq, Hkv, N, d, causal, P)
    (1, 2, 2, 128, 128, True, 1),
    (1, 2, 2, 256, 128, True, 2),
    (1, 2, 2, 512, 128, False, 4),
    (2, 4, 1, 384, 128, True, 3),
    (1, 8, 1, 1024, 128, True, 8),
    (1, 4, 2, 1000, 128, True, 8),     # chunk 125: tiles straddle chunk edges
    (1, 2, 2, 200, 128, True, 2),      # ragged: 200 rows, chunk 100
    (1, 2, 1, 77, 128, False, 1),      # single ragged tile
    (2, 2, 2, 640, 64, True, 5),
    (1, 4, 4, 300, 64, False, 3),
    (1, 2, 2, 1, 128, True, 1),        # one token
    (1, 3, 1, 96, 64, True, 4),        # chunk 24
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,P", PREFILL_CASES)
def test_prefill_bf16(B, Hq, Hkv, N, d, causal, P):
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N, d=d, causal=causal, P=P, seed=N + 7 * P + d)
    check_workload(w)


PACKED_CASES = [
    # Query heads of a KV group packed into one tile (G * N_q <= 128).
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, d, P, causal)
    (1, 8, 1, 16, 16, -1, 128, 2, True),       # packed prefill, G = 8
    (1, 4, 1, 30, 30, -1, 64, 3, True),        # packed prefill, G = 4, chunk 10
    (2, 16, 2, 3, 1024, 1021, 128, 8, True),   # decode, G = 8
    (1, 16, 1, 8, 2048, 2040, 128, 16, True),  # decode, G = 16, 128 rows
    (1, 4, 2, 33, 512, 400, 128, 4, True),     # G = 2, 66 rows, unaligned cache_idx
    (1, 8, 2, 7, 768, 300, 64, 6, False),      # non-causal incremental, G = 4
]


@pytest.mark.parametrize("splits", ["", "1", "5"])
@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,d,P,causal", PACKED_CASES)
def test_packed_heads_bf16(monkeypatch, splits, B, Hq, Hkv, N_q, N_kv, ci, d, P, causal):
    monkeypatch.setenv("RINGATTN_SPLITS", splits)
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=causal, P=P, seed=3 * N_q + Hq)
    check_workload(w)


def test_prefill_bf16_peaky_keys():
    # Keys scaled by 4 (exact) give logits with std ~4: a sharply peaked softmax.
    check_workload(W(Hq=4, Hkv=2, N_q=512, d=128, causal=True, P=4, k_scale=4.0, seed=11))


INCR_CASES = [
    # (B, Hq, Hkv, N_q, N_kv, cache_idx, d, P)
    (1, 4, 1, 1, 1024, 1023, 128, 8),
    (2, 8, 2, 8, 1024, 1016, 128, 8),
    (1, 4, 1, 128, 1024, 896, 128, 8),
    (1, 4, 2, 300, 2048, 1748, 128, 16),
    (1, 4, 4, 64, 1024, 100, 128, 4),     # unaligned cache_idx, keys past the queries masked
    (1, 2, 1, 200, 512, 0, 64, 4),        # queries at the start of the cache
    (1, 4, 1, 5, 640, 635, 64, 5),
]


@pytest.mark.parametrize("splits", ["", "1", "3", "64"])
@pytest.mark.parametrize("B,Hq,Hkv,N_q,N_kv,ci,d,P", INCR_CASES)
def test_cache_idx_bf16(monkeypatch, splits, B, Hq, Hkv, N_q, N_kv, ci, d, P):
    monkeypatch.setenv("RINGATTN_SPLITS", splits)
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, cache_idx=ci, d=d, causal=True, P=P, seed=N_q + ci)
    check_workload(w)


def test_cache_idx_noncausal_bf16():
    check_workload(W(Hq=4, Hkv=1, N_q=32, N_kv=1024, cache_idx=500, d=128, causal=False, P=8, seed=5))


def test_cache_idx_rows_equal_prefill_rows():
    # Invariant: incremental rows equal the matching rows of a causal prefill.
    R = ra()
    w = W(Hq=4, Hkv=2, N_q=1024, d=128, causal=True, P=8, seed=3)
    q, k, v = workloads.make_qkv(w, device="cuda")
    o_full, l_full = R.ring_attn_fwd(q, k, v, causal=True, P=8)
    c = 640
    o_inc, l_inc = R.ring_attn_fwd(q[:, c:].contiguous(), k, v, causal=True, P=8, cache_idx=c)
    torch.cuda.synchronize()
    assert (o_inc.float() - o_full[:, c:].float()).abs().max().item() <= TOL_OUT["bf16"]
    assert (l_inc - l_full[:, :, c:]).abs().max().item() <= TOL_LSE


F32_CASES = [
    (1, 1, 1, 256, 64, False, 4, -1, 0),
    (2, 4, 2, 300, 128, True, 3, -1, 0),
    (1, 2, 1, 64, 64, True, 4, 960, 1024),
    (1, 4, 4, 200, 128, False, 2, -1, 0),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,P,ci,N_kv", F32_CASES)
def test_fwd_f32(B, Hq, Hkv, N, d, causal, P, ci, N_kv):
    w = W(B=B, Hq=Hq, Hkv=Hkv, N_q=N, N_kv=(N_kv or None), cache_idx=ci, d=d, dtype="f32", causal=causal, P=P,
          seed=N + d)
    check_workload(w)


def _block_step_sequence(dtype, order, causal, N=512, P=4, Hq=4, Hkv=2, d=128, seed=21):
    R = ra()
    w = W(Hq=Hq, Hkv=Hkv, N_q=N, d=d, dtype=dtype, causal=causal, P=P, seed=seed)
    q, k, v = workloads.make_qkv(w, device="cuda")
    chunk = N // P
    rng = np.random.default_rng(seed)
    outs, lses = [], []
    for i in range(P):
        if order == "forward":
            seq = [oracle.ring_visit_chunk(i, s, P, 1) for s in range(P)]
        elif order == "backward":
            seq = [oracle.ring_visit_chunk(i, s, P, -1) for s in range(P)]
        else:
            seq = list(rng.permutation(P))
        qi = q[:, i * chunk:(i + 1) * chunk].contiguous()
        acc, m, l = R.init_state(w.B, Hq, chunk, d, "cuda")
        for j in seq:
            kj = k[:, j * chunk:(j + 1) * chunk].contiguous()
            vj = v[:, j * chunk:(j + 1) * chunk].contiguous()
            R.ring_attn_block_step(qi, kj, vj, i * chunk, j * chunk, acc, m, l, causal=causal, scale=w.scale)
        out_dt = torch.float32 if dtype == "f32" else torch.bfloat16
        o, ls = R.ring_attn_finalize(acc, m, l, out_dtype=out_dt)
        outs.append(o)
        lses.append(ls)
    torch.cuda.synchronize()
    assert R.ring_attn_sync_status() == 0
    out = torch.cat(outs, dim=1)
    lse = torch.cat(lses, dim=2)
    ro, rl = oracle.attention_ref(q, k, v, causal=causal, scale=w.scale)
    compare(out, lse, ro, rl, dtype, f"block_step {dtype} {order}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("order", ["forward", "backward", "random"])
@pytest.mark.parametrize("causal", [True, False])
def test_block_step_ring(dtype, order, causal):
    _block_step_sequence(dtype, order, causal)


def test_block_step_ragged_chunks_d64():
    _block_step_sequence("bf16", "forward", True, N=400, P=4, Hq=2, Hkv=1, d=64, seed=5)
    _block_step_sequence("f32", "random", True, N=400, P=4, Hq=2, Hkv=1, d=64, seed=6)


def test_block_step_state_matches_oracle_state():
    # The running (m, l) after a sequence of visits match the oracle's.
    R = ra()
    w = W(Hq=2, Hkv=1, N_q=256, d=128, causal=True, P=2, seed=9)
    q, k, v = workloads.make_qkv(w, device="cuda")
    acc, m, l = R.init_state(1, 2, 128, 128, "cuda")
    qi = q[:, 128:].contiguous()
    sa, sm, sl = oracle.init_state(1, 2, 128, 128)
    for j in (1, 0):
        kj, vj = k[:, j * 128:(j + 1) * 128].contiguous(), v[:, j * 128:(j + 1) * 128].contiguous()
        R.ring_attn_block_step(qi, kj, vj, 128, j * 128, acc, m, l, causal=True, scale=w.scale)
        sa, sm, sl = oracle.block_step_ref(qi, kj, vj, 128, j * 128, sa, sm, sl, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert np.max(np.abs(m.cpu().numpy() - sm)) <= 1e-4
    assert np.max(np.abs(l.cpu().numpy() / sl - 1)) <= 1e-3


def test_block_step_masked_visit_leaves_state():
    R = ra()
    w = W(Hq=2, Hkv=2, N_q=256, d=128, causal=True, P=2, seed=10)
    q, k, v = workloads.make_qkv(w, device="cuda")
    acc, m, l = R.init_state(1, 2, 128, 128, "cuda")
    q0 = q[:, :128].contiguous()
    R.ring_attn_block_step(q0, k[:, :128].contiguous(), v[:, :128].contiguous(), 0, 0, acc, m, l, causal=True)
    a0, m0, l0 = acc.clone(), m.clone(), l.clone()
    # Keys 128..255 are all in the future of rows 0..127.
    for dt in (torch.bfloat16, torch.float32):
        R.ring_attn_block_step(q0.to(dt), k[:, 128:].contiguous().to(dt), v[:, 128:].contiguous().to(dt), 0, 128,
                               acc, m, l, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(acc, a0) and torch.equal(m, m0) and torch.equal(l, l0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("S", [1, 2, 5, 64])
@pytest.mark.parametrize("out_dt", [torch.float32, torch.bfloat16])
def test_lse_merge(d, S, out_dt):
    R = ra()
    g = torch.Generator().manual_seed(S * d)
    B, N_q, Hq = 2, 37, 3
    o_parts = torch.randn((S, B, N_q, Hq, d), generator=g)
    lse_parts = torch.randn((S, B, Hq, N_q), generator=g) * 3
    lse_parts[0, 0, 0, :5] = float("-inf")     # empty partials carry no weight
    if S > 1:
        lse_parts[:, 1, 2, 3] = float("-inf")  # a row with no keys anywhere
        o_parts[:, 1, 3, 2] = 0.0
    ro, rl = oracle.lse_merge_ref(o_parts, lse_parts)
    out, lse = R.lse_merge(o_parts.cuda(), lse_parts.cuda(), out_dtype=out_dt)
    torch.cuda.synchronize()
    tol = 1e-5 if out_dt == torch.float32 else 2e-2
    go = out.float().cpu().numpy()
    assert np.max(np.abs(go - ro)) <= tol
    gl = lse.cpu().numpy()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.max(np.abs(gl[fin] - rl[fin])) <= 1e-5


@pytest.mark.parametrize("d", [64, 128])
def test_finalize(d):
    R = ra()
    g = torch.Generator().manual_seed(d)
    B, Hq, Lq = 2, 3, 45
    acc = torch.randn((B, Hq, Lq, d), generator=g)
    m = torch.randn((B, Hq, Lq), generator=g)
    l = torch.rand((B, Hq, Lq), generator=g) + 0.5
    l[0, 1, :4] = 0.0
    m[0, 1, :4] = float("-inf")
    ro, rl = oracle.finalize_ref(acc, m, l)
    for out_dt, tol in ((torch.float32, 1e-6), (torch.bfloat16, 2e-2)):
        out, lse = R.ring_attn_finalize(acc.cuda(), m.cuda(), l.cuda(), out_dtype=out_dt)
        torch.cuda.synchronize()
        assert np.max(np.abs(out.float().cpu().numpy() - ro)) <= tol * max(1.0, float(np.abs(ro).max()))
        gl = lse.cpu().numpy()
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(gl), fin)
        assert np.max(np.abs(gl[fin] - rl[fin])) <= 1e-5


def test_outputs_fully_written_and_status_clear():
    # NaN-poisoned outputs (run_fwd) must come back finite everywhere.
    w = W(B=2, Hq=4, Hkv=1, N_q=777, d=128, causal=True, P=7, seed=77)
    check_workload(w)
    assert ra().ring_attn_sync_status() == 0


def test_invalid_call_launches_nothing():
    R = ra()
    q = torch.zeros((1, 100, 2, 128), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(R.RingAttnError) as ei:
        R.ring_attn_fwd(q, q, q, causal=True, P=3, chunk=33)
    assert ei.value.status == R.RA_ERR_INVALID_ARG


def test_exp2_poly_error_bound():
    # The FMA-pipe exp2 of the softmax against the hardware exp2 (torch.exp2
    # on CUDA): relative error within the fitted minimax bound 7.5e-5 plus
    # float32 rounding, over the exponent range the softmax uses.
    R = ra()
    g = torch.Generator(device="cuda").manual_seed(0)
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001, device="cuda"),
                   torch.rand(1_000_000, device="cuda", generator=g) * 30 - 25,
                   torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, -124.5, 7.5], device="cuda")])
    y = R.ring_attn_exp2_poly(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref) / ref).abs().max().item()
    assert rel <= 7.6e-5, rel
    # Below the clamp the result is 2^-125 up to the same relative error.
    z = R.ring_attn_exp2_poly(torch.tensor([-200.0, -1e30], device="cuda"))
    assert torch.allclose(z.double(), torch.full((2,), 2.0 ** -125, dtype=torch.float64, device="cuda"),
                          rtol=1e-4, atol=0)
