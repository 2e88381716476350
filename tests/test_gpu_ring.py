"""The ring driver with its default CUDA compute (block step + finalize
kernels) on one GPU: a one-rank group runs the whole sequence as a single
ring step, which must match the float64 oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import workloads
from parity_util import TOL_LSE, TOL_OUT

pytestmark = pytest.mark.gpu


@pytest.fixture
def one_rank_group():
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_driver_cuda_compute(one_rank_group, dtype, causal):
    from long_context_exact_blockwise_b200.ring import ring_attention
    w = workloads.small(B=2, Hq=4, Hkv=2, N_q=384, d=128, dtype=dtype, causal=causal, P=1, seed=90)
    q, k, v = workloads.make_qkv(w, device="cuda")
    out, lse = ring_attention(q, k, v, causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_ref(q, k, v, causal=causal, scale=w.scale)
    assert np.max(np.abs(out.float().cpu().numpy() - ro)) <= TOL_OUT[dtype]
    assert np.max(np.abs(lse.cpu().numpy() - rl)) <= TOL_LSE


@pytest.mark.parametrize("causal", [True, False])
def test_ring_driver_cuda_backward(one_rank_group, causal):
    from long_context_exact_blockwise_b200.ring import ring_attention, ring_attention_bwd
    w = workloads.small(B=2, Hq=4, Hkv=2, N_q=384, d=128, causal=causal, P=1, seed=91)
    q, k, v = workloads.make_qkv(w, device="cuda")
    dout = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(92),
                       device="cuda").to(torch.bfloat16)
    out, lse = ring_attention(q, k, v, causal=causal, scale=w.scale)
    dq, dk, dv = ring_attention_bwd(q, k, v, out, dout, lse, causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    ref = oracle.attention_bwd_ref(q, k, v, dout, causal=causal, scale=w.scale)
    for got, r in zip((dq, dk, dv), ref):
        g = got.float().cpu().numpy()
        assert np.all(np.abs(g - r) <= 2e-2 + 2e-2 * np.abs(r))


@pytest.mark.parametrize("n,offset", [(1, 0), (7, 0), (4096 * 3 + 5, 0), (1000, 1), (12345, 3)])
def test_add_and_clear(n, offset):
    # acc += part, part = 0, on 16-byte aligned buffers (vector path and a
    # tail) and on buffers offset by 1 or 3 floats (scalar path).
    import long_context_exact_blockwise_b200.ringattn as R
    g = torch.Generator(device="cuda").manual_seed(n)
    acc_full = torch.randn(n + offset, generator=g, device="cuda")
    part_full = torch.randn(n + offset, generator=g, device="cuda")
    acc, part = acc_full[offset:], part_full[offset:]
    want = (acc.double() + part.double()).float()
    before_head = acc_full[:offset].clone()
    R.lib.ring_attn_add_and_clear(acc.data_ptr(), part.data_ptr(), n, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.equal(acc, want)
    assert torch.count_nonzero(part).item() == 0
    assert torch.equal(acc_full[:offset], before_head)
