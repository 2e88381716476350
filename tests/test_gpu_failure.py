"""Failure detection on the GPU without faulting it.

Every mbarrier wait in the tensor-core kernel is bounded (2 s of wall time).
RINGATTN_FAULT=device_wait makes the TMA producer issue no copies -- a
barrier nothing completes -- so the MMA thread's wait for Q expires: the
kernel records RA_ERR_DEVICE_TIMEOUT in the device status word, unwinds
(no MMAs issued, TMEM freed) and exits.  The host reads the status, and the
context stays usable: the next normal call is correct.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import TOL_LSE, TOL_OUT, ra

pytestmark = pytest.mark.gpu


# One query tile; two query tiles in one CTA; the CTA-pair kernel (one and
# two pair tiles).
@pytest.mark.parametrize("N,pair", [(128, ""), (256, ""), (256, "1"), (600, "1")])
def test_bounded_wait_expiry_reports_status_and_context_survives(monkeypatch, N, pair):
    monkeypatch.setenv("RINGATTN_PAIR", pair)
    R = ra()
    w = workloads.small(B=1, Hq=1, Hkv=1, N_q=N, d=128, causal=True, P=1, seed=5)
    q, k, v = workloads.make_qkv(w, device="cuda")
    assert R.ring_attn_sync_status() == R.RA_OK
    monkeypatch.setenv("RINGATTN_FAULT", "device_wait")
    R.ring_attn_fwd(q, k, v, causal=True, P=1)        # launches; the error is on the device
    monkeypatch.delenv("RINGATTN_FAULT")
    assert R.ring_attn_sync_status() == R.RA_ERR_DEVICE_TIMEOUT
    assert R.ring_attn_sync_status() == R.RA_OK      # read and cleared
    # The context is intact: a normal call is correct.
    out, lse = R.ring_attn_fwd(q, k, v, causal=True, P=1)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_ref(q, k, v, causal=True, scale=w.scale)
    assert np.max(np.abs(out.float().cpu().numpy() - ro)) <= TOL_OUT["bf16"]
    assert np.max(np.abs(lse.cpu().numpy() - rl)) <= TOL_LSE
    assert R.ring_attn_sync_status() == R.RA_OK


def test_debug_mode_reports_timeout_from_the_call(monkeypatch):
    R = ra()
    w = workloads.small(B=1, Hq=1, Hkv=1, N_q=128, d=64, causal=False, P=1, seed=6)
    q, k, v = workloads.make_qkv(w, device="cuda")
    monkeypatch.setenv("RINGATTN_DEBUG", "1")
    monkeypatch.setenv("RINGATTN_FAULT", "device_wait")
    with pytest.raises(R.RingAttnError) as ei:
        R.ring_attn_fwd(q, k, v, causal=False, P=1)
    assert ei.value.status == R.RA_ERR_DEVICE_TIMEOUT
    monkeypatch.delenv("RINGATTN_FAULT")
    out, _ = R.ring_attn_fwd(q, k, v, causal=False, P=1)   # synchronised, status checked
    assert torch.isfinite(out.float()).all()


def test_workspace_allocation_failure_is_reported(monkeypatch):
    R = ra()
    w = workloads.small(B=1, Hq=4, Hkv=1, N_q=2, N_kv=1024, cache_idx=1022, d=128, causal=True, P=8, seed=7)
    q, k, v = workloads.make_qkv(w, device="cuda")
    monkeypatch.setenv("RINGATTN_SPLITS", "4")
    monkeypatch.setenv("RINGATTN_FAULT", "alloc")
    with pytest.raises(R.RingAttnError) as ei:
        R.ring_attn_fwd(q, k, v, causal=True, P=8, cache_idx=1022)
    assert ei.value.status == R.RA_ERR_OOM
