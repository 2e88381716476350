"""Host-only checks of the C ABI: the library loads, exports every entry point
the header declares, and rejects invalid arguments before touching a device.
No GPU needed: validation runs before any CUDA call, so fake (never
dereferenced) pointers are enough."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "ring_attn.h")


def _lib():
    from long_context_exact_blockwise_b200 import build_lib
    build_lib.build()
    import long_context_exact_blockwise_b200.ringattn as ra
    return ra


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("ring_attn_fwd", "ring_attn_fwd_f32", "ring_attn_block_step", "ring_attn_finalize", "lse_merge",
              "ring_attn_sync_status", "ring_attn_error_string", "ring_attn_last_error", "ring_attn_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    ra = _lib()
    out = subprocess.run(["nm", "-D", "--defined-only", ra.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out.stdout, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert hasattr(ra.lib, n)


def test_error_strings_and_version():
    ra = _lib()
    assert ra.ring_attn_error_string(ra.RA_OK) == "ok"
    for s in range(1, 6):
        assert ra.ring_attn_error_string(s) not in ("", "ok", "unknown status")
    assert ra.ring_attn_error_string(99) == "unknown status"
    assert ra.ring_attn_version() >= 100


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced by validation


def _fwd(ra, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, N_q=512, N_kv=512, d=128, causal=1,
             chunk=128, P=4, cache_idx=-1, scale=0.088, stream=None)
    a.update(kw)
    return ra.lib.ring_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["N_q"],
                                a["N_kv"], a["d"], a["causal"], a["chunk"], a["P"], a["cache_idx"], a["scale"],
                                a["stream"])


@pytest.mark.parametrize("bad", [
    dict(q=None), dict(lse=None), dict(d=96), dict(d=256), dict(Hq=3, Hkv=2), dict(Hkv=0), dict(B=-1),
    dict(P=0), dict(chunk=100), dict(N_kv=500, chunk=125), dict(N_q=256),  # prefill needs N_q == N_kv
    dict(cache_idx=-2), dict(cache_idx=400, N_q=200), dict(causal=2), dict(scale=float("inf")),
    dict(scale=float("nan")), dict(q=ctypes.c_void_p(0x10008)), dict(N_q=2 ** 31, N_kv=2 ** 31, chunk=2 ** 29),
])
def test_fwd_rejects_invalid_arguments(bad):
    ra = _lib()
    assert _fwd(ra, **bad) == ra.RA_ERR_INVALID_ARG


def test_fwd_rejects_length_not_multiple_of_P():
    # The pitfall "sequence length not a multiple of the device count" is an error.
    ra = _lib()
    assert _fwd(ra, N_q=1000, N_kv=1000, P=3, chunk=333) == ra.RA_ERR_INVALID_ARG


def test_empty_inputs_are_noops():
    ra = _lib()
    assert _fwd(ra, B=0) == ra.RA_OK
    assert _fwd(ra, N_q=0, cache_idx=100) == ra.RA_OK


def test_valid_call_without_gpu_reports_unsupported():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    ra = _lib()
    assert _fwd(ra) == ra.RA_ERR_UNSUPPORTED
    assert "device" in ra.lib.ring_attn_last_error().decode()


def test_block_step_finalize_merge_validation():
    ra = _lib()
    L = ra.lib
    ok_args = (FAKE, FAKE, FAKE, 0, 0, FAKE, FAKE, FAKE, 1, 4, 2, 128, 128, 64, 1, 0.1, ra.RA_DTYPE_BF16, None)
    bad = list(ok_args); bad[16] = 7
    assert L.ring_attn_block_step(*bad) == ra.RA_ERR_INVALID_ARG
    bad = list(ok_args); bad[3] = -1
    assert L.ring_attn_block_step(*bad) == ra.RA_ERR_INVALID_ARG
    bad = list(ok_args); bad[5] = ctypes.c_void_p(0x10004)  # acc not 16-byte aligned
    assert L.ring_attn_block_step(*bad) == ra.RA_ERR_INVALID_ARG
    bad = list(ok_args); bad[12] = 0  # Lk == 0: nothing to fold in
    assert L.ring_attn_block_step(*bad) == ra.RA_OK
    assert L.ring_attn_finalize(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 8, 100, 0, None) == ra.RA_ERR_INVALID_ARG
    assert L.ring_attn_finalize(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 8, 64, 5, None) == ra.RA_ERR_INVALID_ARG
    assert L.lse_merge(FAKE, FAKE, 0, FAKE, FAKE, 1, 2, 8, 64, 0, None) == ra.RA_ERR_INVALID_ARG
    assert L.lse_merge(None, FAKE, 2, FAKE, FAKE, 1, 2, 8, 64, 0, None) == ra.RA_ERR_INVALID_ARG
    assert L.lse_merge(FAKE, FAKE, 2, FAKE, FAKE, 1, 2, 0, 64, 0, None) == ra.RA_OK


def test_bwd_block_step_validation():
    ra = _lib()
    L = ra.lib
    # q, k, v, out, dout, lse, q_off, k_off, dq, dk, dv, B, Hq, Hkv, Lq, Lk, d, causal, scale, stream
    ok_args = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 128, FAKE, FAKE, FAKE, 1, 4, 2, 128, 128, 64, 1, 0.1, None)
    assert L.ring_attn_bwd_block_step(*ok_args) == ra.RA_ERR_UNSUPPORTED  # valid, but no GPU here
    for i, val in ((6, -1), (7, -5), (12, 3), (16, 96), (17, 2), (18, float("nan"))):
        bad = list(ok_args); bad[i] = val
        assert L.ring_attn_bwd_block_step(*bad) == ra.RA_ERR_INVALID_ARG, i
    for i in (0, 3, 4, 5, 8, 9, 10):
        bad = list(ok_args); bad[i] = None
        assert L.ring_attn_bwd_block_step(*bad) == ra.RA_ERR_INVALID_ARG, i
    bad = list(ok_args); bad[9] = ctypes.c_void_p(0x10004)  # dk accumulator not 16-byte aligned
    assert L.ring_attn_bwd_block_step(*bad) == ra.RA_ERR_INVALID_ARG
    bad = list(ok_args); bad[15] = 0  # Lk == 0: nothing to add
    assert L.ring_attn_bwd_block_step(*bad) == ra.RA_OK


def test_fp8kv_validation():
    ra = _lib()
    L = ra.lib
    # q, k8, v8, k_scale, v_scale, out, lse, B, Hq, Hkv, N_q, N_kv, d, causal, chunk, P, cache_idx, scale, stream
    ok_args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 1, 256, 128, 1, 128, 2, 255, 0.1, None]
    assert L.ring_attn_fwd_fp8kv(*ok_args) == ra.RA_ERR_UNSUPPORTED  # valid, but no GPU here
    for i in (3, 4):
        bad = list(ok_args); bad[i] = None
        assert L.ring_attn_fwd_fp8kv(*bad) == ra.RA_ERR_INVALID_ARG, i
    bad = list(ok_args); bad[3] = ctypes.c_void_p(0x10002)  # k_scale not 4-byte aligned
    assert L.ring_attn_fwd_fp8kv(*bad) == ra.RA_ERR_INVALID_ARG
    bad = list(ok_args); bad[12] = 96
    assert L.ring_attn_fwd_fp8kv(*bad) == ra.RA_ERR_INVALID_ARG
    bad = list(ok_args); bad[14] = 100  # N_kv != P * chunk
    assert L.ring_attn_fwd_fp8kv(*bad) == ra.RA_ERR_INVALID_ARG


def test_window_anchor_validation():
    ra = _lib()
    L = ra.lib
    # q, k, v, out, lse, B, Hq, Hkv, N, d, chunk, P, window, anchor_period, scale, stream
    ok_args = [FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 1024, 128, 256, 4, 64, 256, 0.1, None]
    assert L.ring_attn_fwd_window_anchor(*ok_args) == ra.RA_ERR_UNSUPPORTED  # valid, but no GPU here
    for i, val in ((12, -1), (13, 0), (13, 100), (13, 384), (9, 96), (10, 100)):
        bad = list(ok_args); bad[i] = val
        assert L.ring_attn_fwd_window_anchor(*bad) == ra.RA_ERR_INVALID_ARG, (i, val)


def test_add_and_clear_validation():
    ra = _lib()
    L = ra.lib
    assert L.ring_attn_add_and_clear(FAKE, ctypes.c_void_p(0x20000), 64, None) == ra.RA_ERR_UNSUPPORTED  # no GPU
    assert L.ring_attn_add_and_clear(FAKE, ctypes.c_void_p(0x20000), 0, None) == ra.RA_OK
    assert L.ring_attn_add_and_clear(FAKE, ctypes.c_void_p(0x20000), -1, None) == ra.RA_ERR_INVALID_ARG
    assert L.ring_attn_add_and_clear(None, FAKE, 8, None) == ra.RA_ERR_INVALID_ARG
    assert L.ring_attn_add_and_clear(FAKE, FAKE, 8, None) == ra.RA_ERR_INVALID_ARG  # the same buffer twice
    assert L.ring_attn_add_and_clear(FAKE, ctypes.c_void_p(0x20002), 8, None) == ra.RA_ERR_INVALID_ARG  # unaligned


def test_nvtx_ranges_switch_keeps_validation(monkeypatch):
    # RINGATTN_NVTX=1 wraps every compute entry point in an NVTX range; with
    # no profiler attached the ranges do nothing and validation is unchanged.
    ra = _lib()
    monkeypatch.setenv("RINGATTN_NVTX", "1")
    L = ra.lib
    assert L.ring_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 128, 128, 96, 1, 128, 1, -1, 0.1, None) == \
        ra.RA_ERR_INVALID_ARG
    assert L.ring_attn_add_and_clear(FAKE, ctypes.c_void_p(0x20000), 0, None) == ra.RA_OK


def test_fwd_host_validation():
    # The host-buffer forward validates like ring_attn_fwd, and its group size
    # must divide Hkv; all of it before any CUDA call.
    ra = _lib()
    L = ra.lib
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 4, 512, 512, 128, 1, 128, 4, -1, 0.088, 0, None]
    for i, val in ((16, -1), (16, 3), (16, 5), (10, 96), (0, None), (5, -1)):
        bad = list(ok); bad[i] = val
        assert L.ring_attn_fwd_host(*bad) == ra.RA_ERR_INVALID_ARG, (i, val)
    zero_b = list(ok); zero_b[5] = 0
    assert L.ring_attn_fwd_host(*zero_b) == ra.RA_OK  # nothing to do: no device needed
    assert L.ring_attn_fwd_host(*ok) == ra.RA_ERR_UNSUPPORTED  # valid, but no GPU here


def test_bwd_host_validation():
    ra = _lib()
    L = ra.lib
    ok = [FAKE] * 9 + [1, 8, 4, 512, 512, 128, 1, -1, 0.088, 0, None]
    for i, val in ((18, -1), (18, 3), (18, 8), (14, 96), (4, None), (8, None), (6, ctypes.c_void_p(0x10008))):
        bad = list(ok); bad[i] = val
        assert L.ring_attn_bwd_host(*bad) == ra.RA_ERR_INVALID_ARG, (i, val)
    zero_b = list(ok); zero_b[9] = 0
    assert L.ring_attn_bwd_host(*zero_b) == ra.RA_OK
    assert L.ring_attn_bwd_host(*ok) == ra.RA_ERR_UNSUPPORTED  # valid, but no GPU here


def test_window_anchor_host_validation():
    ra = _lib()
    L = ra.lib
    ok = [FAKE] * 5 + [1, 8, 4, 1024, 128, 256, 4, 300, 256, 0.088, 0, None]
    for i, val in ((15, -1), (15, 3), (13, 100), (12, -1), (9, 96), (0, None)):
        bad = list(ok); bad[i] = val
        assert L.ring_attn_fwd_window_anchor_host(*bad) == ra.RA_ERR_INVALID_ARG, (i, val)
    assert L.ring_attn_fwd_window_anchor_host(*ok) == ra.RA_ERR_UNSUPPORTED  # valid, but no GPU here
