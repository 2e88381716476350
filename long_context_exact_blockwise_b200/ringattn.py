"""Python binding of libringattn.so (exact blockwise ring attention, B200).

A thin ctypes layer over ``libringattn.so`` (C ABI in ``include/ring_attn.h``).
Each function here has the name of the C entry point it calls and does only
argument marshalling: every step of the computation runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.

If the shared object is missing or cannot be loaded, importing this package
raises ImportError: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "RingAttnError", "lib", "LIB_PATH",
    "ring_attn_fwd", "ring_attn_fwd_f32", "ring_attn_fwd_noalloc", "ring_attn_fwd_fp8kv", "ring_attn_fwd_window_anchor", "ring_attn_bwd", "ring_attn_bwd_block_step", "ring_attn_block_step", "ring_attn_finalize",
    "lse_merge", "ring_attn_sync_status", "ring_attn_error_string", "ring_attn_version", "ring_attn_launch_count", "ring_attn_exp2_poly", "ring_attn_add_and_clear",
    "ring_attn", "init_state",
    "RA_OK", "RA_ERR_INVALID_ARG", "RA_ERR_UNSUPPORTED", "RA_ERR_CUDA", "RA_ERR_DEVICE_TIMEOUT",
    "RA_ERR_OOM", "RA_DTYPE_BF16", "RA_DTYPE_F32",
]

RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_CUDA, RA_ERR_DEVICE_TIMEOUT, RA_ERR_OOM = range(6)
RA_DTYPE_BF16, RA_DTYPE_F32 = 0, 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libringattn.so")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m long_context_exact_blockwise_b200.build_lib` (needs nvcc)")
    try:
        return ctypes.CDLL(LIB_PATH)
    except OSError as e:  # pragma: no cover
        raise ImportError(f"cannot load {LIB_PATH}: {e}") from e


lib = _load()

_p = ctypes.c_void_p
_i = ctypes.c_int
_l = ctypes.c_int64
_f = ctypes.c_float

_SIGS = {
    "ring_attn_fwd": [_p, _p, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _l, _i, _l, _f, _p],
    "ring_attn_fwd_f32": [_p, _p, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _l, _i, _l, _f, _p],
    "ring_attn_fwd_noalloc": [_p, _p, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _l, _i, _l, _f, _p],
    "ring_attn_fwd_host": [_p, _p, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _l, _i, _l, _f, _i, _p],
    "ring_attn_bwd_host": [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _l, _f, _i, _p],
    "ring_attn_fwd_window_anchor": [_p, _p, _p, _p, _p, _i, _i, _i, _l, _i, _l, _i, _l, _l, _f, _p],
    "ring_attn_fwd_window_anchor_host": [_p, _p, _p, _p, _p, _i, _i, _i, _l, _i, _l, _i, _l, _l, _f, _i, _p],
    "ring_attn_fwd_fp8kv": [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _l, _i, _l, _f, _p],
    "ring_attn_bwd": [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _l, _f, _p],
    "ring_attn_bwd_block_step": [_p, _p, _p, _p, _p, _p, _l, _l, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _f, _p],
    "ring_attn_block_step": [_p, _p, _p, _l, _l, _p, _p, _p, _i, _i, _i, _l, _l, _i, _i, _f, _i, _p],
    "ring_attn_finalize": [_p, _p, _p, _p, _p, _i, _i, _l, _i, _i, _p],
    "lse_merge": [_p, _p, _i, _p, _p, _i, _i, _l, _i, _i, _p],
    "ring_attn_sync_status": [_p],
    "ring_attn_error_string": [_i],
    "ring_attn_last_error": [],
    "ring_attn_version": [],
    "ring_attn_launch_count": [],
    "ring_attn_exp2_poly": [_p, _p, _l, _p],
    "ring_attn_add_and_clear": [_p, _p, _l, _p],
}
for _name, _args in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_char_p if _name in ("ring_attn_error_string", "ring_attn_last_error") else _i
lib.ring_attn_launch_count.restype = ctypes.c_int64


class RingAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.ring_attn_error_string(status).decode()
        detail = lib.ring_attn_last_error().decode()
        super().__init__(f"{where}: status {status} ({msg}){': ' + detail if detail else ''}")


def _check(status: int, where: str) -> None:
    if status != RA_OK:
        raise RingAttnError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype: torch.dtype):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def ring_attn_error_string(status: int) -> str:
    return lib.ring_attn_error_string(status).decode()


def ring_attn_version() -> int:
    return lib.ring_attn_version()


def ring_attn_exp2_poly(x: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """2^x by the softmax's FMA-pipe polynomial (for checking its error)."""
    _need(x, "x", torch.float32)
    y = torch.empty_like(x) if out is None else out
    _check(lib.ring_attn_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream, x.device)), "ring_attn_exp2_poly")
    return y


def ring_attn_add_and_clear(acc: torch.Tensor, part: torch.Tensor, stream=None) -> torch.Tensor:
    """acc += part, then part = 0 (float32, same shape): folds one ring
    visit's dk / dv share into the accumulators travelling the ring."""
    _need(acc, "acc", torch.float32)
    _need(part, "part", torch.float32)
    if acc.shape != part.shape or acc.device != part.device:
        raise ValueError("acc and part must have the same shape and device")
    _check(lib.ring_attn_add_and_clear(_ptr(acc), _ptr(part), acc.numel(), _stream(stream, acc.device)),
           "ring_attn_add_and_clear")
    return acc


def ring_attn_launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(lib.ring_attn_launch_count())


def ring_attn_sync_status(stream=None, device=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return lib.ring_attn_sync_status(_stream(stream, device))


def _fwd(fn, dtype, q, k, v, causal, P, chunk, cache_idx, scale, out, lse, stream):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dtype)
    B, N_q, Hq, d = q.shape
    _, N_kv, Hkv, dk = k.shape
    if k.shape != v.shape or dk != d or k.shape[0] != B:
        raise ValueError("k and v must be [B, N_kv, Hkv, d] matching q")
    if chunk is None:
        chunk = N_kv // P if P > 0 else 0
    ci = -1 if cache_idx is None else int(cache_idx)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N_q), device=q.device, dtype=torch.float32)
    _need(out, "out", dtype)
    _need(lse, "lse", torch.float32)
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N_q, N_kv, d, int(bool(causal)),
            int(chunk), int(P), ci, sc, _stream(stream, q.device))
    _check(st, fn.__name__)
    return out, lse


def ring_attn_fwd(q, k, v, *, causal: bool, P: int, chunk: Optional[int] = None, cache_idx=None,
                  scale: Optional[float] = None, out=None, lse=None, stream=None):
    """bf16 forward: q [B,N_q,Hq,d], k/v [B,N_kv,Hkv,d] -> (out bf16, lse f32 [B,Hq,N_q])."""
    return _fwd(lib.ring_attn_fwd, torch.bfloat16, q, k, v, causal, P, chunk, cache_idx, scale, out, lse,
                stream)


def _need_host(t: torch.Tensor, name: str, dtype: torch.dtype):
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a CPU (host) tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def ring_attn_fwd_host(q, k, v, *, causal: bool, P: int, chunk: Optional[int] = None, cache_idx=None,
                       scale: Optional[float] = None, out=None, lse=None, kv_heads_per_group: int = 0,
                       stream=None):
    """bf16 forward for host tensors, copies overlapped with the compute.

    q [B,N_q,Hq,d], k/v [B,N_kv,Hkv,d] are CPU tensors (pinned for overlap);
    out / lse are CPU tensors (pinned ones are allocated if None).  The work is
    queued on `stream` (the current CUDA stream by default): synchronise it
    before reading out and lse.  Returns (out, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need_host(t, n, torch.bfloat16)
    B, N_q, Hq, d = q.shape
    _, N_kv, Hkv, dk = k.shape
    if k.shape != v.shape or dk != d or k.shape[0] != B:
        raise ValueError("k and v must be [B, N_kv, Hkv, d] matching q")
    if chunk is None:
        chunk = N_kv // P if P > 0 else 0
    ci = -1 if cache_idx is None else int(cache_idx)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    if lse is None:
        lse = torch.empty((B, Hq, N_q), dtype=torch.float32).pin_memory()
    _need_host(out, "out", torch.bfloat16)
    _need_host(lse, "lse", torch.float32)
    device = torch.cuda.current_device()
    st = lib.ring_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N_q, N_kv, d,
                                int(bool(causal)), int(chunk), int(P), ci, sc, int(kv_heads_per_group),
                                _stream(stream, device))
    _check(st, "ring_attn_fwd_host")
    return out, lse


def ring_attn_bwd_host(q, k, v, out, dout, lse, *, causal: bool, cache_idx=None, scale: Optional[float] = None,
                       dq=None, dk=None, dv=None, kv_heads_per_group: int = 0, stream=None):
    """Gradients of ring_attn_fwd's output for host tensors, copies overlapped
    with the compute.  Inputs are CPU tensors (pinned for overlap); dq / dk /
    dv are CPU tensors (pinned ones are allocated if None).  Synchronise
    `stream` before reading them.  Returns (dq, dk, dv)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need_host(t, n, torch.bfloat16)
    _need_host(lse, "lse", torch.float32)
    B, N_q, Hq, d = q.shape
    _, N_kv, Hkv, _ = k.shape
    dq = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() if dq is None else dq
    dk = torch.empty(k.shape, dtype=torch.bfloat16).pin_memory() if dk is None else dk
    dv = torch.empty(v.shape, dtype=torch.bfloat16).pin_memory() if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need_host(t, n, torch.bfloat16)
    ci = -1 if cache_idx is None else int(cache_idx)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = lib.ring_attn_bwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                _ptr(dv), B, Hq, Hkv, N_q, N_kv, d, int(bool(causal)), ci, sc,
                                int(kv_heads_per_group), _stream(stream, torch.cuda.current_device()))
    _check(st, "ring_attn_bwd_host")
    return dq, dk, dv


def ring_attn_fwd_f32(q, k, v, *, causal: bool, P: int, chunk: Optional[int] = None, cache_idx=None,
                      scale: Optional[float] = None, out=None, lse=None, stream=None):
    """float32 forward (CUDA-core float32 arithmetic); same layouts as ring_attn_fwd."""
    return _fwd(lib.ring_attn_fwd_f32, torch.float32, q, k, v, causal, P, chunk, cache_idx, scale, out, lse,
                stream)


def ring_attn_fwd_noalloc(q, k, v, *, causal: bool, P: int, cache_idx: int, chunk: Optional[int] = None,
                          scale: Optional[float] = None, out=None, lse=None, stream=None):
    """Incremental-query forward that allocates no device memory inside the
    library (for callers whose memory is owned by their own pool or budget).
    Split-KV partials use a fixed 16 MiB device array shared by all calls:
    calls that may overlap on the GPU race, and over-large calls raise.
    Pass ``out`` and ``lse`` to avoid allocations on the Python side too."""
    return _fwd(lib.ring_attn_fwd_noalloc, torch.bfloat16, q, k, v, causal, P, chunk, cache_idx, scale, out, lse,
                stream)


def ring_attn_fwd_fp8kv(q, k8, v8, k_scale, v_scale, *, causal: bool, P: int, chunk: Optional[int] = None,
                        cache_idx=None, scale: Optional[float] = None, out=None, lse=None, stream=None):
    """Forward over an FP8 E4M3 KV cache: q bf16 [B,N_q,Hq,d]; k8/v8 uint8 codes
    [B,N_kv,Hkv,d]; k_scale/v_scale float32 [B,Hkv] -> (out bf16, lse f32)."""
    _need(q, "q", torch.bfloat16)
    for t, n in ((k8, "k8"), (v8, "v8")):
        _need(t, n, torch.uint8)
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _need(t, n, torch.float32)
    B, N_q, Hq, d = q.shape
    _, N_kv, Hkv, dk = k8.shape
    if k8.shape != v8.shape or dk != d or k8.shape[0] != B:
        raise ValueError("k8 and v8 must be [B, N_kv, Hkv, d] matching q")
    if tuple(k_scale.shape) != (B, Hkv) or tuple(v_scale.shape) != (B, Hkv):
        raise ValueError("k_scale and v_scale must be [B, Hkv]")
    if chunk is None:
        chunk = N_kv // P if P > 0 else 0
    ci = -1 if cache_idx is None else int(cache_idx)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N_q), device=q.device, dtype=torch.float32) if lse is None else lse
    _need(out, "out", torch.bfloat16)
    _need(lse, "lse", torch.float32)
    st = lib.ring_attn_fwd_fp8kv(_ptr(q), _ptr(k8), _ptr(v8), _ptr(k_scale), _ptr(v_scale), _ptr(out), _ptr(lse),
                                 B, Hq, Hkv, N_q, N_kv, d, int(bool(causal)), int(chunk), int(P), ci, sc,
                                 _stream(stream, q.device))
    _check(st, "ring_attn_fwd_fp8kv")
    return out, lse


def ring_attn_fwd_window_anchor(q, k, v, *, window: int, anchor_period: int, P: int = 1,
                                chunk: Optional[int] = None, scale: Optional[float] = None, out=None, lse=None,
                                stream=None):
    """bf16 square prefill under the window-and-anchor sparse mask -> (out, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16)
    B, N, Hq, d = q.shape
    _, N_kv, Hkv, _ = k.shape
    if N_kv != N or v.shape != k.shape:
        raise ValueError("the window-and-anchor mask needs N_q == N_kv")
    chunk = N // P if chunk is None else chunk
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32) if lse is None else lse
    _need(out, "out", torch.bfloat16)
    _need(lse, "lse", torch.float32)
    st = lib.ring_attn_fwd_window_anchor(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d,
                                         int(chunk), int(P), int(window), int(anchor_period), sc,
                                         _stream(stream, q.device))
    _check(st, "ring_attn_fwd_window_anchor")
    return out, lse


def ring_attn_fwd_window_anchor_host(q, k, v, *, window: int, anchor_period: int, P: int = 1,
                                     chunk: Optional[int] = None, scale: Optional[float] = None, out=None, lse=None,
                                     kv_heads_per_group: int = 0, stream=None):
    """ring_attn_fwd_window_anchor for host tensors, copies overlapped with the
    compute (as ring_attn_fwd_host).  Synchronise `stream` before reading
    out and lse.  Returns (out, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need_host(t, n, torch.bfloat16)
    B, N, Hq, d = q.shape
    _, N_kv, Hkv, _ = k.shape
    if N_kv != N or v.shape != k.shape:
        raise ValueError("the window-and-anchor mask needs N_q == N_kv")
    chunk = N // P if chunk is None else chunk
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32).pin_memory() if lse is None else lse
    _need_host(out, "out", torch.bfloat16)
    _need_host(lse, "lse", torch.float32)
    st = lib.ring_attn_fwd_window_anchor_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d,
                                              int(chunk), int(P), int(window), int(anchor_period), sc,
                                              int(kv_heads_per_group), _stream(stream, torch.cuda.current_device()))
    _check(st, "ring_attn_fwd_window_anchor_host")
    return out, lse


def ring_attn_bwd(q, k, v, out, dout, lse, *, causal: bool, cache_idx=None, scale: Optional[float] = None,
                  dq=None, dk=None, dv=None, stream=None):
    """Gradients (dq, dk, dv) of ring_attn_fwd's output for upstream dout (bf16)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, n, torch.bfloat16)
    _need(lse, "lse", torch.float32)
    B, N_q, Hq, d = q.shape
    _, N_kv, Hkv, _ = k.shape
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ci = -1 if cache_idx is None else int(cache_idx)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = lib.ring_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                           _ptr(dv), B, Hq, Hkv, N_q, N_kv, d, int(bool(causal)), ci, sc, _stream(stream, q.device))
    _check(st, "ring_attn_bwd")
    return dq, dk, dv


def ring_attn_bwd_block_step(q_chunk, k_chunk, v_chunk, out_chunk, dout_chunk, lse_chunk, q_off: int, k_off: int,
                             dq_acc, dk_acc, dv_acc, *, causal: bool, scale: Optional[float] = None,
                             stream=None) -> None:
    """Add one ring visit's share of (dq, dk, dv) into float32 accumulators, in place."""
    for t, n in ((q_chunk, "q_chunk"), (k_chunk, "k_chunk"), (v_chunk, "v_chunk"), (out_chunk, "out_chunk"),
                 (dout_chunk, "dout_chunk")):
        _need(t, n, torch.bfloat16)
    for t, n in ((lse_chunk, "lse_chunk"), (dq_acc, "dq_acc"), (dk_acc, "dk_acc"), (dv_acc, "dv_acc")):
        _need(t, n, torch.float32)
    B, Lq, Hq, d = q_chunk.shape
    _, Lk, Hkv, _ = k_chunk.shape
    if dq_acc.shape != q_chunk.shape or dk_acc.shape != k_chunk.shape or dv_acc.shape != v_chunk.shape:
        raise ValueError("accumulator shapes must match q_chunk / k_chunk / v_chunk")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = lib.ring_attn_bwd_block_step(_ptr(q_chunk), _ptr(k_chunk), _ptr(v_chunk), _ptr(out_chunk),
                                      _ptr(dout_chunk), _ptr(lse_chunk), int(q_off), int(k_off), _ptr(dq_acc),
                                      _ptr(dk_acc), _ptr(dv_acc), B, Hq, Hkv, Lq, Lk, d, int(bool(causal)), sc,
                                      _stream(stream, q_chunk.device))
    _check(st, "ring_attn_bwd_block_step")


def ring_attn(q, k, v, *, causal: bool, P: int, cache_idx=None, scale=None, stream=None):
    """Forward pass choosing the entry point by input dtype (bf16 or float32)."""
    if q.dtype == torch.float32:
        return ring_attn_fwd_f32(q, k, v, causal=causal, P=P, cache_idx=cache_idx, scale=scale, stream=stream)
    return ring_attn_fwd(q, k, v, causal=causal, P=P, cache_idx=cache_idx, scale=scale, stream=stream)


def init_state(B: int, Hq: int, Lq: int, d: int, device) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Empty running state for ring_attn_block_step: acc = 0, m = -inf, l = 0."""
    acc = torch.zeros((B, Hq, Lq, d), device=device, dtype=torch.float32)
    m = torch.full((B, Hq, Lq), float("-inf"), device=device, dtype=torch.float32)
    l = torch.zeros((B, Hq, Lq), device=device, dtype=torch.float32)
    return acc, m, l


def ring_attn_block_step(q_chunk, k_chunk, v_chunk, q_off: int, k_off: int, acc, m, l, *, causal: bool,
                         scale: Optional[float] = None, stream=None) -> None:
    """Fold one ring visit into (acc, m, l) in place; dtype from q_chunk (bf16 or float32)."""
    dtype = q_chunk.dtype
    code = {torch.bfloat16: RA_DTYPE_BF16, torch.float32: RA_DTYPE_F32}.get(dtype)
    if code is None:
        raise ValueError("q_chunk must be bf16 or float32")
    for t, n in ((q_chunk, "q_chunk"), (k_chunk, "k_chunk"), (v_chunk, "v_chunk")):
        _need(t, n, dtype)
    for t, n in ((acc, "acc"), (m, "m"), (l, "l")):
        _need(t, n, torch.float32)
    B, Lq, Hq, d = q_chunk.shape
    _, Lk, Hkv, _ = k_chunk.shape
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = lib.ring_attn_block_step(_ptr(q_chunk), _ptr(k_chunk), _ptr(v_chunk), int(q_off), int(k_off), _ptr(acc),
                                  _ptr(m), _ptr(l), B, Hq, Hkv, Lq, Lk, d, int(bool(causal)), sc, code,
                                  _stream(stream, q_chunk.device))
    _check(st, "ring_attn_block_step")


def ring_attn_finalize(acc, m, l, *, out_dtype=torch.bfloat16, out=None, lse=None, stream=None):
    """(acc [B,Hq,Lq,d], m, l) -> (out [B,Lq,Hq,d] out_dtype, lse [B,Hq,Lq])."""
    for t, n in ((acc, "acc"), (m, "m"), (l, "l")):
        _need(t, n, torch.float32)
    B, Hq, Lq, d = acc.shape
    if out is None:
        out = torch.empty((B, Lq, Hq, d), device=acc.device, dtype=out_dtype)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), device=acc.device, dtype=torch.float32)
    code = RA_DTYPE_F32 if out.dtype == torch.float32 else RA_DTYPE_BF16
    st = lib.ring_attn_finalize(_ptr(acc), _ptr(m), _ptr(l), _ptr(out), _ptr(lse), B, Hq, Lq, d, code,
                                _stream(stream, acc.device))
    _check(st, "ring_attn_finalize")
    return out, lse


def lse_merge(o_parts, lse_parts, *, out_dtype=torch.bfloat16, out=None, lse=None, stream=None):
    """o_parts [S,B,N_q,Hq,d], lse_parts [S,B,Hq,N_q] (float32) -> (out, lse)."""
    _need(o_parts, "o_parts", torch.float32)
    _need(lse_parts, "lse_parts", torch.float32)
    S, B, N_q, Hq, d = o_parts.shape
    if out is None:
        out = torch.empty((B, N_q, Hq, d), device=o_parts.device, dtype=out_dtype)
    if lse is None:
        lse = torch.empty((B, Hq, N_q), device=o_parts.device, dtype=torch.float32)
    code = RA_DTYPE_F32 if out.dtype == torch.float32 else RA_DTYPE_BF16
    st = lib.lse_merge(_ptr(o_parts), _ptr(lse_parts), S, _ptr(out), _ptr(lse), B, Hq, N_q, d, code,
                       _stream(stream, o_parts.device))
    _check(st, "lse_merge")
    return out, lse
