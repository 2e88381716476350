"""Seeded synthetic inputs for exact blockwise (ring) attention.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests.  It holds shapes and random-number recipes only: no attention
arithmetic lives here, so neither side can borrow the other's math through it.

Every tensor is drawn as float32 standard normal from a seeded
``torch.Generator`` on the requested device, optionally multiplied by an exact
power of two, then cast (round-to-nearest-even) to the workload's dtype.  The
oracle always consumes the *cast* values, upcast to float64, so both sides see
bit-identical inputs.

Layouts (token-major, row-major contiguous):
  q, out : [B, N_q,  Hq,  d]
  k, v   : [B, N_kv, Hkv, d]
  lse    : [B, Hq, N_q]   (float32, natural log)
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = ["Workload", "CONFIGS", "make_qkv", "make_fp8_kv", "workload", "small"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, ring split and the input recipe."""

    name: str
    B: int
    Hq: int
    Hkv: int
    N_q: int
    N_kv: int
    d: int
    dtype: str            # "bf16" or "f32": element type of q/k/v/out
    causal: bool
    P: int                # number of virtual ring chunks the KV sequence is cut into
    chunk: int            # tokens per chunk; N_kv == P * chunk
    cache_idx: int = -1   # -1: plain prefill (N_q == N_kv); >= 0: queries sit at cache_idx + t
    k_scale: float = 1.0  # exact power-of-two multiplier applied to K before the cast
    seed: int = 0         # q uses seed, k seed+1, v seed+2
    kv_dtype: str = "bf16"  # "fp8": the KV cache is stored as FP8 E4M3 codes with scales (make_fp8_kv)
    window: int = -1        # >= 0: window-and-anchor sparse mask (square prefill) with this window ...
    anchor_period: int = 0  # ... and this anchor period

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"bf16": torch.bfloat16, "f32": torch.float32}[self.dtype]

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five problems the hot path is specified on, plus decode-shaped variants of
# the incremental-query case (same KV cache, 1 or 8 new tokens).
CONFIGS = {
    1: Workload("tiny_exact_f32_N1024", B=1, Hq=1, Hkv=1, N_q=1024, N_kv=1024, d=64,
                dtype="f32", causal=False, P=4, chunk=256, seed=1000),
    2: Workload("llama7b_prefill_N32768", B=1, Hq=32, Hkv=32, N_q=32768, N_kv=32768, d=128,
                dtype="bf16", causal=True, P=8, chunk=4096, seed=2000),
    3: Workload("gqa_prefill_N131072", B=1, Hq=32, Hkv=8, N_q=131072, N_kv=131072, d=128,
                dtype="bf16", causal=True, P=16, chunk=8192, k_scale=2.0, seed=3000),
    4: Workload("prefill_N1048576", B=1, Hq=8, Hkv=1, N_q=1048576, N_kv=1048576, d=128,
                dtype="bf16", causal=True, P=64, chunk=16384, seed=4000),
    5: Workload("cache_idx_query_Nq512_Nkv262144", B=4, Hq=32, Hkv=8, N_q=512, N_kv=262144, d=128,
                dtype="bf16", causal=True, P=64, chunk=4096, cache_idx=262144 - 512, seed=5000),
    "5d1": Workload("cache_idx_decode_Nq1_Nkv262144", B=4, Hq=32, Hkv=8, N_q=1, N_kv=262144, d=128,
                    dtype="bf16", causal=True, P=64, chunk=4096, cache_idx=262144 - 1, seed=5100),
    "5d8": Workload("cache_idx_decode_Nq8_Nkv262144", B=4, Hq=32, Hkv=8, N_q=8, N_kv=262144, d=128,
                    dtype="bf16", causal=True, P=64, chunk=4096, cache_idx=262144 - 8, seed=5200),
    # A quarter-length decode cache (1.07 GB of K/V, still 8x the L2) for
    # profiler captures that must stay small.
    # The full-length decode with its KV cache stored as FP8 E4M3 codes.
    "5d1f8": Workload("cache_idx_decode_fp8kv_Nq1_Nkv262144", B=4, Hq=32, Hkv=8, N_q=1, N_kv=262144, d=128,
                      dtype="bf16", causal=True, P=64, chunk=4096, cache_idx=262144 - 1, seed=5400,
                      kv_dtype="fp8"),
    "5d8f8": Workload("cache_idx_decode_fp8kv_Nq8_Nkv262144", B=4, Hq=32, Hkv=8, N_q=8, N_kv=262144, d=128,
                      dtype="bf16", causal=True, P=64, chunk=4096, cache_idx=262144 - 8, seed=5500,
                      kv_dtype="fp8"),
    # The GQA prefill under the window-and-anchor sparse mask (16K-token window,
    # an anchor every 4096 tokens).
    "wa3": Workload("window_anchor_prefill_N131072_W16384_A4096", B=1, Hq=32, Hkv=8, N_q=131072, N_kv=131072,
                    d=128, dtype="bf16", causal=False, P=16, chunk=8192, seed=3100, window=16384,
                    anchor_period=4096),
    # Quarter-length 8-token decode (1.07 GB of K/V) for profiler captures.
    "5d8s": Workload("cache_idx_decode_Nq8_Nkv65536", B=4, Hq=32, Hkv=8, N_q=8, N_kv=65536, d=128,
                     dtype="bf16", causal=True, P=16, chunk=4096, cache_idx=65536 - 8, seed=5700),
    # Quarter-length FP8 cache (0.54 GB of codes) for profiler captures.
    "5d1f8s": Workload("cache_idx_decode_fp8kv_Nq1_Nkv65536", B=4, Hq=32, Hkv=8, N_q=1, N_kv=65536, d=128,
                       dtype="bf16", causal=True, P=16, chunk=4096, cache_idx=65536 - 1, seed=5600,
                       kv_dtype="fp8"),
    "5d1s": Workload("cache_idx_decode_Nq1_Nkv65536", B=4, Hq=32, Hkv=8, N_q=1, N_kv=65536, d=128,
                     dtype="bf16", causal=True, P=16, chunk=4096, cache_idx=65536 - 1, seed=5300),
}


def workload(key) -> Workload:
    return CONFIGS[key]


def small(B=1, Hq=2, Hkv=1, N_q=200, N_kv=None, d=64, dtype="bf16", causal=True, P=2,
          chunk=None, cache_idx=-1, k_scale=1.0, seed=7, name="small", kv_dtype="bf16", window=-1,
          anchor_period=0) -> Workload:
    """A small problem for parity tests (sizes the CPU oracle finishes quickly)."""
    if N_kv is None:
        N_kv = N_q if cache_idx < 0 else cache_idx + N_q
    if chunk is None:
        chunk = N_kv // P
    return Workload(name, B=B, Hq=Hq, Hkv=Hkv, N_q=N_q, N_kv=N_kv, d=d, dtype=dtype,
                    causal=causal, P=P, chunk=chunk, cache_idx=cache_idx, k_scale=k_scale,
                    seed=seed, kv_dtype=kv_dtype, window=window, anchor_period=anchor_period)


def _randn(shape, seed: int, device, mult: float, dtype: torch.dtype) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if mult != 1.0:
        x.mul_(mult)          # power of two: exact in float32
    return x.to(dtype)


def make_qkv(w: Workload, device="cpu", seed: Optional[int] = None):
    """Return (q, k, v) for workload ``w`` on ``device`` in ``w``'s dtype."""
    s = w.seed if seed is None else seed
    dt = w.torch_dtype
    q = _randn((w.B, w.N_q, w.Hq, w.d), s + 0, device, 1.0, dt)
    k = _randn((w.B, w.N_kv, w.Hkv, w.d), s + 1, device, w.k_scale, dt)
    v = _randn((w.B, w.N_kv, w.Hkv, w.d), s + 2, device, 1.0, dt)
    return q, k, v


E4M3_MAX = 448.0  # largest finite FP8 E4M3 magnitude


def make_fp8_kv(w: Workload, device="cpu", seed: Optional[int] = None):
    """Return (q, k8, v8, k_scale, v_scale) for workload ``w``: an FP8 KV cache.

    q is drawn as in make_qkv.  K and V are drawn as float32 exactly as
    make_qkv draws them, then quantised per (batch, KV head): scale =
    amax / 448 over that head's tokens and channels (1 where the head is all
    zero), codes = round-to-nearest-even of x / scale to FP8 E4M3 (torch's
    float8_e4m3fn cast).  k8, v8 are the codes as uint8 [B, N_kv, Hkv, d];
    k_scale, v_scale are float32 [B, Hkv].  This is input preparation only:
    the codes and scales are the cache both sides read.
    """
    s = w.seed if seed is None else seed
    q = _randn((w.B, w.N_q, w.Hq, w.d), s + 0, device, 1.0, w.torch_dtype)
    out = [q]
    scales = []
    for off, mult in ((1, w.k_scale), (2, 1.0)):
        x = _randn((w.B, w.N_kv, w.Hkv, w.d), s + off, device, mult, torch.float32)
        amax = x.abs().amax(dim=(1, 3))                      # [B, Hkv]
        sc = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
        codes = (x / sc[:, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        out.append(codes.contiguous())
        scales.append(sc.contiguous())
    return out[0], out[1], out[2], scales[0], scales[1]
