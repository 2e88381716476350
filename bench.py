"""Benchmark of the exact blockwise (ring) attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl ours|reference]

One step = one forward pass of the whole path (ring_attn_fwd through the C
ABI) over one batch of synthetic inputs already resident in HBM.  The
default workload is the Llama-7B-like causal prefill (B=1, Hq=Hkv=32,
d=128, N=32768, bf16, P=8 chunks of 4096).  With --gpus N > 1 (launched by
torch.distributed.run) every rank runs its own seeded copy of the workload
(data-parallel replicas, weak scaling, no collective on the data path);
the timed region is bracketed by barriers and its duration is the maximum
over ranks.  Rank 0 prints one JSON line.

The default run (config 2, forward) also times the decode-shaped incremental
queries 5d1 and 5d1f8 (one new token against a 262144-token bf16 or FP8 KV
cache, at least 100 steps each) and attaches them as the line's "decode"
list in GB/s against the measured HBM copy bandwidth.

--ring times the sequence-parallel ring itself (ring.ring_attention with
zigzag chunks across the N ranks, KV exchanged between neighbours every
step; strong scaling at the workload's full sequence) and adds the bytes
exchanged per step to the line.

--impl reference times the CPU float64 oracle on this host's cores on a
bounded sample of the same workload (the reference arm; there is no
reference GPU implementation).  Its ms_per_step is the whole step
extrapolated from the sampled rate ("extrapolated": true).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant
# kernel, from ncu captures (profiles/), keyed by workload, with the hash of
# the kernel sources they were taken on.  A stale hash reports null.
NCU_TRAFFIC = {
    # profiles/fwd_sm100_llama7b_prefill_N32768.md: 0.829952 GB read + 0.254706 GB written.
    "llama7b_prefill_N32768": {"bytes": 1.084657920e9, "src": "d8709868bf1b4f82"},
    # profiles/decode_sm100_Nq1_Nkv65536.md: 1.073960 GB read + 0.005652 GB written.
    "cache_idx_decode_Nq1_Nkv65536": {"bytes": 1.079611648e9, "src": "8331446299cfbe48"},
    # The full-length decodes scale the quarter-length captures by their 4x KV
    # length (traffic is K/V streaming, proportional to N_kv).
    "cache_idx_decode_Nq1_Nkv262144": {"bytes": 4 * 1.079611648e9, "src": "8331446299cfbe48"},
    # profiles/decode_f8_sm100_Nq1_Nkv65536.md (FP8 cache): 0.537050 GB read + 0.003901 GB written.
    "cache_idx_decode_fp8kv_Nq1_Nkv65536": {"bytes": 0.540951296e9, "src": "8331446299cfbe48"},
    "cache_idx_decode_fp8kv_Nq1_Nkv262144": {"bytes": 4 * 0.540951296e9, "src": "8331446299cfbe48"},
    # profiles/bwd_sm100_llama7b_prefill_N32768.md: one backward step, one capture
    # per kernel (prep, dK/dV, dQ): 0.541 + 0.010, 1.087 + 0.509, 1.086 + 0.255 GB
    # read + written.
    "llama7b_prefill_N32768 bwd": {"bytes": 3.487720704e9, "src": "fc202d6b900047b1"},
}


# Sources that do not affect a pass's kernels, left out of its hash.
# The kernel families: "fwd" (the general forward), "decode" (the keys-on-M
# decode kernel, which shares the FP8 converter and cursor code of the
# forward's sources) and "bwd".
_NOT_IN_HASH = {"fwd": {"bwd_sm100.cuh", "decode_sm100.cuh", "decode_f8_sm100.cuh"},
                "decode": {"bwd_sm100.cuh", "fwd_simt.cuh", "fwd2_sm100.cuh"},
                "bwd": {"fwd_sm100.cuh", "fwd_simt.cuh", "merge.cuh", "decode_sm100.cuh", "decode_f8_sm100.cuh",
                        "fwd2_sm100.cuh"}}


def kernel_source_hash(pass_: str = "fwd") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_exact_blockwise_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name in _NOT_IN_HASH[pass_]:
            continue
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    except OSError:
        return dict(FALLBACK_PEAKS), "fallback"


def config_key(s: str):
    return int(s) if s.isdigit() else s


def flops_of(w: workloads.Workload) -> float:
    """Algorithmic FLOPs: 4*d per visible (query, key) pair (QK^T and PV).

    Causal prefill counts half of the square (2*B*Hq*N^2*d); an incremental
    query block counts its exact visible pairs."""
    if w.window >= 0:
        return 4.0 * w.d * w.B * w.Hq * window_anchor_pairs(w.N_q, w.window, w.anchor_period)
    if w.cache_idx < 0:
        pairs = w.N_q * w.N_kv * (0.5 if w.causal else 1.0)
    elif w.causal:
        pairs = w.N_q * (w.cache_idx + 1) + w.N_q * (w.N_q - 1) / 2.0
    else:
        pairs = float(w.N_q * w.N_kv)
    return 4.0 * w.d * w.B * w.Hq * pairs


def kernel_name(w: workloads.Workload, bwd: bool) -> str:
    """The dominant kernel of a step (the library's routing rule for d = 128
    incremental queries with at most 16 packed rows per KV head)."""
    if bwd:
        return "bwd_prep + bwd_dkdv + bwd_dq (whole step)"
    if w.dtype != "bf16":
        return "simt_attn_kernel"
    rows = (w.Hq // w.Hkv) * w.N_q
    if w.d == 128 and w.cache_idx > 0 and w.window < 0:
        if w.kv_dtype == "fp8" and (rows <= 16 or (rows <= 32 and w.Hq // w.Hkv <= 16)):
            return "decode_f8_sm100_kernel (FP8 KV on the 8-bit MMA path)"
        if w.kv_dtype != "fp8" and rows <= 16:
            return "decode_sm100_kernel"
    return "fwd_sm100_kernel" + (" (FP8 KV, converter warpgroup)" if w.kv_dtype == "fp8" else "")


def window_anchor_pairs(n: int, window: int, period: int) -> float:
    """Visible (query, key) pairs of the window-and-anchor mask: each row's
    window [max(0, i - W), i], plus its anchors a, a - 1 (a > 0) and a + A
    (a < n - A) where they fall outside that window."""
    i = np.arange(n, dtype=np.int64)
    lo = np.maximum(0, i - window)
    a = i - i % period
    count = (i - lo + 1).astype(np.float64)
    count += (a < lo)
    count += (a > 0) & (a - 1 < lo)
    count += a < n - period
    return float(count.sum())


def hbm_bytes_of(w: workloads.Workload) -> float:
    """Minimum HBM traffic: q, k, v read once, out written once, lse written
    (an FP8 cache: one byte per K/V element plus its scales)."""
    es = 2 if w.dtype == "bf16" else 4
    kv_es = 1 if w.kv_dtype == "fp8" else es
    kv = kv_es * 2 * w.B * w.N_kv * w.Hkv * w.d + (8 * w.B * w.Hkv if w.kv_dtype == "fp8" else 0)
    return es * 2 * w.B * w.N_q * w.Hq * w.d + kv + 4 * w.B * w.Hq * w.N_q


# ----------------------------------------------------------------- ranks
def rank_seed(w: workloads.Workload, rank: int) -> int:
    """Each replica draws its own inputs."""
    return w.seed + 7919 * rank


def max_over_ranks(value: float, device) -> float:
    """The slowest rank's time (or any maximum) across the process group."""
    if not torch.distributed.is_initialized() or torch.distributed.get_world_size() == 1:
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the work of every replica over the slowest rank's step time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons via NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.h = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self.h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
                "sm_max_mhz": float(self.max_mhz) if self.max_mhz else None,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ our path
def run_ours(args, w, rank, world, device):
    import long_context_exact_blockwise_b200.ringattn as R

    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    fp8 = w.kv_dtype == "fp8"
    if fp8:
        q, k, v, k_sc, v_sc = workloads.make_fp8_kv(w, device=device, seed=rank_seed(w, rank))
    else:
        q, k, v = workloads.make_qkv(w, device=device, seed=rank_seed(w, rank))
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N_q), device=device, dtype=torch.float32)
    ci = None if w.cache_idx < 0 else w.cache_idx
    if fp8:
        def fn(q_, k_, v_, **kw):
            return R.ring_attn_fwd_fp8kv(q_, k_, v_, k_sc, v_sc, **kw)
    elif w.window >= 0:
        def fn(q_, k_, v_, *, causal, P, chunk, cache_idx, scale, out, lse, stream):
            return R.ring_attn_fwd_window_anchor(q_, k_, v_, window=w.window, anchor_period=w.anchor_period, P=P,
                                                 chunk=chunk, scale=scale, out=out, lse=lse, stream=stream)
    else:
        fn = R.ring_attn_fwd_f32 if w.dtype == "f32" else R.ring_attn_fwd

    if args.pass_ == "bwd":
        if w.dtype != "bf16" or fp8:
            raise SystemExit("--pass bwd needs a bf16 workload with a bf16 KV cache")
        fn(q, k, v, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci, scale=w.scale, out=out, lse=lse,
           stream=stream)
        g = torch.Generator(device=device).manual_seed(rank_seed(w, rank) + 99)
        dout = torch.randn(q.shape, generator=g, device=device).to(q.dtype)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def step():
            R.ring_attn_bwd(q, k, v, out, dout, lse, causal=w.causal, cache_idx=ci, scale=w.scale, dq=dq, dk=dk,
                            dv=dv, stream=stream)
    else:
        def step():
            fn(q, k, v, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci, scale=w.scale, out=out, lse=lse,
               stream=stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if R.ring_attn_sync_status(stream) != 0:
        raise RuntimeError("device status word set during warm-up")

    clocks = ClockSampler(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(device)
    launches0 = R.ring_attn_launch_count()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(device)
    clocks.stop()
    barrier()
    launches = R.ring_attn_launch_count() - launches0
    ms_total = max_over_ranks(t0.elapsed_time(t1), device)
    per_launch = [a.elapsed_time(b) for a, b in ev]
    status = R.ring_attn_sync_status(stream)
    if status != 0:
        raise RuntimeError(f"device status word {status} after the timed region")

    # ---- end to end through the public API with host buffers
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    hq = q.cpu().pin_memory()
    hk = k.cpu().pin_memory()
    hv = v.cpu().pin_memory()
    xq, xk, xv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if args.pass_ == "bwd":
        # Inputs: q, k, v, out, dout, lse; results: dq, dk, dv.
        h_in = [hq, hk, hv, out.cpu().pin_memory(), dout.cpu().pin_memory(), lse.cpu().pin_memory()]
        x_in = [xq, xk, xv, torch.empty_like(out), torch.empty_like(dout), torch.empty_like(lse)]
        h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]

        def e2e_step():
            # Host-buffer backward: KV-head groups stream through the device,
            # copies overlapped with the compute.
            R.ring_attn_bwd_host(*h_in, causal=w.causal, cache_idx=ci, scale=w.scale, dq=h_out[0], dk=h_out[1],
                                 dv=h_out[2], stream=stream)
    else:
        h_in = [hq, hk, hv]
        h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                 torch.empty(lse.shape, dtype=lse.dtype).pin_memory()]

        if fp8:
            h_sc = [k_sc.cpu().pin_memory(), v_sc.cpu().pin_memory()]
            x_sc = [k_sc, v_sc]  # the call reads the scales from these device tensors

        if fn is R.ring_attn_fwd:
            # The bf16 forward has a host-buffer entry point that streams
            # KV-head groups through the device, copies overlapped with the
            # compute.
            def e2e_step():
                R.ring_attn_fwd_host(hq, hk, hv, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci,
                                     scale=w.scale, out=h_out[0], lse=h_out[1], stream=stream)
        elif w.window >= 0:
            def e2e_step():
                R.ring_attn_fwd_window_anchor_host(hq, hk, hv, window=w.window, anchor_period=w.anchor_period,
                                                   P=w.P, chunk=w.chunk, scale=w.scale, out=h_out[0], lse=h_out[1],
                                                   stream=stream)
        else:
            def e2e_step():
                xq.copy_(hq, non_blocking=True)
                xk.copy_(hk, non_blocking=True)
                xv.copy_(hv, non_blocking=True)
                if fp8:
                    for x, h in zip(x_sc, h_sc):
                        x.copy_(h, non_blocking=True)
                fn(xq, xk, xv, causal=w.causal, P=w.P, chunk=w.chunk, cache_idx=ci, scale=w.scale, out=out,
                   lse=lse, stream=stream)
                h_out[0].copy_(out, non_blocking=True)
                h_out[1].copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(device)
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e2e_steps, device)
    h2d = sum(x.numel() * x.element_size() for x in h_in) + (16 * w.B * w.Hkv if fp8 else 0)
    d2h = sum(x.numel() * x.element_size() for x in h_out)
    res = dict(ms_total=ms_total, per_launch_ms=per_launch, launches=launches, clocks=clocks.summary(),
               e2e_ms=e2e_ms, h2d=h2d, d2h=d2h,
               host_inputs=(hq, hk, hv) + ((k_sc.cpu(), v_sc.cpu()) if fp8 else ()))
    return res


# ------------------------------------------------------------ the ring itself
def run_ring(args, w, rank, world, device):
    """Time ring.ring_attention (sequence-parallel forward) over the ranks.

    The workload's whole sequence is cut into 2 * world chunks; rank i holds
    chunks i and 2 world - 1 - i (zigzag layout, equal causal work per rank)
    and exchanges KV with its ring neighbours every step (one way, or with
    --bidirectional each of its two chunks in its own direction).  Total work
    is fixed as world grows (strong scaling).  Returns the timing record.
    """
    from long_context_exact_blockwise_b200 import ring
    import long_context_exact_blockwise_b200.ringattn as R

    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    q, k, v = workloads.make_qkv(w, device=device)  # the same seeded sequence on every rank
    qc, kc, vc = (ring.shard(x, rank, world, "zigzag") for x in (q, k, v))
    del q, k, v

    def step():
        return ring.ring_attention(qc, kc, vc, causal=w.causal, scale=w.scale, layout="zigzag",
                                   bidirectional=args.bidirectional)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if R.ring_attn_sync_status(stream) != 0:
        raise RuntimeError("device status word set during warm-up")
    clocks = ClockSampler(device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    launches0 = R.ring_attn_launch_count()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        out, lse = step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    launches = R.ring_attn_launch_count() - launches0
    ms_total = max_over_ranks(t0.elapsed_time(t1), device)
    # End to end: this rank's chunks from pinned host memory, out and lse back.
    hq, hk, hv = (x.cpu().pin_memory() for x in (qc, kc, vc))
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

    def e2e_step():
        for dst, src in ((qc, hq), (kc, hk), (vc, hv)):
            dst.copy_(src, non_blocking=True)
        o, ls = step()
        ho.copy_(o, non_blocking=True)
        hl.copy_(ls, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, min(args.steps, args.e2e_steps))
    a.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, device)
    kv_bytes_rank = 2 * kc.numel() * kc.element_size()
    return dict(ms_total=ms_total, launches=launches, clocks=clocks.summary(), e2e_ms=e2e_ms,
                h2d=sum(x.numel() * x.element_size() for x in (hq, hk, hv)),
                d2h=ho.numel() * ho.element_size() + hl.numel() * hl.element_size(),
                exchange_bytes=world * (world - 1) * kv_bytes_rank)


# ------------------------------------------------------------ CPU oracle legs
def oracle_sample(w, host_qkv, budget_s: float, seed: int = 0):
    """Time the float64 oracle on random (row, head) samples of workload w
    until about budget_s seconds of CPU work are done.  Returns
    (flops_done, seconds, rows_done, threads)."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
    except Exception:  # pragma: no cover
        threadpool_info = None
    q, k, v = host_qkv[:3]
    rng = np.random.default_rng(seed)
    G = w.Hq // w.Hkv
    kf = {}
    if w.kv_dtype == "fp8":
        # Dequantise one KV head of the FP8 cache by the oracle's decoder.
        k_sc, v_sc = (x.double().numpy() for x in host_qkv[3:5])

        def kv_head(hk):
            dk = oracle.decode_e4m3(k[:, :, hk:hk + 1].numpy()) * k_sc[:, None, hk:hk + 1, None]
            dv = oracle.decode_e4m3(v[:, :, hk:hk + 1].numpy()) * v_sc[:, None, hk:hk + 1, None]
            return dk, dv
    else:
        def kv_head(hk):
            return k[:, :, hk:hk + 1].double().numpy(), v[:, :, hk:hk + 1].double().numpy()
    flops = 0.0
    rows_done = 0
    t_start = time.perf_counter()
    elapsed = 0.0
    while elapsed < budget_s and rows_done < w.N_q * w.Hq:
        h = int(rng.integers(0, w.Hq))
        hk = h // G
        if hk not in kf:
            kf[hk] = kv_head(hk)
        r0 = int(rng.integers(0, max(1, w.N_q - 16)))
        nr = min(16, w.N_q - r0)
        qs = q[:, r0:r0 + nr, h:h + 1].double().numpy()
        base = (0 if w.cache_idx < 0 else w.cache_idx) + r0
        t0 = time.perf_counter()
        if w.window >= 0:
            oracle.attention_window_anchor_ref(q[:, :, h:h + 1].double().numpy(), kf[hk][0], kf[hk][1],
                                               window=w.window, anchor_period=w.anchor_period, scale=w.scale,
                                               rows=np.arange(r0, r0 + nr))
        else:
            oracle.attention_ref(qs, kf[hk][0], kf[hk][1], causal=w.causal, scale=w.scale, cache_idx=base)
        elapsed += time.perf_counter() - t0
        if w.window >= 0:
            vis = [min(r0 + i, w.window) + 1 + 2 for i in range(nr)]
        else:
            vis = [(base + i + 1) if w.causal else w.N_kv for i in range(nr)]
        flops += 4.0 * w.d * w.B * sum(min(x, w.N_kv) for x in vis)
        rows_done += nr
        if time.perf_counter() - t_start > 4 * budget_s:
            break
    threads = os.cpu_count()
    if threadpool_info is not None:
        info = threadpool_info()
        if info:
            threads = max(int(x.get("num_threads", 1)) for x in info)
    return flops, elapsed, rows_done, threads


def oracle_bwd_sample(w, host_qkv, budget_s: float, seed: int = 0):
    """Time the float64 gradient oracle on one (batch, KV-head group) of the
    first n tokens of workload w, n doubling from 256 while the budget lasts.
    Returns (flops_done, seconds, description, threads)."""
    import oracle
    q, k, v = host_qkv
    G = w.Hq // w.Hkv
    g = torch.Generator().manual_seed(seed)
    flops, elapsed, n, done, last = 0.0, 0.0, 256, [], 0.0
    # Each doubling of n costs about four times the last size.
    while elapsed + 4.0 * last <= budget_s and n <= min(w.N_q, 1 << 14):
        qs = q[:1, :n, :G].double()
        ks, vs = k[:1, :n, :1].double(), v[:1, :n, :1].double()
        do = torch.randn(qs.shape, generator=g, dtype=torch.float64)
        t0 = time.perf_counter()
        oracle.attention_bwd_ref(qs, ks, vs, do, causal=w.causal, scale=w.scale)
        last = time.perf_counter() - t0
        elapsed += last
        pairs = n * (n + 1) / 2 if w.causal else n * n
        flops += 2.5 * 4.0 * w.d * G * pairs
        done.append(n)
        n *= 2
    return flops, elapsed, done, os.cpu_count()


def decode_line(args, key, rank, world, device, peaks, peak_src):
    """Time one decode-shaped incremental query (the HBM-bound half of the
    metric) on the same GPU, after the main workload: K+V streamed once per
    step, reported as algorithmic GB/s against the measured copy bandwidth."""
    w = workloads.CONFIGS[key]
    sub = argparse.Namespace(**vars(args))
    sub.steps = max(100, args.steps)
    sub.pass_ = "fwd"
    res = run_ours(sub, w, rank, world, device)
    ms = res["ms_total"] / sub.steps
    launch_ms = statistics.mean(res["per_launch_ms"])
    nbytes = hbm_bytes_of(w)
    achieved = nbytes / (launch_ms * 1e-3) / 1e9
    src_hash = kernel_source_hash("decode" if kernel_name(w, False).startswith("decode") else "fwd")
    tr = NCU_TRAFFIC.get(w.name)
    return {"workload": w.name, "kv_cache": "fp8 e4m3 + per-head scales" if w.kv_dtype == "fp8" else w.dtype,
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N_q": w.N_q, "N_kv": w.N_kv, "d": w.d,
            "cache_idx": w.cache_idx, "steps": sub.steps, "warmup": sub.warmup, "ms_per_step": ms,
            "value": nbytes * world / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "tokens_per_s": w.B * w.N_q * world / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"],
                         "traffic": tr["bytes"] if tr and tr.get("src") == src_hash else None,
                         "peak_source": f"{peak_src} (hbm)", "kernel": kernel_name(w, False),
                         "algorithmic_per_launch": nbytes},
            "e2e": {"value": nbytes * world / (res["e2e_ms"] * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
            "gpu_launches": res["launches"], "clocks": res["clocks"]}


def host_inputs(w):
    if w.kv_dtype == "fp8":
        return workloads.make_fp8_kv(w, device="cpu")
    return workloads.make_qkv(w, device="cpu")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="2", help="workload key: 1..5, 5d1, 5d8 (default 2)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd"], default="fwd",
                    help="fwd: the forward pass (default); bwd: the backward pass (dq, dk, dv)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ring", action="store_true",
                    help="time ring.ring_attention across the N ranks (sequence-parallel ring, zigzag chunks, "
                         "strong scaling) instead of data-parallel replicas of the single-GPU kernel")
    ap.add_argument("--bidirectional", action="store_true",
                    help="with --ring: the bidirectional ring (each rank's two chunks travel in opposite "
                         "directions)")
    ap.add_argument("--decode", default="5d1,5d1f8",
                    help="decode workloads timed after the forward prefill of config 2 and reported in the "
                         "line's 'decode' list (comma-separated keys; 'none' to skip)")
    args = ap.parse_args()
    if args.bidirectional and not args.ring:
        ap.error("--bidirectional needs --ring")
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")

    w = workloads.CONFIGS[config_key(args.config)]
    bwd = args.pass_ == "bwd"
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    peaks, peak_src = load_peaks()
    # The backward's algorithmic work is 2.5x the forward's (five GEMMs of the
    # forward's size instead of two); the dQ kernel's recomputation of S and
    # dP is not counted.
    flops = flops_of(w) * (2.5 if bwd else 1.0)
    config = {"workload": w.name,
              "mask": (f"window {w.window} + anchors every {w.anchor_period}" if w.window >= 0 else
                       "causal" if w.causal else "none"),
              "kv_cache": "fp8 e4m3 + per-head scales" if w.kv_dtype == "fp8" else w.dtype,
              "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N_q": w.N_q, "N_kv": w.N_kv, "d": w.d,
              "causal": w.causal, "P": w.P, "chunk": w.chunk, "cache_idx": w.cache_idx, "k_scale": w.k_scale,
              "global_batch": w.B * world, "l2": "inputs larger than the 126 MB L2, no flush"
              if hbm_bytes_of(w) > 126e6 else "inputs fit in L2 (small correctness case)",
              "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}

    if args.impl == "reference":
        if rank != 0:
            return
        hq = host_inputs(w)
        if bwd:
            budget = max(1.0, 60.0 / max(1, args.steps + args.warmup))
            tot_f, tot_s, sizes = 0.0, 0.0, []
            for i in range(args.steps):
                f_, s_, n_, threads = oracle_bwd_sample(w, hq, budget, seed=i + 1)
                tot_f, tot_s, sizes = tot_f + f_, tot_s + s_, sizes + n_
            val = tot_f / tot_s / 1e12
            line = {"impl": "reference", "metric": "attention bwd TFLOP/s", "value": val, "unit": "TFLOP/s",
                    "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                    "ms_per_step": 1e3 * flops / (val * 1e12), "extrapolated": True,
                    "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                    "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                     "sample": f"float64 gradient oracle on one KV-head group of the first "
                                               f"n tokens, n in {sorted(set(sizes))}, {tot_s:.1f} s"},
                    "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
            return
        budget = max(1.0, 60.0 / max(1, args.steps + args.warmup))
        for _ in range(args.warmup):
            oracle_sample(w, hq, budget / 4)
        tot_f, tot_s, tot_rows, threads = 0.0, 0.0, 0, 1
        for i in range(args.steps):
            f_, s_, r_, threads = oracle_sample(w, hq, budget, seed=i + 1)
            tot_f += f_
            tot_s += s_
            tot_rows += r_
        val = tot_f / tot_s / 1e12
        line = {"impl": "reference", "metric": "attention fwd TFLOP/s", "value": val, "unit": "TFLOP/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * flops / (val * 1e12), "extrapolated": True,
                "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                 "sample": f"{tot_rows} random (row, head) query rows in runs of 16, "
                                           f"{tot_s:.1f} s of float64 oracle work over {args.steps} steps"},
                "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1 or args.ring:
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29533")
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank), rank=rank,
                                             world_size=world)
    device = local_rank
    if args.ring:
        if bwd or w.cache_idx >= 0 or w.dtype != "bf16" or w.kv_dtype != "bf16" or w.window >= 0:
            raise SystemExit("--ring times the bf16 prefill forward")
        res = run_ring(args, w, rank, world, device)
        ms_step = res["ms_total"] / args.steps
        value = flops / (ms_step * 1e-3) / 1e12
        config["parallelism"] = (f"sequence-parallel {'bidirectional ' if args.bidirectional else ''}ring x{world} "
                                 "(zigzag chunks)")
        config["global_batch"] = w.B
        line = {"metric": "attention fwd TFLOP/s", "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": config,
                "tokens_per_s": w.B * w.N_q / (ms_step * 1e-3),
                "frac_of_bf16_peak": value / world / peaks["bf16_tflops"],
                "exchange_bytes_per_step": res["exchange_bytes"],
                "e2e": {"value": flops / (res["e2e_ms"] * 1e-3) / 1e12, "unit": "TFLOP/s",
                        "h2d_bytes_per_step": res["h2d"] * world, "d2h_bytes_per_step": res["d2h"] * world},
                "gpu_launches": res["launches"], "clocks": res["clocks"]}
        if rank == 0:
            print(json.dumps(line), flush=True)
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
        return
    res = run_ours(args, w, rank, world, device)
    decode = None
    if not bwd and args.config == "2" and args.decode != "none":
        decode = [decode_line(args, config_key(key), rank, world, device, peaks, peak_src)
                  for key in args.decode.split(",")]
    ms_step = res["ms_total"] / args.steps
    value = aggregate_tflops(flops, world, ms_step)
    launch_ms = statistics.mean(res["per_launch_ms"])
    achieved = flops / (launch_ms * 1e-3) / 1e12
    # A kernel timed alone for a short step is compared with the burst bf16
    # peak; steps of a second or more run under the power cap, so they are
    # compared with the sustained figure.
    long_step = ms_step >= 1000.0
    peak = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    peak_kind = "sustained" if long_step else "burst"
    bound = "tensor"
    unit = "TFLOP/s"
    if w.dtype == "f32":
        bound, unit = "alu", "TFLOP/s"
        # FP32 FFMA peak: 148 SMs x 128 lanes x 2 FLOP x max SM clock.
        peak = 148 * 128 * 2 * (peaks.get("sm_max_mhz", 1965.0) * 1e6) / 1e12
    elif not bwd and w.cache_idx >= 0 and w.N_q * (w.Hq // w.Hkv) <= 64:
        bound, unit = "hbm", "GB/s"
        achieved = hbm_bytes_of(w) / (launch_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
    src_hash = kernel_source_hash("bwd" if bwd else ("decode" if kernel_name(w, bwd).startswith("decode") else "fwd"))
    tr = NCU_TRAFFIC.get(w.name + (" bwd" if bwd else ""))
    traffic = tr["bytes"] if tr and tr.get("src") == src_hash else None
    cpu = None
    if rank == 0 and not args.no_cpu_baseline and bwd:
        f_, s_, n_, threads = oracle_bwd_sample(w, tuple(x.cpu() for x in res["host_inputs"]), args.cpu_budget)
        cpu = {"value": f_ / s_ / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"float64 gradient oracle on one KV-head group of the first n tokens of this "
                         f"workload, n in {n_}, {s_:.1f} s on the host"}
    elif rank == 0 and not args.no_cpu_baseline:
        f_, s_, r_, threads = oracle_sample(w, tuple(x.cpu() for x in res["host_inputs"]), args.cpu_budget)
        cpu = {"value": f_ / s_ / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{r_} random (row, head) query rows in runs of 16 of this workload, {s_:.1f} s of "
                         f"float64 oracle work on the host"}
    e2e_val = aggregate_tflops(flops, world, res["e2e_ms"])
    line = {
        "metric": "attention bwd TFLOP/s" if bwd else "attention fwd TFLOP/s", "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": config,
        "tokens_per_s": w.B * w.N_q * world / (ms_step * 1e-3),
        "hbm_gbs_algorithmic": hbm_bytes_of(w) * world / (ms_step * 1e-3) / 1e9,
        "frac_of_bf16_peak": value / world / peaks["bf16_tflops"],
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} ({peak_kind if bound == 'tensor' else bound})",
                     "kernel": kernel_name(w, bwd),
                     "algorithmic_per_launch": flops if unit == "TFLOP/s" else hbm_bytes_of(w)},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
    }
    if decode is not None:
        line["decode"] = decode
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
