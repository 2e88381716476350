// C ABI of libringattn.so (declared in include/ring_attn.h): argument
// validation, device checks, dispatch to the kernels, stream-ordered
// workspace for the split-KV path, and the device status word.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

// The kernels and their launchers (one translation unit: the status word is
// shared without relocatable device code).
#include "fwd_sm100.cuh"
#include "decode_sm100.cuh"
#include "decode_f8_sm100.cuh"
#include "fwd2_sm100.cuh"
#include "bwd_sm100.cuh"
#include "fwd_simt.cuh"
#include "merge.cuh"

namespace ra {

namespace {

thread_local std::string t_last_error;

int set_cuda_error(cudaError_t e, const char* where) {
  t_last_error = std::string(where) + ": " + cudaGetErrorName(e) + ": " + cudaGetErrorString(e);
  return RA_ERR_CUDA;
}

bool env_flag(const char* name) {
  const char* v = std::getenv(name);
  return v && v[0] && std::strcmp(v, "0") != 0;
}

const char* env_str(const char* name) {
  const char* v = std::getenv(name);
  return v ? v : "";
}

// Longest q or k/v buffer a call accepts (rows); kernels index rows in 32 bits.
constexpr int64_t kMaxTokens = (int64_t(1) << 31) - 8192;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 1 on sm_100 devices; 0 otherwise; -1 if no device could be queried.
int device_is_sm100(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  if (num_sms) *num_sms = sms;
  return (major == 10 && minor == 0) ? 1 : 0;
}

int check_device(int* num_sms) {
  const int r = device_is_sm100(num_sms);
  if (r == 1) return RA_OK;
  t_last_error = r < 0 ? "no CUDA device available" : "device is not sm_100 (B200)";
  return RA_ERR_UNSUPPORTED;
}

// After a launch: report launch errors; in debug mode also synchronise and
// read the device status word.
// RINGATTN_NVTX=1: every compute entry point is an NVTX range named after
// it, for profilers.  NVTX here is header-only: without a profiler attached
// the calls do nothing.
struct NvtxScope {
  bool on;
  explicit NvtxScope(const char* name) : on(env_flag("RINGATTN_NVTX")) {
    if (on) nvtxRangePushA(name);
  }
  ~NvtxScope() {
    if (on) nvtxRangePop();
  }
  NvtxScope(const NvtxScope&) = delete;
  NvtxScope& operator=(const NvtxScope&) = delete;
};

int finish(cudaError_t e, cudaStream_t st, const char* where) {
  if (e != cudaSuccess) return set_cuda_error(e, where);
  if (env_flag("RINGATTN_DEBUG")) {
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return set_cuda_error(e, where);
    int status = 0;
    e = cudaMemcpyFromSymbol(&status, g_status, sizeof(int));
    if (e != cudaSuccess) return set_cuda_error(e, "cudaMemcpyFromSymbol(status)");
    if (status != 0) {
      const int zero = 0;
      cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
      return status;
    }
  }
  return RA_OK;
}

// Common shape checks for the forward entry points.
int validate_fwd(const void* q, const void* k, const void* v, const void* out, const void* lse, int B, int Hq,
                 int Hkv, int64_t N_q, int64_t N_kv, int d, int causal, int64_t chunk, int P, int64_t cache_idx,
                 float scale, bool need_align16) {
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return RA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return RA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID_ARG;
  if (P < 1 || chunk < 1 || N_kv < 1 || N_q < 0) return RA_ERR_INVALID_ARG;
  if (N_kv / P != chunk || N_kv % P != 0) return RA_ERR_INVALID_ARG;  // N_kv == P * chunk
  if (N_q > kMaxTokens || N_kv > kMaxTokens) return RA_ERR_INVALID_ARG;
  if (cache_idx < -1) return RA_ERR_INVALID_ARG;
  if (cache_idx == -1 && N_q != N_kv) return RA_ERR_INVALID_ARG;
  if (cache_idx >= 0 && cache_idx + N_q > N_kv) return RA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return RA_ERR_INVALID_ARG;
  if (need_align16 && !(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out))) return RA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return RA_ERR_INVALID_ARG;
  return RA_OK;
}

// Number of KV splits for an incremental query (`items` CTAs per split, one
// CTA per SM at a time).  RINGATTN_SPLITS overrides.
//   - Decode shapes (at most 64 query rows) stream the KV cache: enough
//     splits for about eight waves of CTAs in flight.
//   - Otherwise every CTA does about the same work (whole ring steps of one
//     query block), so the kernel takes (waves) x (ring steps per CTA).  The
//     count minimising that, with a quarter step of per-CTA overhead, wins;
//     ties go to fewer splits (fewer partials to write and merge).  512
//     queries over 64 steps in 256 CTAs per split: 4 splits (1024 CTAs, 7
//     waves of 16 steps) instead of 2 (512 CTAs, 4 waves of 32 steps, the
//     last wave less than half full).
int choose_splits(long long items, int P, int num_sms, long long n_q) {
  const char* ov = std::getenv("RINGATTN_SPLITS");
  if (ov && ov[0]) {
    int s = std::atoi(ov);
    return s < 1 ? 1 : (s > P ? P : s);
  }
  if (items < 1) items = 1;
  if (n_q <= 64) {
    long long s = (8LL * num_sms + items - 1) / items;
    if (s < 1) s = 1;
    if (s > P) s = P;
    // Whole ring steps per split.
    const int sps = (int)((P + s - 1) / s);
    return (P + sps - 1) / sps;
  }
  constexpr int kMaxSplits = 32;
  int best = 1;
  double best_cost = 0.0;
  for (int sps = P; sps >= 1; --sps) {
    const int s = (P + sps - 1) / sps;
    if (s > kMaxSplits) break;
    const long long waves = (items * s + num_sms - 1) / num_sms;
    const double cost = (double)waves * (sps + 0.25);
    if (sps == P || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

}  // namespace

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace ra

using namespace ra;

extern "C" {

int ring_attn_version(void) { return 100; }

int64_t ring_attn_launch_count(void) { return (int64_t)launch_counter().load(); }

const char* ring_attn_error_string(int status) {
  switch (status) {
    case RA_OK: return "ok";
    case RA_ERR_INVALID_ARG: return "invalid argument";
    case RA_ERR_UNSUPPORTED: return "unsupported device (needs sm_100)";
    case RA_ERR_CUDA: return "CUDA error";
    case RA_ERR_DEVICE_TIMEOUT: return "device-side bounded wait expired";
    case RA_ERR_OOM: return "workspace allocation failed";
    default: return "unknown status";
  }
}

const char* ring_attn_last_error(void) { return t_last_error.c_str(); }

int ring_attn_sync_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return set_cuda_error(e, "cudaStreamSynchronize");
  int status = 0;
  e = cudaMemcpyFromSymbol(&status, g_status, sizeof(int));
  if (e != cudaSuccess) return set_cuda_error(e, "cudaMemcpyFromSymbol(status)");
  if (status != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return set_cuda_error(e, "cudaMemcpyToSymbol(status)");
  }
  return status;
}

}  // extern "C"

namespace {

// The bf16 tensor-core forward (and its FP8-KV variant) for validated
// arguments: one launch for prefill, or split-KV partials merged by their
// log-sum-exp weights for incremental queries.
// a.S == 1: prefill, one launch; a.S == 0: incremental queries, the split
// count is chosen here.
int run_fwd(ProblemArgs a, int num_sms, cudaStream_t st, const char* what) {
  if (a.S == 1) return finish(launch_fwd_sm100(a, kModeFinal, st), st, what);

  // Incremental query: split the ring steps over S CTAs per query block and
  // merge the partials by their log-sum-exp weights.
  const long long items = sm100_geometry(a, kModeSplit).ctas_per_split;
  const int S = choose_splits(items, a.P, num_sms, a.N_q);
  if (S == 1) return finish(launch_fwd_sm100(a, kModeFinal, st), st, what);

  const size_t o_bytes = (size_t)S * a.B * a.N_q * a.Hq * a.d * sizeof(float);
  const size_t l_bytes = (size_t)S * a.B * a.Hq * a.N_q * sizeof(float);
  void* ws = nullptr;
  if (std::strcmp(env_str("RINGATTN_FAULT"), "alloc") == 0) {
    t_last_error = "workspace allocation refused (RINGATTN_FAULT=alloc)";
    return RA_ERR_OOM;
  }
  cudaError_t e = cudaMallocAsync(&ws, o_bytes + l_bytes, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    t_last_error = std::string("cudaMallocAsync: ") + cudaGetErrorString(e);
    return RA_ERR_OOM;
  }
  a.S = S;
  a.o_part = static_cast<float*>(ws);
  a.lse_part = reinterpret_cast<float*>(static_cast<char*>(ws) + o_bytes);
  e = launch_fwd_sm100(a, kModeSplit, st);
  if (e == cudaSuccess) e = launch_lse_merge(a.o_part, a.lse_part, S, a.out, a.lse, a.B, a.Hq, a.N_q, a.d, 0, st);
  cudaError_t ef = cudaFreeAsync(ws, st);
  if (e == cudaSuccess) e = ef;
  return finish(e, st, what);
}

}  // namespace

extern "C" {

int ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                  int64_t N_q, int64_t N_kv, int d, int causal, int64_t chunk, int P, int64_t cache_idx, float scale,
                  void* stream) {
  NvtxScope nvtx_scope("ring_attn_fwd");
  int r = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, N_q, N_kv, d, causal, chunk, P, cache_idx, scale, true);
  if (r != RA_OK) return r;
  if (B == 0 || N_q == 0) return RA_OK;
  int num_sms = 148;
  if ((r = check_device(&num_sms)) != RA_OK) return r;
  ProblemArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = out; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.N_q = N_q; a.N_kv = N_kv;
  a.q_pos0 = cache_idx < 0 ? 0 : cache_idx;
  a.k_pos0 = 0;
  a.causal = causal; a.scale = scale; a.chunk = chunk; a.P = P; a.out_f32 = 0;
  a.S = cache_idx < 0 ? 1 : 0;  // 0: choose a split count
  return run_fwd(a, num_sms, static_cast<cudaStream_t>(stream), "ring_attn_fwd");
}

}  // extern "C"

namespace {

// The host-buffer pipeline's streams on one device (q in, k and v in,
// compute, results out), created once, all or none.  Two copy-in streams let
// the q and the k / v copies of a group run on separate copy engines.
struct PipeStreams {
  cudaStream_t h2d = nullptr, h2d_kv = nullptr, comp = nullptr, d2h = nullptr;
};

int pipe_streams(PipeStreams** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static PipeStreams per_dev[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return RA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  PipeStreams& p = per_dev[dev];
  if (!p.h2d) {
    cudaStream_t s[4] = {nullptr, nullptr, nullptr, nullptr};
    for (int i = 0; i < 4; ++i) {
      e = cudaStreamCreateWithFlags(&s[i], cudaStreamNonBlocking);
      if (e != cudaSuccess) {
        for (int j = 0; j < i; ++j) cudaStreamDestroy(s[j]);
        return set_cuda_error(e, "cudaStreamCreateWithFlags");
      }
    }
    p.h2d = s[0];
    p.h2d_kv = s[1];
    p.comp = s[2];
    p.d2h = s[3];
  }
  *out = &p;
  return RA_OK;
}

// Events of one pipelined call, destroyed when the call returns (a pending
// event's resources are released once it completes).
struct CallEvents {
  std::vector<cudaEvent_t> ev;
  ~CallEvents() {
    for (cudaEvent_t x : ev) cudaEventDestroy(x);
  }
  cudaError_t make(size_t n) {
    ev.reserve(n);
    for (size_t i = 0; i < n; ++i) {
      cudaEvent_t x;
      cudaError_t e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
      if (e != cudaSuccess) return e;
      ev.push_back(x);
    }
    return cudaSuccess;
  }
};

int run_bwd(ra::BwdArgs a, const char* what, cudaStream_t st);  // below

// KV heads per group when the caller passes 0: the fewest that give at most
// sixteen groups (and divide Hkv).  On the 32-head 32K prefill, 16 groups of
// two KV heads measured 17.7 ms per step, 8 of four 17.9, 32 of one 20.4 and
// 4 of eight 20.0 (one copy-in stream).
int default_kv_group(int Hkv) {
  int g = 1;
  while (Hkv / g > 16 || Hkv % g != 0) ++g;
  return g;
}

// One tensor of a host-buffer pipeline.  Group g's part is `rows` rows of
// `row_bytes` bytes starting at byte g * row_bytes of the host tensor, one
// row every `pitch` bytes; on the device it is packed (pitch = row_bytes).
// Inputs go in on copy-in stream `lane` (0 or 1); outputs come back after
// the group's compute.
struct PipeTensor {
  const void* in;   // host input, or nullptr
  void* out;        // host output, or nullptr
  size_t row_bytes, pitch, rows;
  int lane;
};

// Streams the groups of a host-buffer call through two device staging slots:
// while group g computes, group g + 1 is copied in and group g - 1 copied out.
// compute(g, dev, comp_stream) launches group g's work on the packed device
// tensors dev[i] (same order as t) and returns an ra status.
template <class F>
int run_host_pipeline(int n_groups, const PipeTensor* t, int n_t, cudaStream_t st, const char* what, F&& compute) {
  constexpr int kMaxTensors = 12;
  if (n_t > kMaxTensors) return RA_ERR_INVALID_ARG;
  PipeStreams* ps = nullptr;
  int r = pipe_streams(&ps);
  if (r != RA_OK) return r;
  const int n_slots = n_groups > 1 ? 2 : 1;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  size_t off[kMaxTensors];
  size_t slot_bytes = 0;
  for (int i = 0; i < n_t; ++i) {
    off[i] = slot_bytes;
    slot_bytes += up(t[i].row_bytes * t[i].rows);
  }
  cudaStream_t lanes[2] = {ps->h2d, ps->h2d_kv};

  // Events: start, then per group (in on each lane, computed, out), then the
  // four streams' ends.
  CallEvents evs;
  cudaError_t e = evs.make(1 + 4 * (size_t)n_groups + 4);
  if (e != cudaSuccess) return set_cuda_error(e, "cudaEventCreateWithFlags");
  cudaEvent_t ev_start = evs.ev[0];
  auto ev_in = [&](int g, int lane) { return evs.ev[1 + 4 * g + lane]; };
  auto ev_comp = [&](int g) { return evs.ev[3 + 4 * g]; };
  auto ev_out = [&](int g) { return evs.ev[4 + 4 * g]; };
  cudaEvent_t* ev_end = &evs.ev[1 + 4 * n_groups];

  if (std::strcmp(env_str("RINGATTN_FAULT"), "alloc") == 0) {
    t_last_error = "workspace allocation refused (RINGATTN_FAULT=alloc)";
    return RA_ERR_OOM;
  }
  void* ws = nullptr;
  e = cudaMallocAsync(&ws, slot_bytes * n_slots, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    t_last_error = std::string("cudaMallocAsync: ") + cudaGetErrorString(e);
    return RA_ERR_OOM;
  }
  // The pipeline starts after the work already queued on the caller's stream.
  e = cudaEventRecord(ev_start, st);
  cudaStream_t pipes[4] = {ps->h2d, ps->h2d_kv, ps->comp, ps->d2h};
  for (cudaStream_t s : pipes)
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_start, 0);

  int status = RA_OK;
  for (int g = 0; g < n_groups && e == cudaSuccess && status == RA_OK; ++g) {
    char* base = static_cast<char*>(ws) + (size_t)(g % n_slots) * slot_bytes;
    void* dev[kMaxTensors];
    for (int i = 0; i < n_t; ++i) dev[i] = base + off[i];
    // In, once the compute of the group that used the slot before is done.
    for (int lane = 0; lane < 2 && e == cudaSuccess; ++lane)
      if (g >= n_slots) e = cudaStreamWaitEvent(lanes[lane], ev_comp(g - n_slots), 0);
    for (int i = 0; i < n_t && e == cudaSuccess; ++i)
      if (t[i].in)
        e = cudaMemcpy2DAsync(dev[i], t[i].row_bytes, static_cast<const char*>(t[i].in) + (size_t)g * t[i].row_bytes,
                              t[i].pitch, t[i].row_bytes, t[i].rows, cudaMemcpyHostToDevice, lanes[t[i].lane]);
    for (int lane = 0; lane < 2 && e == cudaSuccess; ++lane) {
      e = cudaEventRecord(ev_in(g, lane), lanes[lane]);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(ps->comp, ev_in(g, lane), 0);
    }
    // Compute, once the slot's previous results have been copied out.
    if (e == cudaSuccess && g >= n_slots) e = cudaStreamWaitEvent(ps->comp, ev_out(g - n_slots), 0);
    if (e != cudaSuccess) break;
    status = compute(g, dev, ps->comp);
    if (status != RA_OK) break;
    e = cudaEventRecord(ev_comp(g), ps->comp);
    // Out.
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ps->d2h, ev_comp(g), 0);
    for (int i = 0; i < n_t && e == cudaSuccess; ++i)
      if (t[i].out)
        e = cudaMemcpy2DAsync(static_cast<char*>(t[i].out) + (size_t)g * t[i].row_bytes, t[i].pitch, dev[i],
                              t[i].row_bytes, t[i].row_bytes, t[i].rows, cudaMemcpyDeviceToHost, ps->d2h);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out(g), ps->d2h);
  }
  // Join: the caller's stream waits for all four streams (also after a
  // failure, so the staging is freed only once nothing uses it).
  cudaError_t ej = cudaSuccess;
  for (int i = 0; i < 4; ++i) {
    if (ej == cudaSuccess) ej = cudaEventRecord(ev_end[i], pipes[i]);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, ev_end[i], 0);
  }
  if (ej != cudaSuccess) {
    // The join could not be queued: wait for the pipeline on the host.
    for (cudaStream_t s : pipes) cudaStreamSynchronize(s);
  }
  cudaError_t ef = cudaFreeAsync(ws, st);
  if (status != RA_OK) return status;
  if (e == cudaSuccess) e = ej;
  if (e == cudaSuccess) e = ef;
  return finish(e, st, what);
}

// Host-tensor descriptors of one group: token-major [B, N, H, d] rows (the
// group's `heads` of every token row) and [B, H, N] float32 rows (the group's
// heads of every batch entry).
PipeTensor token_rows(const void* in, void* out, int heads, int H, int d, size_t esz, long long BN, int lane) {
  return PipeTensor{in, out, (size_t)heads * d * esz, (size_t)H * d * esz, (size_t)BN, lane};
}
PipeTensor head_rows(const void* in, void* out, int heads, int H, long long N, int B, int lane) {
  return PipeTensor{in, out, (size_t)heads * N * 4, (size_t)H * N * 4, (size_t)B, lane};
}

}  // namespace

extern "C" {

int ring_attn_fwd_host(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                       int64_t N_q, int64_t N_kv, int d, int causal, int64_t chunk, int P, int64_t cache_idx,
                       float scale, int kv_heads_per_group, void* stream) {
  NvtxScope nvtx_scope("ring_attn_fwd_host");
  int r = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, N_q, N_kv, d, causal, chunk, P, cache_idx, scale, true);
  if (r != RA_OK) return r;
  if (kv_heads_per_group < 0 || kv_heads_per_group > Hkv ||
      (kv_heads_per_group > 0 && Hkv % kv_heads_per_group != 0))
    return RA_ERR_INVALID_ARG;
  if (B == 0 || N_q == 0) return RA_OK;
  int num_sms = 148;
  if ((r = check_device(&num_sms)) != RA_OK) return r;
  const int kvg = kv_heads_per_group > 0 ? kv_heads_per_group : default_kv_group(Hkv);
  const int hg = kvg * (Hq / Hkv);  // query heads per group
  const PipeTensor t[5] = {
      token_rows(q, nullptr, hg, Hq, d, 2, (long long)B * N_q, 0),
      token_rows(k, nullptr, kvg, Hkv, d, 2, (long long)B * N_kv, 1),
      token_rows(v, nullptr, kvg, Hkv, d, 2, (long long)B * N_kv, 1),
      token_rows(nullptr, out, hg, Hq, d, 2, (long long)B * N_q, 0),
      head_rows(nullptr, lse, hg, Hq, N_q, B, 0),
  };
  auto compute = [&](int, void** dev, cudaStream_t cs) {
    // The group is an independent problem of hg query heads over kvg KV heads.
    ProblemArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = dev[0]; a.k = dev[1]; a.v = dev[2]; a.out = dev[3]; a.lse = static_cast<float*>(dev[4]);
    a.B = B; a.Hq = hg; a.Hkv = kvg; a.d = d;
    a.N_q = N_q; a.N_kv = N_kv;
    a.q_pos0 = cache_idx < 0 ? 0 : cache_idx;
    a.k_pos0 = 0;
    a.causal = causal; a.scale = scale; a.chunk = chunk; a.P = P; a.out_f32 = 0;
    a.S = cache_idx < 0 ? 1 : 0;
    return run_fwd(a, num_sms, cs, "ring_attn_fwd_host");
  };
  return run_host_pipeline(Hkv / kvg, t, 5, static_cast<cudaStream_t>(stream), "ring_attn_fwd_host", compute);
}

int ring_attn_bwd_host(const void* q, const void* k, const void* v, const void* out, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int64_t N_q,
                       int64_t N_kv, int d, int causal, int64_t cache_idx, float scale, int kv_heads_per_group,
                       void* stream) {
  NvtxScope nvtx_scope("ring_attn_bwd_host");
  if (!dout || !dq || !dk || !dv) return RA_ERR_INVALID_ARG;
  if (!(aligned16(dout) && aligned16(dq) && aligned16(dk) && aligned16(dv))) return RA_ERR_INVALID_ARG;
  int r = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, N_q, N_kv, d, causal, N_kv, 1, cache_idx, scale, true);
  if (r != RA_OK) return r;
  if (kv_heads_per_group < 0 || kv_heads_per_group > Hkv ||
      (kv_heads_per_group > 0 && Hkv % kv_heads_per_group != 0))
    return RA_ERR_INVALID_ARG;
  if (B == 0 || N_q == 0) return RA_OK;
  if ((r = check_device(nullptr)) != RA_OK) return r;
  const int kvg = kv_heads_per_group > 0 ? kv_heads_per_group : default_kv_group(Hkv);
  const int hg = kvg * (Hq / Hkv);
  const long long BNq = (long long)B * N_q, BNk = (long long)B * N_kv;
  const PipeTensor t[9] = {
      token_rows(q, nullptr, hg, Hq, d, 2, BNq, 0),      token_rows(k, nullptr, kvg, Hkv, d, 2, BNk, 1),
      token_rows(v, nullptr, kvg, Hkv, d, 2, BNk, 1),    token_rows(out, nullptr, hg, Hq, d, 2, BNq, 0),
      token_rows(dout, nullptr, hg, Hq, d, 2, BNq, 1),   head_rows(lse, nullptr, hg, Hq, N_q, B, 0),
      token_rows(nullptr, dq, hg, Hq, d, 2, BNq, 0),     token_rows(nullptr, dk, kvg, Hkv, d, 2, BNk, 0),
      token_rows(nullptr, dv, kvg, Hkv, d, 2, BNk, 0),
  };
  auto compute = [&](int, void** dev, cudaStream_t cs) {
    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = dev[0]; a.k = dev[1]; a.v = dev[2]; a.out = dev[3]; a.dout = dev[4];
    a.lse = static_cast<const float*>(dev[5]);
    a.dq = dev[6]; a.dk = dev[7]; a.dv = dev[8];
    a.B = B; a.Hq = hg; a.Hkv = kvg; a.d = d;
    a.N_q = N_q; a.N_kv = N_kv;
    a.q_pos0 = cache_idx < 0 ? 0 : cache_idx;
    a.k_pos0 = 0;
    a.causal = causal; a.scale = scale;
    a.accumulate = 0;
    return run_bwd(a, "ring_attn_bwd_host", cs);
  };
  return run_host_pipeline(Hkv / kvg, t, 9, static_cast<cudaStream_t>(stream), "ring_attn_bwd_host", compute);
}

int ring_attn_fwd_window_anchor(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                                int Hkv, int64_t N, int d, int64_t chunk, int P, int64_t window,
                                int64_t anchor_period, float scale, void* stream) {
  NvtxScope nvtx_scope("ring_attn_fwd_window_anchor");
  if (window < 0 || window > kMaxTokens || anchor_period <= 0 || anchor_period % 256 != 0 ||
      anchor_period > kMaxTokens)
    return RA_ERR_INVALID_ARG;
  int r = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, N, N, d, 0, chunk, P, -1, scale, true);
  if (r != RA_OK) return r;
  if (B == 0 || N == 0) return RA_OK;
  int num_sms = 148;
  if ((r = check_device(&num_sms)) != RA_OK) return r;
  ProblemArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = out; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.N_q = N; a.N_kv = N;
  a.q_pos0 = 0; a.k_pos0 = 0;
  a.causal = 0; a.scale = scale; a.chunk = chunk; a.P = P; a.out_f32 = 0; a.S = 1;
  a.wa_window = (int)window;
  a.wa_period = (int)anchor_period;
  return run_fwd(a, num_sms, static_cast<cudaStream_t>(stream), "ring_attn_fwd_window_anchor");
}

int ring_attn_fwd_window_anchor_host(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                     int Hq, int Hkv, int64_t N, int d, int64_t chunk, int P, int64_t window,
                                     int64_t anchor_period, float scale, int kv_heads_per_group, void* stream) {
  NvtxScope nvtx_scope("ring_attn_fwd_window_anchor_host");
  if (window < 0 || window > kMaxTokens || anchor_period <= 0 || anchor_period % 256 != 0 ||
      anchor_period > kMaxTokens)
    return RA_ERR_INVALID_ARG;
  int r = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, N, N, d, 0, chunk, P, -1, scale, true);
  if (r != RA_OK) return r;
  if (kv_heads_per_group < 0 || kv_heads_per_group > Hkv ||
      (kv_heads_per_group > 0 && Hkv % kv_heads_per_group != 0))
    return RA_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return RA_OK;
  int num_sms = 148;
  if ((r = check_device(&num_sms)) != RA_OK) return r;
  const int kvg = kv_heads_per_group > 0 ? kv_heads_per_group : default_kv_group(Hkv);
  const int hg = kvg * (Hq / Hkv);
  const long long BN = (long long)B * N;
  const PipeTensor t[5] = {
      token_rows(q, nullptr, hg, Hq, d, 2, BN, 0),  token_rows(k, nullptr, kvg, Hkv, d, 2, BN, 1),
      token_rows(v, nullptr, kvg, Hkv, d, 2, BN, 1), token_rows(nullptr, out, hg, Hq, d, 2, BN, 0),
      head_rows(nullptr, lse, hg, Hq, N, B, 0),
  };
  auto compute = [&](int, void** dev, cudaStream_t cs) {
    ProblemArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = dev[0]; a.k = dev[1]; a.v = dev[2]; a.out = dev[3]; a.lse = static_cast<float*>(dev[4]);
    a.B = B; a.Hq = hg; a.Hkv = kvg; a.d = d;
    a.N_q = N; a.N_kv = N;
    a.q_pos0 = 0; a.k_pos0 = 0;
    a.causal = 0; a.scale = scale; a.chunk = chunk; a.P = P; a.out_f32 = 0; a.S = 1;
    a.wa_window = (int)window;
    a.wa_period = (int)anchor_period;
    return run_fwd(a, num_sms, cs, "ring_attn_fwd_window_anchor_host");
  };
  return run_host_pipeline(Hkv / kvg, t, 5, static_cast<cudaStream_t>(stream), "ring_attn_fwd_window_anchor_host",
                           compute);
}

int ring_attn_fwd_fp8kv(const void* q, const void* k8, const void* v8, const float* k_scale, const float* v_scale,
                        void* out, float* lse, int B, int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d, int causal,
                        int64_t chunk, int P, int64_t cache_idx, float scale, void* stream) {
  NvtxScope nvtx_scope("ring_attn_fwd_fp8kv");
  if (!k_scale || !v_scale) return RA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_scale) | reinterpret_cast<uintptr_t>(v_scale)) & 3u) return RA_ERR_INVALID_ARG;
  int r = validate_fwd(q, k8, v8, out, lse, B, Hq, Hkv, N_q, N_kv, d, causal, chunk, P, cache_idx, scale, true);
  if (r != RA_OK) return r;
  if (B == 0 || N_q == 0) return RA_OK;
  int num_sms = 148;
  if ((r = check_device(&num_sms)) != RA_OK) return r;
  ProblemArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k8; a.v = v8; a.out = out; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.N_q = N_q; a.N_kv = N_kv;
  a.q_pos0 = cache_idx < 0 ? 0 : cache_idx;
  a.k_pos0 = 0;
  a.causal = causal; a.scale = scale; a.chunk = chunk; a.P = P; a.out_f32 = 0;
  a.kv8 = 1; a.k_scale = k_scale; a.v_scale = v_scale;
  a.S = cache_idx < 0 ? 1 : 0;
  return run_fwd(a, num_sms, static_cast<cudaStream_t>(stream), "ring_attn_fwd_fp8kv");
}

int ring_attn_fwd_f32(const float* q, const float* k, const float* v, float* out, float* lse, int B, int Hq,
                      int Hkv, int64_t N_q, int64_t N_kv, int d, int causal, int64_t chunk, int P, int64_t cache_idx,
                      float scale, void* stream) {
  NvtxScope nvtx_scope("ring_attn_fwd_f32");
  int r = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, N_q, N_kv, d, causal, chunk, P, cache_idx, scale, false);
  if (r != RA_OK) return r;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
       reinterpret_cast<uintptr_t>(out)) & 3u)
    return RA_ERR_INVALID_ARG;
  if (B == 0 || N_q == 0) return RA_OK;
  if ((r = check_device(nullptr)) != RA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProblemArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = out; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.N_q = N_q; a.N_kv = N_kv;
  a.q_pos0 = cache_idx < 0 ? 0 : cache_idx;
  a.k_pos0 = 0;
  a.causal = causal; a.scale = scale; a.chunk = chunk; a.P = P; a.S = 1; a.out_f32 = 1;
  return finish(launch_fwd_simt_f32(a, kModeFinal, st), st, "ring_attn_fwd_f32");
}

int ring_attn_block_step(const void* q_chunk, const void* k_chunk, const void* v_chunk, int64_t q_off,
                         int64_t k_off, float* acc, float* m, float* l, int B, int Hq, int Hkv, int64_t Lq,
                         int64_t Lk, int d, int causal, float scale, int dtype, void* stream) {
  NvtxScope nvtx_scope("ring_attn_block_step");
  if (!q_chunk || !k_chunk || !v_chunk || !acc || !m || !l) return RA_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return RA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return RA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID_ARG;
  if (Lq < 0 || Lk < 0 || Lq > kMaxTokens || Lk > kMaxTokens) return RA_ERR_INVALID_ARG;
  if (q_off < 0 || k_off < 0) return RA_ERR_INVALID_ARG;
  if (dtype != RA_DTYPE_BF16 && dtype != RA_DTYPE_F32) return RA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return RA_ERR_INVALID_ARG;
  if (!aligned16(acc) || (reinterpret_cast<uintptr_t>(m) & 3u) || (reinterpret_cast<uintptr_t>(l) & 3u))
    return RA_ERR_INVALID_ARG;
  if (dtype == RA_DTYPE_BF16 && !(aligned16(q_chunk) && aligned16(k_chunk) && aligned16(v_chunk)))
    return RA_ERR_INVALID_ARG;
  if (B == 0 || Lq == 0 || Lk == 0) return RA_OK;
  int r = check_device(nullptr);
  if (r != RA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProblemArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q_chunk; a.k = k_chunk; a.v = v_chunk;
  a.acc = acc; a.m = m; a.l = l;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.N_q = Lq; a.N_kv = Lk;
  a.q_pos0 = q_off; a.k_pos0 = k_off;
  a.causal = causal; a.scale = scale; a.chunk = Lk; a.P = 1; a.S = 1;
  cudaError_t e = dtype == RA_DTYPE_BF16 ? launch_fwd_sm100(a, kModeState, st) : launch_fwd_simt_f32(a, kModeState, st);
  return finish(e, st, "ring_attn_block_step");
}

int ring_attn_finalize(const float* acc, const float* m, const float* l, void* out, float* lse, int B, int Hq,
                       int64_t Lq, int d, int out_dtype, void* stream) {
  NvtxScope nvtx_scope("ring_attn_finalize");
  if (!acc || !m || !l || !out || !lse) return RA_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Lq < 0 || (d != 64 && d != 128)) return RA_ERR_INVALID_ARG;
  if (out_dtype != RA_DTYPE_BF16 && out_dtype != RA_DTYPE_F32) return RA_ERR_INVALID_ARG;
  if (!aligned16(acc) || !aligned16(out)) return RA_ERR_INVALID_ARG;
  if (B == 0 || Lq == 0) return RA_OK;
  int r = check_device(nullptr);
  if (r != RA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return finish(launch_finalize(acc, m, l, out, lse, B, Hq, Lq, d, out_dtype == RA_DTYPE_F32, st), st,
                "ring_attn_finalize");
}

int lse_merge(const float* o_parts, const float* lse_parts, int S, void* out, float* lse, int B, int Hq,
              int64_t N_q, int d, int out_dtype, void* stream) {
  NvtxScope nvtx_scope("lse_merge");
  if (!o_parts || !lse_parts || !out || !lse) return RA_ERR_INVALID_ARG;
  if (S < 1 || B < 0 || Hq < 1 || N_q < 0 || (d != 64 && d != 128)) return RA_ERR_INVALID_ARG;
  if (out_dtype != RA_DTYPE_BF16 && out_dtype != RA_DTYPE_F32) return RA_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(out)) return RA_ERR_INVALID_ARG;
  if (B == 0 || N_q == 0) return RA_OK;
  int r = check_device(nullptr);
  if (r != RA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return finish(launch_lse_merge(o_parts, lse_parts, S, out, lse, B, Hq, N_q, d, out_dtype == RA_DTYPE_F32, st), st,
                "lse_merge");
}

}  // extern "C"

namespace {

// Workspace (lse * log2 e and D per query row, padded to 128 rows), then the
// three backward kernels.  Arguments are already validated.
int run_bwd(ra::BwdArgs a, const char* what, cudaStream_t st) {
  a.Npad = (a.N_q + 127) / 128 * 128;
  const size_t ws_bytes = (size_t)2 * a.B * a.Hq * a.Npad * sizeof(float);
  if (std::strcmp(env_str("RINGATTN_FAULT"), "alloc") == 0) {
    t_last_error = "workspace allocation refused (RINGATTN_FAULT=alloc)";
    return RA_ERR_OOM;
  }
  void* ws = nullptr;
  cudaError_t e = cudaMallocAsync(&ws, ws_bytes, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    t_last_error = std::string("cudaMallocAsync: ") + cudaGetErrorString(e);
    return RA_ERR_OOM;
  }
  a.ws_lse2 = static_cast<float*>(ws);
  a.ws_d = a.ws_lse2 + (size_t)a.B * a.Hq * a.Npad;
  e = launch_bwd_sm100(a, st);
  cudaError_t ef = cudaFreeAsync(ws, st);
  if (e == cudaSuccess) e = ef;
  return finish(e, st, what);
}

}  // namespace

extern "C" {

int ring_attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d, int causal,
                  int64_t cache_idx, float scale, void* stream) {
  NvtxScope nvtx_scope("ring_attn_bwd");
  if (!dout || !dq || !dk || !dv) return RA_ERR_INVALID_ARG;
  if (!(aligned16(dout) && aligned16(dq) && aligned16(dk) && aligned16(dv))) return RA_ERR_INVALID_ARG;
  // Same shape rules as ring_attn_fwd (one chunk spanning the sequence).
  int r = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, N_q, N_kv, d, causal, N_kv, 1, cache_idx, scale, true);
  if (r != RA_OK) return r;
  if (B == 0 || N_q == 0) return RA_OK;
  if ((r = check_device(nullptr)) != RA_OK) return r;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = out; a.dout = dout; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.N_q = N_q; a.N_kv = N_kv;
  a.q_pos0 = cache_idx < 0 ? 0 : cache_idx;
  a.k_pos0 = 0;
  a.causal = causal; a.scale = scale;
  a.accumulate = 0;
  return run_bwd(a, "ring_attn_bwd", static_cast<cudaStream_t>(stream));
}

int ring_attn_bwd_block_step(const void* q_chunk, const void* k_chunk, const void* v_chunk, const void* out_chunk,
                             const void* dout_chunk, const float* lse_chunk, int64_t q_off, int64_t k_off,
                             float* dq_acc, float* dk_acc, float* dv_acc, int B, int Hq, int Hkv, int64_t Lq,
                             int64_t Lk, int d, int causal, float scale, void* stream) {
  NvtxScope nvtx_scope("ring_attn_bwd_block_step");
  if (!q_chunk || !k_chunk || !v_chunk || !out_chunk || !dout_chunk || !lse_chunk) return RA_ERR_INVALID_ARG;
  if (!dq_acc || !dk_acc || !dv_acc) return RA_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return RA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return RA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID_ARG;
  if (Lq < 0 || Lk < 0 || Lq > kMaxTokens || Lk > kMaxTokens) return RA_ERR_INVALID_ARG;
  if (q_off < 0 || k_off < 0) return RA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return RA_ERR_INVALID_ARG;
  if (!(aligned16(q_chunk) && aligned16(k_chunk) && aligned16(v_chunk) && aligned16(out_chunk) &&
        aligned16(dout_chunk) && aligned16(dq_acc) && aligned16(dk_acc) && aligned16(dv_acc)))
    return RA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse_chunk) & 3u) return RA_ERR_INVALID_ARG;
  if (B == 0 || Lq == 0 || Lk == 0) return RA_OK;
  int r = check_device(nullptr);
  if (r != RA_OK) return r;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q_chunk; a.k = k_chunk; a.v = v_chunk; a.out = out_chunk; a.dout = dout_chunk; a.lse = lse_chunk;
  a.dq = dq_acc; a.dk = dk_acc; a.dv = dv_acc;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.N_q = Lq; a.N_kv = Lk;
  a.q_pos0 = q_off;
  a.k_pos0 = k_off;
  a.causal = causal; a.scale = scale;
  a.accumulate = 1;
  return run_bwd(a, "ring_attn_bwd_block_step", static_cast<cudaStream_t>(stream));
}

int ring_attn_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  NvtxScope nvtx_scope("ring_attn_exp2_poly");
  if (!x || !y || n < 0) return RA_ERR_INVALID_ARG;
  if (n == 0) return RA_OK;
  int r = check_device(nullptr);
  if (r != RA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return finish(launch_exp2_poly(x, y, n, st), st, "ring_attn_exp2_poly");
}

int ring_attn_add_and_clear(float* acc, float* part, int64_t n, void* stream) {
  NvtxScope nvtx_scope("ring_attn_add_and_clear");
  if (n < 0) return RA_ERR_INVALID_ARG;
  if (n == 0) return RA_OK;
  if (!acc || !part || acc == part) return RA_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(acc) | reinterpret_cast<uintptr_t>(part)) & 3u) != 0) return RA_ERR_INVALID_ARG;
  int num_sms = 148;
  int r = check_device(&num_sms);
  if (r != RA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return finish(launch_add_clear(acc, part, n, num_sms, st), st, "ring_attn_add_and_clear");
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Allocation-free incremental query (ring_attn_fwd_noalloc).
//
// Some callers cannot let a library allocate device memory: serving stacks
// whose pool allocator owns the whole HBM budget up front, and latency-critical
// loops where an allocation could fail, fragment that budget or stall on the
// allocator.  For them the split-KV partials live in a fixed, file-scope device
// array instead of a stream-ordered workspace.  Every GPU that loads this
// library reserves the array until the process exits.
// ----------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char ra_noalloc_scratch[kNoAllocScratchBytes];

namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_scratch_ptr[256] = {};  // device address of the array, per device ordinal

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress once per device (with that device current) and
// cached.
int noalloc_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= 256) {
    t_last_error = "ring_attn_fwd_noalloc: device ordinal out of range";
    return RA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, ra_noalloc_scratch);
    if (e != cudaSuccess) return set_cuda_error(e, "cudaGetSymbolAddress(ra_noalloc_scratch)");
    g_noalloc_scratch_ptr[dev] = p;
  }
  *out = g_noalloc_scratch_ptr[dev];
  return RA_OK;
}

}  // namespace

extern "C" int ring_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                     int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d, int causal, int64_t chunk,
                                     int P, int64_t cache_idx, float scale, void* stream) {
  NvtxScope nvtx_scope("ring_attn_fwd_noalloc");
  int r = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, N_q, N_kv, d, causal, chunk, P, cache_idx, scale, true);
  if (r != RA_OK) return r;
  if (cache_idx < 0) {
    t_last_error = "ring_attn_fwd_noalloc serves incremental queries only (cache_idx >= 0)";
    return RA_ERR_INVALID_ARG;
  }
  if (B == 0 || N_q == 0) return RA_OK;
  int num_sms = 148;
  if ((r = check_device(&num_sms)) != RA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  ProblemArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = out; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.N_q = N_q; a.N_kv = N_kv;
  a.q_pos0 = cache_idx;
  a.k_pos0 = 0;
  a.causal = causal; a.scale = scale; a.chunk = chunk; a.P = P; a.S = 1; a.out_f32 = 0;

  // Same split count as ring_attn_fwd, so both produce the same partials.
  const long long items = sm100_geometry(a, kModeSplit).ctas_per_split;
  const int S = choose_splits(items, P, num_sms, N_q);
  if (S == 1) return finish(launch_fwd_sm100(a, kModeFinal, st), st, "ring_attn_fwd_noalloc");

  const size_t o_bytes = (size_t)S * B * N_q * Hq * d * sizeof(float);
  const size_t l_bytes = (size_t)S * B * Hq * N_q * sizeof(float);
  if (o_bytes + l_bytes > kNoAllocScratchBytes) {
    t_last_error = "ring_attn_fwd_noalloc: this call needs " + std::to_string(o_bytes + l_bytes) +
                   " bytes of split-KV scratch; the static scratch holds " + std::to_string(kNoAllocScratchBytes) +
                   " bytes (use ring_attn_fwd, or fewer rows B*N_q*Hq)";
    return RA_ERR_INVALID_ARG;
  }
  void* base = nullptr;
  if ((r = noalloc_scratch_address(&base)) != RA_OK) return r;
  // Every partial row and lse the merge reads is written by the split kernel
  // of this same call, so nothing in the scratch needs clearing first.
  a.S = S;
  a.o_part = static_cast<float*>(base);
  a.lse_part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + o_bytes);
  cudaError_t e = launch_fwd_sm100(a, kModeSplit, st);
  if (e == cudaSuccess) e = launch_lse_merge(a.o_part, a.lse_part, S, out, lse, B, Hq, N_q, d, 0, st);
  return finish(e, st, "ring_attn_fwd_noalloc");
}
