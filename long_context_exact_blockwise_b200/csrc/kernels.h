// Host-side launchers of the library's kernels (internal; not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace ra {

// Kernels this process has launched through the library (all devices).
inline std::atomic<long long>& launch_counter() {
  static std::atomic<long long> n{0};
  return n;
}
inline cudaError_t count_launch(cudaError_t e) {
  if (e == cudaSuccess) launch_counter().fetch_add(1, std::memory_order_relaxed);
  return e;
}

// Output modes of the forward kernels.
enum FwdMode : int {
  kModeFinal = 0,  // normalised out (bf16/f32) + lse
  kModeSplit = 1,  // normalised float32 partial + lse per KV split (merged by lse_merge)
  kModeState = 2,  // running (acc, m, l) read and written in place (one ring visit)
};

// One blockwise attention problem as seen by a kernel.  Query row t of the q
// buffer sits at global position q_pos0 + t; key row j of the k/v buffers at
// k_pos0 + j.  The k rows are cut into P chunks of `chunk` rows; a tile of
// query rows homed at chunk i visits chunk (i + s) mod P at step s.
struct ProblemArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;        // kModeFinal: [B, N_q, Hq, d]
  float* lse;       // kModeFinal: [B, Hq, N_q]
  float* o_part;    // kModeSplit: [S, B, N_q, Hq, d]
  float* lse_part;  // kModeSplit: [S, B, Hq, N_q]
  float* acc;       // kModeState: [B, Hq, N_q, d]
  float* m;         // kModeState: [B, Hq, N_q]
  float* l;         // kModeState: [B, Hq, N_q]
  int B, Hq, Hkv, d;
  long long N_q, N_kv;
  long long q_pos0, k_pos0;
  int causal;
  float scale;
  long long chunk;
  int P;
  int S;            // KV splits (kModeSplit), 1 otherwise
  int out_f32;      // kModeFinal: 1 = float32 out, 0 = bf16 out
  int kv8;          // 1: k and v are FP8 E4M3 codes, dequantised by k_scale / v_scale [B, Hkv]
  const float* k_scale;
  const float* v_scale;
  int wa_window;    // window-and-anchor mask (square prefill, causal = 0): window W and
  int wa_period;    // anchor period A (a multiple of 256); wa_period = 0: no such mask
};

// Tensor-core path (tcgen05 + TMEM + TMA), bf16 inputs, d in {64, 128}.
cudaError_t launch_fwd_sm100(const ProblemArgs& a, int mode, cudaStream_t stream);

// Pair (cta_group::2) kernel for long query blocks (d = 128, bf16, final or
// split-KV output): whether it takes a problem, and its launcher.
// launch_fwd_sm100 routes such problems to it when RINGATTN_PAIR=1 (off by
// default: it measured slower than the single-CTA kernel).
bool fwd2_applies(const ProblemArgs& a, int mode);
cudaError_t launch_fwd2_sm100(const ProblemArgs& a, int mode, cudaStream_t stream);

// Keys-on-M decode kernel (d = 128, incremental queries with G * N_q <= 32
// rows per KV head): rows per block it would use (16 or 32; 0 = not
// applicable), and its launcher.  launch_fwd_sm100 routes such problems to it.
int decode_rows(const ProblemArgs& a, int mode);
cudaError_t launch_decode_sm100(const ProblemArgs& a, int mode, cudaStream_t stream);

// CTA geometry the tensor-core path uses for a problem: query heads packed
// per tile (gpack), tokens per tile, one or two query tiles per CTA, and the
// number of CTAs per KV split.
struct Sm100Geometry {
  int gpack, gshift, tpt;
  bool two;
  int n_qblk;
  long long ctas_per_split;
};
Sm100Geometry sm100_geometry(const ProblemArgs& a, int mode);

// CUDA-core float32 path (also serves float32 block steps).
cudaError_t launch_fwd_simt_f32(const ProblemArgs& a, int mode, cudaStream_t stream);

// out = acc / l, lse = m + ln l.
cudaError_t launch_finalize(const float* acc, const float* m, const float* l, void* out, float* lse,
                            int B, int Hq, long long Lq, int d, int out_f32, cudaStream_t stream);

// Log-sum-exp merge of S normalised partials.
cudaError_t launch_lse_merge(const float* o_parts, const float* lse_parts, int S, void* out, float* lse,
                             int B, int Hq, long long N_q, int d, int out_f32, cudaStream_t stream);

// Backward pass (bf16 tensors, float32 workspace of 2 * B * Hq * Npad floats).
struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* out;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* ws_lse2;  // [B, Hq, Npad]
  float* ws_d;     // [B, Hq, Npad]
  int B, Hq, Hkv, d;
  long long N_q, N_kv, Npad;
  long long q_pos0, k_pos0;  // global positions of q row 0 and k row 0
  int causal;
  int accumulate;  // 0: dq, dk, dv are bf16 outputs; 1: float32 accumulators (+=)
  float scale;
};
cudaError_t launch_bwd_sm100(const BwdArgs& a, cudaStream_t stream);

// dst += src, then src = 0 (float32, n elements).
cudaError_t launch_add_clear(float* dst, float* src, long long n, int num_sms, cudaStream_t stream);

// y = exp2_poly2(x) elementwise (the FMA-pipe exp2 of the softmax), for tests.
cudaError_t launch_exp2_poly(const float* x, float* y, long long n, cudaStream_t stream);

// Resolve cuTensorMapEncodeTiled through the runtime (no link-time libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace ra
