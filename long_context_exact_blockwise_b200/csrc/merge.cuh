// Global normalisation kernels ("From hundreds of milliseconds to a million
// tokens", system layer 4: the fusion layer normalises the softmax over all
// local outputs):
//   finalize : out = acc / l, lse = m + ln l           (one running state)
//   lse_merge: out = sum_s w_s O_s / sum_s w_s,        (S normalised partials)
//              w_s = exp(lse_s - max_s lse_s)
// Both are HBM-bound: one warp per output row, 16-byte loads along d.
#pragma once

#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace ra {

namespace {

constexpr int kRowsPerBlock = 8;  // one warp per row

template <int D>
struct Vec;
template <>
struct Vec<128> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float (&x)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
};
template <>
struct Vec<64> {
  static constexpr int N = 2;
  __device__ static void load(const float* p, float (&x)[2]) {
    const float2 v = __ldg(reinterpret_cast<const float2*>(p));
    x[0] = v.x; x[1] = v.y;
  }
};

template <int N>
__device__ __forceinline__ void store_row(void* out, long long off, int lane, const float (&x)[N], int out_f32) {
  if (out_f32) {
    float* o = static_cast<float*>(out) + off + lane * N;
    if constexpr (N == 4) {
      *reinterpret_cast<float4*>(o) = make_float4(x[0], x[1], x[2], x[3]);
    } else {
      *reinterpret_cast<float2*>(o) = make_float2(x[0], x[1]);
    }
  } else {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out) + off + lane * N;
    if constexpr (N == 4) {
      __nv_bfloat162 p0 = __floats2bfloat162_rn(x[0], x[1]);
      __nv_bfloat162 p1 = __floats2bfloat162_rn(x[2], x[3]);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&p0);
      u.y = *reinterpret_cast<uint32_t*>(&p1);
      *reinterpret_cast<uint2*>(o) = u;
    } else {
      __nv_bfloat162 p0 = __floats2bfloat162_rn(x[0], x[1]);
      *reinterpret_cast<__nv_bfloat162*>(o) = p0;
    }
  }
}

// Rows are enumerated in the output layout [B, N_q, Hq].
template <int D>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
lse_merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int S, void* out,
                 float* lse, int B, int Hq, long long N_q, int out_f32) {
  constexpr int N = Vec<D>::N;
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  const long long rows = (long long)B * N_q * Hq;
  if (r >= rows) return;
  const int h = (int)(r % Hq);
  const long long t = (r / Hq) % N_q;
  const int b = (int)(r / ((long long)Hq * N_q));
  const long long lse_stride = (long long)B * Hq * N_q;  // between splits
  const long long lse_idx = ((long long)b * Hq + h) * N_q + t;
  const long long o_stride = rows * D;

  // Row maximum of the partial lse values, lanes striding over the splits.
  float M = -INFINITY;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, __ldg(lse_parts + s * lse_stride + lse_idx));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float base = (M == -INFINITY) ? 0.f : M;

  float acc[N];
#pragma unroll
  for (int i = 0; i < N; ++i) acc[i] = 0.f;
  float W = 0.f;
  for (int s = 0; s < S; ++s) {
    const float ls = __ldg(lse_parts + s * lse_stride + lse_idx);
    const float w = expf(ls - base);
    if (w > 0.f) {
      float x[N];
      Vec<D>::load(o_parts + s * o_stride + r * D + lane * N, x);
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = fmaf(w, x[i], acc[i]);
      W += w;
    }
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) acc[i] *= inv;
  store_row<N>(out, r * D, lane, acc, out_f32);
  if (lane == 0) lse[lse_idx] = W > 0.f ? base + logf(W) : -INFINITY;
}

// Rows are enumerated in the state layout [B, Hq, Lq].
template <int D>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
finalize_kernel(const float* __restrict__ acc, const float* __restrict__ m, const float* __restrict__ l, void* out,
                float* lse, int B, int Hq, long long Lq, int out_f32) {
  constexpr int N = Vec<D>::N;
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  const long long rows = (long long)B * Hq * Lq;
  if (r >= rows) return;
  const long long t = r % Lq;
  const int h = (int)((r / Lq) % Hq);
  const int b = (int)(r / ((long long)Hq * Lq));
  const float lr = __ldg(l + r);
  const float mr = __ldg(m + r);
  float x[N];
  Vec<D>::load(acc + r * D + lane * N, x);
  const float inv = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) x[i] = lr > 0.f ? x[i] * inv : 0.f;
  const long long ooff = (((long long)b * Lq + t) * Hq + h) * D;
  store_row<N>(out, ooff, lane, x, out_f32);
  if (lane == 0) lse[r] = lr > 0.f ? mr + logf(lr) : -INFINITY;
}

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

// dst += src, then src = 0, over n floats: 16-byte vectors over the first
// n4 * 4 elements (n4 = 0 when a pointer is not 16-byte aligned), then the
// scalar tail.  Grid-stride.
__global__ void add_clear_kernel(float* __restrict__ dst, float* __restrict__ src, long long n, long long n4) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  float4* d4 = reinterpret_cast<float4*>(dst);
  float4* s4 = reinterpret_cast<float4*>(src);
  for (long long i = t0; i < n4; i += stride) {
    float4 a = d4[i];
    const float4 b = s4[i];
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    d4[i] = a;
    s4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (long long i = 4 * n4 + t0; i < n; i += stride) {
    dst[i] += src[i];
    src[i] = 0.f;
  }
}

}  // namespace

cudaError_t launch_add_clear(float* dst, float* src, long long n, int num_sms, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const bool vec = ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15u) == 0;
  const long long n4 = vec ? n / 4 : 0;
  const long long work = n4 + (n - 4 * n4);
  long long blocks = (work + 255) / 256;
  const long long cap = 4LL * num_sms;  // a few resident blocks per SM, grid-stride beyond
  if (blocks > cap) blocks = cap;
  add_clear_kernel<<<(unsigned)blocks, 256, 0, st>>>(dst, src, n, n4);
  return count_launch(cudaGetLastError());
}

cudaError_t launch_exp2_poly(const float* x, float* y, long long n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const long long pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, st>>>(x, y, n);
  return count_launch(cudaGetLastError());
}

cudaError_t launch_lse_merge(const float* o_parts, const float* lse_parts, int S, void* out, float* lse, int B,
                             int Hq, long long N_q, int d, int out_f32, cudaStream_t st) {
  const long long rows = (long long)B * N_q * Hq;
  if (rows <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock);
  if (d == 64)
    lse_merge_kernel<64><<<grid, 32 * kRowsPerBlock, 0, st>>>(o_parts, lse_parts, S, out, lse, B, Hq, N_q, out_f32);
  else
    lse_merge_kernel<128><<<grid, 32 * kRowsPerBlock, 0, st>>>(o_parts, lse_parts, S, out, lse, B, Hq, N_q, out_f32);
  return count_launch(cudaGetLastError());
}

cudaError_t launch_finalize(const float* acc, const float* m, const float* l, void* out, float* lse, int B, int Hq,
                            long long Lq, int d, int out_f32, cudaStream_t st) {
  const long long rows = (long long)B * Hq * Lq;
  if (rows <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock);
  if (d == 64)
    finalize_kernel<64><<<grid, 32 * kRowsPerBlock, 0, st>>>(acc, m, l, out, lse, B, Hq, Lq, out_f32);
  else
    finalize_kernel<128><<<grid, 32 * kRowsPerBlock, 0, st>>>(acc, m, l, out, lse, B, Hq, Lq, out_f32);
  return count_launch(cudaGetLastError());
}

}  // namespace ra
