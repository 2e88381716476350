// Float32 blockwise attention on CUDA cores (FFMA), for the float32 entry
// points: ring_attn_fwd_f32 and ring_attn_block_step with float32 chunks.
//
// TF32 tensor cores would miss the 1e-4 absolute bound the float32 path is
// held to, so this path stays in exact float32 arithmetic (only exp2 is the
// hardware approximation, relative error ~2^-22).
//
// Mapping: D/32 threads share one query row; thread `sub` owns elements
// e = i * TPR + sub (i < 32) of the row, so the threads of a row read
// adjacent shared-memory banks.  A CTA of 128 threads holds 128 / TPR rows
// and walks the KV chunks in ring order (i + s) mod P ("Ring Attention: the
// secret of million-token context", §2.2), streaming 32-key tiles through
// shared memory and folding each tile into running (m, l, o) statistics
// (§3.1 inner loop).
#pragma once

#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace ra {

namespace {

constexpr int kSimtThreads = 128;
constexpr int kSimtKeys = 32;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kSimtThreads) simt_attn_kernel(ProblemArgs a) {
  constexpr int TPR = D / 32;
  constexpr int ROWS = kSimtThreads / TPR;
  constexpr int KT = kSimtKeys;
  __shared__ float sK[KT][D];
  __shared__ float sV[KT][D];

  const int tid = threadIdx.x;
  const int sub = tid % TPR;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int hk = h / (a.Hq / a.Hkv);
  const long long row0 = (long long)blockIdx.x * ROWS;
  const long long row = row0 + tid / TPR;
  const bool valid = row < a.N_q;
  const long long pos = a.q_pos0 + row;
  const float sl = a.scale * kLog2e;

  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* V = static_cast<const T*>(a.v);

  float qv[32], o[32];
  float m2 = -INFINITY, l = 0.f;
  float m_in_nat = -INFINITY;
  {
    const long long qoff = (((long long)b * a.N_q + (valid ? row : 0)) * a.Hq + h) * D;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      qv[i] = valid ? to_f<T>(Q[qoff + i * TPR + sub]) : 0.f;
      o[i] = 0.f;
    }
  }
  if (MODE == kModeState && valid) {
    const long long srow = ((long long)b * a.Hq + h) * a.N_q + row;
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = a.acc[srow * D + i * TPR + sub];
    m_in_nat = a.m[srow];
    m2 = m_in_nat * kLog2e;
    l = a.l[srow];
  }
  const float m2_in = m2;

  // Keys past the CTA's last query position are invisible to all its rows.
  const long long last_row = min(row0 + ROWS, a.N_q) - 1;
  long long lim = a.N_kv;
  if (a.causal) lim = min(lim, a.q_pos0 + last_row - a.k_pos0 + 1);
  long long first_rel = a.q_pos0 + row0 - a.k_pos0;
  int home = 0;
  if (first_rel > 0) home = (int)min((long long)(a.P - 1), first_rel / a.chunk);

  for (int s = 0; s < a.P; ++s) {
    const int c = (home + s) % a.P;
    const long long cb = (long long)c * a.chunk;
    const long long ce = min(cb + a.chunk, lim);
    for (long long kt = cb; kt < ce; kt += KT) {
      const int nk = (int)min((long long)KT, ce - kt);
      __syncthreads();
      for (int idx = tid; idx < KT * D; idx += kSimtThreads) {
        const int j = idx / D, e = idx % D;
        float kx = 0.f, vx = 0.f;
        if (j < nk) {
          const long long g = (((long long)b * a.N_kv + kt + j) * a.Hkv + hk) * D + e;
          kx = to_f<T>(K[g]);
          vx = to_f<T>(V[g]);
        }
        sK[j][e] = kx;
        sV[j][e] = vx;
      }
      __syncthreads();
      float sc[KT];
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < KT; ++j) {
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) part = fmaf(qv[i], sK[j][i * TPR + sub], part);
#pragma unroll
        for (int off = 1; off < TPR; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        const long long kpos = a.k_pos0 + kt + j;
        const bool vis = (j < nk) && (!a.causal || kpos <= pos);
        sc[j] = vis ? part * sl : -INFINITY;
        mx = fmaxf(mx, sc[j]);
      }
      const float m_new = fmaxf(m2, mx);
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m2 - base);
      l *= alpha;
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] *= alpha;
#pragma unroll
      for (int j = 0; j < KT; ++j) {
        const float pj = ex2(sc[j] - base);
        l += pj;
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = fmaf(pj, sV[j][i * TPR + sub], o[i]);
      }
      m2 = m_new;
    }
  }

  if (!valid) return;
  if (MODE == kModeFinal) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const long long ooff = (((long long)b * a.N_q + row) * a.Hq + h) * D;
    if (a.out_f32) {
      float* out = static_cast<float*>(a.out);
#pragma unroll
      for (int i = 0; i < 32; ++i) out[ooff + i * TPR + sub] = o[i] * inv;
    } else {
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
#pragma unroll
      for (int i = 0; i < 32; ++i) out[ooff + i * TPR + sub] = __float2bfloat16_rn(o[i] * inv);
    }
    if (sub == 0)
      a.lse[((long long)b * a.Hq + h) * a.N_q + row] = l > 0.f ? (m2 + log2f(l)) * kLn2 : -INFINITY;
  } else {  // kModeState
    const long long srow = ((long long)b * a.Hq + h) * a.N_q + row;
#pragma unroll
    for (int i = 0; i < 32; ++i) a.acc[srow * D + i * TPR + sub] = o[i];
    if (sub == 0) {
      a.m[srow] = (m2 == m2_in) ? m_in_nat : m2 * kLn2;
      a.l[srow] = l;
    }
  }
}

template <typename T, int D, int MODE>
cudaError_t launch_t(const ProblemArgs& a, cudaStream_t st) {
  constexpr int ROWS = kSimtThreads / (D / 32);
  dim3 grid((unsigned)((a.N_q + ROWS - 1) / ROWS), (unsigned)a.Hq, (unsigned)a.B);
  simt_attn_kernel<T, D, MODE><<<grid, kSimtThreads, 0, st>>>(a);
  return count_launch(cudaGetLastError());
}

}  // namespace

cudaError_t launch_fwd_simt_f32(const ProblemArgs& a, int mode, cudaStream_t st) {
  if (a.N_q <= 0 || a.B <= 0) return cudaSuccess;
  if (a.d == 64) {
    return mode == kModeState ? launch_t<float, 64, kModeState>(a, st) : launch_t<float, 64, kModeFinal>(a, st);
  }
  return mode == kModeState ? launch_t<float, 128, kModeState>(a, st) : launch_t<float, 128, kModeFinal>(a, st);
}

}  // namespace ra
