// Decode-shaped forward over an FP8 E4M3 KV cache on the tensor cores'
// 8-bit path: the cache codes are MMA operands exactly as they sit in memory,
// with no conversion pass.
//
// The same exact blockwise attention as fwd_sm100.cuh and decode_sm100.cuh
// ("Ring Attention: the secret of million-token context": chunks visited in
// ring order, §2.2; the flash inner loop over 128-key tiles, §3.1; one
// global normalisation at the end), over the quantised cache that "Billion-
// token context window engineering" (production parameters: 4-/8-bit KV
// quantisation) asks for in serving.  Keys sit on the MMA's M side, as in
// decode_sm100.cuh, for a block of R <= NR packed query rows:
//   S^T (128 keys x 2NR)  = K8 (128 x 128) . [Q_hi | Q_lo]^T          M = 128
//   O^T (128 ch  x 2NR)  += V8^T (128 x 128 keys) . [P_hi | P_lo]^T    M = 128
// with tcgen05.mma kind::f8f6f4 (E4M3 x E4M3 -> f32).  The 8-bit MMA needs
// both operands in E4M3, so the bf16 queries and the float probabilities are
// each written as two E4M3 planes, x = hi + lo / 16 (hi = x rounded to E4M3,
// lo = the remainder times 16 rounded to E4M3):
//   - a bf16 q has 8 significant bits; hi holds the top 4 and the remainder
//     is a multiple of q's last bit below hi's half-ulp, so lo holds it
//     exactly: after a per-row power-of-two scale that puts the row's largest
//     |q| in [224, 448], q = hi + lo / 16 exactly for every |q| >= 2^-6 of
//     that range (smaller entries are off by at most 2^-14 of it);
//   - p in [0, 2^8] (the exponent base trails the row max by at most 8)
//     is kept to 8 significant bits, as much as the bf16 P of the other
//     kernels.
// Products of two E4M3 values are exact and accumulate in float32, so the
// scores carry the full cache values; the dequantisation scales fold into
// the score scale (k_scale) and the epilogue (v_scale).
//
// Against the converter kernels this drops the per-tile decode of 32 KB of
// codes into 64 KB of bf16 (shared-memory traffic and issue slots), and the
// CTA is small enough for two per SM, whose per-tile softmax chains then
// overlap.
//
// CTA organisation (one CTA = one (batch, KV head, row block, KV split)):
//   warp 0       TMA producer: the bf16 Q block once, then K/V code tiles
//                (128 keys x 128 bytes, 128-byte swizzle) into an NSLOT ring.
//   warp 1       MMA issuer: S^T_j two tiles ahead into one of two TMEM
//                buffers; O^T += V^T_j P^T_j once the P planes are written.
//   warp 2       TMEM allocator.
//   warp 3       writes the Q planes and per-row scales once, from the bf16
//                block in shared memory.
//   warps 4-11   softmax as in decode_sm100.cuh (thread = key; column maxima
//                exchanged through shared memory under an mbarrier; running
//                base per row with a slack), then the P planes as E4M3 bytes;
//                epilogue with thread = channel.
// Every mbarrier wait is bounded; an expired wait unwinds the CTA.
#pragma once

#include <cuda_fp16.h>

#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace ra {

namespace {

// Two floats -> two E4M3 codes, round to nearest even, saturating at +-448:
// byte 0 holds x0's code, byte 1 x1's.
__device__ __forceinline__ uint32_t e4m3x2_rn(float x0, float x1) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(x1), "f"(x0));
  return d;
}

// Two E4M3 codes (byte 0, byte 1) -> their values (exact in f16).
__device__ __forceinline__ float2 e4m3x2_value(uint32_t codes) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)codes));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// x = hi + lo / 16 for a pair (x0, x1): hi, lo hold byte 0 for x0, byte 1 for x1.
__device__ __forceinline__ void split_e4m3x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = e4m3x2_rn(x0, x1);
  const float2 h = e4m3x2_value(hi);
  lo = e4m3x2_rn((x0 - h.x) * 16.f, (x1 - h.y) * 16.f);
}

// Maximum of x over the 32 lanes of the warp (one reduction instruction).
__device__ __forceinline__ float warp_max_f32(float x) {
  float m;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(x));
  return m;
}

// 4 x 4 byte transpose among the four lanes of a lane quad: lane i of the quad
// holds byte r of word x for (its key, row r); on return it holds byte k for
// (key k of the quad, row i).  Two exchanges, each followed by a byte select.
__device__ __forceinline__ uint32_t quad_byte_transpose(uint32_t x, int lane) {
  const uint32_t sel1 = (lane & 1) ? 0x3715u : 0x6240u;  // odd: y1 x1 y3 x3; even: x0 y0 x2 y2
  const uint32_t sel2 = (lane & 2) ? 0x3276u : 0x5410u;  // upper pair: y2 y3 x2 x3; lower: x0 x1 y0 y1
  uint32_t y = __shfl_xor_sync(0xFFFFFFFFu, x, 1);
  x = __byte_perm(x, y, sel1);
  y = __shfl_xor_sync(0xFFFFFFFFu, x, 2);
  return __byte_perm(x, y, sel2);
}

// Instruction descriptor, kind::f8f6f4 with E4M3 A and B and an f32
// accumulator (A / B formats 0 = E4M3); a_mn / b_mn: operand is MN-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                      // D format: f32
         | ((uint32_t)a_mn << 15)       // A major-ness
         | ((uint32_t)b_mn << 16)       // B major-ness
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// D(tmem) (+)= A(smem desc) * B(smem desc)^T, kind::f8f6f4 (K = 32 per instruction).
__device__ __forceinline__ void umma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Ring depth and CTAs per SM of the 16-row configuration.
#ifndef RA_DF8_NSLOT
#define RA_DF8_NSLOT 5
#endif
#ifndef RA_DF8_MINB
#define RA_DF8_MINB 2
#endif

template <int NR, int NSLOT>
struct DecF8Layout {
  static constexpr int kQ16Bytes = NR * kDecD * 2;  // bf16 Q block: two 64-channel halves of NR x 128 B
  static constexpr int kQ8Bytes = 2 * NR * kDecD;   // E4M3 planes: 2NR rows x 128 B
  static constexpr int kTileBytes = kTileN * kDecD;  // one code tile: 128 keys x 128 B
  static constexpr int kPBytes = 2 * NR * kTileN;    // P planes: 2NR rows x 128 keys
  static constexpr int kQ16Off = 0;
  static constexpr int kQ8Off = 1024 * ((kQ16Bytes + 1023) / 1024);
  static constexpr int kKVOff = kQ8Off + 1024 * ((kQ8Bytes + 1023) / 1024);
  static constexpr int kPOff = kKVOff + NSLOT * kTileBytes;
  // [3][NR][4 lane quarters] floats: column maxima (two tile-parity buffers),
  // then the row sums of the epilogue; then NR per-row score factors 2^-k.
  static constexpr int kRedOff = kPOff + 2 * kPBytes;
  static constexpr int kInvSigOff = kRedOff + 3 * 4 * NR * 4;
  static constexpr int kBarOff = kInvSigOff + NR * 4;
  // q, q8, kv_full[NSLOT], kv_empty[NSLOT], s[2], p[2], pv[2], red[2][2], done, sum
  static constexpr int kNumBars = 2 + 2 * NSLOT + 10 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 6 * NR <= 128 ? 128 : 256;
};

template <int NR, int NSLOT, int MODE, int MINB>
__global__ void __launch_bounds__(384, MINB) decode_f8_sm100_kernel(const __grid_constant__ DecParams p) {
  using L = DecF8Layout<NR, NSLOT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  const uint32_t BAR_Q = bar0;        // bf16 Q block landed
  const uint32_t BAR_Q8 = bar0 + 8u;  // Q planes and row scales written
  auto BAR_KV_FULL = [&](int i) { return bar0 + 8u * (2 + i); };
  auto BAR_KV_EMPTY = [&](int i) { return bar0 + 8u * (2 + NSLOT + i); };
  auto BAR_S = [&](int i) { return bar0 + 8u * (2 + 2 * NSLOT + i); };    // S^T buffer i ready
  auto BAR_P = [&](int i) { return bar0 + 8u * (4 + 2 * NSLOT + i); };    // P planes i written
  auto BAR_PV = [&](int i) { return bar0 + 8u * (6 + 2 * NSLOT + i); };   // PV reading P planes i done
  // Column maxima of buffer i written by the four warps of row-column half h.
  auto BAR_RED = [&](int i, int h) { return bar0 + 8u * (8 + 2 * NSLOT + 2 * i + h); };
  const uint32_t BAR_DONE = bar0 + 8u * (12 + 2 * NSLOT);
  const uint32_t BAR_SUM = bar0 + 8u * (13 + 2 * NSLOT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
  float* inv_sigma = reinterpret_cast<float*>(smem + L::kInvSigOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: KV heads innermost, then splits, row blocks, batch.
  long long x = blockIdx.x;
  const int hk = (int)(x % p.Hkv);
  x /= p.Hkv;
  const int sigma = (int)(x % p.S);
  x /= p.S;
  const int qblk = (int)(x % p.n_qblk);
  const int b = (int)(x / p.n_qblk);
  const int tok0 = qblk * p.tpb;
  const int ntok = (int)min((long long)p.tpb, p.N_q - tok0);
  const int nrows = ntok * p.G;
  const long long qk_delta = p.q_pos0 - p.k_pos0;
  const int pos_first = clamp_key(qk_delta + tok0);
  const int pos_last = clamp_key(qk_delta + tok0 + ntok - 1);
  int lim = (int)p.N_kv;
  if (p.causal) lim = max(0, min(lim, pos_last + 1));
  const int home = pos_first > 0 ? (int)min((long long)(p.P - 1), (long long)pos_first / p.chunk) : 0;
  const int s_begin = sigma * p.steps_per_split;
  const int s_end = min(p.P, s_begin + p.steps_per_split);

  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    mbar_init(BAR_Q8, 1);
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(BAR_KV_FULL(i), 1);
      mbar_init(BAR_KV_EMPTY(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR_S(i), 1);
      mbar_init(BAR_P(i), 8);  // one arrival per softmax warp
      mbar_init(BAR_PV(i), 1);
      mbar_init(BAR_RED(i, 0), 4);
      mbar_init(BAR_RED(i, 1), 4);
    }
    mbar_init(BAR_DONE, 1);
    mbar_init(BAR_SUM, 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S^T buffers [0, 2NR) and [2NR, 4NR), O^T [4NR, 6NR); in each,
  // the first NR columns belong to the hi plane and the next NR to the lo plane.
  auto T_S = [&](int i) { return tmem + (uint32_t)(2 * NR * i); };
  const uint32_t T_O = tmem + 4 * NR;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    if (lane == 0 && !p.skip_loads) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_k);
      prefetch_tmap(&p.tm_v);
      mbar_arrive_expect_tx(BAR_Q, L::kQ16Bytes);
      for (int hf = 0; hf < 2; ++hf)
        tma_load_4d(sbase + L::kQ16Off + hf * (NR * 128), &p.tm_q, BAR_Q, hf * 64, hk * p.G, tok0, b);
      KvCursor<false> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t issued = 0;
      bool ok = true;
      while (ok && cur.valid()) {
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const uint32_t slot = issued % NSLOT;
          if (!(ok = mbar_wait_idle(BAR_KV_EMPTY(slot), ((issued / NSLOT) & 1u) ^ 1u, abort_flag))) break;
          mbar_arrive_expect_tx(BAR_KV_FULL(slot), L::kTileBytes);
          tma_load_4d(sbase + L::kKVOff + slot * L::kTileBytes, kv == 0 ? &p.tm_k : &p.tm_v, BAR_KV_FULL(slot), 0,
                      hk, cur.k0, b);
          ++issued;
        }
        cur.next();
      }
      // Let the last fills land before the CTA can exit.
      for (uint32_t f = issued > NSLOT ? issued - NSLOT : 0; f < issued; ++f) {
        volatile int no_abort = 0;
        mbar_wait_idle(BAR_KV_FULL(f % NSLOT), (f / NSLOT) & 1u, &no_abort);
      }
      volatile int no_abort = 0;
      mbar_wait_idle(BAR_Q, 0, &no_abort);
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      bool ok = mbar_wait_idle(BAR_Q8, 0, abort_flag);
      tc_fence_after();
      const uint64_t qdesc = smem_desc_sw128(sbase + L::kQ8Off, 16, 1024);
      auto kv_addr = [&](uint32_t f) { return sbase + L::kKVOff + (f % NSLOT) * L::kTileBytes; };
      auto full = [&](uint32_t f) { return mbar_wait_idle(BAR_KV_FULL(f % NSLOT), (f / NSLOT) & 1u, abort_flag); };
      // S^T_j = K_j [Q_hi | Q_lo]^T (both K-major; a K step of 32 codes is 32
      // bytes inside the 128-byte swizzle row).
      auto issue_s = [&](uint32_t j) {
        constexpr uint32_t idesc = idesc_e4m3_f32(kTileN, 2 * NR, 0, 0);
        const uint64_t kdesc = smem_desc_sw128(kv_addr(2 * j), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kDecD / 32; ++kk)
          umma_f8_ss(T_S(j & 1), kdesc + ((kk * 32) >> 4), qdesc + ((kk * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
        tc_commit(BAR_S(j & 1));
        tc_commit(BAR_KV_EMPTY((2 * j) % NSLOT));
      };
      KvCursor<false> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t n_tiles = 0;
      for (KvCursor<false> c = cur; c.valid(); c.next()) ++n_tiles;
      for (uint32_t j = 0; j < 2 && j < n_tiles && ok; ++j) {
        if (!(ok = full(2 * j))) break;
        tc_fence_after();
        issue_s(j);
      }
      for (uint32_t j = 0; j < n_tiles && ok; ++j) {
        if (!(ok = mbar_wait_idle(BAR_P(j & 1), (j >> 1) & 1u, abort_flag))) break;
        if (!(ok = full(2 * j + 1))) break;
        tc_fence_after();
        // O^T += V^T_j [P_hi | P_lo]^T: A = the V code tile read MN-major
        // (channels contiguous; 8-key groups 1024 bytes apart, a K step of 32
        // keys = 4096 bytes), B = the P planes (K-major).
        constexpr uint32_t idesc = idesc_e4m3_f32(kDecD, 2 * NR, 1, 0);
        const uint64_t vdesc = smem_desc_sw128(kv_addr(2 * j + 1), kTileN * 128, 1024);
        const uint64_t pdesc = smem_desc_sw128(sbase + L::kPOff + (j & 1) * L::kPBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kTileN / 32; ++kk)
          umma_f8_ss(T_O, vdesc + ((kk * 4096) >> 4), pdesc + ((kk * 32) >> 4), idesc, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(BAR_PV(j & 1));
        tc_commit(BAR_KV_EMPTY((2 * j + 1) % NSLOT));
        if (j + 2 < n_tiles) {
          if (!(ok = full(2 * j + 4))) break;
          tc_fence_after();
          issue_s(j + 2);
        }
      }
      tc_commit(BAR_DONE);
      volatile int no_abort = 0;
      mbar_wait_idle(BAR_DONE, 0, &no_abort);
    }
  } else if (warp == 3) {
    // ======================= Q planes and row scales =======================
    // Row r of the bf16 block (64-channel half hf at r * 128 bytes, 16-byte
    // chunk j stored at j ^ (r mod 8)); lane l takes channels 4l .. 4l + 3.
    bool ok = mbar_wait_idle(BAR_Q, 0, abort_flag);
    if (ok) {
      const int hf = lane >> 4, jc = (lane & 15) >> 1;
      for (int r = 0; r < NR; ++r) {
        const uint8_t* src = smem + L::kQ16Off + hf * (NR * 128) + r * 128 + ((jc ^ (r & 7)) << 4) + (lane & 1) * 8;
        const uint2 raw = *reinterpret_cast<const uint2*>(src);
        const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        float amax = fmaxf(fmaxf(fabsf(q01.x), fabsf(q01.y)), fmaxf(fabsf(q23.x), fabsf(q23.y)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        // 2^k with amax * 2^k in [224, 448]: amax = m 2^e (1 <= m < 2) and
        // 448 = 1.75 * 2^8, so k = 8 - e when m <= 1.75, else 7 - e.
        int k = 0;
        if (amax > 0.f) {
          const uint32_t bits = __float_as_uint(amax);
          const int e = (int)((bits >> 23) & 0xFFu) - 127;
          k = ((bits & 0x7FFFFFu) > 0x600000u ? 7 : 8) - e;
          k = max(-126, min(126, k));
        }
        const float sig = __uint_as_float((uint32_t)(k + 127) << 23);
        uint32_t h0, l0, h1, l1;
        split_e4m3x2(q01.x * sig, q01.y * sig, h0, l0);
        split_e4m3x2(q23.x * sig, q23.y * sig, h1, l1);
        // Planes: row n at n * 128 bytes, 16-byte chunk (ch / 16) ^ (n mod 8).
        const int ch16 = lane >> 2, boff = (lane & 3) * 4;
        const int rh = r, rl = NR + r;
        *reinterpret_cast<uint32_t*>(smem + L::kQ8Off + rh * 128 + ((ch16 ^ (rh & 7)) << 4) + boff) = h0 | (h1 << 16);
        *reinterpret_cast<uint32_t*>(smem + L::kQ8Off + rl * 128 + ((ch16 ^ (rl & 7)) << 4) + boff) = l0 | (l1 << 16);
        if (lane == 0) inv_sigma[r] = __uint_as_float((uint32_t)(127 - k) << 23);
      }
      // The planes are read by the tensor cores (async proxy).
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_Q8);
    }
  } else if (warp >= 4 && warp < 12) {
    // ============================ softmax ============================
    constexpr int CH = NR / 2;                // row columns of this warp
    const int quad = warp & 3;                // TMEM lane quarter
    const int hh = (warp - 4) >> 2;           // row-column half of this warp
    const int c0 = hh * CH;                   // first row column of this warp
    const int row = quad * 32 + lane;         // key of the tile; channel d in the epilogue
    const uint32_t lb = (uint32_t)(quad * 32) << 16;
    auto last_key = [&](int c) {
      const int r = c0 + c;
      return r < nrows ? (p.causal ? pos_first + (r >> p.gshift) : 0x7FFFFFFF) : -1;
    };
    float m2[CH], lsum[CH], fac[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      m2[c] = -INFINITY;
      lsum[c] = 0.f;
    }
    bool ok = mbar_wait_idle(BAR_Q8, 0, abort_flag);
    {
      // Score in log2 units = scale * log2(e) * k_scale * 2^-k_row * (S_hi + S_lo / 16).
      const float sl = p.scale_log2 * p.k_scale[b * p.Hkv + hk];
#pragma unroll
      for (int c = 0; c < CH; ++c) fac[c] = sl * inv_sigma[c0 + c];
    }
    const bool pad_only = c0 >= nrows;  // all of this warp's row columns are padding
    KvCursor<false> cur;
    cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
    uint32_t j = 0;
    while (ok && cur.valid()) {
      const int bsel = (int)(j & 1);
      if (!(ok = mbar_wait_idle(BAR_S(bsel), (j >> 1) & 1u, abort_flag))) break;
      tc_fence_after();
      float xv[CH];
      float* rb = red + bsel * 4 * NR;
      if (!pad_only) {
        float xh[CH], xl[CH];
        tmem_ld_ch<CH>(T_S(bsel) + lb + c0, xh);
        tmem_ld_ch<CH>(T_S(bsel) + lb + NR + c0, xl);
        tc_wait_ld();
        const bool masked = (cur.kend - cur.k0 < kTileN) || (p.causal && cur.kend - 1 > pos_first);
        const int key = cur.k0 + row;
        const bool kvalid = key < cur.kend;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const float sx = fmaf(xl[c], 0.0625f, xh[c]) * fac[c];
          xv[c] = (!masked || (kvalid && key <= last_key(c))) ? sx : -INFINITY;
        }
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const float m = warp_max_f32(xv[c]);
          if (lane == 0) rb[(c0 + c) * 4 + quad] = m;
        }
      }
      __syncwarp();
      // Only the four lane quarters of the same row columns exchange maxima;
      // the wait is short and on the critical path, so it polls.
      if (lane == 0) mbar_arrive(BAR_RED(bsel, hh));
      if (!(ok = mbar_wait(BAR_RED(bsel, hh), (j >> 1) & 1u, abort_flag))) break;
      if (pad_only) {
        // Only keeps pace on the barriers: its P columns feed O^T columns that
        // are never written.
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR_P(bsel));
        ++j;
        cur.next();
        continue;
      }
      // Running base per row (log2 units), trailing its max by at most
      // kRescaleSlack; O^T and the partial sums follow it when it moves.
      bool grow = false;
      float alpha[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const float4 q4 = *reinterpret_cast<const float4*>(rb + (c0 + c) * 4);
        const float tm = fmaxf(fmaxf(q4.x, q4.y), fmaxf(q4.z, q4.w));
        alpha[c] = 1.f;
        if (tm > m2[c] + kRescaleSlack) {
          alpha[c] = ex2(m2[c] - tm);  // 0 while the row had no key
          m2[c] = tm;
          grow = true;
        }
      }
      if (grow) {
#pragma unroll
        for (int c = 0; c < CH; ++c) lsum[c] *= alpha[c];
        if (j > 0) {
          // O^T holds earlier tiles: once the last PV has landed, rescale this
          // warp's columns (both planes) of its lanes (channels).
          if (!(ok = mbar_wait_idle(BAR_PV((j - 1) & 1), ((j - 1) >> 1) & 1u, abort_flag))) break;
          tc_fence_after();
          float oh[CH], ol[CH];
          tmem_ld_ch<CH>(T_O + lb + c0, oh);
          tmem_ld_ch<CH>(T_O + lb + NR + c0, ol);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            oh[c] *= alpha[c];
            ol[c] *= alpha[c];
          }
          tmem_st_ch<CH>(T_O + lb + c0, oh);
          tmem_st_ch<CH>(T_O + lb + NR + c0, ol);
          tc_wait_st();
        }
      }
      // P planes of buffer bsel (last read by PV_{j-2}): K-major, 128-byte
      // swizzle; row n, key k at n * 128 + ((k / 16) ^ (n mod 8)) * 16 +
      // k mod 16.  A thread's codes for 4 consecutive rows form one word; a
      // byte transpose in each lane quad turns them into 4 consecutive keys
      // of one row, stored as one 32-bit word.
      uint32_t whi[CH / 4], wlo[CH / 4];
#pragma unroll
      for (int c = 0; c < CH; c += 2) {
        const float p0 = ex2(xv[c] - (m2[c] == -INFINITY ? 0.f : m2[c]));
        const float p1 = ex2(xv[c + 1] - (m2[c + 1] == -INFINITY ? 0.f : m2[c + 1]));
        lsum[c] += p0;
        lsum[c + 1] += p1;
        uint32_t hi, lo;
        split_e4m3x2(p0, p1, hi, lo);
        if ((c & 2) == 0) {
          whi[c / 4] = hi;
          wlo[c / 4] = lo;
        } else {
          whi[c / 4] |= hi << 16;
          wlo[c / 4] |= lo << 16;
        }
      }
      if (j >= 2 && !(ok = mbar_wait_idle(BAR_PV(bsel), ((j - 2) >> 1) & 1u, abort_flag))) break;
      uint8_t* pbuf = smem + L::kPOff + bsel * L::kPBytes;
      const int k4 = quad * 32 + 4 * (lane >> 2);  // first of the quad's 4 keys
#pragma unroll
      for (int h = 0; h < CH / 4; ++h) {
        const int nh = c0 + 4 * h + (lane & 3), nl = NR + nh;
        const uint32_t th = quad_byte_transpose(whi[h], lane), tl = quad_byte_transpose(wlo[h], lane);
        *reinterpret_cast<uint32_t*>(pbuf + nh * 128 + (((k4 >> 4) ^ (nh & 7)) << 4) + (k4 & 15)) = th;
        *reinterpret_cast<uint32_t*>(pbuf + nl * 128 + (((k4 >> 4) ^ (nl & 7)) << 4) + (k4 & 15)) = tl;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_P(bsel));
      ++j;
      cur.next();
    }
    // ------------------------------ epilogue ------------------------------
    if (ok) ok = mbar_wait_idle(BAR_DONE, 0, abort_flag);
    float* rs = red + 2 * 4 * NR;
    if (ok) {
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        float v = lsum[c];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if (lane == 0) rs[(c0 + c) * 4 + quad] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_SUM);
      ok = mbar_wait_idle(BAR_SUM, 0, abort_flag);
    }
    if (ok) {
      tc_fence_after();
      float oh[CH], ol[CH];
      if (j > 0) {
        tmem_ld_ch<CH>(T_O + lb + c0, oh);
        tmem_ld_ch<CH>(T_O + lb + NR + c0, ol);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < CH; ++c) oh[c] = ol[c] = 0.f;
      }
      const float v_mul = p.v_scale[b * p.Hkv + hk];
      const int dch = row;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int r = c0 + c;
        if (r >= nrows) continue;
        const float4 s4 = *reinterpret_cast<const float4*>(rs + r * 4);
        const float l = (s4.x + s4.y) + (s4.z + s4.w);
        const float inv = l > 0.f ? v_mul / l : 0.f;
        const float val = fmaf(ol[c], 0.0625f, oh[c]) * inv;
        const long long t = tok0 + (r >> p.gshift);
        const int h = hk * p.G + (r & (p.G - 1));
        const float lse_v = l > 0.f ? (m2[c] + log2f(l)) * kLn2 : -INFINITY;
        if (MODE == kModeSplit) {
          p.o_part[(((long long)(sigma * p.B + b) * p.N_q + t) * p.Hq + h) * kDecD + dch] = val;
          if (row == 0) p.lse_part[((long long)(sigma * p.B + b) * p.Hq + h) * p.N_q + t] = lse_v;
        } else {
          static_cast<__nv_bfloat16*>(p.out)[(((long long)b * p.N_q + t) * p.Hq + h) * kDecD + dch] =
              __float2bfloat16_rn(val);
          if (row == 0) p.lse[((long long)b * p.Hq + h) * p.N_q + t] = lse_v;
        }
      }
    }
  }

  // ---- tear-down: every role has finished (MMAs drained) before TMEM is freed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, L::kTmemCols);
}

template <int NR, int NSLOT, int MODE, int MINB>
cudaError_t launch_df8_cfg(const DecParams& prm, long long grid, cudaStream_t st) {
  using L = DecF8Layout<NR, NSLOT>;
  // At most 227 KB per CTA; MINB CTAs (each with 1 KB reserved) in the
  // SM's 228 KB.
  static_assert(L::kAlloc <= 232448 && MINB * (L::kAlloc + 1024) <= 233472, "shared memory budget exceeded");
  auto kern = decode_f8_sm100_kernel<NR, NSLOT, MODE, MINB>;
  static unsigned long long attr_set_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_set_mask, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&attr_set_mask, bit, __ATOMIC_RELEASE);
  }
  kern<<<(unsigned)grid, 384, L::kAlloc, st>>>(prm);
  return count_launch(cudaGetLastError());
}

}  // namespace

// The FP8-cache decode on the 8-bit MMA path: same parameters and routing
// as the keys-on-M kernel, for NR = 16 or 32 packed rows.
cudaError_t launch_decode_f8_sm100(const DecParams& prm, int NR, int mode, long long grid, cudaStream_t st) {
  if (NR == 16)
    return mode == kModeSplit ? launch_df8_cfg<16, RA_DF8_NSLOT, kModeSplit, RA_DF8_MINB>(prm, grid, st)
                              : launch_df8_cfg<16, RA_DF8_NSLOT, kModeFinal, RA_DF8_MINB>(prm, grid, st);
  // 32 rows: 16 row columns per softmax warp need more than the 80 registers
  // of two CTAs per SM, so one CTA with a deeper ring.
  return mode == kModeSplit ? launch_df8_cfg<32, 6, kModeSplit, 1>(prm, grid, st)
                            : launch_df8_cfg<32, 6, kModeFinal, 1>(prm, grid, st);
}

}  // namespace ra
