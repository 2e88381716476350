// Decode-shaped forward (few query rows against a long KV cache) on B200
// tensor cores, with keys on the MMA's M side.
//
// The same exact blockwise attention as fwd_sm100.cuh ("Ring Attention: the
// secret of million-token context": chunks visited in ring order, §2.2;
// the flash inner loop over 128-key tiles, §3.1; global normalisation at the
// end), for an incremental-query block of R <= NR packed rows (the G query
// heads of one KV head times the new tokens).  With 128 query rows per MMA
// most of the tensor work on such a block multiplies padding; here the roles
// of queries and keys swap:
//   S^T (128 keys x NR rows)  = K (128 x d) . Q^T            M = 128, N = NR
//   O^T (d x NR rows)        += V^T (d x 128 keys) . P^T     M = d,   N = NR
// so a KV tile costs 2 * 128 * NR * d multiply-adds instead of 2 * 128^2 * d.
//
// CTA organisation (one CTA = one (batch, KV head, row block, KV split)):
//   warp 0       TMA producer: the Q block once, then K/V tiles into an
//                NSLOT-deep ring (K_j -> fill 2j, V_j -> fill 2j + 1); with an
//                FP8 cache the raw codes go to an FP8 ring instead.
//   warp 1       MMA issuer: S^T_j into one of two TMEM buffers (two tiles
//                ahead), O^T += V^T_j P^T_j once P^T_j is in shared memory.
//   warp 2       TMEM allocator.
//   warps 4-11   softmax: thread = key of the tile (TMEM lane); warp w takes
//                lane quarter w mod 4 and half of the NR row columns, so two
//                warps per SM sub-partition hide each other's latency.  Per
//                tile: the column maxima over the 128 keys (warp reductions,
//                then the four lane quarters through shared memory), the
//                running base per row (rescaling O^T in TMEM when it moves
//                past a slack), P^T as bf16 into shared memory, per-thread
//                partial row sums.  Epilogue: thread = channel d of O^T.
//   warps 12-15  (FP8 cache) converters, as in fwd_sm100.cuh.
// Every mbarrier wait is bounded; the warpgroup's exchange of column maxima
// also goes through an mbarrier, so an expired wait anywhere unwinds the CTA.
#pragma once

#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace ra {

namespace {

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(taddr));
}

// 32 lanes x 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&r)[8]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&r)[8]) {
  const uint32_t* u = reinterpret_cast<const uint32_t*>(r);
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(u[0]),
               "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
               : "memory");
}

// CH = 8 or 16 columns of this thread's lane.
template <int CH>
__device__ __forceinline__ void tmem_ld_ch(uint32_t taddr, float (&r)[CH]) {
  static_assert(CH == 8 || CH == 16, "8 or 16 columns per warp");
  if constexpr (CH == 8)
    tmem_ld8(taddr, r);
  else
    tmem_ld16(taddr, r);
}
template <int CH>
__device__ __forceinline__ void tmem_st_ch(uint32_t taddr, const float (&r)[CH]) {
  if constexpr (CH == 8)
    tmem_st8(taddr, r);
  else
    tmem_st16(taddr, *reinterpret_cast<const uint32_t(*)[16]>(r));
}

// Floats as signed integers with the same order (non-NaN), for the warp's
// integer max reduction; the map is its own inverse.
__device__ __forceinline__ int f2ord(float f) {
  const int u = __float_as_int(f);
  return u >= 0 ? u : u ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float ord2f(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7FFFFFFF); }

// Instruction descriptor, kind::f16, bf16 A and B, f32 D, A MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_amn(int M, int N) {
  return idesc_bf16_f32(M, N, 0) | (1u << 15);
}

constexpr int kDecD = 128;  // channels (the decode kernel serves d = 128)
// Work order: KV heads innermost (1, measured faster on the bf16 cache) or
// splits innermost (0).
#ifndef RA_DEC_HEADS_INNER
#define RA_DEC_HEADS_INNER 1
#endif
// Warps whose row columns are all padding skip their arithmetic (1, measured
// faster: they leave issue slots to the others) or not (0).
#ifndef RA_DEC_IDLE_PAD
#define RA_DEC_IDLE_PAD 1
#endif
// Column maxima by shuffle trees (1, measured faster) or integer warp
// reductions (0).
#ifndef RA_DEC_SHFL_MAX
#define RA_DEC_SHFL_MAX 1
#endif
// CTAs per SM the decode kernel is compiled for.
#ifndef RA_DEC_MINB
#define RA_DEC_MINB 1
#endif
// Ring depth of the 16-row bf16 configuration.
#ifndef RA_DEC_NSLOT
#define RA_DEC_NSLOT 6
#endif
// Ring depths of the 16-row FP8 configuration (bf16 slots, FP8 slots).
#ifndef RA_DEC8_NSLOT
#define RA_DEC8_NSLOT 5
#endif
#ifndef RA_DEC8_NSLOT8
#define RA_DEC8_NSLOT8 3
#endif

template <int NR, int NSLOT, int NSLOT8>
struct DecLayout {
  static constexpr int kQBytes = NR * kDecD * 2;      // Q block: two 64-channel halves of NR x 128 B
  static constexpr int kTileBytes = kTileN * kDecD * 2;
  static constexpr int kF8Bytes = kTileN * kDecD;
  static constexpr int kPBytes = NR * kTileN * 2;     // P^T: two 64-key halves of NR x 128 B
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 1024 * ((kQBytes + 1023) / 1024);
  static constexpr int kPOff = kKVOff + NSLOT * kTileBytes;
  static constexpr int kF8Off = kPOff + 2 * kPBytes;
  // [3][NR][4 lane quarters] floats: column maxima (two tile-parity
  // buffers), then the row sums of the epilogue.
  static constexpr int kRedOff = kF8Off + NSLOT8 * kF8Bytes;
  static constexpr int kBarOff = kRedOff + 3 * 4 * NR * 4;
  // q, kv_full[NSLOT], kv_empty[NSLOT], s[2], p[2], pv[2], red[2], done, sum,
  // f8_full[NSLOT8], f8_empty[NSLOT8]
  static constexpr int kNumBars = 1 + 2 * NSLOT + 8 + 2 + 2 * NSLOT8;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 3 * NR <= 32 ? 32 : (3 * NR <= 64 ? 64 : 128);
};

struct DecParams {
  CUtensorMap tm_q;  // box {64, G, NR / G, 1}: rows = token-major, head within the group
  CUtensorMap tm_k;  // bf16 (box {64, 1, 128, 1}, 128-byte swizzle) or FP8 codes (box {128, 1, 128, 1})
  CUtensorMap tm_v;
  void* out;         // kModeFinal: [B, N_q, Hq, d] bf16
  float* lse;        // kModeFinal: [B, Hq, N_q]
  float* o_part;     // kModeSplit: [S, B, N_q, Hq, d]
  float* lse_part;   // kModeSplit: [S, B, Hq, N_q]
  const float* k_scale;  // FP8 cache: [B, Hkv]
  const float* v_scale;
  int B, Hq, Hkv, G;
  long long N_q, N_kv;
  long long q_pos0, k_pos0;
  int causal;
  float scale_log2;
  long long chunk;
  int P, S, steps_per_split, n_qblk;
  int tpb;         // tokens per row block: NR / G
  int gshift;      // log2(G)
  int skip_loads;  // failure-detection test: no copies are issued
};

template <int NR, int NSLOT, int MODE, int NSLOT8>
__global__ void __launch_bounds__(NSLOT8 > 0 ? 512 : 384, RA_DEC_MINB) decode_sm100_kernel(const __grid_constant__ DecParams p) {
  using L = DecLayout<NR, NSLOT, NSLOT8>;
  constexpr bool kKV8 = NSLOT8 > 0;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  const uint32_t BAR_Q = bar0;
  auto BAR_KV_FULL = [&](int i) { return bar0 + 8u * (1 + i); };
  auto BAR_KV_EMPTY = [&](int i) { return bar0 + 8u * (1 + NSLOT + i); };
  auto BAR_S = [&](int i) { return bar0 + 8u * (1 + 2 * NSLOT + i); };    // S^T buffer i ready
  auto BAR_P = [&](int i) { return bar0 + 8u * (3 + 2 * NSLOT + i); };    // P^T buffer i written
  auto BAR_PV = [&](int i) { return bar0 + 8u * (5 + 2 * NSLOT + i); };   // PV reading P^T buffer i done
  auto BAR_RED = [&](int i) { return bar0 + 8u * (7 + 2 * NSLOT + i); };  // column maxima buffer i written
  const uint32_t BAR_DONE = bar0 + 8u * (9 + 2 * NSLOT);
  const uint32_t BAR_SUM = bar0 + 8u * (10 + 2 * NSLOT);
  auto BAR_F8_FULL = [&](int i) { return bar0 + 8u * (11 + 2 * NSLOT + i); };
  auto BAR_F8_EMPTY = [&](int i) { return bar0 + 8u * (11 + 2 * NSLOT + NSLOT8 + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item.
#if RA_DEC_HEADS_INNER
  // KV heads innermost: the CTAs of one (batch, split, row block) run side by
  // side and read neighbouring slices of the same token rows.
  long long x = blockIdx.x;
  const int hk = (int)(x % p.Hkv);
  x /= p.Hkv;
  const int sigma = (int)(x % p.S);
  x /= p.S;
  const int qblk = (int)(x % p.n_qblk);
  const int b = (int)(x / p.n_qblk);
#else
  // Splits innermost, then row blocks, KV heads, batch.
  long long x = blockIdx.x;
  const int sigma = (int)(x % p.S);
  x /= p.S;
  const int qblk = (int)(x % p.n_qblk);
  x /= p.n_qblk;
  const int hk = (int)(x % p.Hkv);
  const int b = (int)(x / p.Hkv);
#endif
  const int tok0 = qblk * p.tpb;
  const int ntok = (int)min((long long)p.tpb, p.N_q - tok0);
  const int nrows = ntok * p.G;
  const long long qk_delta = p.q_pos0 - p.k_pos0;
  const int pos_first = clamp_key(qk_delta + tok0);              // key row of the first token's position
  const int pos_last = clamp_key(qk_delta + tok0 + ntok - 1);
  int lim = (int)p.N_kv;
  if (p.causal) lim = max(0, min(lim, pos_last + 1));
  const int home = pos_first > 0 ? (int)min((long long)(p.P - 1), (long long)pos_first / p.chunk) : 0;
  const int s_begin = sigma * p.steps_per_split;
  const int s_end = min(p.P, s_begin + p.steps_per_split);

  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(BAR_KV_FULL(i), kKV8 ? 4 : 1);
      mbar_init(BAR_KV_EMPTY(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR_S(i), 1);
      mbar_init(BAR_P(i), 8);    // one arrival per softmax warp
      mbar_init(BAR_PV(i), 1);
      mbar_init(BAR_RED(i), 8);
    }
    mbar_init(BAR_DONE, 1);
    mbar_init(BAR_SUM, 8);
    for (int i = 0; i < NSLOT8; ++i) {
      mbar_init(BAR_F8_FULL(i), 1);
      mbar_init(BAR_F8_EMPTY(i), 4);
    }
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
  // TMEM columns: S^T buffers [0, NR) and [NR, 2 NR), O^T [2 NR, 3 NR).
  auto T_S = [&](int i) { return tmem + (uint32_t)(NR * i); };
  const uint32_t T_O = tmem + 2 * NR;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    if (lane == 0 && !p.skip_loads) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_k);
      prefetch_tmap(&p.tm_v);
      mbar_arrive_expect_tx(BAR_Q, L::kQBytes);
      for (int hf = 0; hf < 2; ++hf)
        tma_load_4d(sbase + L::kQOff + hf * (NR * 128), &p.tm_q, BAR_Q, hf * 64, hk * p.G, tok0, b);
      KvCursor<false> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t issued = 0;
      bool ok = true;
      while (ok && cur.valid()) {
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const CUtensorMap* map = kv == 0 ? &p.tm_k : &p.tm_v;
          if constexpr (kKV8) {
            const uint32_t slot8 = issued % NSLOT8;
            if (!(ok = mbar_wait_idle(BAR_F8_EMPTY(slot8), ((issued / NSLOT8) & 1u) ^ 1u, abort_flag))) break;
            mbar_arrive_expect_tx(BAR_F8_FULL(slot8), L::kF8Bytes);
            tma_load_4d(sbase + L::kF8Off + slot8 * L::kF8Bytes, map, BAR_F8_FULL(slot8), 0, hk, cur.k0, b);
          } else {
            const uint32_t slot = issued % NSLOT;
            if (!(ok = mbar_wait_idle(BAR_KV_EMPTY(slot), ((issued / NSLOT) & 1u) ^ 1u, abort_flag))) break;
            mbar_arrive_expect_tx(BAR_KV_FULL(slot), L::kTileBytes);
            for (int hf = 0; hf < 2; ++hf)
              tma_load_4d(sbase + L::kKVOff + slot * L::kTileBytes + hf * (kTileN * 128), map, BAR_KV_FULL(slot),
                          hf * 64, hk, cur.k0, b);
          }
          ++issued;
        }
        cur.next();
      }
      // Let the last fills land before the CTA can exit.
      constexpr uint32_t kRing = kKV8 ? NSLOT8 : NSLOT;
      for (uint32_t f = issued > kRing ? issued - kRing : 0; f < issued; ++f) {
        volatile int no_abort = 0;
        if constexpr (kKV8)
          mbar_wait_idle(BAR_F8_FULL(f % NSLOT8), (f / NSLOT8) & 1u, &no_abort);
        else
          mbar_wait_idle(BAR_KV_FULL(f % NSLOT), (f / NSLOT) & 1u, &no_abort);
      }
      volatile int no_abort = 0;
      mbar_wait_idle(BAR_Q, 0, &no_abort);
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      bool ok = mbar_wait_idle(BAR_Q, 0, abort_flag);
      tc_fence_after();
      const uint64_t qdesc = smem_desc_sw128(sbase + L::kQOff, 16, 1024);
      auto kv_addr = [&](uint32_t f) { return sbase + L::kKVOff + (f % NSLOT) * L::kTileBytes; };
      auto full = [&](uint32_t f) { return mbar_wait_idle(BAR_KV_FULL(f % NSLOT), (f / NSLOT) & 1u, abort_flag); };
      // S^T_j = K_j Q^T into buffer j & 1 (K-major A = K tile, K-major B = Q block).
      auto issue_s = [&](uint32_t j) {
        constexpr uint32_t idesc = idesc_bf16_f32(kTileN, NR, 0);
        const uint64_t kdesc = smem_desc_sw128(kv_addr(2 * j), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kDecD / 16; ++kk) {
          const uint32_t ka = (kk / 4) * (kTileN * 128) + (kk % 4) * 32;
          const uint32_t qa = (kk / 4) * (NR * 128) + (kk % 4) * 32;
          umma_ss(T_S(j & 1), kdesc + (ka >> 4), qdesc + (qa >> 4), idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(BAR_S(j & 1));
        tc_commit(BAR_KV_EMPTY((2 * j) % NSLOT));
      };
      KvCursor<false> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      // Count the tiles (the cursor is cheap to walk).
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
        // O^T += V^T_j P^T_j: A = V tile as MN-major (d contiguous), B = P^T (K-major).
        constexpr uint32_t idesc = idesc_bf16_f32_amn(kDecD, NR);
        const uint64_t vdesc = smem_desc_sw128(kv_addr(2 * j + 1), kTileN * 128, 1024);
        const uint64_t pdesc = smem_desc_sw128(sbase + L::kPOff + (j & 1) * L::kPBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk) {
          const uint32_t pa = (kk / 4) * (NR * 128) + (kk % 4) * 32;
          umma_ss(T_O, vdesc + ((kk * 2048) >> 4), pdesc + (pa >> 4), idesc, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(BAR_PV(j & 1));
        tc_commit(BAR_KV_EMPTY((2 * j + 1) % NSLOT));
        // S^T_{j+2} into the buffer S^T_j used (the softmax finished reading it
        // before publishing P^T_j).
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
  } else if (warp >= 4 && warp < 12) {
    // ============================ softmax ============================
    constexpr int CH = NR / 2;                // row columns of this warp
    const int quad = warp & 3;                // TMEM lane quarter
    const int c0 = ((warp - 4) >> 2) * CH;    // first row column of this warp
    const int row = quad * 32 + lane;         // key of the tile; channel d in the epilogue
    const uint32_t lb = (uint32_t)(quad * 32) << 16;
    const float k_mul = kKV8 ? p.k_scale[b * p.Hkv + hk] * kFp8Bias : 1.f;
    const float sl = p.scale_log2 * k_mul;    // score -> log2 units
    // Last key row packed row c0 + c sees: pos_first + ((c0 + c) >> gshift)
    // under the causal mask (-1 for padding rows).
    auto last_key = [&](int c) {
      const int r = c0 + c;
      return r < nrows ? (p.causal ? pos_first + (r >> p.gshift) : 0x7FFFFFFF) : -1;
    };
    float m2[CH], lsum[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      m2[c] = -INFINITY;
      lsum[c] = 0.f;
    }
    KvCursor<false> cur;
    cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
    uint32_t j = 0;
    bool ok = true;
    while (cur.valid()) {
      const int bsel = (int)(j & 1);
      if (!(ok = mbar_wait_idle(BAR_S(bsel), (j >> 1) & 1u, abort_flag))) break;
      tc_fence_after();
      float x[CH];
#if RA_DEC_IDLE_PAD
      // A warp whose row columns are all padding only keeps pace on the
      // barriers (its P^T columns feed O^T columns that are never written).
      const bool pad_only = c0 >= nrows;
#else
      const bool pad_only = false;
#endif
      if (!pad_only) {
      tmem_ld_ch<CH>(T_S(bsel) + lb + c0, x);
      tc_wait_ld();
      // Masking only where some key is past a row's position or beyond the
      // chunk's end.  Padding rows need none: their Q rows are zero-filled
      // and their P^T columns only feed O^T columns that are never written.
      const bool masked = (cur.kend - cur.k0 < kTileN) || (p.causal && cur.kend - 1 > pos_first);
      if (masked) {
        const int key = cur.k0 + row;
        const bool kvalid = key < cur.kend;
#pragma unroll
        for (int c = 0; c < CH; ++c) x[c] = (kvalid && key <= last_key(c)) ? x[c] * sl : -INFINITY;
      } else {
#pragma unroll
        for (int c = 0; c < CH; ++c) x[c] *= sl;
      }
      }
      // Column maxima over the tile's 128 keys: each warp, then the four lane
      // quarters ([column][quarter] in shared memory).
      float* rb = red + bsel * 4 * NR;
      if (!pad_only) {
#if RA_DEC_SHFL_MAX
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        float m = x[c];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) rb[(c0 + c) * 4 + quad] = m;
      }
#else
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int m = __reduce_max_sync(0xFFFFFFFFu, f2ord(x[c]));
        if (lane == 0) rb[(c0 + c) * 4 + quad] = ord2f(m);
      }
#endif
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_RED(bsel));
      if (!(ok = mbar_wait_idle(BAR_RED(bsel), (j >> 1) & 1u, abort_flag))) break;
      if (pad_only) {
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR_P(bsel));
        ++j;
        cur.next();
        continue;
      }
      // The base of each row's exponentials trails its running max by at most
      // kRescaleSlack; O^T and the partial sums follow a base that moves.
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
          // warp's columns of its lanes (channels) in place.
          if (!(ok = mbar_wait_idle(BAR_PV((j - 1) & 1), ((j - 1) >> 1) & 1u, abort_flag))) break;
          tc_fence_after();
          float o[CH];
          tmem_ld_ch<CH>(T_O + lb + c0, o);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < CH; ++c) o[c] *= alpha[c];
          tmem_st_ch<CH>(T_O + lb + c0, o);
          tc_wait_st();
        }
      }
      // P^T as bf16 into buffer bsel (last read by PV_{j-2}), 128-byte
      // swizzled K-major: query row r, key `row` at row r * 128 bytes of the
      // key's 64-key half, 16-byte chunk (key / 8) ^ (r mod 8).
      if (j >= 2 && !(ok = mbar_wait_idle(BAR_PV(bsel), ((j - 2) >> 1) & 1u, abort_flag))) break;
      uint8_t* half = smem + L::kPOff + bsel * L::kPBytes + (row >> 6) * (NR * 128);
      const int kh = row & 63;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int r = c0 + c;
        const float pe = ex2(x[c] - (m2[c] == -INFINITY ? 0.f : m2[c]));
        lsum[c] += pe;
        *reinterpret_cast<__nv_bfloat16*>(half + r * 128 + (((kh >> 3) ^ (r & 7)) << 4) + (kh & 7) * 2) =
            __float2bfloat16_rn(pe);
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
      float o[CH];
      if (j > 0) {
        tmem_ld_ch<CH>(T_O + lb + c0, o);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < CH; ++c) o[c] = 0.f;
      }
      const float v_mul = kKV8 ? p.v_scale[b * p.Hkv + hk] : 1.f;
      const int dch = row;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int r = c0 + c;
        if (r >= nrows) continue;
        const float4 s4 = *reinterpret_cast<const float4*>(rs + r * 4);
        const float l = (s4.x + s4.y) + (s4.z + s4.w);
        const float inv = l > 0.f ? v_mul / l : 0.f;
        const float val = (kKV8 ? o[c] * kFp8Bias : o[c]) * inv;
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
  } else if (kKV8 && warp >= 12) {
    // ============================ FP8 converters ============================
    if constexpr (kKV8) {
      const int ct = (int)threadIdx.x - 384;
      KvCursor<false> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t f = 0;
      bool ok = true;
      while (ok && cur.valid()) {
        for (int kv = 0; kv < 2; ++kv) {
          const uint32_t slot8 = f % NSLOT8, slot = f % NSLOT;
          if (!(ok = mbar_wait_idle(BAR_F8_FULL(slot8), (f / NSLOT8) & 1u, abort_flag))) break;
          if (!(ok = mbar_wait_idle(BAR_KV_EMPTY(slot), ((f / NSLOT) & 1u) ^ 1u, abort_flag))) break;
          convert_fp8_tile<kDecD>(smem + L::kF8Off + slot8 * L::kF8Bytes, smem + L::kKVOff + slot * L::kTileBytes,
                                  ct);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(BAR_KV_FULL(slot));
            mbar_arrive(BAR_F8_EMPTY(slot8));
          }
          ++f;
        }
        cur.next();
      }
    }
  }

  // ---- tear-down: every role has finished (MMAs drained) before TMEM is freed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, L::kTmemCols);
}

template <int NR, int NSLOT, int MODE, int NSLOT8>
cudaError_t launch_dec_cfg(const DecParams& prm, long long grid, cudaStream_t st) {
  using L = DecLayout<NR, NSLOT, NSLOT8>;
  static_assert(L::kAlloc <= 232448, "shared memory budget exceeded");
  auto kern = decode_sm100_kernel<NR, NSLOT, MODE, NSLOT8>;
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
  kern<<<(unsigned)grid, NSLOT8 > 0 ? 512 : 384, L::kAlloc, st>>>(prm);
  return count_launch(cudaGetLastError());
}

// bf16 [B, N, H, d] map whose box is 64 channels x box_heads heads x box_rows tokens.
CUresult encode_map_box(CUtensorMap* m, const void* base, int d, int H, long long N, int B, int box_heads,
                        int box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return CUDA_ERROR_NOT_FOUND;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)N * H * d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace

// The FP8-cache decode on the 8-bit MMA path (decode_f8_sm100.cuh).
cudaError_t launch_decode_f8_sm100(const DecParams& prm, int NR, int mode, long long grid, cudaStream_t st);

// FP8 caches go to the 8-bit MMA kernel (1) or to the converter variant of
// this kernel (0).
#ifndef RA_DEC8_NATIVE
#define RA_DEC8_NATIVE 1
#endif

// Rows per KV head of an incremental-query block (G heads x N_q tokens) that
// the keys-on-M decode kernels take: 16 or 32 (0: they do not apply).
int decode_rows(const ProblemArgs& a, int mode) {
  if (mode == kModeState || a.d != kDecD || a.wa_period > 0 || a.q_pos0 <= 0) return 0;
  // RINGATTN_DECODE: "0" never; "all" up to 32 rows in one block; default up
  // to 16 rows for a bf16 cache (at 32 rows the general kernel measured
  // faster).  An FP8 cache takes up to 32 rows by default, as 16-row blocks
  // (two CTAs per SM; the row blocks of one KV head share its tiles in L2).
  const char* ov = std::getenv("RINGATTN_DECODE");
  if (ov && ov[0] == '0') return 0;
  const bool all = ov && std::strcmp(ov, "all") == 0;
  const long long G = a.Hq / a.Hkv;
  const long long rows = G * a.N_q;
  const bool f8_blocks = a.kv8 && RA_DEC8_NATIVE && !all && rows <= 32;
  const int nr = (rows <= 16 || f8_blocks) ? 16 : (rows <= 32 && all ? 32 : 0);
  if (nr == 0 || G > nr || nr % G != 0) return 0;
  return nr;
}

cudaError_t launch_decode_sm100(const ProblemArgs& a, int mode, cudaStream_t st) {
  const int NR = decode_rows(a, mode);
  if (NR == 0) return cudaErrorInvalidValue;
  DecParams prm;
  memset(&prm, 0, sizeof(prm));
  const int G = a.Hq / a.Hkv;
  if (encode_map_box(&prm.tm_q, a.q, a.d, a.Hq, a.N_q, a.B, G, NR / G) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (a.kv8) {
    if (encode_map_u8(&prm.tm_k, a.k, a.d, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS ||
        encode_map_u8(&prm.tm_v, a.v, a.d, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else if (encode_map(&prm.tm_k, a.k, a.d, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS ||
             encode_map(&prm.tm_v, a.v, a.d, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS) {
    return cudaErrorInvalidValue;
  }
  prm.out = a.out;
  prm.lse = a.lse;
  prm.o_part = a.o_part;
  prm.lse_part = a.lse_part;
  prm.k_scale = a.k_scale;
  prm.v_scale = a.v_scale;
  prm.B = a.B;
  prm.Hq = a.Hq;
  prm.Hkv = a.Hkv;
  prm.G = G;
  prm.N_q = a.N_q;
  prm.N_kv = a.N_kv;
  prm.q_pos0 = a.q_pos0;
  prm.k_pos0 = a.k_pos0;
  prm.causal = a.causal;
  prm.scale_log2 = a.scale * kLog2e;
  prm.chunk = a.chunk;
  prm.P = a.P;
  prm.S = mode == kModeSplit ? a.S : 1;
  prm.steps_per_split = (a.P + prm.S - 1) / prm.S;
  prm.tpb = NR / G;
  prm.gshift = 0;
  while ((1 << prm.gshift) < G) ++prm.gshift;
  prm.n_qblk = (int)((a.N_q + prm.tpb - 1) / prm.tpb);
  {
    const char* f = std::getenv("RINGATTN_FAULT");
    prm.skip_loads = (f && std::strcmp(f, "device_wait") == 0) ? 1 : 0;
  }
  const long long grid = (long long)a.B * a.Hkv * prm.n_qblk * prm.S;
  if (a.kv8 && RA_DEC8_NATIVE) return launch_decode_f8_sm100(prm, NR, mode, grid, st);
  if (a.kv8) {
    if (NR == 16)
      return mode == kModeSplit ? launch_dec_cfg<16, RA_DEC8_NSLOT, kModeSplit, RA_DEC8_NSLOT8>(prm, grid, st)
                                : launch_dec_cfg<16, RA_DEC8_NSLOT, kModeFinal, RA_DEC8_NSLOT8>(prm, grid, st);
    return mode == kModeSplit ? launch_dec_cfg<32, 4, kModeSplit, 4>(prm, grid, st)
                              : launch_dec_cfg<32, 4, kModeFinal, 4>(prm, grid, st);
  }
  if (NR == 16) return mode == kModeSplit ? launch_dec_cfg<16, RA_DEC_NSLOT, kModeSplit, 0>(prm, grid, st)
                                          : launch_dec_cfg<16, RA_DEC_NSLOT, kModeFinal, 0>(prm, grid, st);
  return mode == kModeSplit ? launch_dec_cfg<32, 6, kModeSplit, 0>(prm, grid, st)
                            : launch_dec_cfg<32, 6, kModeFinal, 0>(prm, grid, st);
}

}  // namespace ra
