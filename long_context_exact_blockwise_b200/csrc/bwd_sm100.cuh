// Backward pass of exact attention on B200 tensor cores (bf16 inputs and
// gradients, float32 accumulation).
//
// The pages define the forward only; the backward is its gradient:
//   D_t   = dout_t . out_t
//   p_tj  = exp(scale q_t . k_j - lse_t)         (visible pairs, else 0)
//   ds_tj = p_tj (dout_t . v_j - D_t)
//   dv_j  = sum_t p_tj dout_t,   dk_j = scale sum_t ds_tj q_t,
//   dq_t  = scale sum_j ds_tj k_j
// summed over the query heads of a GQA group for dk, dv.
//
// Three kernels:
//   bwd_prep_kernel : D and lse * log2(e) per query row, written to a
//                     workspace whose rows are padded to 128 (padding holds
//                     lse = +inf, so padded queries get p = 0, and D = 0).
//   bwd_dkdv_kernel : one CTA per (batch, KV head, 128-key tile); loops over
//                     the group's query heads and query tiles; S^T = K Q^T
//                     and dP^T = V dout^T into TMEM, elementwise P^T, dS^T
//                     (bf16, written back over S^T / dP^T), then
//                     dV += P^T dout and dK += dS^T Q accumulate in TMEM.
//   bwd_dq_kernel   : one CTA per (batch, query head, 128-query tile); loops
//                     over KV tiles; S = Q K^T, dP = dout V^T, dS, then
//                     dQ += dS K in TMEM.
// Warp roles in both: warp 0 TMA, warp 1 MMA issue (one thread), warp 2
// TMEM allocation, warps 4.. the elementwise warps.  An elementwise thread
// owns one TMEM lane (tile row) and one column group.  dK/dV runs two warps
// per lane quarter, one per half of the tile's 128 columns, so two warps per
// SM sub-partition overlap their exponential chains; dQ runs one warp per
// quarter over all 128 columns.  Every mbarrier wait is bounded as in the
// forward.
#pragma once

#include <cstdlib>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace ra {

namespace {

constexpr int kBT = 128;  // tile rows (queries or keys)

// Elementwise warps of each kernel: 4 (one per TMEM lane quarter) or 8 (two
// per quarter, one per column half).
#ifndef RA_BWD_EW_DKDV
#define RA_BWD_EW_DKDV 8
#endif
#ifndef RA_BWD_EW_DQ
#define RA_BWD_EW_DQ 4
#endif

template <int EW>
struct EwSplit {
  static_assert(EW == 4 || EW == 8, "elementwise warps: one or two per TMEM lane quarter");
  static constexpr int kNH = EW / 4;        // column groups per tile row
  static constexpr int kCW = kBT / kNH;     // columns per group
  static constexpr int kThreads = 128 + 32 * EW;
  // A column group g writes its bf16 pairs (16 columns per 32 values) over
  // the start of its own fp32 columns [g kCW, (g+1) kCW), so no group
  // overwrites values another has yet to read.  TMEM column of the packed
  // operand's 16 contraction elements kk (as A of an MMA from TMEM):
  static __device__ __forceinline__ constexpr uint32_t packed_col(int kk) {
    return (uint32_t)((kk / (kCW / 16)) * kCW + (kk % (kCW / 16)) * 8);
  }
};
constexpr int kEwDkdv = RA_BWD_EW_DKDV, kEwDq = RA_BWD_EW_DQ;

// 1-D bulk copy global -> shared, completion on an mbarrier (16-byte aligned
// addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  const float* lse2;  // [B, Hq, Npad]: lse * log2(e), +inf on padding
  const float* dD;    // [B, Hq, Npad]: dout . out, 0 on padding
  void* dq;
  void* dk;
  void* dv;
  int B, Hq, Hkv, G;
  long long N_q, N_kv, Npad;
  long long q_pos0, k_pos0;  // global positions of q row 0 and k row 0
  int causal;
  int accumulate;  // 0: write dq, dk, dv as bf16; 1: add into float32 dq, dk, dv
  float scale;
  float scale_log2;
  int n_qt, n_kt;  // query / key tiles
};

// Smem descriptors of a 128-row x D tile staged by TMA (boxes of 64
// elements, 128-byte swizzle).  As a K-major operand (contraction over d):
// SBO 1024 between 8-row groups; as an MN-major operand (N = d, K = rows):
// LBO = one 64-element block (128 rows x 128 bytes) apart, SBO 1024.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) { return smem_desc_sw128(addr, 16, 1024); }
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t addr) { return smem_desc_sw128(addr, kBT * 128, 1024); }

// D(tmem, M=128 x N=128) = A(128 x D) B(128 x D)^T, both K-major tiles.
template <int D>
__device__ __forceinline__ void mma_rows_x_rows(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBT, kBT, 0);
  const uint64_t ad = kmajor_desc(a_addr), bd = kmajor_desc(b_addr);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * (kBT * 128) + (kk % 4) * 32;
    umma_ss(d_tmem, ad + (off >> 4), bd + (off >> 4), idesc, kk > 0 ? 1u : 0u);
  }
}

// D(tmem, M=128 x N=D) (+)= A(tmem, bf16 128 x 128 packed by column group)
// B(128 rows x D, MN-major).
template <int D, int EW>
__device__ __forceinline__ void mma_tmem_x_tile(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_addr, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBT, D, 1);
  const uint64_t bd = mnmajor_desc(b_addr);
#pragma unroll
  for (int kk = 0; kk < kBT / 16; ++kk)
    umma_ts(d_tmem, a_tmem + EwSplit<EW>::packed_col(kk), bd + ((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// D(tmem, M=128 x N=D) (+)= A(smem, 128 x 128, K-major in two 64-column
// blocks) B(128 rows x D, MN-major).
template <int D>
__device__ __forceinline__ void mma_rows_x_rows_mn(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBT, D, 1);
  const uint64_t ad = kmajor_desc(a_addr), bd = mnmajor_desc(b_addr);
#pragma unroll
  for (int kk = 0; kk < kBT / 16; ++kk) {
    const uint32_t aoff = (kk / 4) * (kBT * 128) + (kk % 4) * 32;
    umma_ss(d_tmem, ad + (aoff >> 4), bd + ((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar, int D, int head, int row,
                                         int b) {
  for (int hf = 0; hf < D / 64; ++hf) tma_load_4d(dst + hf * (kBT * 128), map, bar, hf * 64, head, row, b);
}

// ---------------------------------------------------------------- prep
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ out,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse, float* lse2, float* dD, int B,
                                                       int Hq, long long N_q, long long Npad) {
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);  // row of [B, Hq, Npad]
  if (r >= (long long)B * Hq * Npad) return;
  const long long t = r % Npad;
  const int h = (int)((r / Npad) % Hq);
  const int b = (int)(r / (Npad * Hq));
  float acc = 0.f;
  if (t < N_q) {
    const long long off = (((long long)b * N_q + t) * Hq + h) * D;
#pragma unroll
    for (int e = lane; e < D; e += 32) acc += __bfloat162float(out[off + e]) * __bfloat162float(dout[off + e]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    dD[r] = t < N_q ? acc : 0.f;
    lse2[r] = t < N_q ? lse[((long long)b * Hq + h) * N_q + t] * kLog2e : INFINITY;
  }
}

// ---------------------------------------------------------------- dK, dV
template <int D>
struct DkdvLayout {
  static constexpr int kTile = kBT * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kStage0 = kV + kTile;  // per stage: Q, dout, lse2[128], D[128]
  static constexpr int kStageBytes = 2 * kTile + 2 * kBT * 4;
  // P^T as bf16, the A operand of dV += P^T dout: 128 key rows x 128 query
  // columns, K-major, two 64-column blocks with the 128-byte swizzle.
  static constexpr int kP = kStage0 + 2 * kStageBytes;
  static constexpr int kBars = kP + kBT * kBT * 2;  // kv_full, qf[2], qe[2], s, p, done, drain, dp, ds, sfree, pfree
  static constexpr int kMisc = kBars + 13 * 8;
  static constexpr int kBytes = kMisc + 16;
  // The tiles need 1024-byte alignment.  At D = 128 the layout leaves room
  // for 896 bytes of padding only, so the kernel requires a dynamic
  // shared-memory base aligned to 128 bytes (it checks, and reports
  // RA_ERR_UNSUPPORTED otherwise).  More than half the SM's shared memory:
  // one CTA per SM, so the 512-column TMEM allocation never waits.
  static constexpr int kSlack = 1024 - 128;
  static constexpr int kAlloc = kBytes + kSlack < 120 * 1024 ? 120 * 1024 : kBytes + kSlack;
};

template <int D>
__global__ void __launch_bounds__(EwSplit<kEwDkdv>::kThreads, 1) bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using L = DkdvLayout<D>;
  constexpr int kEw = kEwDkdv, kNH = EwSplit<kEw>::kNH, kCW = EwSplit<kEw>::kCW;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 127u) {  // see DkdvLayout::kSlack
    if (threadIdx.x == 0) atomicExch(&g_status, (int)RA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBars;
  const uint32_t BAR_KV = bar0;
  auto BAR_QF = [&](int s) { return bar0 + 8u * (1 + s); };
  auto BAR_QE = [&](int s) { return bar0 + 8u * (3 + s); };
  const uint32_t BAR_S = bar0 + 8u * 5, BAR_P = bar0 + 8u * 6, BAR_DONE = bar0 + 8u * 7, BAR_DRAIN = bar0 + 8u * 8;
  const uint32_t BAR_DP = bar0 + 8u * 9, BAR_DS = bar0 + 8u * 10, BAR_SFREE = bar0 + 8u * 11;
  const uint32_t BAR_PFREE = bar0 + 8u * 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  auto stage_q = [&](int s) { return sbase + L::kStage0 + s * L::kStageBytes; };
  auto stage_do = [&](int s) { return stage_q(s) + L::kTile; };
  auto stage_lse = [&](int s) {
    return reinterpret_cast<const float*>(smem + L::kStage0 + s * L::kStageBytes + 2 * L::kTile);
  };
  auto stage_d = [&](int s) { return stage_lse(s) + kBT; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Head-major order, key tiles ascending inside a head: the CTAs resident
  // at one time share one KV head's Q / dout stream in L2 (an order across
  // heads measured 15x the DRAM traffic), and under a causal mask a key
  // tile's work falls with its index, so each head's longest CTAs go first.
  const int jt = (int)(blockIdx.x % p.n_kt);
  const int hk = (int)((blockIdx.x / p.n_kt) % p.Hkv);
  const int b = (int)(blockIdx.x / ((long long)p.n_kt * p.Hkv));
  const int j0 = jt * kBT;
  // First query tile with a query that sees key j0 (causal), else 0.
  int it0 = 0;
  if (p.causal) {
    const long long tmin = (long long)j0 + (p.k_pos0 - p.q_pos0);
    it0 = tmin <= 0 ? 0 : (int)min((long long)p.n_qt, tmin / kBT);
  }
  const int n_it = p.n_qt - it0;
  const int n_work = n_it * p.G;  // (head, query tile) iterations

  if (threadIdx.x == 0) {
    mbar_init(BAR_KV, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR_QF(s), 1);
      mbar_init(BAR_QE(s), 1 + kEw);  // MMA commit + one arrival per elementwise warp
    }
    mbar_init(BAR_S, 1);
    mbar_init(BAR_P, kEw);
    mbar_init(BAR_DONE, 1);
    mbar_init(BAR_DRAIN, 1);
    mbar_init(BAR_DP, 1);
    mbar_init(BAR_DS, kEw);
    mbar_init(BAR_SFREE, kEw);
    mbar_init(BAR_PFREE, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S^T [0,128), dP^T [128,256), dV [256, 256+D), dK [256+D, 256+2D)
  const uint32_t T_ST = tmem, T_DPT = tmem + 128, T_DV = tmem + 256, T_DK = tmem + 256 + D;

  auto work = [&](int w, int& head, int& qt) {
    head = hk * p.G + w / n_it;
    qt = it0 + w % n_it;
  };

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_k);
      prefetch_tmap(&p.tm_v);
      prefetch_tmap(&p.tm_do);
      mbar_arrive_expect_tx(BAR_KV, 2 * L::kTile);
      tma_tile(sbase + L::kK, &p.tm_k, BAR_KV, D, hk, j0, b);
      tma_tile(sbase + L::kV, &p.tm_v, BAR_KV, D, hk, j0, b);
      for (int w = 0; w < n_work; ++w) {
        const int s = w & 1;
        if (!mbar_wait(BAR_QE(s), ((w >> 1) & 1) ^ 1, abort_flag)) break;
        int head, qt;
        work(w, head, qt);
        mbar_arrive_expect_tx(BAR_QF(s), 2 * L::kTile + 2 * kBT * 4);
        tma_tile(stage_q(s), &p.tm_q, BAR_QF(s), D, head, qt * kBT, b);
        tma_tile(stage_do(s), &p.tm_do, BAR_QF(s), D, head, qt * kBT, b);
        const long long roff = ((long long)b * p.Hq + head) * p.Npad + (long long)qt * kBT;
        bulk_load(smem_u32(stage_lse(s)), p.lse2 + roff, kBT * 4, BAR_QF(s));
        bulk_load(smem_u32(stage_d(s)), p.dD + roff, kBT * 4, BAR_QF(s));
      }
      // Let in-flight copies land before the CTA can exit.
      volatile int no_abort = 0;
      mbar_wait(BAR_KV, 0, &no_abort);
      for (int w = n_work > 2 ? n_work - 2 : 0; w < n_work; ++w) mbar_wait(BAR_QF(w & 1), (w >> 1) & 1, &no_abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // Software pipeline over iterations w (one query tile of one head):
      //   S^T_{w+1}, dV_w += P^T_w dout_w  |  dK_w += dS^T_w Q_w  |  dP^T_{w+1}
      // P^T goes to shared memory, so S^T_{w+1} may overwrite S^T_w as soon
      // as the elementwise warps hold S^T_w in registers (SFREE): the tensor
      // pipe computes the next scores while they form P^T_w.  dP^T_{w+1}
      // overwrites the columns dK_w reads dS^T_w from: tcgen05 MMAs of one
      // thread run in issue order.  Each S / dP commit comes after the
      // elementwise warps have passed the previous wait on the same barrier,
      // so no barrier runs two phases ahead of its waiters.
      bool ok = mbar_wait(BAR_KV, 0, abort_flag);
      tc_fence_after();
      if (ok && n_work > 0 && (ok = mbar_wait(BAR_QF(0), 0, abort_flag))) {
        tc_fence_after();
        mma_rows_x_rows<D>(T_ST, sbase + L::kK, stage_q(0));    // S^T = K Q^T
        tc_commit(BAR_S);
        mma_rows_x_rows<D>(T_DPT, sbase + L::kV, stage_do(0));  // dP^T = V dout^T
        tc_commit(BAR_DP);
      }
      for (int w = 0; w < n_work && ok; ++w) {
        const int s = w & 1;
        const bool more = w + 1 < n_work;
        // S^T_{w+1} (once the warps hold S^T_w and Q_{w+1} has landed) and
        // dV_w (once P^T_w is written) go out in the order their inputs
        // arrive, S^T first when both are ready: a late Q tile must not hold
        // up dV_w, whose completion frees the P^T buffer.
        if (more && !(ok = mbar_wait(BAR_SFREE, w & 1, abort_flag))) break;
        bool s_todo = more, v_todo = true;
        const uint32_t qpar = ((w + 1) >> 1) & 1;
        const unsigned long long t0 = globaltimer_ns();
        for (uint32_t i = 1; s_todo || v_todo; ++i) {
          if (s_todo && mbar_test(BAR_QF(s ^ 1), qpar)) {
            tc_fence_after();
            mma_rows_x_rows<D>(T_ST, sbase + L::kK, stage_q(s ^ 1));  // S^T_{w+1}
            tc_commit(BAR_S);
            s_todo = false;
          } else if (v_todo && mbar_test(BAR_P, w & 1)) {
            tc_fence_after();
            mma_rows_x_rows_mn<D>(T_DV, sbase + L::kP, stage_do(s), w > 0);  // dV += P^T dout
            tc_commit(BAR_PFREE);
            v_todo = false;
          } else if ((i & 255u) == 0u) {
            if (*abort_flag) {
              ok = false;
              break;
            }
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
              *abort_flag = 1;
              atomicExch(&g_status, (int)RA_ERR_DEVICE_TIMEOUT);
              ok = false;
              break;
            }
          }
        }
        if (!ok) break;
        if (!(ok = mbar_wait(BAR_DS, w & 1, abort_flag))) break;
        tc_fence_after();
        mma_tmem_x_tile<D, kEw>(T_DK, T_DPT, stage_q(s), w > 0);   // dK += dS^T Q
        tc_commit(BAR_QE(s));
        if (more) {
          mma_rows_x_rows<D>(T_DPT, sbase + L::kV, stage_do(s ^ 1));
          tc_commit(BAR_DP);
        }
      }
      tc_commit(BAR_DONE);
      tc_commit(BAR_DRAIN);
      volatile int no_abort = 0;
      mbar_wait(BAR_DRAIN, 0, &no_abort);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int grp = (warp - 4) >> 2;  // query columns [grp kCW, (grp+1) kCW)
    const int g0 = grp * kCW;
    const int r = quad * 32 + lane;  // key row of the tile
    const uint32_t lq = (uint32_t)(quad * 32) << 16;
    const uint32_t lb = lq + (uint32_t)g0;
    const long long key = (long long)j0 + r;
    const float sl = p.scale_log2;
    // This thread's row of the P^T buffer (K-major, 128-byte swizzle).
    uint8_t* prow = smem + L::kP + r * 128;
    bool ok = true;
    for (int w = 0; w < n_work; ++w) {
      const int s = w & 1;
      int head, qt;
      work(w, head, qt);
      if (!(ok = mbar_wait(BAR_S, w & 1, abort_flag))) break;
      // The stage's lse / D came in by bulk copy: wait on its own barrier
      // (already complete) so the loads below observe the copied data.
      if (!(ok = mbar_wait(BAR_QF(s), (w >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const float* lse2 = stage_lse(s) + g0;
      const float* dD = stage_d(s) + g0;
      // Causal: query column c is visible to this key iff
      // q_pos0 + qt*128 + c >= k_pos0 + key, i.e. c >= cmin.
      long long cm = p.causal ? (key + p.k_pos0 - p.q_pos0) - (long long)qt * kBT : -1;
      const int cmin = (int)(cm < 0 ? 0 : (cm > kBT ? kBT : cm));
      // Phase 1: P^T (kept in registers for phase 2), bf16 to shared memory.
      // The first 32 columns' exponentials overlap the load of the rest.
      float pv[kCW];
      tmem_ld32(T_ST + lb, *reinterpret_cast<float(*)[32]>(pv));
      tc_wait_ld();
#pragma unroll
      for (int c = 1; c < kCW / 32; ++c) tmem_ld32(T_ST + lb + c * 32, *reinterpret_cast<float(*)[32]>(pv + c * 32));
      // Only warps on the causal diagonal mask columns; the others skip the
      // selects (a warp-uniform choice, so no lanes diverge).
      const bool diag = __any_sync(0xffffffffu, cmin > g0);
      auto exps = [&](auto lo_c, auto hi_c, auto masked) {
#pragma unroll
        for (int l = decltype(lo_c)::value * 32; l < decltype(hi_c)::value * 32; ++l) {
          float e = ex2(fmaf(pv[l], sl, -lse2[l]));
          if constexpr (decltype(masked)::value) {
            if (g0 + l < cmin) e = 0.f;
          }
          pv[l] = e;
        }
      };
      using C0 = std::integral_constant<int, 0>;
      using C1 = std::integral_constant<int, 1>;
      using CN = std::integral_constant<int, kCW / 32>;
      if (diag)
        exps(C0{}, C1{}, std::true_type{});
      else
        exps(C0{}, C1{}, std::false_type{});
      tc_wait_ld();
      // S^T_w is in registers: the next tile's scores may overwrite it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_SFREE);
      if (diag)
        exps(C1{}, CN{}, std::true_type{});
      else
        exps(C1{}, CN{}, std::false_type{});
      // dV_{w-1} must have read the buffer before it is overwritten.
      if (w > 0 && !(ok = mbar_wait(BAR_PFREE, (w - 1) & 1, abort_flag))) break;
#pragma unroll
      for (int c = 0; c < kCW / 8; ++c) {
        // 8 query columns = one 16-byte chunk of the row's 64-column block.
        const int q8 = (g0 + c * 8) >> 3;
        *reinterpret_cast<uint4*>(prow + (q8 >> 3) * (kBT * 128) + (((q8 & 7) ^ (r & 7)) << 4)) =
            make_uint4(pack_bf16x2(pv[c * 8], pv[c * 8 + 1]), pack_bf16x2(pv[c * 8 + 2], pv[c * 8 + 3]),
                       pack_bf16x2(pv[c * 8 + 4], pv[c * 8 + 5]), pack_bf16x2(pv[c * 8 + 6], pv[c * 8 + 7]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_P);
      // Phase 2: dS^T = P^T (dP^T - D), bf16 over dP^T.
      if (!(ok = mbar_wait(BAR_DP, w & 1, abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kCW / 32; ++c) {
        float dpt[32];
        tmem_ld32(T_DPT + lb + c * 32, dpt);
        tc_wait_ld();
        uint32_t uds[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int l0 = c * 32 + i;
          uds[i / 2] = pack_bf16x2(pv[l0] * (dpt[i] - dD[l0]), pv[l0 + 1] * (dpt[i + 1] - dD[l0 + 1]));
        }
        tmem_st16(T_DPT + lb + c * 16, uds);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(BAR_DS);
        mbar_arrive(BAR_QE(s));  // this warp is done with the stage's lse / D
      }
    }
    if (ok) ok = mbar_wait(BAR_DONE, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const bool valid = key < p.N_kv;
      const long long off = (((long long)b * p.N_kv + (valid ? key : 0)) * p.Hkv + hk) * D;
      const int e0 = grp * (D / kNH);  // this warp's dV / dK columns
      if (p.accumulate) {
        // dv += P^T dout, dk += scale dS^T Q into the caller's float32 rows
        // (a key no query of this call sees is left as it was).
        float* dv = static_cast<float*>(p.dv) + off + e0;
        float* dk = static_cast<float*>(p.dk) + off + e0;
#pragma unroll
        for (int c = 0; c < D / 32 / kNH; ++c) {
          float a[32], g[32];
          tmem_ld32(T_DV + lq + e0 + c * 32, a);
          tmem_ld32(T_DK + lq + e0 + c * 32, g);
          tc_wait_ld();
          if (!valid || n_work == 0) continue;
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 ov = *reinterpret_cast<float4*>(dv + c * 32 + i);
            float4 ok4 = *reinterpret_cast<float4*>(dk + c * 32 + i);
            ov.x += a[i]; ov.y += a[i + 1]; ov.z += a[i + 2]; ov.w += a[i + 3];
            ok4.x = fmaf(g[i], p.scale, ok4.x);
            ok4.y = fmaf(g[i + 1], p.scale, ok4.y);
            ok4.z = fmaf(g[i + 2], p.scale, ok4.z);
            ok4.w = fmaf(g[i + 3], p.scale, ok4.w);
            *reinterpret_cast<float4*>(dv + c * 32 + i) = ov;
            *reinterpret_cast<float4*>(dk + c * 32 + i) = ok4;
          }
        }
      } else {
        __nv_bfloat16* dv = static_cast<__nv_bfloat16*>(p.dv) + off + e0;
        __nv_bfloat16* dk = static_cast<__nv_bfloat16*>(p.dk) + off + e0;
#pragma unroll
        for (int c = 0; c < D / 32 / kNH; ++c) {
          float a[32], g[32];
          tmem_ld32(T_DV + lq + e0 + c * 32, a);
          tmem_ld32(T_DK + lq + e0 + c * 32, g);
          tc_wait_ld();
          if (!valid) continue;
          // A key no query sees gets a zero gradient (TMEM was never written).
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            a[i] = n_work > 0 ? a[i] : 0.f;
            g[i] = n_work > 0 ? g[i] * p.scale : 0.f;
          }
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 wv, wk;
            wv.x = pack_bf16x2(a[i], a[i + 1]);
            wv.y = pack_bf16x2(a[i + 2], a[i + 3]);
            wv.z = pack_bf16x2(a[i + 4], a[i + 5]);
            wv.w = pack_bf16x2(a[i + 6], a[i + 7]);
            wk.x = pack_bf16x2(g[i], g[i + 1]);
            wk.y = pack_bf16x2(g[i + 2], g[i + 3]);
            wk.z = pack_bf16x2(g[i + 4], g[i + 5]);
            wk.w = pack_bf16x2(g[i + 6], g[i + 7]);
            *reinterpret_cast<uint4*>(dv + c * 32 + i) = wv;
            *reinterpret_cast<uint4*>(dk + c * 32 + i) = wk;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- dQ
template <int D>
struct DqLayout {
  // K_j is read by S_j and, last, by dQ_j; V_j only by dP_j.  Three K slots
  // let K_{j+1} load while dQ_{j-1} still holds its slot (two stages put a
  // whole load latency in front of S_{j+1}); V needs two.
  static constexpr int kKSlots = 3, kVSlots = 2;
  static constexpr int kTile = kBT * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kDo = kQ + kTile;
  static constexpr int kK0 = kDo + kTile;
  static constexpr int kV0 = kK0 + kKSlots * kTile;
  // q_full, kf[3], ke[3], vf[2], ve[2], s[2], ds, done, drain, dp
  static constexpr int kBars = kV0 + kVSlots * kTile;
  static constexpr int kMisc = kBars + 17 * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024 < 120 * 1024 ? 120 * 1024 : kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(EwSplit<kEwDq>::kThreads, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using L = DqLayout<D>;
  constexpr int kEw = kEwDq, kNH = EwSplit<kEw>::kNH, kCW = EwSplit<kEw>::kCW;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBars;
  const uint32_t BAR_Q = bar0;
  auto BAR_KF = [&](int i) { return bar0 + 8u * (1 + i); };
  auto BAR_KE = [&](int i) { return bar0 + 8u * (4 + i); };
  auto BAR_VF = [&](int i) { return bar0 + 8u * (7 + i); };
  auto BAR_VE = [&](int i) { return bar0 + 8u * (9 + i); };
  auto BAR_S = [&](int s) { return bar0 + 8u * (11 + s); };
  const uint32_t BAR_DS = bar0 + 8u * 13, BAR_DONE = bar0 + 8u * 14, BAR_DRAIN = bar0 + 8u * 15, BAR_DP = bar0 + 8u * 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  constexpr int KS = L::kKSlots, VS = L::kVSlots;
  auto slot_k = [&](int j) { return sbase + L::kK0 + (j % KS) * L::kTile; };  // K_j
  auto slot_v = [&](int j) { return sbase + L::kV0 + (j % VS) * L::kTile; };  // V_j

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Head-major order (the resident CTAs share one KV head's K / V in L2),
  // query tiles from the last inside a head: under a causal mask a query
  // tile's work grows with its index, so each head's longest CTAs go first.
  const int qt = p.n_qt - 1 - (int)(blockIdx.x % p.n_qt);
  const int h = (int)((blockIdx.x / p.n_qt) % p.Hq);
  const int b = (int)(blockIdx.x / ((long long)p.n_qt * p.Hq));
  const int hk = h / p.G;
  const int t0 = qt * kBT;
  // Key tiles with a key some query of this tile sees.
  int n_jt = p.n_kt;
  if (p.causal) {
    const long long last_q = min((long long)t0 + kBT, p.N_q) - 1;
    const long long kmax = last_q + (p.q_pos0 - p.k_pos0);  // last visible key row
    n_jt = kmax < 0 ? 0 : (int)min((long long)p.n_kt, kmax / kBT + 1);
  }

  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(BAR_KF(i), 1);
      mbar_init(BAR_KE(i), 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(BAR_VF(i), 1);
      mbar_init(BAR_VE(i), 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(BAR_S(s), 1);
    mbar_init(BAR_DS, kEw);
    mbar_init(BAR_DONE, 1);
    mbar_init(BAR_DRAIN, 1);
    mbar_init(BAR_DP, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S (two buffers) [0,128) and [128,256), dP [256,384), dQ [384, 384+D)
  auto T_S = [&](int s) { return tmem + 128u * s; };
  const uint32_t T_DP = tmem + 256, T_DQ = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_k);
      prefetch_tmap(&p.tm_v);
      prefetch_tmap(&p.tm_do);
      mbar_arrive_expect_tx(BAR_Q, 2 * L::kTile);
      tma_tile(sbase + L::kQ, &p.tm_q, BAR_Q, D, h, t0, b);
      tma_tile(sbase + L::kDo, &p.tm_do, BAR_Q, D, h, t0, b);
      for (int j = 0; j < n_jt; ++j) {
        if (!mbar_wait(BAR_KE(j % KS), ((j / KS) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(BAR_KF(j % KS), L::kTile);
        tma_tile(slot_k(j), &p.tm_k, BAR_KF(j % KS), D, hk, j * kBT, b);
        if (!mbar_wait(BAR_VE(j % VS), ((j / VS) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(BAR_VF(j % VS), L::kTile);
        tma_tile(slot_v(j), &p.tm_v, BAR_VF(j % VS), D, hk, j * kBT, b);
      }
      // Let in-flight copies land before the CTA can exit.
      volatile int no_abort = 0;
      mbar_wait(BAR_Q, 0, &no_abort);
      for (int j = n_jt > KS ? n_jt - KS : 0; j < n_jt; ++j) mbar_wait(BAR_KF(j % KS), (j / KS) & 1, &no_abort);
      for (int j = n_jt > VS ? n_jt - VS : 0; j < n_jt; ++j) mbar_wait(BAR_VF(j % VS), (j / VS) & 1, &no_abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // Software pipeline over key tiles j, S double-buffered in TMEM:
      //   S_{j+1}  |  dQ += dS_j K_j  |  dP_{j+1}
      // so S_{j+1} (and the elementwise warps' exponentials for it) overlap
      // dS_j.  S_{j+1} goes to the buffer dQ_{j-1} read dS_{j-1} from, and
      // dP_{j+1} over dP_j, which the warps finished with at dS_j: tcgen05
      // MMAs of one thread run in issue order.  Each S buffer has its own
      // barrier, and S_{j+2} is committed only after dS_j, so neither runs
      // two phases ahead of the elementwise warps.
      bool ok = mbar_wait(BAR_Q, 0, abort_flag);
      tc_fence_after();
      auto issue_dp = [&](int j) {  // dP_j = dout V_j^T, then V_j's slot is free
        mma_rows_x_rows<D>(T_DP, sbase + L::kDo, slot_v(j));
        tc_commit(BAR_DP);
        tc_commit(BAR_VE(j % VS));
      };
      if (ok && n_jt > 0 && (ok = mbar_wait(BAR_KF(0), 0, abort_flag))) {
        tc_fence_after();
        mma_rows_x_rows<D>(T_S(0), sbase + L::kQ, slot_k(0));   // S = Q K^T
        tc_commit(BAR_S(0));
        if ((ok = mbar_wait(BAR_VF(0), 0, abort_flag))) {
          tc_fence_after();
          issue_dp(0);
        }
      }
      for (int j = 0; j < n_jt && ok; ++j) {
        const int s = j & 1;
        const bool more = j + 1 < n_jt;
        if (more) {
          if (!(ok = mbar_wait(BAR_KF((j + 1) % KS), ((j + 1) / KS) & 1, abort_flag))) break;
          tc_fence_after();
          mma_rows_x_rows<D>(T_S(s ^ 1), sbase + L::kQ, slot_k(j + 1));
          tc_commit(BAR_S(s ^ 1));
        }
        if (!(ok = mbar_wait(BAR_DS, j & 1, abort_flag))) break;
        tc_fence_after();
        mma_tmem_x_tile<D, kEw>(T_DQ, T_S(s), slot_k(j), j > 0);    // dQ += dS K
        tc_commit(BAR_KE(j % KS));
        if (more) {
          if (!(ok = mbar_wait(BAR_VF((j + 1) % VS), ((j + 1) / VS) & 1, abort_flag))) break;
          tc_fence_after();
          issue_dp(j + 1);
        }
      }
      tc_commit(BAR_DONE);
      tc_commit(BAR_DRAIN);
      volatile int no_abort = 0;
      mbar_wait(BAR_DRAIN, 0, &no_abort);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int grp = (warp - 4) >> 2;  // key columns [grp kCW, (grp+1) kCW)
    const int g0 = grp * kCW;
    const int r = quad * 32 + lane;  // query row of the tile
    const uint32_t lq = (uint32_t)(quad * 32) << 16;
    const uint32_t lb = lq + (uint32_t)g0;
    const long long t = (long long)t0 + r;
    const bool valid = t < p.N_q;
    const long long srow = ((long long)b * p.Hq + h) * p.Npad + t;
    const float lse2 = p.lse2[srow];  // +inf on padded rows: p = 0
    const float Dt = p.dD[srow];
    const float sl = p.scale_log2;
    // Last key row this query sees (causal), relative to the k buffer.
    const long long klast_abs = p.causal ? t + (p.q_pos0 - p.k_pos0) : p.N_kv - 1;
    bool ok = true;
    for (int j = 0; j < n_jt; ++j) {
      const int s = j & 1;
      if (!(ok = mbar_wait(BAR_S(s), (j >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      // Last visible column of this group (relative to g0): -1 = none.
      const long long kl = min(klast_abs, p.N_kv - 1) - (long long)j * kBT - g0;
      const int klast = (int)(kl < -1 ? -1 : (kl > kCW ? kCW : kl));
      // P first (while dP may still be in the tensor pipe), then dS over S.
      float pv[kCW];
#pragma unroll
      for (int c = 0; c < kCW / 32; ++c) tmem_ld32(T_S(s) + lb + c * 32, *reinterpret_cast<float(*)[32]>(pv + c * 32));
      tc_wait_ld();
      // Warps whose rows see every key of their columns skip the selects.
      if (__all_sync(0xffffffffu, klast >= kCW - 1)) {
#pragma unroll
        for (int i = 0; i < kCW; ++i) pv[i] = ex2(fmaf(pv[i], sl, -lse2));
      } else {
#pragma unroll
        for (int i = 0; i < kCW; ++i) {
          const float pe = ex2(fmaf(pv[i], sl, -lse2));
          pv[i] = i > klast ? 0.f : pe;
        }
      }
      if (!(ok = mbar_wait(BAR_DP, j & 1, abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kCW / 32; ++c) {
        float dp[32];
        tmem_ld32(T_DP + lb + c * 32, dp);
        tc_wait_ld();
        uint32_t uds[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int k0 = c * 32 + i;
          uds[i / 2] = pack_bf16x2(pv[k0] * (dp[i] - Dt), pv[k0 + 1] * (dp[i + 1] - Dt));
        }
        tmem_st16(T_S(s) + lb + c * 16, uds);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR_DS);
    }
    if (ok) ok = mbar_wait(BAR_DONE, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const long long off = (((long long)b * p.N_q + (valid ? t : 0)) * p.Hq + h) * D;
      const int e0 = grp * (D / kNH);  // this warp's dQ columns
      if (p.accumulate) {
        // dq += scale dS K into the caller's float32 row (unchanged when no
        // key of this call is visible to the tile).
        float* dq = static_cast<float*>(p.dq) + off + e0;
#pragma unroll
        for (int c = 0; c < D / 32 / kNH; ++c) {
          float a[32];
          tmem_ld32(T_DQ + lq + e0 + c * 32, a);
          tc_wait_ld();
          if (!valid || n_jt == 0) continue;
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 o = *reinterpret_cast<float4*>(dq + c * 32 + i);
            o.x = fmaf(a[i], p.scale, o.x);
            o.y = fmaf(a[i + 1], p.scale, o.y);
            o.z = fmaf(a[i + 2], p.scale, o.z);
            o.w = fmaf(a[i + 3], p.scale, o.w);
            *reinterpret_cast<float4*>(dq + c * 32 + i) = o;
          }
        }
      } else {
        __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(p.dq) + off + e0;
#pragma unroll
        for (int c = 0; c < D / 32 / kNH; ++c) {
          float a[32];
          tmem_ld32(T_DQ + lq + e0 + c * 32, a);
          tc_wait_ld();
          if (!valid) continue;
          // A query that sees no key gets a zero gradient (TMEM never written).
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = n_jt > 0 ? a[i] * p.scale : 0.f;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w;
            w.x = pack_bf16x2(a[i], a[i + 1]);
            w.y = pack_bf16x2(a[i + 2], a[i + 3]);
            w.z = pack_bf16x2(a[i + 4], a[i + 5]);
            w.w = pack_bf16x2(a[i + 6], a[i + 7]);
            *reinterpret_cast<uint4*>(dq + c * 32 + i) = w;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

CUresult encode_bwd_map(CUtensorMap* m, const void* base, int d, int H, long long N, int B) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return CUDA_ERROR_NOT_FOUND;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)N * H * d * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Sets the dynamic shared-memory limit of `kern` once per device.  TAG
// distinguishes kernels of the same type (each gets its own cache).
template <int TAG, typename K>
cudaError_t set_smem_attr(K kern, int bytes) {
  static unsigned long long mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&mask, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&mask, bit, __ATOMIC_RELEASE);
  }
  return cudaSuccess;
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs& a, cudaStream_t st) {
  static_assert(DkdvLayout<D>::kAlloc <= 232448 && DqLayout<D>::kAlloc <= 232448, "shared memory budget exceeded");
  BwdParams prm;
  memset(&prm, 0, sizeof(prm));
  if (encode_bwd_map(&prm.tm_q, a.q, D, a.Hq, a.N_q, a.B) != CUDA_SUCCESS ||
      encode_bwd_map(&prm.tm_do, a.dout, D, a.Hq, a.N_q, a.B) != CUDA_SUCCESS ||
      encode_bwd_map(&prm.tm_k, a.k, D, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS ||
      encode_bwd_map(&prm.tm_v, a.v, D, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  prm.lse2 = a.ws_lse2;
  prm.dD = a.ws_d;
  prm.dq = a.dq;
  prm.dk = a.dk;
  prm.dv = a.dv;
  prm.B = a.B;
  prm.Hq = a.Hq;
  prm.Hkv = a.Hkv;
  prm.G = a.Hq / a.Hkv;
  prm.N_q = a.N_q;
  prm.N_kv = a.N_kv;
  prm.Npad = a.Npad;
  prm.q_pos0 = a.q_pos0;
  prm.k_pos0 = a.k_pos0;
  prm.causal = a.causal;
  prm.accumulate = a.accumulate;
  prm.scale = a.scale;
  prm.scale_log2 = a.scale * kLog2e;
  prm.n_qt = (int)((a.N_q + kBT - 1) / kBT);
  prm.n_kt = (int)((a.N_kv + kBT - 1) / kBT);

  const long long rows = (long long)a.B * a.Hq * a.Npad;
  bwd_prep_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(a.out), static_cast<const __nv_bfloat16*>(a.dout), a.lse, a.ws_lse2, a.ws_d,
      a.B, a.Hq, a.N_q, a.Npad);
  cudaError_t e = count_launch(cudaGetLastError());
  if (e != cudaSuccess) return e;
  if ((e = set_smem_attr<2 * D + 0>(bwd_dkdv_kernel<D>, DkdvLayout<D>::kAlloc)) != cudaSuccess) return e;
  if ((e = set_smem_attr<2 * D + 1>(bwd_dq_kernel<D>, DqLayout<D>::kAlloc)) != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<(unsigned)((long long)prm.n_kt * a.Hkv * a.B), EwSplit<kEwDkdv>::kThreads, DkdvLayout<D>::kAlloc, st>>>(prm);
  if ((e = count_launch(cudaGetLastError())) != cudaSuccess) return e;
  bwd_dq_kernel<D><<<(unsigned)((long long)prm.n_qt * a.Hq * a.B), EwSplit<kEwDq>::kThreads, DqLayout<D>::kAlloc, st>>>(prm);
  return count_launch(cudaGetLastError());
}

}  // namespace

cudaError_t launch_bwd_sm100(const BwdArgs& a, cudaStream_t st) {
  if (a.B <= 0 || a.N_q <= 0) return cudaSuccess;
  return a.d == 64 ? launch_bwd_d<64>(a, st) : launch_bwd_d<128>(a, st);
}

}  // namespace ra
