// Blockwise (ring) attention forward for long query blocks on pairs of SMs:
// tcgen05 MMAs with cta_group::2, bf16 inputs, float32 logits and
// accumulators, d = 128.
//
// What it computes is the same as fwd_sm100.cuh ("Ring Attention: the secret
// of million-token context": chunks visited in ring order, §2.2; the flash
// inner loop over 128-key tiles, §3.1; the next KV tile fetched while the
// current one is computed, §3.2; one global normalisation at the end).  How:
//
// A cluster of two CTAs (a CTA pair on two SMs) owns 512 query rows of one
// head: two pair tiles of 256 rows, each split as 128 rows per CTA.  One
// thread of the even CTA (the leader) issues every MMA for both:
//   S_t  = Q_t K_j^T   M = 256 (each CTA's 128 rows of Q), N = 128 keys
//   O_t += P_t V_j     M = 256 (each CTA's 128 rows of P),  N = 128 channels
// With cta_group::2 each CTA holds half of every B operand: keys
// [64 r, 64 r + 64) of each K tile and channels [64 r, 64 r + 64) of each V
// tile (r = the CTA's rank in the pair), so per SM the MMAs read half of B
// from shared memory and the K/V ring takes half the space.  The space goes
// to one P buffer per pair tile: the softmax writes P (bf16) to shared
// memory instead of over S in TMEM, so S_t(j + 1) is issued as soon as the
// softmax has S_t(j) in registers and the next tile's scores are ready when
// its softmax ends.  The softmax and the PV / S MMAs are no longer one chain
// per tile.
//
// CTA organisation (both CTAs of the pair):
//   warp 0       TMA producer: this CTA's two Q tiles once, then its halves of
//                K_j and V_j into two rings; completion is counted on the
//                leader's full barriers (cta_group::2 loads, no multicast).
//   warp 1       leader only: the MMA issuer.  Commits signal barriers in
//                both CTAs (tcgen05.commit multicast).
//   warp 2       TMEM allocation for the pair.
//   warps 4..11  one softmax warpgroup per pair tile: thread = query row
//                (TMEM lane).  Per visible KV tile: wait S, load it, tell the
//                leader S may be overwritten, exponentials with the running
//                base, P into shared memory (after the previous PV has read
//                the buffer), tell the leader P is ready.  Epilogue as in
//                fwd_sm100.cuh.
// TMEM (512 columns in each CTA): S_t at [128 t, +128), O_t at [256 + 128 t, +128).
//
// Every mbarrier wait is bounded; an expired wait sets the device status
// word and the CTA unwinds, so the other CTA's waits expire too.
#pragma once

#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace ra {

namespace {

// Pause of the MMA issuer's loop when none of its four streams can go
// (nanoseconds; 0 = poll continuously).
// MMA issue order: fixed per KV tile with suspending waits (1, measured
// faster: 8.74 ms against 11.2 ms on the 32K causal prefill), or whichever
// stream is ready, tested without blocking (0).
#ifndef RA_PAIR_STATIC
#define RA_PAIR_STATIC 1
#endif
#ifndef RA_PAIR_SLEEP_NS
#define RA_PAIR_SLEEP_NS 100
#endif

constexpr int kPairQTileBytes = 128 * 128 * 2;  // 128 rows x 128 channels (two 64-channel halves)
constexpr int kPairKHalfBytes = 64 * 128 * 2;   // 64 keys x 128 channels (two 64-channel halves)
constexpr int kPairVHalfBytes = 128 * 64 * 2;   // 128 keys x 64 channels
constexpr int kPairPBytes = 128 * 128 * 2;      // 128 rows x 128 keys (two 64-key halves)

template <int NK, int NV>
struct PairLayout {
  static constexpr int kQOff = 0;                                // 2 Q tiles
  static constexpr int kPOff = kQOff + 2 * kPairQTileBytes;      // 2 P tiles
  static constexpr int kKOff = kPOff + 2 * kPairPBytes;          // NK K halves
  static constexpr int kVOff = kKOff + NK * kPairKHalfBytes;     // NV V halves
  static constexpr int kBarOff = kVOff + NV * kPairVHalfBytes;
  // q, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s[2], sc[2], p[2],
  // pfree[2], o[2], drain
  static constexpr int kNumBars = 1 + 2 * NK + 2 * NV + 10 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // 1024-byte alignment of the swizzled tiles
};

// P = exp2(sl * s - base) for keys [64 H, 64 H + 64) of row r, as bf16 into
// the row's part of 64-key block H of a K-major, 128-byte-swizzled P tile
// (rows 128 bytes apart, 16-byte chunk c of row r at c ^ (r mod 8)); returns
// the sum of the float values.  `before_store` runs once, after the first 32
// keys' exponentials and before the first store (the wait for the buffer).
template <int H, class F>
__device__ __forceinline__ float softmax_p_to_smem(const float (&s)[128], float sl, float base, uint8_t* pblk, int r,
                                                   F&& before_store) {
  const float2 sl2 = make_float2(sl, sl);
  const float2 nb2 = make_float2(-base, -base);
  float2 sum0 = make_float2(0.f, 0.f), sum1 = sum0, sum2 = sum0, sum3 = sum0;
  uint8_t* prow = pblk + H * (128 * 128) + r * 128;
  uint4 w[4];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int key = 64 * H + 8 * c + 2 * k;
      float2 e = __ffma2_rn(make_float2(s[key], s[key + 1]), sl2, nb2);
      e = make_float2(ex2(e.x), ex2(e.y));
      u[k] = pack_bf16x2(e.x, e.y);
      if (k == 0) sum0 = __fadd2_rn(sum0, e);
      if (k == 1) sum1 = __fadd2_rn(sum1, e);
      if (k == 2) sum2 = __fadd2_rn(sum2, e);
      if (k == 3) sum3 = __fadd2_rn(sum3, e);
    }
    const uint4 v = make_uint4(u[0], u[1], u[2], u[3]);
    if (c < 4) {
      w[c] = v;
      if (c == 3) {
        before_store();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) = w[cc];
      }
    } else {
      *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = v;
    }
  }
  const float2 sa = __fadd2_rn(__fadd2_rn(sum0, sum1), __fadd2_rn(sum2, sum3));
  return sa.x + sa.y;
}

// Geometry of one CTA's part of a pair tile, or of a whole pair tile
// (rows = 256): first token, valid rows, and the key rows of the first and
// last valid token's positions (see QTile).
__device__ __forceinline__ QTile pair_qtile(long long tok0, int rows, long long N_q, long long qk_delta) {
  QTile q;
  q.tok0 = (int)tok0;
  const long long nt = N_q - tok0;
  const int ntok = (int)(nt < 0 ? 0 : (nt > rows ? rows : nt));
  q.nv = ntok;
  q.kmin = clamp_key(qk_delta + tok0);
  q.kmax = clamp_key(qk_delta + tok0 + (ntok > 0 ? ntok - 1 : 0));
  return q;
}

template <int NK, int NV, int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    fwd2_sm100_kernel(const __grid_constant__ Sm100Params p) {
  using L = PairLayout<NK, NV>;
  constexpr int D = 128;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  const uint32_t BAR_Q = bar0;
  auto BAR_K_FULL = [&](int i) { return bar0 + 8u * (1 + i); };
  auto BAR_K_EMPTY = [&](int i) { return bar0 + 8u * (1 + NK + i); };
  auto BAR_V_FULL = [&](int i) { return bar0 + 8u * (1 + 2 * NK + i); };
  auto BAR_V_EMPTY = [&](int i) { return bar0 + 8u * (1 + 2 * NK + NV + i); };
  auto BAR_S = [&](int t) { return bar0 + 8u * (1 + 2 * NK + 2 * NV + t); };       // S_t in TMEM (both CTAs)
  auto BAR_SC = [&](int t) { return bar0 + 8u * (3 + 2 * NK + 2 * NV + t); };      // S_t read (leader; 8 warps)
  auto BAR_P = [&](int t) { return bar0 + 8u * (5 + 2 * NK + 2 * NV + t); };       // P_t written (leader; 8 warps)
  auto BAR_PFREE = [&](int t) { return bar0 + 8u * (7 + 2 * NK + 2 * NV + t); };   // PV_t done (both CTAs)
  auto BAR_O = [&](int t) { return bar0 + 8u * (9 + 2 * NK + 2 * NV + t); };       // last PV_t done (both)
  const uint32_t BAR_DRAIN = bar0 + 8u * (11 + 2 * NK + 2 * NV);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  // ---- work item of the pair: KV head outermost, then the heaviest query
  // blocks of 512 rows first, then the G heads of the group, then splits.
  long long x = blockIdx.x >> 1;
  const int sigma = (int)(x % p.S);
  x /= p.S;
  const int g = (int)(x % p.G);
  x /= p.G;
  const int qblk = p.n_qblk - 1 - (int)(x % p.n_qblk);
  x /= p.n_qblk;
  const int hk = (int)(x % p.Hkv);
  const int b = (int)(x / p.Hkv);
  const int h = hk * p.G + g;

  const long long qk_delta = p.q_pos0 - p.k_pos0;
  QTile pq[2], own[2];  // pair tiles (visibility) and this CTA's rows of them (masks, epilogue)
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const long long t0 = (long long)qblk * 512 + 256 * t;
    pq[t] = pair_qtile(t0, 256, p.N_q, qk_delta);
    own[t] = pair_qtile(t0 + 128 * rank, 128, p.N_q, qk_delta);
  }
  const int kmax_last = pq[1].nv > 0 ? pq[1].kmax : pq[0].kmax;
  int lim = (int)p.N_kv;
  if (p.causal) lim = max(0, min(lim, kmax_last + 1));
  const long long first_rel = qk_delta + (long long)qblk * 512;
  const int home = first_rel > 0 ? (int)min((long long)(p.P - 1), first_rel / p.chunk) : 0;
  const int s_begin = sigma * p.steps_per_split;
  const int s_end = min(p.P, s_begin + p.steps_per_split);

  // ---- set-up
  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(BAR_K_FULL(i), 1);
      mbar_init(BAR_K_EMPTY(i), 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(BAR_V_FULL(i), 1);
      mbar_init(BAR_V_EMPTY(i), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR_S(t), 1);
      mbar_init(BAR_SC(t), 8);
      mbar_init(BAR_P(t), 8);
      mbar_init(BAR_PFREE(t), 1);
      mbar_init(BAR_O(t), 1);
    }
    mbar_init(BAR_DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // Both CTAs' barriers are initialised before any arrival crosses the pair.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) reg_dealloc<kRegsControl>();
  if (warp == 0) {
    // =========================== TMA producer ===========================
    if (lane == 0 && !p.skip_loads) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_k);
      prefetch_tmap(&p.tm_v);
      // Both CTAs' Q tiles (zero-filled past N_q) are counted on the
      // leader's barrier: 2 CTAs x 2 tiles x 32 KB.
      if (leader) mbar_arrive_expect_tx(BAR_Q, 4 * kPairQTileBytes);
      const uint32_t cq = mapa_shared(BAR_Q, 0);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          tma_load_4d_pair(sbase + L::kQOff + t * kPairQTileBytes + hf * (128 * 128), &p.tm_q, cq, hf * 64, h,
                           own[t].tok0, b);
      KvCursor<false> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t j = 0;
      bool ok = true;
      while (ok && cur.valid()) {
        {
          const uint32_t slot = j % NK, use = j / NK;
          if (!(ok = mbar_wait(BAR_K_EMPTY(slot), (use & 1u) ^ 1u, abort_flag))) break;
          if (leader) mbar_arrive_expect_tx(BAR_K_FULL(slot), 2 * kPairKHalfBytes);
          const uint32_t cb = mapa_shared(BAR_K_FULL(slot), 0);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            tma_load_4d_pair(sbase + L::kKOff + slot * kPairKHalfBytes + hf * (64 * 128), &p.tm_k, cb, hf * 64, hk,
                             cur.k0 + 64 * (int)rank, b);
        }
        {
          const uint32_t slot = j % NV, use = j / NV;
          if (!(ok = mbar_wait(BAR_V_EMPTY(slot), (use & 1u) ^ 1u, abort_flag))) break;
          if (leader) mbar_arrive_expect_tx(BAR_V_FULL(slot), 2 * kPairVHalfBytes);
          tma_load_4d_pair(sbase + L::kVOff + slot * kPairVHalfBytes, &p.tm_v, mapa_shared(BAR_V_FULL(slot), 0),
                           64 * (int)rank, hk, cur.k0, b);
        }
        ++j;
        cur.next();
      }
      if (leader) {
        // Let the last fills of both CTAs land before the pair can exit
        // (normally long consumed; this matters when unwinding after a
        // timeout).  The cluster barrier at the end holds the other CTA.
        volatile int no_abort = 0;
        for (uint32_t f = j > NK ? j - NK : 0; f < j; ++f) mbar_wait(BAR_K_FULL(f % NK), (f / NK) & 1u, &no_abort);
        for (uint32_t f = j > NV ? j - NV : 0; f < j; ++f) mbar_wait(BAR_V_FULL(f % NV), (f / NV) & 1u, &no_abort);
        mbar_wait(BAR_Q, 0, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (leader && lane == 0) {
      bool ok = mbar_wait(BAR_Q, 0, abort_flag);
      tc_fence_after();
      constexpr uint32_t idesc_s = idesc_bf16_f32(256, 128, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(256, D, 1);
      auto issue_s = [&](int t, uint32_t kslot) {
        const uint64_t qdesc = smem_desc_sw128(sbase + L::kQOff + t * kPairQTileBytes, 16, 1024);
        const uint64_t kdesc = smem_desc_sw128(sbase + L::kKOff + kslot * kPairKHalfBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = (kk / 4) * (128 * 128) + (kk % 4) * 32;
          const uint32_t ko = (kk / 4) * (64 * 128) + (kk % 4) * 32;
          umma_ss_pair(tmem + 128 * t, qdesc + (qo >> 4), kdesc + (ko >> 4), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit_pair(BAR_S(t));
      };
      auto issue_pv = [&](int t, uint32_t vslot, bool acc) {
        const uint64_t pdesc = smem_desc_sw128(sbase + L::kPOff + t * kPairPBytes, 16, 1024);
        const uint64_t vdesc = smem_desc_sw128(sbase + L::kVOff + vslot * kPairVHalfBytes, 128 * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          const uint32_t po = (kk / 4) * (128 * 128) + (kk % 4) * 32;
          umma_ss_pair(tmem + 256 + 128 * t, pdesc + (po >> 4), vdesc + ((kk * 2048) >> 4), idesc_o,
                       (acc || kk > 0) ? 1u : 0u);
        }
        tc_commit_pair(BAR_PFREE(t));
      };
#if RA_PAIR_STATIC
      // Fixed order per KV tile: the next tile's S for both pair tiles (each
      // once its softmax holds the previous S), then the current tile's PVs.
      auto wait_m = [&](uint32_t bar, uint32_t par) { return mbar_wait_idle(bar, par, abort_flag); };
      uint32_t n_s[2] = {0, 0}, n_sc[2] = {0, 0}, n_p[2] = {0, 0};
      KvCursor<false> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t j = 0;
      if (ok && cur.valid()) {
        ok = wait_m(BAR_K_FULL(0), 0);
        tc_fence_after();
        if (ok) {
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (tile_visible<false>(pq[t], cur.k0, cur.kend, p.causal)) {
              issue_s(t, 0);
              ++n_s[t];
            }
          tc_commit_pair(BAR_K_EMPTY(0));
        }
      }
      while (ok && cur.valid()) {
        KvCursor<false> nxt = cur;
        nxt.next();
        if (nxt.valid()) {
          const uint32_t kf = j + 1, kslot = kf % NK;
          if (!(ok = wait_m(BAR_K_FULL(kslot), (kf / NK) & 1u))) break;
          tc_fence_after();
#pragma unroll
          for (int t = 0; t < 2 && ok; ++t) {
            if (!tile_visible<false>(pq[t], nxt.k0, nxt.kend, p.causal)) continue;
            if (n_s[t] > n_sc[t]) {
              if (!(ok = wait_m(BAR_SC(t), n_sc[t] & 1u))) break;
              ++n_sc[t];
              tc_fence_after();
            }
            issue_s(t, kslot);
            ++n_s[t];
          }
          if (!ok) break;
          tc_commit_pair(BAR_K_EMPTY(kslot));
        }
        const uint32_t vslot = j % NV;
        if (!(ok = wait_m(BAR_V_FULL(vslot), (j / NV) & 1u))) break;
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < 2 && ok; ++t) {
          if (!tile_visible<false>(pq[t], cur.k0, cur.kend, p.causal)) continue;
          if (!(ok = wait_m(BAR_P(t), n_p[t] & 1u))) break;
          tc_fence_after();
          issue_pv(t, vslot, n_p[t] > 0);
          ++n_p[t];
        }
        if (!ok) break;
        tc_commit_pair(BAR_V_EMPTY(vslot));
        cur = nxt;
        ++j;
      }
#else
      // The four streams (S and PV of each pair tile) are served in the
      // order their inputs become ready: each pass tests, without blocking,
      // whether a PV can go (its P is in shared memory and its V tile has
      // landed) and whether an S can go (its K tile has landed and the
      // softmax holds the previous S in registers).  PVs go first: the next
      // softmax waits for its P buffer, while the next S is needed only when
      // the current softmax ends.  Each stream walks the KV tiles in ring
      // order, skipping the ones its pair tile does not see; j counts the
      // fills of the shared K / V rings.
      struct Stream {
        KvCursor<false> c;
        uint32_t j;
      };
      auto skip_invisible = [&](Stream& st, int t) {
        while (st.c.valid() && !tile_visible<false>(pq[t], st.c.k0, st.c.kend, p.causal)) {
          st.c.next();
          ++st.j;
        }
      };
      Stream sS[2], sP[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        sS[t].c.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
        sS[t].j = 0;
        skip_invisible(sS[t], t);
        sP[t] = sS[t];
      }
      uint32_t n_s[2] = {0, 0}, n_p[2] = {0, 0};
      uint32_t rel_k = 0, rel_v = 0;  // ring fills handed back to the producers
      unsigned long long t_last = globaltimer_ns();
      uint32_t idle = 0;
      while (ok) {
        bool left = false, progressed = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!sP[t].c.valid()) continue;
          left = true;
          const uint32_t f = sP[t].j, vs = f % NV;
          if (n_p[t] < n_s[t] && mbar_test(BAR_P(t), n_p[t] & 1u) && mbar_test(BAR_V_FULL(vs), (f / NV) & 1u)) {
            tc_fence_after();
            issue_pv(t, vs, n_p[t] > 0);
            ++n_p[t];
            sP[t].c.next();
            ++sP[t].j;
            skip_invisible(sP[t], t);
            progressed = true;
          }
        }
        // V fills both tiles are past, once landed: their last reader was issued.
        while (rel_v < min(sP[0].j, sP[1].j) && mbar_test(BAR_V_FULL(rel_v % NV), (rel_v / NV) & 1u)) {
          tc_commit_pair(BAR_V_EMPTY(rel_v % NV));
          ++rel_v;
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!sS[t].c.valid()) continue;
          left = true;
          const uint32_t f = sS[t].j, ks = f % NK;
          if (mbar_test(BAR_K_FULL(ks), (f / NK) & 1u) && (n_s[t] == 0 || mbar_test(BAR_SC(t), (n_s[t] - 1) & 1u))) {
            tc_fence_after();
            issue_s(t, ks);
            ++n_s[t];
            sS[t].c.next();
            ++sS[t].j;
            skip_invisible(sS[t], t);
            progressed = true;
          }
        }
        while (rel_k < min(sS[0].j, sS[1].j) && mbar_test(BAR_K_FULL(rel_k % NK), (rel_k / NK) & 1u)) {
          tc_commit_pair(BAR_K_EMPTY(rel_k % NK));
          ++rel_k;
        }
        if (!left) break;
        if (progressed) {
          t_last = globaltimer_ns();
          idle = 0;
        } else if (RA_PAIR_SLEEP_NS > 0) {
          // Nothing was ready: leave the issue slots of this sub-partition
          // to the softmax warps for a moment.
          __nanosleep(RA_PAIR_SLEEP_NS);
          if ((++idle & 15u) == 0u) {
            if (*abort_flag) {
              ok = false;
            } else if (globaltimer_ns() - t_last > kWaitLimitNs) {
              *abort_flag = 1;
              atomicExch(&g_status, (int)RA_ERR_DEVICE_TIMEOUT);
              ok = false;
            }
          }
        } else if ((++idle & 255u) == 0u) {
          // The same wall-clock bound as every other wait.
          if (*abort_flag) {
            ok = false;
          } else if (globaltimer_ns() - t_last > kWaitLimitNs) {
            *abort_flag = 1;
            atomicExch(&g_status, (int)RA_ERR_DEVICE_TIMEOUT);
            ok = false;
          }
        }
      }
#endif
#pragma unroll
      for (int t = 0; t < 2; ++t) tc_commit_pair(BAR_O(t));
      tc_commit_pair(BAR_DRAIN);
    }
  } else if (warp >= 4) {
    // ========================= softmax warpgroups =========================
    reg_alloc<kRegsSoftmax>();
    const int t = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int rloc = quad * 32 + lane;  // row inside this CTA's 128 == TMEM lane
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + 128 * t;
    const uint32_t o_tmem = tmem + lane_base + 256 + 128 * t;
    const QTile q = own[t];
    const bool row_valid = rloc < q.nv;
    const bool warp_active = quad * 32 < q.nv;
    const long long row = (long long)q.tok0 + rloc;
    uint8_t* pblk = smem + L::kPOff + t * kPairPBytes;
    const uint32_t c_sc = mapa_shared(BAR_SC(t), 0), c_p = mapa_shared(BAR_P(t), 0);
    const float scale_l2 = p.scale_log2;
    const bool fold = scale_l2 > 0.f;
    const float sl = fold ? scale_l2 : 1.f;
    float m2 = -INFINITY, l = 0.f;

    KvCursor<false> cur;
    cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
    uint32_t n = 0;
    bool ok = true;
    while (ok && cur.valid()) {
      if (!tile_visible<false>(pq[t], cur.k0, cur.kend, p.causal)) {
        cur.next();
        continue;
      }
      if (!(ok = mbar_wait(BAR_S(t), n & 1u, abort_flag))) break;
      tc_fence_after();
      float s[128];
      if (warp_active) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_tmem + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        tc_wait_ld();
      }
      // S is in registers: the leader may overwrite it with the next tile's scores.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(c_sc);
      // The P buffer is free once the previous PV of this tile has read it
      // (that also makes O stable for a rescale).
      bool freed = n == 0;
      auto wait_free = [&]() {
        if (!freed) {
          ok = mbar_wait(BAR_PFREE(t), (n - 1) & 1u, abort_flag);
          tc_fence_after();
          freed = true;
        }
      };
      if (warp_active) {
        if (!fold) {
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] *= scale_l2;
        }
        const bool masked = tile_needs_mask<false>(q, cur.k0, cur.kend, p.causal);
        if (masked) {
          const int kvis = cur.kend - cur.k0;
          const long long kc = p.causal ? (long long)q.kmin + rloc - cur.k0 : (long long)kTileN;
          const int kcausal = (int)(kc < -1 ? -1 : (kc > kTileN ? kTileN : kc));
          const int klast = min(kvis - 1, kcausal);
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = (c <= klast) ? s[c] : -INFINITY;
        }
        auto row_max = [&]() {
          float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
          for (int c = 4; c < 128; c += 8) {
            mx0 = fmax3(mx0, s[c], s[c + 1]);
            mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
            mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
            mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
          }
          return fmax3(fmaxf(mx0, mx1), mx2, mx3) * sl;
        };
        auto compute_p = [&](float base) {
          float r = softmax_p_to_smem<0>(s, sl, base, pblk, rloc, wait_free);
          r += softmax_p_to_smem<1>(s, sl, base, pblk, rloc, [] {});
          return r;
        };
        // One pass with the current base after a row's first tile; the max
        // (and a redo with a new base) only when the row sum shows that some
        // entry may exceed 2^kRescaleSlack.  P is published only after that
        // check, so a redo simply overwrites the buffer.
        float rs = 0.f, alpha = 1.f;
        const bool max_first = n == 0 || __any_sync(0xffffffffu, m2 == -INFINITY);
        bool redo = max_first;
        if (!max_first) {
          rs = compute_p(m2);
          if (__any_sync(0xffffffffu, !(rs <= kSlackSum))) {
            const float m_tile = row_max();
            if (m_tile > m2 + kRescaleSlack) {
              alpha = ex2(m2 - m_tile);
              m2 = m_tile;
              l *= alpha;
            }
            redo = __any_sync(0xffffffffu, alpha != 1.f);
          }
        } else {
          const float m_tile = row_max();
          if (m_tile > m2 + kRescaleSlack) {
            alpha = ex2(m2 - m_tile);  // 0 when m2 = -inf
            m2 = m_tile;
            l *= alpha;
          }
        }
        if (redo) {
          if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            // Rare: the max jumped past the slack; rescale O (stable: the
            // previous PV has completed) before the new P is published.
            wait_free();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              float r[32];
              tmem_ld32(o_tmem + c * 32, r);
              tc_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] *= alpha;
              tmem_st32(o_tmem + c * 32, *reinterpret_cast<const uint32_t(*)[32]>(r));
            }
            tc_wait_st();
          }
          rs = compute_p((m2 == -INFINITY) ? 0.f : m2);
        }
        l += rs;
      } else {
        wait_free();  // keep the same waits as the active warps
      }
      if (!ok) break;
      // P (generic-proxy stores) is read by the tensor cores (async proxy).
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(c_p);
      ++n;
      cur.next();
    }

    // ------------------------------ epilogue ------------------------------
    if (ok && n > 0) ok = mbar_wait(BAR_O(t), 0, abort_flag);
    if (ok && warp_active) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const long long ooff = (((long long)(MODE == kModeSplit ? sigma * p.B + b : b) * p.N_q + row) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float r[32];
        if (n > 0) {
          tmem_ld32(o_tmem + c * 32, r);
          tc_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0.f;
        }
        if (!row_valid) continue;
        if (MODE == kModeSplit) {
          float* dst = p.o_part + ooff + c * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(r[i] * inv, r[i + 1] * inv, r[i + 2] * inv, r[i + 3] * inv);
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + ooff + c * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w;
            w.x = pack_bf16x2(r[i] * inv, r[i + 1] * inv);
            w.y = pack_bf16x2(r[i + 2] * inv, r[i + 3] * inv);
            w.z = pack_bf16x2(r[i + 4] * inv, r[i + 5] * inv);
            w.w = pack_bf16x2(r[i + 6] * inv, r[i + 7] * inv);
            *reinterpret_cast<uint4*>(dst + i) = w;
          }
        }
      }
      if (row_valid) {
        const float lse_v = l > 0.f ? (m2 + log2f(l)) * kLn2 : -INFINITY;
        if (MODE == kModeSplit)
          p.lse_part[(((long long)sigma * p.B + b) * p.Hq + h) * p.N_q + row] = lse_v;
        else
          p.lse[((long long)b * p.Hq + h) * p.N_q + row] = lse_v;
      }
    }
  }

  // ---- tear-down: the pair's MMAs have drained before TMEM is freed, and
  // neither CTA leaves while the other may still touch its shared memory.
  if (warp == 2) {
    volatile int no_abort = 0;
    mbar_wait(BAR_DRAIN, 0, &no_abort);
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tmem, 512);
}

template <int NK, int NV, int MODE>
cudaError_t launch_fwd2_cfg(const Sm100Params& prm, long long grid, cudaStream_t st) {
  using L = PairLayout<NK, NV>;
  static_assert(L::kAlloc <= 232448, "shared memory budget exceeded");
  auto kern = fwd2_sm100_kernel<NK, NV, MODE>;
  // The in-kernel register split assumes exactly kLaunchRegs per thread.
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    cudaError_t e0 = cudaFuncGetAttributes(&fa, kern);
    if (e0 != cudaSuccess) return e0;
    regs = fa.numRegs;
  }
  if (regs != kLaunchRegs) return cudaErrorInvalidConfiguration;
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

// Off by default: on the 32K causal prefill it measured 8.74 ms against
// 8.25 ms for the single-CTA kernel (same box).  RINGATTN_PAIR=1 selects it.
bool fwd2_applies(const ProblemArgs& a, int mode) {
  if (a.d != 128 || a.kv8 || a.wa_period > 0 || (mode != kModeFinal && mode != kModeSplit)) return false;
  if (a.N_q <= kTileM) return false;  // one query tile: the single-CTA kernel
  const char* ov = std::getenv("RINGATTN_PAIR");
  return ov && ov[0] == '1';
}

cudaError_t launch_fwd2_sm100(const ProblemArgs& a, int mode, cudaStream_t st) {
  Sm100Params prm;
  memset(&prm, 0, sizeof(prm));
  if (encode_map(&prm.tm_q, a.q, a.d, a.Hq, a.N_q, a.B, 1) != CUDA_SUCCESS ||
      encode_map_box(&prm.tm_k, a.k, a.d, a.Hkv, a.N_kv, a.B, 1, 64) != CUDA_SUCCESS ||
      encode_map(&prm.tm_v, a.v, a.d, a.Hkv, a.N_kv, a.B, 1) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  prm.out = a.out;
  prm.lse = a.lse;
  prm.o_part = a.o_part;
  prm.lse_part = a.lse_part;
  prm.B = a.B;
  prm.Hq = a.Hq;
  prm.Hkv = a.Hkv;
  prm.G = a.Hq / a.Hkv;
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
  prm.gpack = 1;
  prm.gshift = 0;
  prm.tpt = kTileM;
  {
    const char* f = std::getenv("RINGATTN_FAULT");
    prm.skip_loads = (f && std::strcmp(f, "device_wait") == 0) ? 1 : 0;
  }
  prm.n_qblk = (int)((a.N_q + 511) / 512);  // query blocks of one CTA pair
  const long long grid = 2LL * prm.n_qblk * a.B * a.Hkv * prm.G * prm.S;
  if (mode == kModeSplit) return launch_fwd2_cfg<3, 3, kModeSplit>(prm, grid, st);
  return launch_fwd2_cfg<3, 3, kModeFinal>(prm, grid, st);
}

}  // namespace ra
