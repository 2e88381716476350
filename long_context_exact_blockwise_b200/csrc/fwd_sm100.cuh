// Blockwise (ring) attention forward on B200 tensor cores: bf16 inputs,
// float32 logits and accumulators.
//
// What it computes follows "Ring Attention: the secret of million-token
// context": the KV sequence is cut into P chunks (§2.1); a tile of query
// rows homed at chunk i visits chunk (i + s) mod P at step s (§2.2 figure);
// each visit runs the flash-attention inner loop over 128-key tiles held in
// on-chip memory (§3.1), and the next KV tile is fetched while the current
// one is computed (§3.2 double buffering, here a TMA ring of smem slots).
// The partial results are merged by a running max / sum (online softmax)
// and normalised once over all keys at the end.
//
// CTA organisation (one CTA owns NQT query tiles of 128 rows of one head):
//   warp 0       TMA producer: Q tiles once, then K/V tiles into an
//                NSLOT-deep ring of shared-memory slots (K_j -> slot 2j,
//                V_j -> slot 2j+1, modulo NSLOT).
//   warp 1       MMA issuer (one thread): S_t = Q_t K_j^T into TMEM
//                (tcgen05.mma, A and B from smem), then O_t += P_t V_j with
//                P_t read from TMEM.  Q tiles ping-pong: S for one tile is
//                computed while the other tile's softmax runs.  (One issuer
//                for both tiles measured faster than one per tile: MMAs of
//                two threads interleave in the tensor pipe.)
//   warp 2       TMEM allocator.
//   warps 4..    one softmax warpgroup per query tile: thread = query row
//                (TMEM lane).  Reads S with tcgen05.ld, masks (only tiles
//                that straddle the causal diagonal or a chunk edge), runs the
//                exp2 online softmax, writes P (bf16) back over S, rescales O
//                in TMEM when the row max grew, and writes the epilogue.
//   warps 8..11  (FP8 KV cache only, single-tile CTAs) converters: the
//                producer's TMA brings raw E4M3 tiles into their own ring of
//                NSLOT8 slots; these warps decode each tile to bf16 in the
//                128-byte-swizzled layout the MMAs read and publish it in the
//                bf16 ring.  k_scale folds into the exponent scale, v_scale
//                into the epilogue.
// TMEM columns: S_t at [128 t, 128 t + 128) (P_t aliases its first 64
// columns), O_t at [128 NQT + D t, ... + D).
//
// Every mbarrier wait is bounded (common.cuh); an expired wait sets the
// device status word and the CTA unwinds without trapping.
#include <algorithm>
#include <cstdio>
#include <cstdlib>

#pragma once

#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace ra {

namespace {

constexpr int kTileM = 128;  // query rows per tile (TMEM lanes)
// The exponent base may trail the running row max by up to this much (log2
// units) before O is rescaled: P entries stay <= 2^8, far inside bf16 range.
constexpr float kRescaleSlack = 8.f;
// Row sum of one tile's P with every entry <= 2^kRescaleSlack is at most
// 128 * 2^8; a sum at most 2^8 guarantees every entry is, so the one-pass
// path checks the sum against 2^8.
constexpr float kSlackSum = 256.f;
// Which of every 8 exponential pairs of an unmasked tile go to the FMA pipe
// (bit i: pairs with index i mod 8).
#ifndef RA_EXP2_POLY_MASK
#define RA_EXP2_POLY_MASK 0x00
#endif
constexpr int kExp2PolyMask = RA_EXP2_POLY_MASK;
// FP8-KV kernel ring depths at d = 128 (bf16 slots, FP8 slots).
#ifndef RA_KV8_NSLOT
#define RA_KV8_NSLOT 4
#endif
#ifndef RA_KV8_NSLOT8
#define RA_KV8_NSLOT8 4
#endif

// Register split of the two-query-tile kernel (384 threads at 168 registers).
constexpr int kLaunchRegs = 168;
constexpr int kRegsControl = 88;   // warps 0-3: TMA, MMA issue, TMEM allocation
constexpr int kRegsSoftmax = 208;  // warps 4-11: the two softmax warpgroups
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= 384 * kLaunchRegs, "register split exceeds the launch");
// Register split of the FP8-KV kernel (one query tile + a converter
// warpgroup: 384 threads at 168 registers).
constexpr int kRegsControl8 = 80;   // warps 0-3
constexpr int kRegsSoftmax8 = 248;  // warps 4-7
constexpr int kRegsConvert8 = 80;   // warps 8-11
static_assert(128 * (kRegsControl8 + kRegsSoftmax8 + kRegsConvert8) <= 384 * kLaunchRegs,
              "register split exceeds the launch");
constexpr int kTileN = 128;  // keys per KV tile

struct Sm100Params {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  void* out;
  float* lse;
  float* o_part;
  float* lse_part;
  float* acc;
  float* m_state;
  float* l_state;
  int B, Hq, Hkv, G;
  long long N_q, N_kv;
  long long q_pos0, k_pos0;
  int causal;
  float scale_log2;
  long long chunk;
  int P;
  int S;
  int steps_per_split;
  int n_qblk;
  int out_f32;
  int gpack;   // query heads packed into one tile (1, or G for incremental queries)
  int gshift;  // log2(gpack)
  int skip_loads;  // failure-detection test: the producer issues no copies, so the
                   // consumers' bounded waits expire and the kernel unwinds
  int tpt;     // tokens per tile: 128 / gpack
  const float* k_scale;  // FP8 KV cache: [B, Hkv] dequantisation scales
  const float* v_scale;
  int wa_window;  // window-and-anchor mask: window W (keys i - W .. i) ...
  int wa_period;  // ... and anchor period A; 0: no such mask
};

// The window-and-anchor sparse mask as seen by one CTA: keys [lo, hi] hold
// the local windows of its query rows, and a0, am1, ap its anchor keys
// (a, a - 1, a + A; -1 when absent).  All of a CTA's rows share one anchor
// period (A is a multiple of its row span).
// It lives in shared memory (written once per CTA), so the roles' cursors
// carry no registers for it; kernels without the mask never touch it.
struct WinAnchor {
  int W, lo, hi, a0, am1, ap;
};
__shared__ WinAnchor s_wa;

__device__ __forceinline__ bool wa_has_anchor(int k0, int kend) {
  return (s_wa.a0 >= k0 && s_wa.a0 < kend) || (s_wa.am1 >= k0 && s_wa.am1 < kend) ||
         (s_wa.ap >= k0 && s_wa.ap < kend);
}
// Does any row of the CTA see a key in [k0, kend)?
template <bool WA>
__device__ __forceinline__ bool wa_live(int k0, int kend) {
  if constexpr (!WA) return true;
  return (kend - 1 >= s_wa.lo && k0 <= s_wa.hi) || wa_has_anchor(k0, kend);
}

// The sequence of KV tiles one CTA visits: chunks in ring order from `home`,
// 128-key tiles inside each chunk, keys clipped to [0, lim).  Indices are
// k-buffer rows; the host caps buffers well below 2^31 rows, so 32 bits hold
// every sum formed here.
//
// Under the window-and-anchor mask the cursor yields only tiles some row of
// the CTA sees (chunks and tiles outside the windows and anchors are
// skipped); every role walks the same cursor, so they stay in step.
template <bool WA>
struct KvCursor {
  int chunk, lim, P, home, s, s_end;
  int k0, kend, cend;

  // First live tile of chunk step s or a later one.
  __device__ __forceinline__ void load_chunk() {
    while (s < s_end) {
      const int c = (home + s) % P;
      const int cb = c * chunk;
      const int ce = min(cb + chunk, lim);
      if (cb < ce && wa_live<WA>(cb, ce)) {
        cend = ce;
        for (k0 = cb; k0 < ce; k0 += kTileN) {
          kend = min(k0 + kTileN, ce);
          if (wa_live<WA>(k0, kend)) return;
        }
      }
      ++s;
    }
  }
  __device__ __forceinline__ void init(int chunk_, int lim_, int P_, int home_, int s0, int s1) {
    chunk = chunk_;
    lim = lim_;
    P = P_;
    home = home_;
    s = s0;
    s_end = s1;
    load_chunk();
  }
  __device__ __forceinline__ bool valid() const { return s < s_end; }
  __device__ __forceinline__ void next() {
    for (k0 += kTileN; k0 < cend; k0 += kTileN) {
      kend = min(k0 + kTileN, cend);
      if (wa_live<WA>(k0, kend)) return;
    }
    ++s;
    load_chunk();
  }
};

// Geometry of one query tile of the CTA.  A tile holds tpt tokens x gpack
// heads; tile row r is token tok0 + (r >> gshift) of head h + (r & (gpack-1)).
// kmin / kmax: the k-buffer row whose global position equals that of the
// tile's first / last valid token, so under causal masking token tok0 + i
// sees keys k <= kmin + i.  Clamped to [-2^30, 2^31 - 4096]: beyond either
// end the answer is the same.
struct QTile {
  int tok0;  // first token in the q buffer
  int nv;    // valid rows (0..128)
  int kmin;
  int kmax;
};

constexpr long long kKeyClampLo = -(1ll << 30);
constexpr long long kKeyClampHi = (1ll << 31) - 4096;

__device__ __forceinline__ int clamp_key(long long x) {
  return (int)(x < kKeyClampLo ? kKeyClampLo : (x > kKeyClampHi ? kKeyClampHi : x));
}

template <int D, int NQT, int NSLOT, int NSLOT8 = 0>
struct Layout {
  static constexpr int kTileBytes = kTileM * D * 2;  // one bf16 tile of 128 rows x D
  static constexpr int kF8Bytes = kTileN * D;        // one FP8 tile of 128 keys x D
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kQOff + NQT * kTileBytes;
  static constexpr int kF8Off = kKVOff + NSLOT * kTileBytes;
  static constexpr int kBarOff = kF8Off + NSLOT8 * kF8Bytes;
  // barriers: q, kv_full[NSLOT], kv_empty[NSLOT], s[NQT], s_consumed[NQT],
  // p_lo[NQT], p_hi[NQT], o[NQT], drain, f8_full[NSLOT8], f8_empty[NSLOT8]
  static constexpr int kNumBars = 1 + 2 * NSLOT + 5 * NQT + 1 + 2 * NSLOT8;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr uint32_t kTmemCols = (NQT * (128 + D) <= 256) ? 256 : 512;
  // 1024 bytes of slack for the 1024-byte alignment of the swizzled tiles.  A
  // CTA that takes all 512 TMEM columns also takes more than half of the
  // SM's shared memory, so a second CTA never waits on the allocator.
  static constexpr int kAlloc = (kTmemCols == 512 && kBytes + 1024 < 120 * 1024) ? 120 * 1024 : kBytes + 1024;
};

template <int NQT>
__device__ __forceinline__ QTile make_qtile(int qblk, int t, long long N_q, long long qk_delta, int tpt,
                                           int gshift) {
  QTile q;
  q.tok0 = qblk * (NQT * tpt) + t * tpt;
  const long long nt = N_q - q.tok0;
  const int ntok = (int)(nt < 0 ? 0 : (nt > tpt ? tpt : nt));
  q.nv = ntok << gshift;
  q.kmin = clamp_key(qk_delta + q.tok0);
  q.kmax = clamp_key(qk_delta + q.tok0 + (ntok > 0 ? ntok - 1 : 0));
  return q;
}

template <bool WA>
__device__ __forceinline__ bool tile_visible(const QTile& q, int k0, int kend, int causal) {
  if constexpr (WA) return q.nv > 0 && ((kend - 1 >= q.kmin - s_wa.W && k0 <= q.kmax) || wa_has_anchor(k0, kend));
  return q.nv > 0 && (!causal || k0 <= q.kmax);
}

template <bool WA>
__device__ __forceinline__ bool tile_needs_mask(const QTile& q, int k0, int kend, int causal) {
  if constexpr (WA) return (kend - k0 < kTileN) || k0 < q.kmax - s_wa.W || kend - 1 > q.kmin;
  return (kend - k0 < kTileN) || (causal && kend - 1 > q.kmin);
}

// P = exp2(sl * s - base) for keys [64 H, 64 H + 64) of one row, written as
// bf16 pairs to TMEM columns [32 H, 32 H + 32) of S; returns the sum of the
// float values.  Bit i of EMU set: pairs whose index is i mod 8 use
// exp2_poly2 (FMA pipe) instead of ex2 (MUFU).  EMU is a compile-time
// constant so each pair's choice is fixed in the generated code.
template <int EMU, int H>
__device__ __forceinline__ float softmax_p_half(const float (&s)[128], float sl, float base, uint32_t s_tmem) {
  const float2 sl2 = make_float2(sl, sl);
  const float2 nb2 = make_float2(-base, -base);
  float2 sum0 = make_float2(0.f, 0.f), sum1 = sum0, sum2 = sum0, sum3 = sum0;
#pragma unroll
  for (int c = 2 * H; c < 2 * H + 2; ++c) {
    uint32_t u[16];
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
      float2 e[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        e[k] = __ffma2_rn(make_float2(s[c * 32 + 2 * (i + k)], s[c * 32 + 2 * (i + k) + 1]), sl2, nb2);
        if ((EMU >> ((i + k) & 7)) & 1)
          e[k] = exp2_poly2(e[k]);
        else
          e[k] = make_float2(ex2(e[k].x), ex2(e[k].y));
        u[i + k] = pack_bf16x2(e[k].x, e[k].y);
      }
      sum0 = __fadd2_rn(sum0, e[0]);
      sum1 = __fadd2_rn(sum1, e[1]);
      sum2 = __fadd2_rn(sum2, e[2]);
      sum3 = __fadd2_rn(sum3, e[3]);
    }
    tmem_st16(s_tmem + c * 16, u);
  }
  const float2 sa = __fadd2_rn(__fadd2_rn(sum0, sum1), __fadd2_rn(sum2, sum3));
  return sa.x + sa.y;
}

// S (+)= Q K^T for keys [64 H0, 64 H1) of a 128-key K tile at smem address
// `kaddr`, into TMEM columns [64 H0, 64 H1) of the S tile at `s_tmem`.
// Q and K are K-major with 128-byte swizzle: a K-step of 16 elements is 32
// bytes inside a swizzle row, every 64 elements move to the next
// 128-row x 128-byte block, and key row r starts r * 128 bytes into a block.
template <int D, int H0, int H1>
__device__ __forceinline__ void mma_qk(uint32_t s_tmem, uint64_t qdesc, uint32_t kaddr) {
  constexpr uint32_t idesc = idesc_bf16_f32(kTileM, (H1 - H0) * 64, 0);
  const uint64_t kdesc = smem_desc_sw128(kaddr + H0 * 64 * 128, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * (kTileM * 128) + (kk % 4) * 32;
    umma_ss(s_tmem + 64 * H0, qdesc + (off >> 4), kdesc + (off >> 4), idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V for keys [64 HALF, 64 HALF + 64) of a 128-key V tile at `vaddr`.
// P (bf16 pairs) is read from TMEM at `p_tmem`: 16 keys = 8 columns.  For
// B = V (N = d, K = keys) the tile is MN-major: 64-element blocks of d are
// kTileN * 128 bytes apart (LBO), groups of 8 keys 1024 bytes apart (SBO),
// 16 keys = 2048 bytes.
template <int D, int HALF>
__device__ __forceinline__ void mma_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t vaddr, bool accumulate_first) {
  constexpr uint32_t idesc = idesc_bf16_f32(kTileM, D, 1);
  const uint64_t vdesc = smem_desc_sw128(vaddr, kTileN * 128, 1024);
#pragma unroll
  for (int kk = 4 * HALF; kk < 4 * HALF + 4; ++kk)
    umma_ts(o_tmem, p_tmem + kk * 8, vdesc + ((kk * 2048) >> 4), idesc, (accumulate_first || kk > 0) ? 1u : 0u);
}

// Signal a per-warp barrier after this thread's tcgen05 operations: every
// thread waits for and fences its own, the warp synchronises, one lane arrives.
__device__ __forceinline__ void warp_arrive_after_tc(uint32_t bar, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// Four E4M3 codes (bytes of w, lowest address first) to two bf16x2 words
// holding each code's value times 2^-120 (kFp8Bias), with integer operations
// only.  An E4M3 code s.eeee.mmm placed in a bf16 word as s.0000eeee.mmm0000
// reads as 2^(e-127) (1 + m/8) = 2^-120 * 2^(e-7) (1 + m/8) for e >= 1, and
// as the subnormal 2^-126 * m/8 = 2^-120 * 2^-6 * m/8 for e = 0: exact for
// every finite code.  The 2^120 goes back in through the scales.
constexpr float kFp8Bias = 1.329227995784916e36f;  // 2^120
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w, uint32_t sel) {
  // Two codes into the low bytes of the two 16-bit halves: 0000 0000 seee emmm.
  const uint32_t x = __byte_perm(w, 0, sel);
  // Moving the sign from bit 7 to bit 15 while the code moves up 4 bits:
  // 16 * (x + 15 * sign) = (code << 4) - (sign << 4) + (sign << 8), as two
  // multiply-adds (FMA pipe) and one mask (ALU pipe).
  const uint32_t sgn = x & 0x00800080u;
  return __umul24(sgn, 15u) * 16u + x * 16u;
}
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  lo = e4m3x2_to_bf16x2(w, 0x4140);  // codes 0, 1
  hi = e4m3x2_to_bf16x2(w, 0x4342);  // codes 2, 3
}

// Decode one FP8 tile (128 keys x D codes) into a bf16 tile in the layout a
// TMA copy with 128-byte swizzle produces: 64-element column blocks of
// 128 rows x 128 bytes, the 16-byte chunk j of row r stored at j ^ (r mod 8).
// Thread ct of the converter warpgroup converts 16-code chunks.
//
// d = 128: the FP8 tile also arrives 128-byte swizzled (its 16-code chunk c
// of row r at c ^ (r mod 8)).  Eight consecutive threads (one shared-memory
// phase of a 16-byte access) take the same chunk column of eight
// consecutive rows, so their loads and their stores fall on eight distinct
// bank groups.  d = 64: row-major codes, threads along the row.
// Every chunk of a thread has the same column and the same row mod 8, so all
// its addresses are one base plus constants.
template <int D>
__device__ __forceinline__ void convert_fp8_tile(const uint8_t* src, uint8_t* dst, int ct) {
  constexpr int kChunksPerRow = D / 16;
  constexpr int kPerThread = kTileN * kChunksPerRow / 128;
  int r0, cc, row_step, src_chunk;
  if constexpr (D == 128) {
    const int a = ct >> 3, b = ct & 7;
    cc = a & 7;
    r0 = b + 8 * (a >> 3);  // rows r0 + 16 i
    row_step = 16;
    src_chunk = cc ^ b;     // swizzled position of chunk cc in row r0 (r0 mod 8 = b)
  } else {
    r0 = ct / kChunksPerRow;
    cc = ct % kChunksPerRow;
    row_step = 128 / kChunksPerRow;
    src_chunk = cc;
  }
  const uint8_t* s0 = src + r0 * D + src_chunk * 16;
  const int j0 = (cc % 4) * 2;  // 16 codes = 32 bytes of bf16: chunks j0, j0 + 1
  uint8_t* d0 = dst + (cc / 4) * (kTileN * 128) + r0 * 128;
  const int a0 = (j0 ^ (r0 & 7)) << 4, a1 = ((j0 + 1) ^ (r0 & 7)) << 4;
  // All of this thread's loads first, so their latencies overlap.
  uint4 w[kPerThread];
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) w[i] = *reinterpret_cast<const uint4*>(s0 + i * row_step * D);
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    uint4 o0, o1;
    e4m3x4_to_bf16x4(w[i].x, o0.x, o0.y);
    e4m3x4_to_bf16x4(w[i].y, o0.z, o0.w);
    e4m3x4_to_bf16x4(w[i].z, o1.x, o1.y);
    e4m3x4_to_bf16x4(w[i].w, o1.z, o1.w);
    *reinterpret_cast<uint4*>(d0 + i * row_step * 128 + a0) = o0;
    *reinterpret_cast<uint4*>(d0 + i * row_step * 128 + a1) = o1;
  }
}

template <int D, int NQT, int NSLOT, int MODE, int NSLOT8 = 0, bool WA = false>
__global__ void __launch_bounds__(128 + 128 * NQT + (NSLOT8 > 0 ? 128 : 0), 1)
    fwd_sm100_kernel(const __grid_constant__ Sm100Params p) {
  using L = Layout<D, NQT, NSLOT, NSLOT8>;
  constexpr bool kKV8 = NSLOT8 > 0;
  static_assert(!kKV8 || NQT == 1, "the FP8-KV kernel has one query tile");
  constexpr int kHalves = D / 64;  // 64-element (128-byte) swizzle columns per tile
  // Single-tile CTAs (short or packed queries) have no second tile to keep
  // the tensor pipe busy during a softmax, so they overlap inside the tile:
  // the next S is computed in two halves (keys 64..127 while the softmax
  // runs) and P is published in two halves (PV on keys 0..63 overlaps the
  // rest of the softmax).  Two-tile CTAs ping-pong instead; the extra
  // signalling measured slower there.
  constexpr bool kSplitS = (NQT == 1);
  constexpr bool kSplitPV = (NQT == 1);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto BAR_Q = [&]() { return bar0; };
  auto BAR_KV_FULL = [&](int i) { return bar0 + 8u * (1 + i); };
  auto BAR_KV_EMPTY = [&](int i) { return bar0 + 8u * (1 + NSLOT + i); };
  auto BAR_S = [&](int t) { return bar0 + 8u * (1 + 2 * NSLOT + t); };             // S_t in TMEM
  auto BAR_SC = [&](int t) { return bar0 + 8u * (1 + 2 * NSLOT + NQT + t); };      // S_t read by softmax
  auto BAR_PA = [&](int t) { return bar0 + 8u * (1 + 2 * NSLOT + 2 * NQT + t); };  // P_t keys 0..63
  auto BAR_PB = [&](int t) { return bar0 + 8u * (1 + 2 * NSLOT + 3 * NQT + t); };  // P_t keys 64..127, O ready
  auto BAR_O = [&](int t) { return bar0 + 8u * (1 + 2 * NSLOT + 4 * NQT + t); };
  const uint32_t BAR_DRAIN = bar0 + 8u * (1 + 2 * NSLOT + 5 * NQT);
  auto BAR_F8_FULL = [&](int i) { return bar0 + 8u * (2 + 2 * NSLOT + 5 * NQT + i); };
  auto BAR_F8_EMPTY = [&](int i) { return bar0 + 8u * (2 + 2 * NSLOT + 5 * NQT + NSLOT8 + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item.  KV head outermost so that the CTAs resident at one time
  // share the same K/V in L2; inside it the heaviest query blocks first
  // (causal work grows with the block index), then the G query heads of the
  // group and the KV splits.
  long long x = blockIdx.x;
  const int sigma = (int)(x % p.S);
  x /= p.S;
  const int g_iter = p.gpack > 1 ? 1 : p.G;  // packed tiles hold the whole group
  const int g = (int)(x % g_iter);
  x /= g_iter;
  const int qblk = p.n_qblk - 1 - (int)(x % p.n_qblk);
  x /= p.n_qblk;
  const int hk = (int)(x % p.Hkv);
  const int b = (int)(x / p.Hkv);
  const int h = hk * p.G + g;

  QTile qt[NQT];
  const long long qk_delta = p.q_pos0 - p.k_pos0;
#pragma unroll
  for (int t = 0; t < NQT; ++t) qt[t] = make_qtile<NQT>(qblk, t, p.N_q, qk_delta, p.tpt, p.gshift);
  // Keys past the block's last query position are invisible to every row.
  int kmax_last = qt[0].kmax;
#pragma unroll
  for (int t = 1; t < NQT; ++t)
    if (qt[t].nv > 0) kmax_last = qt[t].kmax;
  int lim = (int)p.N_kv;
  if (p.causal) lim = max(0, min(lim, kmax_last + 1));
  if (WA && threadIdx.x == 0) {
    // Square prefill: query t sits at position t, key j at j.  Published by
    // the set-up barrier below.
    s_wa.W = p.wa_window;
    s_wa.lo = max(0, qt[0].kmin - p.wa_window);
    s_wa.hi = kmax_last;
    const int a = (qt[0].tok0 / p.wa_period) * p.wa_period;
    s_wa.a0 = a;
    s_wa.am1 = a > 0 ? a - 1 : -1;
    s_wa.ap = (long long)a + p.wa_period < p.N_kv ? a + p.wa_period : -1;
  }
  const long long first_rel = qk_delta + qt[0].tok0;
  const int home = first_rel > 0 ? (int)min((long long)(p.P - 1), first_rel / p.chunk) : 0;
  const int s_begin = sigma * p.steps_per_split;
  const int s_end = min(p.P, s_begin + p.steps_per_split);

  // ---- set-up
  if (threadIdx.x == 0) {
    mbar_init(BAR_Q(), 1);
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(BAR_KV_FULL(i), kKV8 ? 4 : 1);  // FP8: one arrival per converter warp
      mbar_init(BAR_KV_EMPTY(i), 1);
    }
    for (int i = 0; i < NSLOT8; ++i) {
      mbar_init(BAR_F8_FULL(i), 1);
      mbar_init(BAR_F8_EMPTY(i), 4);
    }
    for (int t = 0; t < NQT; ++t) {
      // One arrival per softmax warp that holds valid rows.
      const int active_warps = min(4, (qt[t].nv + 31) / 32);
      mbar_init(BAR_S(t), 1);
      mbar_init(BAR_SC(t), max(1, active_warps));
      mbar_init(BAR_PA(t), max(1, active_warps));
      mbar_init(BAR_PB(t), max(1, active_warps));
      mbar_init(BAR_O(t), 1);
    }
    mbar_init(BAR_DRAIN, 1);
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

  // Two query tiles: registers move from the producer/MMA warpgroup to the
  // softmax warpgroups at the head of each role's branch.  The block is
  // launched with kLaunchRegs per thread (checked on the host before
  // launch): 128 * 88 + 256 * 208 = 384 * 168.
  if (warp < 4) {
    if constexpr (NQT == 2) reg_dealloc<kRegsControl>();
    if constexpr (kKV8) reg_dealloc<kRegsControl8>();
  }
  if (warp == 0) {
    // =========================== TMA producer ===========================
    if (lane == 0 && !p.skip_loads) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_k);
      prefetch_tmap(&p.tm_v);
      uint32_t qbytes = 0;
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (qt[t].nv > 0) qbytes += L::kTileBytes;
      mbar_arrive_expect_tx(BAR_Q(), qbytes);
#pragma unroll
      for (int t = 0; t < NQT; ++t) {
        if (qt[t].nv == 0) continue;
#pragma unroll
        for (int hf = 0; hf < kHalves; ++hf)
          tma_load_4d(sbase + L::kQOff + t * L::kTileBytes + hf * (kTileM * 128), &p.tm_q, BAR_Q(), hf * 64, h,
                      qt[t].tok0, b);
      }
      KvCursor<WA> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t issued = 0;  // slot fills issued (2 per KV tile)
      bool ok = true;
      while (ok && cur.valid()) {
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
          const CUtensorMap* map = kv == 0 ? &p.tm_k : &p.tm_v;
          if constexpr (kKV8) {
            // Raw E4M3 tile (no swizzle) into the FP8 ring; the converters
            // fill the bf16 slot.
            const uint32_t slot8 = issued % NSLOT8;
            if (!mbar_wait(BAR_F8_EMPTY(slot8), ((issued / NSLOT8) & 1u) ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(BAR_F8_FULL(slot8), L::kF8Bytes);
            tma_load_4d(sbase + L::kF8Off + slot8 * L::kF8Bytes, map, BAR_F8_FULL(slot8), 0, hk, (int)cur.k0, b);
          } else {
            const uint32_t slot = issued % NSLOT;
            const uint32_t use = issued / NSLOT;
            if (!mbar_wait(BAR_KV_EMPTY(slot), (use & 1u) ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(BAR_KV_FULL(slot), L::kTileBytes);
#pragma unroll
            for (int hf = 0; hf < kHalves; ++hf)
              tma_load_4d(sbase + L::kKVOff + slot * L::kTileBytes + hf * (kTileN * 128), map, BAR_KV_FULL(slot),
                          hf * 64, hk, (int)cur.k0, b);
          }
          ++issued;
        }
        cur.next();
      }
      // Let the last fills land before the CTA can exit (normally already
      // consumed; this matters only when unwinding after a timeout).
      constexpr uint32_t kRing = kKV8 ? NSLOT8 : NSLOT;
      const uint32_t first = issued > kRing ? issued - kRing : 0;
      for (uint32_t f = first; f < issued; ++f) {
        volatile int no_abort = 0;
        if constexpr (kKV8)
          mbar_wait(BAR_F8_FULL(f % NSLOT8), (f / NSLOT8) & 1u, &no_abort);
        else
          mbar_wait(BAR_KV_FULL(f % NSLOT), (f / NSLOT) & 1u, &no_abort);
      }
      mbar_wait(BAR_Q(), 0, abort_flag);
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      bool ok = mbar_wait(BAR_Q(), 0, abort_flag);
      tc_fence_after();
      uint64_t qdesc[NQT];
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        qdesc[t] = smem_desc_sw128(sbase + L::kQOff + t * L::kTileBytes, 16, 1024);
      auto kv_addr = [&](uint32_t slot) { return sbase + L::kKVOff + slot * L::kTileBytes; };
      uint32_t n_seen[NQT];  // visible tiles of query tile t handled so far
      bool o_live[NQT];
#pragma unroll
      for (int t = 0; t < NQT; ++t) {
        n_seen[t] = 0;
        o_live[t] = (MODE == kModeState);
      }
      KvCursor<WA> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t j = 0;  // KV tile index
      if (ok && cur.valid()) {
        ok = mbar_wait(BAR_KV_FULL(0), 0, abort_flag);
        tc_fence_after();
        if (ok) {
#pragma unroll
          for (int t = 0; t < NQT; ++t)
            if (tile_visible<WA>(qt[t], cur.k0, cur.kend, p.causal)) {
              mma_qk<D, 0, 2>(tmem + 128 * t, qdesc[t], kv_addr(0));
              tc_commit(BAR_S(t));
            }
          tc_commit(BAR_KV_EMPTY(0));
        }
      }
      // Per query tile t and KV tile j (both visible), in issue order:
      //   [softmax read S(j)]  S(j+1) keys 64..127 -> S columns 64..127
      //                        (single-tile CTAs only: with two tiles the
      //                        other tile's work fills the tensor pipe)
      //   [P keys 0..63]       PV(j) keys 0..63
      //   [P keys 64..127]     PV(j) keys 64..127, then S(j+1) (keys 0..63
      //                        only if the other half went early) into the
      //                        S columns, after PV has read P.

      while (ok && cur.valid()) {
        KvCursor<WA> nxt = cur;
        nxt.next();
        const bool has_next = nxt.valid();
        const uint32_t vfill = 2 * j + 1, kfill = 2 * j + 2;
        const uint32_t vslot = vfill % NSLOT, kslot = kfill % NSLOT;
        ok = mbar_wait(BAR_KV_FULL(vslot), (vfill / NSLOT) & 1u, abort_flag);
        tc_fence_after();
        bool k_ready = false;
        auto wait_k = [&]() {
          if (!k_ready) {
            ok = mbar_wait(BAR_KV_FULL(kslot), (kfill / NSLOT) & 1u, abort_flag);
            tc_fence_after();
            k_ready = true;
          }
          return ok;
        };
#pragma unroll
        for (int t = 0; t < NQT && ok; ++t) {
          const bool vc = tile_visible<WA>(qt[t], cur.k0, cur.kend, p.causal);
          const bool vn = has_next && tile_visible<WA>(qt[t], nxt.k0, nxt.kend, p.causal);
          if (vc) {
            const uint32_t par = n_seen[t] & 1u;
            ++n_seen[t];
            if (kSplitS && vn) {
              if (!wait_k()) break;
              if (!(ok = mbar_wait(BAR_SC(t), par, abort_flag))) break;
              tc_fence_after();
              mma_qk<D, 1, 2>(tmem + 128 * t, qdesc[t], kv_addr(kslot));
            }
            if (kSplitPV) {
              if (!(ok = mbar_wait(BAR_PA(t), par, abort_flag))) break;
              tc_fence_after();
              mma_pv<D, 0>(tmem + 128 * NQT + D * t, tmem + 128 * t, kv_addr(vslot), o_live[t]);
            }
            if (!(ok = mbar_wait(BAR_PB(t), par, abort_flag))) break;
            tc_fence_after();
            if (!kSplitPV) mma_pv<D, 0>(tmem + 128 * NQT + D * t, tmem + 128 * t, kv_addr(vslot), o_live[t]);
            mma_pv<D, 1>(tmem + 128 * NQT + D * t, tmem + 128 * t, kv_addr(vslot), true);
            o_live[t] = true;
            if (vn) {
              if (kSplitS) {
                mma_qk<D, 0, 1>(tmem + 128 * t, qdesc[t], kv_addr(kslot));
              } else {
                if (!wait_k()) break;
                mma_qk<D, 0, 2>(tmem + 128 * t, qdesc[t], kv_addr(kslot));
              }
              tc_commit(BAR_S(t));
            }
          } else if (vn) {
            // S_t is free: its last P was consumed by a PV issued earlier.
            if (!wait_k()) break;
            mma_qk<D, 0, 2>(tmem + 128 * t, qdesc[t], kv_addr(kslot));
            tc_commit(BAR_S(t));
          }
        }
        if (!ok) break;
        tc_commit(BAR_KV_EMPTY(vslot));
        if (has_next) {
          if (!wait_k()) break;  // every tile the cursor yields is visible to some query tile
          tc_commit(BAR_KV_EMPTY(kslot));
        }
        cur = nxt;
        ++j;
      }
#pragma unroll
      for (int t = 0; t < NQT; ++t) tc_commit(BAR_O(t));
      // Drain: all MMAs issued above have completed once this arrives.
      tc_commit(BAR_DRAIN);
      volatile int no_abort = 0;
      mbar_wait(BAR_DRAIN, 0, &no_abort);
    }
  } else if (kKV8 && warp >= 4 + 4 * NQT) {
    // ============================ FP8 converters ============================
    if constexpr (kKV8) {
      reg_dealloc<kRegsConvert8>();
      const int ct = (int)threadIdx.x - (128 + 128 * NQT);
      KvCursor<WA> cur;
      cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
      uint32_t f = 0;  // fills converted, in the producer's order (K_j, V_j, ...)
      bool ok = true;
      while (ok && cur.valid()) {
        for (int kv = 0; kv < 2; ++kv) {
          const uint32_t slot8 = f % NSLOT8, slot = f % NSLOT;
          if (!(ok = mbar_wait(BAR_F8_FULL(slot8), (f / NSLOT8) & 1u, abort_flag))) break;
          if (!(ok = mbar_wait(BAR_KV_EMPTY(slot), ((f / NSLOT) & 1u) ^ 1u, abort_flag))) break;
          convert_fp8_tile<D>(smem + L::kF8Off + slot8 * L::kF8Bytes, smem + L::kKVOff + slot * L::kTileBytes, ct);
          // The bf16 tile is read by the tensor cores (async proxy).
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
  } else if (warp >= 4) {
    // ========================= softmax warpgroups =========================
    if constexpr (NQT == 2) reg_alloc<kRegsSoftmax>();
    if constexpr (kKV8) reg_alloc<kRegsSoftmax8>();
    const int t = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int rloc = quad * 32 + lane;  // row inside the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + 128 * t;
    const uint32_t o_tmem = tmem + lane_base + 128 * NQT + D * t;
    const QTile q = make_qtile<NQT>(qblk, t, p.N_q, p.q_pos0 - p.k_pos0, p.tpt, p.gshift);
    const bool row_valid = rloc < q.nv;
    const int tl = rloc >> p.gshift;                   // token inside the tile
    const int head = h + (rloc & (p.gpack - 1));       // query head of this row
    const long long row = (long long)q.tok0 + tl;      // token in the q buffer
    // Warps whose 32 rows are all empty (short incremental queries) sit out.
    const bool warp_active = quad * 32 < q.nv;
    // With scale > 0 the row max is taken on raw scores and the scale is
    // folded into the exponent's FMA; otherwise scores are scaled first.
    // FP8 KV cache: k = code * k_scale folds into the score scale, v = code *
    // v_scale into the final normalisation.
    // The decoded tiles hold code values times 2^-120: the scores come back
    // up through the score scale (finite while scale * k_scale < 177), the
    // output through the epilogue (O * 2^120 first, then v_scale / l).
    const float k_mul = kKV8 ? p.k_scale[b * p.Hkv + hk] * kFp8Bias : 1.f;
    const float v_mul = kKV8 ? p.v_scale[b * p.Hkv + hk] : 1.f;
    const float scale_l2 = p.scale_log2 * k_mul;
    const bool fold = scale_l2 > 0.f;
    const float sl = fold ? scale_l2 : 1.f;

    // m2: the base of the exponentials (log2 units); it trails the true row
    // max by at most kRescaleSlack, so exp2(x - m2) <= 2^kRescaleSlack and O
    // needs rescaling only when the max jumps past that.  O, l and m2 always
    // describe the same sum, so the final out and lse are exact.
    float m2 = -INFINITY, l = 0.f, m_in_nat = -INFINITY;
    const long long srow = ((long long)b * p.Hq + head) * p.N_q + (row_valid ? row : 0);
    if (MODE == kModeState) {
      if (row_valid) {
        m_in_nat = p.m_state[srow];
        m2 = m_in_nat * kLog2e;
        l = p.l_state[srow];
      }
#pragma unroll
      for (int c = 0; c < D / 32 && warp_active; ++c) {
        uint32_t u[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          u[i] = row_valid ? __float_as_uint(p.acc[srow * D + c * 32 + i]) : 0u;
        tmem_st32(o_tmem + c * 32, u);
      }
      tc_wait_st();
    }
    const float m2_in = m2;
    float m_true = m2;  // true running max (kept for the state epilogue)

    KvCursor<WA> cur;
    cur.init((int)p.chunk, lim, p.P, home, s_begin, s_end);
    uint32_t n = 0;
    bool ok = true;
    while (warp_active && cur.valid()) {
      if (tile_visible<WA>(q, cur.k0, cur.kend, p.causal)) {
        if (!mbar_wait(BAR_S(t), n & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float (&r)[32] = *reinterpret_cast<float(*)[32]>(&s[c * 32]);
          tmem_ld32(s_tmem + c * 32, r);
        }
        tc_wait_ld();
        // S is in registers: the issuer may now overwrite its columns 64..127
        // with the next tile's scores (the first 64 columns get P).
        if constexpr (kSplitS) warp_arrive_after_tc(BAR_SC(t), lane);
        if (!fold) {
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] *= scale_l2;
        }
        const bool masked = tile_needs_mask<WA>(q, cur.k0, cur.kend, p.causal);
        if (WA && masked) {
          // This row's window [pos - W, pos] and the CTA's anchors, inside
          // the keys of this tile (tile-relative).
          const int kvis = cur.kend - cur.k0;
          const int pos = q.kmin + tl;
          const int kf = max(0, pos - s_wa.W - cur.k0);
          const int kl = min(kvis - 1, pos - cur.k0);
          // 128 visibility bits for this row: the window [kf, kl], then
          // the anchors that fall inside the tile's keys.
          uint32_t vm[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int lo = min(max(kf - 32 * w, 0), 32), hi = min(max(kl + 1 - 32 * w, 0), 32);
            vm[w] = hi > lo ? (uint32_t)((((1ull << hi) - 1ull) >> lo) << lo) : 0u;
          }
          const int xs[3] = {s_wa.a0 - cur.k0, s_wa.am1 - cur.k0, s_wa.ap - cur.k0};
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            const int x = xs[i];
            const bool in = (i == 0 || (i == 1 ? s_wa.am1 >= 0 : s_wa.ap >= 0)) && x >= 0 && x < kvis;
#pragma unroll
            for (int w = 0; w < 4; ++w) vm[w] |= (in && (x >> 5) == w) ? (1u << (x & 31)) : 0u;
          }
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = ((vm[c >> 5] >> (c & 31)) & 1u) ? s[c] : -INFINITY;
        } else if (masked) {
          const int kvis = cur.kend - cur.k0;  // keys inside the chunk / range
          // Last key (tile-relative) this row sees under causal masking.
          const long long kc = p.causal ? (long long)q.kmin + tl - cur.k0 : (long long)kTileN;
          const int kcausal = (int)(kc < -1 ? -1 : (kc > kTileN ? kTileN : kc));
          const int klast = min(kvis - 1, kcausal);
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = (c <= klast) ? s[c] : -INFINITY;
        }
        // After a row's first tile the exponentials use the current base m2
        // directly: every P <= 2^kRescaleSlack exactly when the row sum is,
        // and only a larger sum (rare) makes the tile compute its max and,
        // if the max did jump past the slack, redo P with a new base before
        // P is published.  A row's first tile, and single-tile CTAs (which
        // publish half of P early), take the max first.
        auto row_max = [&]() {
          // Four independent chains of 3-input max.
          float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
          for (int c = 4; c < 128; c += 8) {
            mx0 = fmax3(mx0, s[c], s[c + 1]);
            mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
            mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
            mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
          }
          return fmax3(fmaxf(mx0, mx1), mx2, mx3) * sl;  // -inf stays -inf (sl > 0)
        };
        auto compute_p = [&](float base) {
          // P in two halves (published separately for single-tile CTAs).
          // Unmasked tiles may evaluate part of their exponentials on the
          // FMA pipe; masked tiles use ex2 so masked keys give exactly 0.
          float r = masked ? softmax_p_half<0, 0>(s, sl, base, s_tmem)
                           : softmax_p_half<kExp2PolyMask, 0>(s, sl, base, s_tmem);
          if constexpr (kSplitPV) {
            tc_wait_st();
            warp_arrive_after_tc(BAR_PA(t), lane);
          }
          r += masked ? softmax_p_half<0, 1>(s, sl, base, s_tmem)
                      : softmax_p_half<kExp2PolyMask, 1>(s, sl, base, s_tmem);
          return r;
        };
        // After a row's first tile, P is computed directly with the current
        // base m2.  Every entry of P is <= 2^kRescaleSlack whenever the row
        // sum is, so only a larger sum (rare) makes the tile compute its max;
        // if that max did pass m2 + slack, O and l are rescaled and P is
        // redone with the new base before it is published.  A row's first
        // tile, and single-tile CTAs (which publish half of P early), take
        // the max first.
        float rs = 0.f;
        float alpha = 1.f;
        bool max_first = kSplitPV || n == 0 || __any_sync(0xffffffffu, m2 == -INFINITY);
        bool redo = max_first;
        if (!max_first) {
          rs = compute_p(m2);
          if (__any_sync(0xffffffffu, !(rs <= kSlackSum))) {
            const float m_tile = row_max();
            m_true = fmaxf(m_true, m_tile);
            if (m_tile > m2 + kRescaleSlack) {
              alpha = ex2(m2 - m_tile);
              m2 = m_tile;
              l *= alpha;
            }
            redo = __any_sync(0xffffffffu, alpha != 1.f);
          } else if (MODE == kModeState) {
            m_true = fmaxf(m_true, row_max());  // to hand the state back at the true max
          }
        } else {
          const float m_tile = row_max();
          m_true = fmaxf(m_true, m_tile);
          if (m_tile > m2 + kRescaleSlack) {
            alpha = ex2(m2 - m_tile);  // 0 when m2 = -inf
            m2 = m_tile;
            l *= alpha;
          }
        }
        if (redo) {
          // O must be rescaled before P is published: PV accumulates into it.
          const bool o_has_data = (MODE == kModeState) || n > 0;
          if (o_has_data && __any_sync(0xffffffffu, alpha != 1.f)) {
            // Rare (the max must jump past the slack): one 32-column chunk at
            // a time, in place, while the scores still occupy registers.
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              float r[32];
              tmem_ld32(o_tmem + c * 32, r);
              tc_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] *= alpha;
              tmem_st32(o_tmem + c * 32, *reinterpret_cast<const uint32_t(*)[32]>(r));
            }
          }
          rs = compute_p((m2 == -INFINITY) ? 0.f : m2);
        }
        tc_wait_st();
        warp_arrive_after_tc(BAR_PB(t), lane);
        l += rs;
        ++n;
      }
      cur.next();
    }

    // ------------------------------ epilogue ------------------------------
    if (ok && n > 0) ok = mbar_wait(BAR_O(t), 0, abort_flag);
    if (ok && warp_active) {
      tc_fence_after();
      if (MODE == kModeFinal || MODE == kModeSplit) {
        const float inv = l > 0.f ? v_mul / l : 0.f;
        const long long ooff =
            (((long long)(MODE == kModeSplit ? sigma * p.B + b : b) * p.N_q + row) * p.Hq + head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float r[32];
          if (n > 0) {
            tmem_ld32(o_tmem + c * 32, r);
            tc_wait_ld();
            if constexpr (kKV8) {
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] *= kFp8Bias;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = 0.f;
          }
          if (!row_valid) continue;
          if (MODE == kModeSplit || p.out_f32) {
            float* dst = (MODE == kModeSplit ? p.o_part : static_cast<float*>(p.out)) + ooff + c * 32;
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
            p.lse_part[(((long long)sigma * p.B + b) * p.Hq + head) * p.N_q + row] = lse_v;
          else
            p.lse[((long long)b * p.Hq + head) * p.N_q + row] = lse_v;
        }
      } else if (n > 0) {  // kModeState with at least one visible tile
        // Hand back the state relative to the true running max.
        const float fix = (m_true > m2) ? ex2(m2 - m_true) : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float r[32];
          tmem_ld32(o_tmem + c * 32, r);
          tc_wait_ld();
          if (!row_valid) continue;
          float* dst = p.acc + srow * D + c * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(r[i] * fix, r[i + 1] * fix, r[i + 2] * fix, r[i + 3] * fix);
        }
        if (row_valid) {
          p.m_state[srow] = (m_true == m2_in) ? m_in_nat : m_true * kLn2;
          p.l_state[srow] = l * fix;
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

template <int D, int NQT, int NSLOT, int MODE, int NSLOT8 = 0, bool WA = false>
cudaError_t launch_cfg(const Sm100Params& prm, long long grid, cudaStream_t st) {
  using L = Layout<D, NQT, NSLOT, NSLOT8>;
  auto kern = fwd_sm100_kernel<D, NQT, NSLOT, MODE, NSLOT8, WA>;
  static_assert(L::kAlloc <= 232448, "shared memory budget exceeded");
  constexpr int kThreads = 128 + 128 * NQT + (NSLOT8 > 0 ? 128 : 0);
  if constexpr (NQT == 2 || NSLOT8 > 0) {
    // The in-kernel register split assumes exactly kLaunchRegs per thread.
    static int regs = -1;
    if (regs < 0) {
      cudaFuncAttributes fa;
      cudaError_t e0 = cudaFuncGetAttributes(&fa, kern);
      if (e0 != cudaSuccess) return e0;
      regs = fa.numRegs;
    }
    if (regs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  }
  // The attribute is per device: set it on every device this instance runs on.
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
  kern<<<(unsigned)grid, kThreads, L::kAlloc, st>>>(prm);
  return count_launch(cudaGetLastError());
}

// FP8 codes, one row of d bytes per (token, head): 128-key boxes, 128-byte
// swizzled at d = 128 (the converters read them conflict-free), plain at
// d = 64.
CUresult encode_map_u8(CUtensorMap* m, const void* base, int d, int H, long long N, int B) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return CUDA_ERROR_NOT_FOUND;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d, (cuuint64_t)H * d, (cuuint64_t)N * H * d};
  cuuint32_t box[4] = {(cuuint32_t)d, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_map(CUtensorMap* m, const void* base, int d, int H, long long N, int B, int box_heads = 1) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return CUDA_ERROR_NOT_FOUND;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)N * H * d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_heads, (cuuint32_t)(128 / box_heads), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace

Sm100Geometry sm100_geometry(const ProblemArgs& a, int mode) {
  Sm100Geometry g;
  const int G = a.Hq / a.Hkv;
  // Pack the G query heads of a KV head into one tile when all of a KV
  // head's query rows fit: one CTA then streams that KV once for the group.
  const bool pack = mode != kModeState && G > 1 && (128 % G) == 0 && a.N_q * G <= kTileM;
  g.gpack = pack ? G : 1;
  g.gshift = 0;
  while ((1 << g.gshift) < g.gpack) ++g.gshift;
  g.tpt = kTileM / g.gpack;
  // Two query tiles per CTA share each K/V tile (not with an FP8 cache,
  // whose CTAs carry a converter warpgroup instead).
  g.two = a.N_q * g.gpack > kTileM && !a.kv8;
  const long long tok_per_cta = (long long)(g.two ? 2 : 1) * g.tpt;
  g.n_qblk = (int)((a.N_q + tok_per_cta - 1) / tok_per_cta);
  g.ctas_per_split = (long long)g.n_qblk * a.B * a.Hkv * (pack ? 1 : G);
  return g;
}

cudaError_t launch_fwd_sm100(const ProblemArgs& a, int mode, cudaStream_t st) {
  if (a.B <= 0 || a.N_q <= 0) return cudaSuccess;
  if (decode_rows(a, mode) > 0) return launch_decode_sm100(a, mode, st);
  const Sm100Geometry geo = sm100_geometry(a, mode);
  if (geo.two && fwd2_applies(a, mode)) return launch_fwd2_sm100(a, mode, st);
  Sm100Params prm;
  memset(&prm, 0, sizeof(prm));
  if (encode_map(&prm.tm_q, a.q, a.d, a.Hq, a.N_q, a.B, geo.gpack) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (a.kv8) {
    if (mode == kModeState || encode_map_u8(&prm.tm_k, a.k, a.d, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS ||
        encode_map_u8(&prm.tm_v, a.v, a.d, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    prm.k_scale = a.k_scale;
    prm.v_scale = a.v_scale;
  } else if (encode_map(&prm.tm_k, a.k, a.d, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS ||
             encode_map(&prm.tm_v, a.v, a.d, a.Hkv, a.N_kv, a.B) != CUDA_SUCCESS) {
    return cudaErrorInvalidValue;
  }
  prm.out = a.out;
  prm.lse = a.lse;
  prm.o_part = a.o_part;
  prm.lse_part = a.lse_part;
  prm.acc = a.acc;
  prm.m_state = a.m;
  prm.l_state = a.l;
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
  prm.out_f32 = a.out_f32;
  prm.gpack = geo.gpack;
  prm.gshift = geo.gshift;
  {
    // Host-side fault injection for the failure-detection test (see ringattn.cu).
    const char* f = std::getenv("RINGATTN_FAULT");
    prm.skip_loads = (f && std::strcmp(f, "device_wait") == 0) ? 1 : 0;
  }
  prm.tpt = geo.tpt;
  prm.n_qblk = geo.n_qblk;
  prm.wa_window = a.wa_window;
  prm.wa_period = a.wa_period;
  const bool two = geo.two;
  const long long grid = geo.ctas_per_split * prm.S;
  // K/V ring depth: as many 128-key slots as shared memory allows
  // (d=128: 2 query tiles + 5 slots = 224 KB; 1 tile + 6 slots).
#define RA_LAUNCH(D_, NQT_, NS_)                                                  \
  switch (mode) {                                                               \
    case kModeFinal: return launch_cfg<D_, NQT_, NS_, kModeFinal>(prm, grid, st); \
    case kModeSplit: return launch_cfg<D_, NQT_, NS_, kModeSplit>(prm, grid, st); \
    default: return launch_cfg<D_, NQT_, NS_, kModeState>(prm, grid, st);        \
  }
  if (a.wa_period > 0) {
    // Window-and-anchor mask: square prefill, one launch.
    if (mode != kModeFinal) return cudaErrorInvalidValue;
    if (a.d == 64) {
      if (two) return launch_cfg<64, 2, 8, kModeFinal, 0, true>(prm, grid, st);
      return launch_cfg<64, 1, 8, kModeFinal, 0, true>(prm, grid, st);
    }
    if (two) return launch_cfg<128, 2, 5, kModeFinal, 0, true>(prm, grid, st);
    return launch_cfg<128, 1, 6, kModeFinal, 0, true>(prm, grid, st);
  }
  if (a.kv8) {
    // One query tile, bf16 ring, FP8 ring (d=128: 32 + 4 x 32 + 4 x 16 = 224 KB).
    if (a.d == 64) {
      if (mode == kModeFinal) return launch_cfg<64, 1, 6, kModeFinal, 8>(prm, grid, st);
      return launch_cfg<64, 1, 6, kModeSplit, 8>(prm, grid, st);
    }
    if (mode == kModeFinal) return launch_cfg<128, 1, RA_KV8_NSLOT, kModeFinal, RA_KV8_NSLOT8>(prm, grid, st);
    return launch_cfg<128, 1, RA_KV8_NSLOT, kModeSplit, RA_KV8_NSLOT8>(prm, grid, st);
  }
  if (a.d == 64) {
    if (two) { RA_LAUNCH(64, 2, 8) } else { RA_LAUNCH(64, 1, 8) }
  } else {
    if (two) { RA_LAUNCH(128, 2, 5) } else { RA_LAUNCH(128, 1, 6) }
  }
#undef RA_LAUNCH
}

}  // namespace ra
