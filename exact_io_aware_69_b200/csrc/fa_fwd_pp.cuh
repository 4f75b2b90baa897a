// fa_fwd_pp.cuh -- exact attention forward for sm_100a, two query tiles per CTA.
//
// One CTA owns two consecutive 128-row query tiles of one (batch, head) and walks the
// key/value tiles they see, block by block, with the online softmax of josueisai.com
// "flash-attention", section "El truco: trocear y llevar la cuenta del softmax": per
// row a running maximum m and running sum l; when m grows the partial output is
// rescaled, and after the last block the output is divided by l once. The score and
// probability tiles live only in tensor memory (TMEM); every K and V tile is read
// from HBM (or L2) once per CTA and used by both query tiles.
//
// Warp roles (384 threads = 3 warpgroups; at launch every thread may hold 168
// registers, then warpgroup 2 hands registers to warpgroups 0 and 1 with setmaxnreg):
//   warps 0-3  softmax of query tile 0 (warpgroup 0), warps 4-7 of query tile 1
//              (warpgroup 1): thread r of a warpgroup owns query row r (TMEM lane r)
//              and the whole 128-column score row, so its row maximum needs no
//              exchange between threads.
//   warp 8     TMA producer: both Q tiles once, then K_j into a 3-stage ring and V_j
//              into a 2-stage ring, K one tile ahead of V.
//   warps 10-11 idle (they complete warpgroup 2, which runs on 56 registers).
//   warp 9     MMA issuer and TMEM owner, in the order
//                S0_j0 S1_j0 | PV0_j0 S0_j0+1 PV1_j0 S1_j0+1 | PV0_j0+1 S0_j0+2 ...
//              so that while one warpgroup exponentiates its scores the tensor core
//              multiplies the other's (ping-pong): the two warps that share a
//              sub-partition are never in the same phase, and MUFU (exp2) and the
//              tensor pipe work at once.
//
// TMEM (512 columns at d = 128): S/P of warpgroup 0 at column 0, of warpgroup 1 at
// column 128, O of warpgroup 0 at 256, O of warpgroup 1 at 256 + d. S_g,j+1 is issued
// after PV_g,j (which reads P_g,j from the same columns); tcgen05 MMAs of one thread run
// in issue order, so when S_g,j+1 has completed, PV_g,j has too, and O_g may be
// rescaled without a further wait.
//
// Scores are kept in the base-2 domain: s' = s * scale * log2(e), p = 2^(s' - m'). The
// running reference m' is only moved when the row maximum exceeds it by more than
// kRescaleSlack (so exponentials stay <= 2^kRescaleSlack); the result is the same
// because l, O and L all share whatever reference is current. Two row sums are kept:
// l_o adds up the 16-bit-rounded p, the very values the P V product multiplies, and
// normalises O, so that O is an exact convex combination of V rows with those weights;
// l adds up the unrounded p and gives L, the log-sum-exp of the scores themselves.
//
// Optional second output O_res: the rounding residual of O in the same 16-bit type,
// O_res = dtype(O_fp32 - O). O + O_res carries O to about 2^-17 relative, and the
// backward uses it for D = rowsum(dO * O).
#pragma once

#include <type_traits>

#include "fa_band.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kPpThreads = 384;
constexpr int kPpProducerWarp = 8;
constexpr int kPpMmaWarp = 9;
// Registers per thread: 168 at launch (the most 384 threads can have: each
// sub-partition holds one warp of each warpgroup and 16K registers); then
// 2 x 224 (softmax) + 56 (producer, MMA) = 3 x 168 per sub-partition.
constexpr int kPpLaunchRegs = 168;
constexpr int kPpSoftmaxRegs = 224;
constexpr int kPpSmallRegs = 56;
static_assert(2 * kPpSoftmaxRegs + kPpSmallRegs == 3 * kPpLaunchRegs, "register split");
constexpr float kPpRescaleSlack = 8.0f;
// Of every 16 exponential pairs of a softmax thread, how many go to the FMA pipe on
// tiles without a mask (a power of two up to 16; 0 = MUFU only).
#ifndef FA_PP_POLY_PAIRS
#define FA_PP_POLY_PAIRS 2
#endif
// At d = 64 (half the MMA work per key tile) its own count: there the polynomial's
// extra issue slots cost more than the MUFU time it saves (B1 H16 N16384 d64 non-causal
// on one box, 0 / 2 / 4 / 8 pairs: 1.603 / 1.667 / 1.723 / 1.866 ms), so MUFU only.
#ifndef FA_PP_POLY_PAIRS_D64
#define FA_PP_POLY_PAIRS_D64 0
#endif
static_assert(FA_PP_POLY_PAIRS >= 0 && FA_PP_POLY_PAIRS <= 16 &&
                  (FA_PP_POLY_PAIRS & (FA_PP_POLY_PAIRS - 1)) == 0 && FA_PP_POLY_PAIRS_D64 >= 0 &&
                  FA_PP_POLY_PAIRS_D64 <= 16 && (FA_PP_POLY_PAIRS_D64 & (FA_PP_POLY_PAIRS_D64 - 1)) == 0,
              "poly pairs: a power of two up to 16, or 0");
#ifndef FA_PP_RES_IN_K
#define FA_PP_RES_IN_K 1
#endif
constexpr int kPpKStages = 3;
constexpr int kPpVStages = 2;

template <int D>
struct PpLayout {
  static constexpr uint32_t kTileBytes = kTile * D * 2;  // 128 rows x D 16-bit values
  static constexpr uint32_t kChunkBytes = kTile * 128;   // 128 rows x 64 values
  static constexpr uint32_t kQ = 0;                      // 2 tiles
  static constexpr uint32_t kK = kQ + 2 * kTileBytes;
  static constexpr uint32_t kV = kK + kPpKStages * kTileBytes;
  static constexpr uint32_t kBar = kV + kPpVStages * kTileBytes;
  static constexpr int kNumBars = 20;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 8;
  static constexpr uint32_t kBytes = kAbort + 8 + 1024;  // + alignment slack
  static constexpr uint32_t tS = 0;                       // + 128 * warpgroup
  static constexpr uint32_t tO = 256;                     // + D * warpgroup
};

enum : int {
  kPbQFull = 0,                            // both Q tiles
  kPbKFull = 1,                            // + K stage
  kPbKEmpty = kPbKFull + kPpKStages,       // + K stage
  kPbVFull = kPbKEmpty + kPpKStages,       // + V stage
  kPbVEmpty = kPbVFull + kPpVStages,       // + V stage
  kPbSFull = kPbVEmpty + kPpVStages,       // + warpgroup
  kPbPFull = kPbSFull + 2,                 // + warpgroup (128 arrivals): all of P_g,j
  kPbPHalf = kPbPFull + 2,                 // + warpgroup (128 arrivals): P_g,j of keys 0-63
  kPbODone = kPbPHalf + 2,                 // + warpgroup: its last P V has completed
  kPpNumBars = kPbODone + 2,
};
static_assert(kPpNumBars <= 20, "barrier area");

// BAND = false: every key visible (but the end of a ragged last key
// tile); true = the key window [wl, wr] around the bottom-right diagonal. Tensors are
// seen through 4-D tensor maps (column, row, head, batch); L is [B][H][Nq].
template <int D, bool BAND, bool BF16>
__global__ void __launch_bounds__(kPpThreads, 1)
    fa_fwd_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const __grid_constant__ CUtensorMap tmOres, bool has_res,
                     float* __restrict__ Lse, int Nq, int Nk, int H, int wl, int wr,
                     float scale_log2, int group) {
  using Lay = PpLayout<D>;
  constexpr int kPpPolyPairs = D == 64 ? FA_PP_POLY_PAIRS_D64 : FA_PP_POLY_PAIRS;
  constexpr int kPpPolyStride = kPpPolyPairs > 0 ? 16 / kPpPolyPairs : 16;
  // P_g,j V_j in two halves at d = 64 (see the MMA issuer)
  constexpr bool kPpSplitPV = D == 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;

  FA_TRACE_CTA(0);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntq = (Nq + kTile - 1) / kTile;  // query tiles per head
  const int ntk = (Nk + kTile - 1) / kTile;  // key / value tiles per head
  const int npairs = (ntq + 1) / 2;          // CTAs per head
  // band: heaviest pairs first, heads in groups (band_order); otherwise head-major
  int bh, pr;
  if (BAND) {
    band_order(blockIdx.x, npairs, gridDim.x / npairs, group, &bh, &pr);
  } else {
    bh = blockIdx.x / npairs;
    pr = blockIdx.x - bh * npairs;
  }
  const int hh = bh % H;
  const int bb = bh / H;
  const int pair = BAND ? (npairs - 1 - pr) : pr;  // causal: heaviest pairs first
  // Query tiles 2 pair and 2 pair + 1 (the second may not exist when ntq is odd), and
  // the key tiles each one visits: R_g = [a_g, a_g + n_g).
  int a[2], n[2];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const int t = 2 * pair + g;
    const TileRange r = t >= ntq ? TileRange{0, 0}
                        : BAND   ? kv_tiles_of_query_tile(t, kTile, Nq, Nk, wl, wr)
                                 : TileRange{0, ntk};
    a[g] = r.first;
    n[g] = r.count;
  }
  // The tiles the CTA loads: the union of the two ranges, which is contiguous (two
  // adjacent query tiles' windows overlap or touch).
  const int J0 = n[0] == 0 ? a[1] : (n[1] == 0 ? a[0] : min(a[0], a[1]));
  const int J1 = max(n[0] ? a[0] + n[0] : 0, n[1] ? a[1] + n[1] : 0);  // one past the last
  const int nj = n[0] + n[1] == 0 ? 0 : J1 - J0;
  const int off = Nk - Nq;
  const int last_keys = Nk - (ntk - 1) * kTile;  // valid keys in the last KV tile
  // per-warpgroup ranges as scalars (a runtime index into a[] would live in memory)
  const int a0 = a[0], n0 = n[0], a1 = a[1], n1 = n[1];

  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kAbort);
  auto first_of = [&](int g) -> int { return g ? a1 : a0; };
  auto count_of = [&](int g) -> int { return g ? n1 : n0; };
  auto in_range = [&](int g, int j) -> bool {
    return j >= first_of(g) && j < first_of(g) + count_of(g);
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(kPbQFull), 1);
    for (int s = 0; s < kPpKStages; ++s) {
      mbar_init(bar(kPbKFull + s), 1);
      mbar_init(bar(kPbKEmpty + s), 1);
    }
    for (int s = 0; s < kPpVStages; ++s) {
      mbar_init(bar(kPbVFull + s), 1);
      mbar_init(bar(kPbVEmpty + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(kPbSFull + g), 1);
      mbar_init(bar(kPbPFull + g), 128);
      mbar_init(bar(kPbPHalf + g), 128);
      mbar_init(bar(kPbODone + g), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kPpMmaWarp) {
    tmem_alloc(sbase + Lay::kTmemSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  FA_TRACE_BEGIN();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Lay::kTmemSlot);

  if (warp >= 8) setmaxnreg_dec<kPpSmallRegs>();  // every warp of warpgroup 2
  if (warp == kPpProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nj > 0) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      // Only the Q tile of a warpgroup that visits a key tile is loaded: one that visits
      // none stages its (zero) output in its Q buffer without waiting for anything.
      mbar_expect_tx(bar(kPbQFull), ((n0 > 0) + (n1 > 0)) * Lay::kTileBytes);
      for (int g = 0; g < 2; ++g)
        if (count_of(g) > 0)
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sbase + Lay::kQ + g * Lay::kTileBytes + c * Lay::kChunkBytes, &tmQ,
                        c * 64, (2 * pair + g) * kTile, hh, bb, bar(kPbQFull));
      // step s loads K of tile J0 + s and V of tile J0 + s - 1
      for (int step = 0; step <= nj; ++step) {
        if (step < nj) {
          const int ks = step % kPpKStages;
          if (step >= kPpKStages &&
              !mbar_wait(bar(kPbKEmpty + ks), static_cast<uint32_t>(step / kPpKStages - 1) & 1,
                         abort_flag))
            break;
          mbar_expect_tx(bar(kPbKFull + ks), Lay::kTileBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sbase + Lay::kK + ks * Lay::kTileBytes + c * Lay::kChunkBytes, &tmK,
                        c * 64, (J0 + step) * kTile, hh, bb, bar(kPbKFull + ks));
          FA_TRACE_EVENT(step, 10);
        }
        if (step >= 1) {
          const int i = step - 1;
          const int vs = i % kPpVStages;
          if (i >= kPpVStages &&
              !mbar_wait(bar(kPbVEmpty + vs), static_cast<uint32_t>(i / kPpVStages - 1) & 1,
                         abort_flag))
            break;
          mbar_expect_tx(bar(kPbVFull + vs), Lay::kTileBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sbase + Lay::kV + vs * Lay::kTileBytes + c * Lay::kChunkBytes, &tmV,
                        c * 64, (J0 + i) * kTile, hh, bb, bar(kPbVFull + vs));
          FA_TRACE_EVENT(i, 11);
        }
      }
    }
  } else if (warp == kPpMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0 && nj > 0) {
      constexpr uint32_t idesc_s = idesc_f16_f32(kTile, kTile, BF16, false, false);
      constexpr uint32_t idesc_o = idesc_f16_f32(kTile, D, BF16, false, true);
      bool ok = mbar_wait(bar(kPbQFull), 0, abort_flag);
      // step j (J0 <= j <= J1): P V of tile j - 1 and S of tile j, warpgroup 0 first
      for (int j = J0; ok && j <= J1; ++j) {
        const int i = j - J0;  // ring position of tile j
        bool v_waited = false;
        bool k_waited = false;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          if (in_range(g, j - 1)) {  // PV_g,j-1: O_g += P_g,j-1 V_j-1
            const int u = j - 1 - first_of(g);  // use count of this warpgroup's buffers
            // At d = 64 in two halves: keys 0-63 as soon as their P is in TMEM (the
            // softmax is then still on keys 64-127), keys 64-127 with the rest of P. At
            // d = 128 (twice the MMA work per key) the split measured no gain.
            if (!mbar_wait(bar((kPpSplitPV ? kPbPHalf : kPbPFull) + g), static_cast<uint32_t>(u) & 1,
                           abort_flag)) {
              ok = false;
              break;
            }
            const int vs = (i - 1) % kPpVStages;
            if (!v_waited &&
                !mbar_wait(bar(kPbVFull + vs), static_cast<uint32_t>((i - 1) / kPpVStages) & 1,
                           abort_flag)) {
              ok = false;
              break;
            }
            v_waited = true;
            tc_fence_after();
            const uint64_t dv = sdesc_sw128(sbase + Lay::kV + vs * Lay::kTileBytes,
                                            Lay::kChunkBytes, 1024);
            const uint32_t a_p = tmem + Lay::tS + g * 128;  // P packed in 64 columns
            const uint32_t d_o = tmem + Lay::tO + g * D;
#pragma unroll
            for (int k = 0; k < kTile / 32; ++k)
              mma_ts(d_o, a_p + k * 8, sdesc_step(dv, k * 2048), idesc_o,
                     (u > 0 || k > 0) ? 1u : 0u);
            if (kPpSplitPV) {
              if (!mbar_wait(bar(kPbPFull + g), static_cast<uint32_t>(u) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
#pragma unroll
            for (int k = kTile / 32; k < kTile / 16; ++k)
              mma_ts(d_o, a_p + k * 8, sdesc_step(dv, k * 2048), idesc_o, 1u);
            if (j == first_of(g) + count_of(g)) mma_commit(bar(kPbODone + g));  // its last P V
            FA_TRACE_EVENT(i, 2 * g);
          }
          if (in_range(g, j)) {  // S_g,j = Q_g K_j^T
            const int ks = i % kPpKStages;
            if (!k_waited &&
                !mbar_wait(bar(kPbKFull + ks), static_cast<uint32_t>(i / kPpKStages) & 1,
                           abort_flag)) {
              ok = false;
              break;
            }
            k_waited = true;
            tc_fence_after();
            const uint64_t dq = sdesc_sw128(sbase + Lay::kQ + g * Lay::kTileBytes, 16, 1024);
            const uint64_t dk = sdesc_sw128(sbase + Lay::kK + ks * Lay::kTileBytes, 16, 1024);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t koff = (k >> 2) * Lay::kChunkBytes + (k & 3) * 32;
              mma_ss(tmem + Lay::tS + g * 128, sdesc_step(dq, koff), sdesc_step(dk, koff),
                     idesc_s, k > 0 ? 1u : 0u);
            }
            mma_commit(bar(kPbSFull + g));
            FA_TRACE_EVENT(i, 2 * g + 1);
          }
        }
        if (!ok) break;
        if (j < J1) mma_commit(bar(kPbKEmpty + i % kPpKStages));           // K_j read
        if (j > J0) mma_commit(bar(kPbVEmpty + (i - 1) % kPpVStages));     // V_j-1 read
      }
    }
  } else if (warp < 8) {
    // ----------------------------------------------------------------- softmax
    setmaxnreg_inc<kPpSoftmaxRegs>();
    const int g = warp >> 2;  // warpgroup = query tile 2 pair + g
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const int t = 2 * pair + g;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t s_cols = Lay::tS + g * 128;
    const uint32_t o_cols = Lay::tO + g * D;
    const int gbar = 1 + g;  // named barrier of this warpgroup
    const int ga = first_of(g), gn = count_of(g);
    float m = -INFINITY;     // running reference, base-2 scaled units
    float l = 0.f;           // row sum of p
    float l_o = 0.f;         // row sum of the 16-bit-rounded p
    const uint64_t c2 = f2_pack(scale_log2, scale_log2);
    bool ok = true;
    for (int u = 0; u < gn && ok; ++u) {
      const int jt = ga + u;  // key tile
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar(kPbSFull + g), static_cast<uint32_t>(u) & 1, abort_flag));
      if (!ok) break;
      if (r == 0) FA_TRACE_EVENT(u, 4 + 3 * g);
      tc_fence_after();
      float s[128];
      {
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + s_cols + c * 32, sr + c * 32);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) reg_fence32(sr + c * 32);
#pragma unroll
        for (int e = 0; e < 128; ++e) s[e] = __uint_as_float(sr[e]);
      }
      // band: key column c of the tile is visible to row r when
      // r + delta - wl <= c <= r + delta + wr; last tile: keys >= Nk are masked
      const int delta = t * kTile + off - jt * kTile;
      const bool hmask = BAND && delta + wr < kTile - 1;
      const bool lmask = BAND && delta - wl > -(kTile - 1);
      const bool kmask = jt == ntk - 1 && last_keys < kTile;
      if (hmask || lmask || kmask) {
        int hi = kmask ? last_keys - 1 : kTile - 1;
        if (hmask) hi = min(hi, r + delta + wr);
        const int lo = lmask ? r + delta - wl : 0;
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = (c > hi || c < lo) ? -INFINITY : s[c];
      }
      // row maximum over four independent chains (a single chain of 64 dependent
      // 3-input maxima would cost its whole latency)
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) mq[k] = fmax3(mq[k], s[c + 2 * k], s[c + 2 * k + 1]);
      }
      const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      if (r == 0) FA_TRACE_EVENT(u, 5 + 3 * g);
      const float cand = mx * scale_log2;
      const float m_new = (cand > m + kPpRescaleSlack) ? cand : m;
      // A row that sees no key keeps m = -inf: it takes alpha = 1 and subtracts 0, so
      // that its p = 2^-inf = 0 and no inf - inf appears.
      const bool empty_row = m_new == -INFINITY;
      const float alpha = empty_row ? 1.f : ex2_approx(m - m_new);  // 0 on the first tile
      const float m_sub = empty_row ? 0.f : m_new;
      const uint64_t nm2 = f2_pack(-m_sub, -m_sub);
      // O_g holds P_g,j-1 V_j-1 already (S_g,j completing implies it); it is rescaled,
      // only when a row's reference moved, before any of P_g,j V_j is issued: ahead of the
      // exponentials where the first half of P V goes at the PHalf signal, else after
      // them, where the TMEM round trip no longer delays the P stores
      auto rescale_o = [&]() {
        if (u > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + o_cols + c * 32, o);
            tmem_wait_ld();
            reg_fence32(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(lane_base + o_cols + c * 32, o);
          }
        }
      };
      if (kPpSplitPV) rescale_o();
      // packed fp32 pairs, two independent accumulators per sum (16-deep chains)
      uint64_t sum2[2] = {0, 0}, sum2_o[2] = {0, 0};  // packed +0.0f
      // Exponentials on MUFU; on tiles without a mask, kPpPolyPairs of every 16 pairs
      // on the FMA pipe instead (ex2_poly_pair), which shortens a warp's exponential
      // phase when it has its sub-partition's MUFU to itself. Masked tiles stay on
      // MUFU, which returns exact zeros for masked scores.
      auto exps = [&](auto poly_tag) {
        constexpr bool kPoly = decltype(poly_tag)::value;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int e = h * 32 + 2 * c;
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), c2, nm2), x0, x1);
            float p0, p1;
            if (kPoly && c % kPpPolyStride == kPpPolyStride - 1) {
              ex2_poly_pair(x0, x1, p0, p1);
            } else {
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            pk[c] = pack2<BF16>(p0, p1);
            float r0, r1;
            unpack2<BF16>(pk[c], r0, r1);
            sum2[c & 1] = f2_add(sum2[c & 1], f2_pack(p0, p1));
            sum2_o[c & 1] = f2_add(sum2_o[c & 1], f2_pack(r0, r1));
          }
          // P packed over the first 64 columns of the S buffer; this thread owns the
          // row, and all of S is in registers already
          tmem_st16(lane_base + s_cols + h * 16, pk);
          if (kPpSplitPV && h == 1) {  // keys 0-63 (and a rescaled O) in TMEM: their P V may go
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(kPbPHalf + g));
          }
        }
      };
      if (kPpPolyPairs > 0 && !(hmask || lmask || kmask))
        exps(std::integral_constant<bool, true>{});
      else
        exps(std::integral_constant<bool, false>{});
      float a0, a1, b0, b1;
      f2_unpack(f2_add(sum2[0], sum2[1]), a0, a1);
      f2_unpack(f2_add(sum2_o[0], sum2_o[1]), b0, b1);
      l = l * alpha + (a0 + a1);
      l_o = l_o * alpha + (b0 + b1);
      if (!kPpSplitPV) rescale_o();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kPbPFull + g));
      if (r == 0) FA_TRACE_EVENT(u, 6 + 3 * g);
      m = m_new;
    }
    // epilogue: O / l_o and O's rounding residual, staged in shared memory and written
    // with TMA stores. O goes to this warpgroup's Q tile (free: its last S MMA has
    // completed). O_res goes at the same time to the K stage of key tile J1 - 2 + g when
    // nothing touches that stage any more once this warpgroup's last P V has completed:
    // warpgroup 1's range must end at J1 (its last P V is then the CTA's last MMA) and
    // warpgroup 0's at J1 - 1 or J1 (its last P V then follows both S MMAs of tile
    // J1 - 2); no K load goes past tile J1 - 1. Otherwise O_res follows O through the
    // Q tile once O has left it.
    ok = __all_sync(0xffffffffu, ok && (gn == 0 || mbar_wait(bar(kPbODone + g), 0, abort_flag)));
    const bool live = t < ntq;
    ok = named_bar_and(gbar, 128, ok) && live;
    if (ok) {
      tc_fence_after();
      const float inv_l = l_o > 0.f ? 1.f / l_o : 0.f;  // rows that see no key: O = 0
      const uint32_t st = sbase + Lay::kQ + g * Lay::kTileBytes;
      const int res_tile = J1 - 2 + g;
      const bool res_k = FA_PP_RES_IN_K && has_res && gn > 0 && res_tile >= J0 &&
                         (g == 1 ? ga + gn == J1 : ga + gn >= J1 - 1);
      const uint32_t st_res =
          res_k ? sbase + Lay::kK + static_cast<uint32_t>((res_tile - J0) % kPpKStages) * Lay::kTileBytes
                : st;
      const int sw = r & 7;
      uint32_t lw[D / 2];  // O_res, kept until O has left shared memory (when st_res = st)
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (gn > 0) {  // with no KV tile, O in TMEM was never written
          tmem_ld32(lane_base + o_cols + c * 32, o);
          tmem_wait_ld();
          reg_fence32(o);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        uint32_t hw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = __uint_as_float(o[2 * e]) * inv_l;
          const float x1 = __uint_as_float(o[2 * e + 1]) * inv_l;
          hw[e] = pack2<BF16>(x0, x1);
          float h0, h1;
          unpack2<BF16>(hw[e], h0, h1);
          lw[c * 16 + e] = pack2<BF16>(x0 - h0, x1 - h1);  // exact difference, then rounded
        }
        const int col = c * 32;
        const uint32_t chunk = static_cast<uint32_t>(col / 64) * Lay::kChunkBytes + r * 128;
        const int u0 = (col % 64) / 8;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           st + chunk + static_cast<uint32_t>(((u0 + uu) ^ sw) * 16)),
                       "r"(hw[4 * uu]), "r"(hw[4 * uu + 1]), "r"(hw[4 * uu + 2]), "r"(hw[4 * uu + 3])
                       : "memory");
        if (res_k) {
#pragma unroll
          for (int uu = 0; uu < 4; ++uu)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             st_res + chunk + static_cast<uint32_t>(((u0 + uu) ^ sw) * 16)),
                         "r"(lw[c * 16 + 4 * uu]), "r"(lw[c * 16 + 4 * uu + 1]),
                         "r"(lw[c * 16 + 4 * uu + 2]), "r"(lw[c * 16 + 4 * uu + 3])
                         : "memory");
        }
      }
      fence_async_smem();
      if (t * kTile + r < Nq)
        Lse[static_cast<long>(bh) * Nq + t * kTile + r] =
            (m + log2f(l)) * 0.69314718055994530942f;
      named_bar_sync(gbar, 128);
      if (r == 0) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_store_4d(&tmO, st + c * Lay::kChunkBytes, c * 64, t * kTile, hh, bb);
        if (res_k) {
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_store_4d(&tmOres, st_res + c * Lay::kChunkBytes, c * 64, t * kTile, hh, bb);
        }
        bulk_commit();
        bulk_wait_read_all();  // the staging tiles are read before O_res overwrites O's
      }
      if (has_res && !res_k) {
        named_bar_sync(gbar, 128);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const int col = c * 32;
          const uint32_t chunk = static_cast<uint32_t>(col / 64) * Lay::kChunkBytes + r * 128;
          const int u0 = (col % 64) / 8;
#pragma unroll
          for (int uu = 0; uu < 4; ++uu)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             st + chunk + static_cast<uint32_t>(((u0 + uu) ^ sw) * 16)),
                         "r"(lw[c * 16 + 4 * uu]), "r"(lw[c * 16 + 4 * uu + 1]),
                         "r"(lw[c * 16 + 4 * uu + 2]), "r"(lw[c * 16 + 4 * uu + 3])
                         : "memory");
        }
        fence_async_smem();
        named_bar_sync(gbar, 128);
        if (r == 0) {
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_store_4d(&tmOres, st + c * Lay::kChunkBytes, c * 64, t * kTile, hh, bb);
          bulk_commit();
          bulk_wait_read_all();
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kPpMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  FA_TRACE_CTA(1);
}

}  // namespace fa
