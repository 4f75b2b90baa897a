// fa_fwd_d256.cuh -- exact attention forward for sm_100a at head dimension 256.
//
// The same method as fa_fwd_pp.cuh (josueisai.com "flash-attention", section "El truco:
// trocear y llevar la cuenta del softmax": per row a running maximum m and running sum
// l, the partial output rescaled when m grows, one division by l at the end), laid out
// for d = 256, where two query tiles' accumulators (2 x (128 + 256) columns) do not fit
// the 512 columns of tensor memory. One CTA owns one 128-row query tile of one
// (batch, head).
//
// Warp roles (352 threads):
//   warps 0-7  softmax, in pairs: warps w and w+4 share TMEM lane quarter w % 4, so
//              thread r of the pair's two warps owns query row r = 32 (w % 4) + lane;
//              warp w < 4 takes score columns 0-63 and O columns [0, 128), warp w+4
//              columns 64-127 and [128, 256). The pair exchanges its two partial row
//              maxima through shared memory once per key tile; each half keeps its
//              own partial row sums until the epilogue.
//   warp 8     TMA loads of Q (once) and of K_j (one 64 KB stage).
//   warp 10    TMA loads of V_j (one 64 KB stage).
//   warp 9     MMA issuer and TMEM owner, in the order S_0 | S_1 PV_0 | S_2 PV_1 | ...:
//              S_j = Q K_j^T (16 shared x shared MMAs over d) runs one key tile ahead
//              of O += P_j V_j (8 MMAs of N = 256, P from TMEM, V from shared memory).
//
// TMEM (512 columns x 128 lanes of 32 bit): score buffers at columns 0 and 128 (S_j in
// buffer j mod 2; P_j, packed 16-bit, over the first 64 columns of the same buffer),
// O at columns 256-511. tcgen05 MMAs of one thread run in issue order, so S_{j+2}
// overwrites P_j only after P_j V_j has read it.
//
// Shared memory: Q 64 KB, one K stage and one V stage of 64 KB each (d = 256 leaves no
// room for a second); the epilogue stages O in the K stage and O_res in the V stage.
//
// Scores in the base-2 domain with a lazily moved reference (kWRescaleSlack), the two
// row sums (l_o of the 16-bit-rounded p normalises O, l gives L) and the optional
// rounding residual O_res as in fa_fwd_pp.cuh.
#pragma once

#include "fa_band.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kWThreads = 352;
constexpr int kWKLoadWarp = 8;
constexpr int kWMmaWarp = 9;
constexpr int kWVLoadWarp = 10;
constexpr float kWRescaleSlack = 8.0f;
constexpr int kWD = 256;     // head dimension
constexpr int kWSBufs = 2;   // score buffers in TMEM

struct WideLayout {
  static constexpr uint32_t kTileBytes = kTile * kWD * 2;  // 128 rows x 256 16-bit values
  static constexpr uint32_t kChunkBytes = kTile * 128;     // 128 rows x 64 values (one swizzle column)
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTileBytes;
  static constexpr uint32_t kV = kK + kTileBytes;
  // [2 parity][2 half][128] fp32 row-maximum exchange; in the epilogue also the two
  // row sums of each half
  static constexpr uint32_t kRed = kV + kTileBytes;
  static constexpr uint32_t kBar = kRed + 2 * 2 * 2 * 128 * 4;
  static constexpr int kNumBars = 16;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 8;
  static constexpr uint32_t kBytes = kAbort + 8 + 1024;  // + alignment slack
  static constexpr uint32_t tO = kWSBufs * 128;          // O accumulator columns
  static_assert(tO + kWD <= 512, "score buffers and O must fit in TMEM");
};

// barrier indices
enum : int {
  kWbQFull = 0,
  kWbKFull = 1,
  kWbKEmpty = 2,
  kWbVFull = 3,
  kWbVEmpty = 4,
  kWbSFull = 5,                   // + score buffer
  kWbPFull = kWbSFull + kWSBufs,  // + score buffer (256 arrivals)
  kWbODone = kWbPFull + kWSBufs,  // + score buffer of the P that P V read
  kWNumBars = kWbODone + kWSBufs,
};
static_assert(kWNumBars <= 16, "barrier area");

// BAND = false: every key is visible (no mask but the end of a ragged last key tile);
// BAND = true: the key window [wl, wr] around the bottom-right diagonal (fa_band.cuh),
// the causal mask being wl = kUnbounded, wr = 0. Tensors are seen through 4-D tensor
// maps (column, row, head, batch); L is [B][H][Nq].
template <bool BAND, bool BF16>
__global__ void __launch_bounds__(kWThreads, 1)
    fa_fwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ CUtensorMap tmOres, bool has_res,
                       float* __restrict__ Lse, int Nq, int Nk, int H, int wl, int wr,
                       float scale_log2, int group) {
  constexpr int D = kWD;
  using Lay = WideLayout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;

  FA_TRACE_CTA(0);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntq = (Nq + kTile - 1) / kTile;  // query tiles per head (one CTA each)
  const int ntk = (Nk + kTile - 1) / kTile;  // key / value tiles per head
  // band: heaviest tiles first, heads in groups (band_order); otherwise head-major
  int bh, tr;
  if (BAND) {
    band_order(blockIdx.x, ntq, gridDim.x / ntq, group, &bh, &tr);
  } else {
    bh = blockIdx.x / ntq;
    tr = blockIdx.x - bh * ntq;
  }
  const int hh = bh % H;  // head
  const int bb = bh / H;  // batch
  const int t = BAND ? (ntq - 1 - tr) : tr;  // causal: heaviest tiles first
  // The key/value tiles this query tile visits: all of them, or the band's. A tile of
  // only rows that see no key visits none (O = 0, L = -inf).
  const TileRange kv = BAND ? kv_tiles_of_query_tile(t, kTile, Nq, Nk, wl, wr)
                            : TileRange{0, ntk};
  const int j0 = kv.first;
  const int nkv = kv.count;
  const int off = Nk - Nq;
  // Rows and keys of a last tile past Nq / Nk come in as zeros from the tensor maps;
  // the keys are masked below, the rows are not stored.
  const int last_keys = Nk - (ntk - 1) * kTile;  // valid keys in the last KV tile

  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar(kWbQFull), 1);
    mbar_init(bar(kWbKFull), 1);
    mbar_init(bar(kWbKEmpty), 1);
    mbar_init(bar(kWbVFull), 1);
    mbar_init(bar(kWbVEmpty), 1);
    for (int s = 0; s < kWSBufs; ++s) {
      mbar_init(bar(kWbSFull + s), 1);
      mbar_init(bar(kWbPFull + s), 256);
      mbar_init(bar(kWbODone + s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWMmaWarp) {
    tmem_alloc(sbase + Lay::kTmemSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  FA_TRACE_BEGIN();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Lay::kTmemSlot);

  if (warp == kWKLoadWarp) {
    // ------------------------------------------------------- TMA loads: Q and K
    if (lane == 0) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmK);
      mbar_expect_tx(bar(kWbQFull), Lay::kTileBytes);
      for (int c = 0; c < D / 64; ++c)
        tma_load_4d(sbase + Lay::kQ + c * Lay::kChunkBytes, &tmQ, c * 64, t * kTile, hh, bb,
                    bar(kWbQFull));
      for (int j = 0; j < nkv; ++j) {
        // the single K stage is free once S_j-1 has completed
        if (j > 0 && !mbar_wait(bar(kWbKEmpty), static_cast<uint32_t>(j - 1) & 1, abort_flag))
          break;
        mbar_expect_tx(bar(kWbKFull), Lay::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Lay::kK + c * Lay::kChunkBytes, &tmK, c * 64, (j0 + j) * kTile, hh,
                      bb, bar(kWbKFull));
        FA_TRACE_EVENT(j, 8);
      }
    }
  } else if (warp == kWVLoadWarp) {
    // ------------------------------------------------------------ TMA loads: V
    if (lane == 0) {
      tma_prefetch(&tmV);
      for (int j = 0; j < nkv; ++j) {
        // the single V stage is free once P_j-1 V_j-1 has completed
        if (j > 0 && !mbar_wait(bar(kWbVEmpty), static_cast<uint32_t>(j - 1) & 1, abort_flag))
          break;
        mbar_expect_tx(bar(kWbVFull), Lay::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Lay::kV + c * Lay::kChunkBytes, &tmV, c * 64, (j0 + j) * kTile, hh,
                      bb, bar(kWbVFull));
        FA_TRACE_EVENT(j, 9);
      }
    }
  } else if (warp == kWMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16_f32(kTile, kTile, BF16, false, false);
      constexpr uint32_t idesc_o = idesc_f16_f32(kTile, D, BF16, false, true);
      const uint64_t dq = sdesc_sw128(sbase + Lay::kQ, 16, 1024);
      const uint64_t dk = sdesc_sw128(sbase + Lay::kK, 16, 1024);
      const uint64_t dv = sdesc_sw128(sbase + Lay::kV, Lay::kChunkBytes, 1024);
      bool ok = mbar_wait(bar(kWbQFull), 0, abort_flag);
      for (int j = 0; ok && j < nkv + 1; ++j) {
        if (j < nkv) {
          const int sb = j & 1;  // S_j's buffer: P_j-2 V_j-2, which read it, went before
          if (!mbar_wait(bar(kWbKFull), static_cast<uint32_t>(j) & 1, abort_flag)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t koff = (k >> 2) * Lay::kChunkBytes + (k & 3) * 32;
            mma_ss(tmem + sb * 128, sdesc_advance(dq, koff), sdesc_advance(dk, koff), idesc_s,
                   k > 0 ? 1u : 0u);
          }
          mma_commit(bar(kWbKEmpty));
          mma_commit(bar(kWbSFull + sb));
          FA_TRACE_EVENT(j, 0);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int pb = jj & 1;
          if (!mbar_wait(bar(kWbPFull + pb), static_cast<uint32_t>(jj >> 1) & 1, abort_flag))
            break;
          FA_TRACE_EVENT(jj, 1);
          if (!mbar_wait(bar(kWbVFull), static_cast<uint32_t>(jj) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t a_p = tmem + pb * 128;  // P packed in the first 64 columns
#pragma unroll
          for (int k = 0; k < kTile / 16; ++k)
            mma_ts(tmem + Lay::tO, a_p + k * 8, sdesc_advance(dv, k * 2048), idesc_o,
                   (jj > 0 || k > 0) ? 1u : 0u);
          mma_commit(bar(kWbVEmpty));
          mma_commit(bar(kWbODone + pb));
          FA_TRACE_EVENT(jj, 2);
        }
      }
    }
  } else if (warp < 8) {
    // ----------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int r = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t o_cols = Lay::tO + half * (D / 2);
    float* red = reinterpret_cast<float*>(smem + Lay::kRed);  // [parity][half][row]
    const int pair_bar = 1 + quarter;                          // named barrier of the pair
    float m = -INFINITY;  // running reference, base-2 scaled units (same in both halves)
    float l = 0.f;        // this half's share of the row sum of p
    float l_o = 0.f;      // ... and of the 16-bit-rounded p
    const uint64_t c2 = f2_pack(scale_log2, scale_log2);
    // `ok` turns false (warp-uniformly) when a wait gives up; the loop then runs on
    // without work so that both warps of a pair still meet at every named barrier.
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int b = j & 1;  // score buffer of tile j
      const int par = j & 1;
      ok = __all_sync(0xffffffffu,
                      ok && mbar_wait(bar(kWbSFull + b), static_cast<uint32_t>(j >> 1) & 1,
                                      abort_flag));
      if (threadIdx.x == 0) FA_TRACE_EVENT(j, 3);
      float s[64];
      float mx = -INFINITY;
      if (ok) {
        tc_fence_after();
        {
          uint32_t sr[64];
          tmem_ld32(lane_base + b * 128 + half * 64, sr);
          tmem_ld32(lane_base + b * 128 + half * 64 + 32, sr + 32);
          tmem_wait_ld();
          reg_fence32(sr);
          reg_fence32(sr + 32);
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c]);
        }
        // band: key column c of the tile is visible to row r when
        // r + delta - wl <= c <= r + delta + wr; last tile: keys >= Nk are masked
        const int jt = j0 + j;  // the key tile itself
        const int delta = t * kTile + off - jt * kTile;
        const bool hmask = BAND && delta + wr < kTile - 1;     // upper edge crosses the tile
        const bool lmask = BAND && delta - wl > -(kTile - 1);  // lower edge crosses it
        const bool kmask = jt == ntk - 1 && last_keys < kTile;
        if (hmask || lmask || kmask) {
          int hi = kmask ? last_keys - 1 : kTile - 1;
          if (hmask) hi = min(hi, r + delta + wr);
          const int lo = (lmask ? r + delta - wl : 0) - half * 64;
          hi -= half * 64;
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = (c > hi || c < lo) ? -INFINITY : s[c];
        }
        // four independent chains of 3-input maxima
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k) mq[k] = fmax3(mq[k], s[c + 2 * k], s[c + 2 * k + 1]);
        }
        mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      }
      red[(par * 2 + half) * 128 + r] = mx;
      named_bar_sync(pair_bar, 64);
      mx = fmaxf(mx, red[(par * 2 + (half ^ 1)) * 128 + r]);
      if (threadIdx.x == 0) FA_TRACE_EVENT(j, 4);
      if (!ok) continue;
      const float cand = mx * scale_log2;
      const float m_new = (cand > m + kWRescaleSlack) ? cand : m;
      // A row that sees no key keeps m = -inf: it takes alpha = 1 and subtracts 0, so
      // that its p = 2^-inf = 0 and no inf - inf appears.
      const bool empty_row = m_new == -INFINITY;
      const float alpha = empty_row ? 1.f : ex2_approx(m - m_new);  // 0 on the first tile
      const float m_sub = empty_row ? 0.f : m_new;
      const uint64_t nm2 = f2_pack(-m_sub, -m_sub);
      // packed fp32 pairs, two independent accumulators per sum
      uint64_t sum2[2] = {0, 0}, sum2_o[2] = {0, 0};  // packed +0.0f
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int e = h2 * 32 + 2 * c;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), c2, nm2), x0, x1);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          pk[c] = pack2<BF16>(p0, p1);
          float r0, r1;
          unpack2<BF16>(pk[c], r0, r1);
          sum2[c & 1] = f2_add(sum2[c & 1], f2_pack(p0, p1));
          sum2_o[c & 1] = f2_add(sum2_o[c & 1], f2_pack(r0, r1));
        }
        // P of this half's 64 keys over 32 columns; the partner half has loaded its
        // scores before the exchange above, so columns 32-63 are free to overwrite
        tmem_st16(lane_base + b * 128 + half * 32 + h2 * 16, pk);
      }
      float a0, a1, b0, b1;
      f2_unpack(f2_add(sum2[0], sum2[1]), a0, a1);
      f2_unpack(f2_add(sum2_o[0], sum2_o[1]), b0, b1);
      l = l * alpha + (a0 + a1);
      l_o = l_o * alpha + (b0 + b1);
      if (threadIdx.x == 0) FA_TRACE_EVENT(j, 5);
      // O is touched only when a row's reference moved (rare after the first tiles);
      // then P_{j-1} V_{j-1} must have landed first. One barrier per score buffer makes
      // the skipped waits safe: S_j, complete by now, was issued after P_{j-2} V_{j-2},
      // so the barrier of P_{j-1} V_{j-1} (the one of P_{j-3} V_{j-3} before it) is at
      // most one phase away from the one waited.
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        const int pj = j - 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kWbODone + (pj & 1)),
                                               static_cast<uint32_t>(pj >> 1) & 1, abort_flag));
        if (!ok) continue;
        if (threadIdx.x == 0) FA_TRACE_EVENT(j, 6);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + o_cols + c * 32, o);
          tmem_wait_ld();
          reg_fence32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_base + o_cols + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kWbPFull + b));
      if (threadIdx.x == 0) FA_TRACE_EVENT(j, 7);
      m = m_new;
    }
    // the last P V
    ok = __all_sync(0xffffffffu,
                    ok && (nkv == 0 || mbar_wait(bar(kWbODone + ((nkv - 1) & 1)),
                                                 static_cast<uint32_t>((nkv - 1) >> 1) & 1,
                                                 abort_flag)));
    // both halves' sums: reuse the exchange buffer of parity (nkv & 1), which the pair
    // last used two tiles ago
    red[((nkv & 1) * 2 + half) * 128 + r] = l;
    red[((nkv & 1) * 2 + half) * 128 + r + 512] = l_o;
    named_bar_sync(pair_bar, 64);
    const float l_row = l + red[((nkv & 1) * 2 + (half ^ 1)) * 128 + r];
    const float l_o_row = l_o + red[((nkv & 1) * 2 + (half ^ 1)) * 128 + r + 512];
    // O and its rounding residual go out through shared memory and TMA stores (whole
    // 128-byte lines): O staged in the K stage, which the finished last S MMA has
    // freed, O_res in the V stage, which the finished last P V MMA has freed; the
    // 128-row x 64-column chunk c at + c * kChunkBytes, in the 128-byte-swizzled layout
    // of the tensor maps.
    if (ok) {
      tc_fence_after();
      const float inv_l = l_o_row > 0.f ? 1.f / l_o_row : 0.f;  // rows that see no key: O = 0
      const uint32_t st_o = sbase + Lay::kK;
      const uint32_t st_r = sbase + Lay::kV;
      const int sw = r & 7;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t o[32];
        if (nkv > 0) {  // with no KV tile, O in TMEM was never written
          tmem_ld32(lane_base + o_cols + c * 32, o);
          tmem_wait_ld();
          reg_fence32(o);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        uint32_t hw[16], lw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = __uint_as_float(o[2 * e]) * inv_l;
          const float x1 = __uint_as_float(o[2 * e + 1]) * inv_l;
          hw[e] = pack2<BF16>(x0, x1);
          float h0, h1;
          unpack2<BF16>(hw[e], h0, h1);
          lw[e] = pack2<BF16>(x0 - h0, x1 - h1);  // exact difference, then rounded
        }
        // this thread's 32 columns: half * D/2 + 32 c .. +31
        const int col = half * (D / 2) + c * 32;
        const uint32_t chunk = static_cast<uint32_t>(col / 64) * Lay::kChunkBytes + r * 128;
        const int u0 = (col % 64) / 8;  // first 16-byte unit within the 128-byte row
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t so = chunk + static_cast<uint32_t>(((u0 + u) ^ sw) * 16);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(st_o + so),
                       "r"(hw[4 * u]), "r"(hw[4 * u + 1]), "r"(hw[4 * u + 2]), "r"(hw[4 * u + 3])
                       : "memory");
          if (has_res)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(st_r + so),
                         "r"(lw[4 * u]), "r"(lw[4 * u + 1]), "r"(lw[4 * u + 2]),
                         "r"(lw[4 * u + 3])
                         : "memory");
        }
      }
      fence_async_smem();
      if (half == 0 && t * kTile + r < Nq)
        Lse[static_cast<long>(bh) * Nq + t * kTile + r] =
            (m + log2f(l_row)) * 0.69314718055994530942f;
    }
    // all 256 softmax threads have staged their part (or all gave up together)
    if (named_bar_and(5, 256, ok) && threadIdx.x == 0) {
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_store_4d(&tmO, sbase + Lay::kK + c * Lay::kChunkBytes, c * 64, t * kTile, hh, bb);
        if (has_res)
          tma_store_4d(&tmOres, sbase + Lay::kV + c * Lay::kChunkBytes, c * 64, t * kTile, hh,
                       bb);
      }
      bulk_commit();
      bulk_wait_read_all();  // shared memory is read before the CTA releases it
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  FA_TRACE_CTA(1);
}

}  // namespace fa
