// fa_bwd_dq.cuh -- dQ as a separate pass over the keys, summed in a fixed order.
//
// The gradient dQ_i = scale * sum_j dS_ij k_j (josueisai.com "flash-attention",
// section "Recomputar sale mas barato que recordar": the backward recomputes the
// scores from Q, K and V) is formed here by one CTA per 128-row query tile, which
// walks the key/value tiles of its band in increasing order and accumulates dQ in
// tensor memory. Every element of dQ is therefore the same sequence of fp32 additions
// on every run: repeated calls give identical bits, unlike the dK/dV kernel's
// reduce-adds of dQ partials, whose order depends on which CTA finishes first. The
// dK/dV kernel then runs without its dQ work.
//
// Per key tile j, with the row statistics of the preprocess kernel (-L log2 e, -D):
//   S = Q K_j^T,  dP = dO V_j^T                       (SMEM x SMEM -> TMEM, fp32)
//   P = 2^(S scale log2 e - L log2 e),  dS = P * (dP - D)   (thread = query row)
//   dQ += dS K_j                                      (dS from TMEM, K_j from SMEM)
//
// Warp roles (320 threads):
//   warps 0-7  compute, in pairs: warps w and w+4 share TMEM lane quarter w % 4 (thread
//              = query row); warp w < 4 takes key columns 0-63, warp w+4 columns
//              64-127. dS goes back into TMEM over the S columns as packed 16-bit
//              values, as the forward does with P.
//   warp 8     TMA producer: Q and dO once, K_j into a 3-stage ring (a stage is held
//              until the dQ MMA of its tile completes), V_j into a 2-stage ring.
//   warp 9     MMA issuer and TMEM owner: S_0 dP_0 | S_1 dQ_0 dP_1 | S_2 dQ_1 dP_2 | ...
//
// TMEM: S/dS buffers at columns 0 and 128, dP at 256, dQ at 384 (d columns).
#pragma once

#include "fa_band.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kDqThreads = 320;
constexpr int kDqProducerWarp = 8;
constexpr int kDqMmaWarp = 9;
constexpr int kDqKStages = 3;
constexpr int kDqVStages = 2;

template <int D>
struct DqLayout {
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr uint32_t kChunkBytes = kTile * 128;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kDO = kQ + kTileBytes;
  static constexpr uint32_t kK = kDO + kTileBytes;
  static constexpr uint32_t kV = kK + kDqKStages * kTileBytes;
  static constexpr uint32_t kBar = kV + kDqVStages * kTileBytes;
  static constexpr int kNumBars = 20;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 8;
  static constexpr uint32_t kBytes = kAbort + 8 + 1024;  // + alignment slack
  // TMEM columns
  static constexpr uint32_t tS = 0;  // + 128 * buffer
  static constexpr uint32_t tDP = 256;
  static constexpr uint32_t tDQ = 384;
};

enum : int {
  kDbQFull = 0,                          // Q and dO
  kDbKFull = 1,                          // + K stage
  kDbKEmpty = kDbKFull + kDqKStages,     // + K stage
  kDbVFull = kDbKEmpty + kDqKStages,     // + V stage
  kDbVEmpty = kDbVFull + kDqVStages,     // + V stage
  kDbSFull = kDbVEmpty + kDqVStages,     // + S buffer
  kDbDPFull = kDbSFull + 2,
  kDbDSReady = kDbDPFull + 1,            // + S buffer: dS of that buffer is in TMEM
  kDbDone = kDbDSReady + 2,
  kDqNumBars = kDbDone + 1,
};
static_assert(kDqNumBars <= 20, "barrier area");

// Ls, Dv: the preprocess kernel's -L log2(e) and -D, [B*H][ntq * 128] fp32.
template <int D, bool BAND, bool BF16>
__global__ void __launch_bounds__(kDqThreads, 1)
    fa_bwd_dq_pass_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmDO,
                          const __grid_constant__ CUtensorMap tmDQ, const float* __restrict__ Ls,
                          const float* __restrict__ Dv, int Nq, int Nk, int H, int wl, int wr,
                          float scale, float scale_log2, int group) {
  using Lay = DqLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntq = (Nq + kTile - 1) / kTile;
  const int ntk = (Nk + kTile - 1) / kTile;
  // band: heaviest tiles first, heads in groups (band_order); otherwise head-major
  int bh, tr;
  if (BAND) {
    band_order(blockIdx.x, ntq, gridDim.x / ntq, group, &bh, &tr);
  } else {
    bh = blockIdx.x / ntq;
    tr = blockIdx.x - bh * ntq;
  }
  const int hh = bh % H;
  const int bb = bh / H;
  const int t = BAND ? (ntq - 1 - tr) : tr;  // causal: heaviest tiles first
  const TileRange kv = BAND ? kv_tiles_of_query_tile(t, kTile, Nq, Nk, wl, wr)
                            : TileRange{0, ntk};
  const int j0 = kv.first;
  const int nkv = kv.count;
  const int off = Nk - Nq;
  const int last_keys = Nk - (ntk - 1) * kTile;

  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar(kDbQFull), 1);
    for (int s = 0; s < kDqKStages; ++s) {
      mbar_init(bar(kDbKFull + s), 1);
      mbar_init(bar(kDbKEmpty + s), 1);
    }
    for (int s = 0; s < kDqVStages; ++s) {
      mbar_init(bar(kDbVFull + s), 1);
      mbar_init(bar(kDbVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kDbSFull + s), 1);
      mbar_init(bar(kDbDSReady + s), 256);
    }
    mbar_init(bar(kDbDPFull), 1);
    mbar_init(bar(kDbDone), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kDqMmaWarp) {
    tmem_alloc(sbase + Lay::kTmemSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Lay::kTmemSlot);

  if (warp == kDqProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nkv > 0) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      tma_prefetch(&tmDO);
      mbar_expect_tx(bar(kDbQFull), 2 * Lay::kTileBytes);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_4d(sbase + Lay::kQ + c * Lay::kChunkBytes, &tmQ, c * 64, t * kTile, hh, bb,
                    bar(kDbQFull));
        tma_load_4d(sbase + Lay::kDO + c * Lay::kChunkBytes, &tmDO, c * 64, t * kTile, hh, bb,
                    bar(kDbQFull));
      }
      for (int j = 0; j < nkv; ++j) {
        const int ks = j % kDqKStages;
        if (j >= kDqKStages &&
            !mbar_wait(bar(kDbKEmpty + ks), static_cast<uint32_t>(j / kDqKStages - 1) & 1,
                       abort_flag))
          break;
        mbar_expect_tx(bar(kDbKFull + ks), Lay::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Lay::kK + ks * Lay::kTileBytes + c * Lay::kChunkBytes, &tmK, c * 64,
                      (j0 + j) * kTile, hh, bb, bar(kDbKFull + ks));
        const int vs = j % kDqVStages;
        if (j >= kDqVStages &&
            !mbar_wait(bar(kDbVEmpty + vs), static_cast<uint32_t>(j / kDqVStages - 1) & 1,
                       abort_flag))
          break;
        mbar_expect_tx(bar(kDbVFull + vs), Lay::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Lay::kV + vs * Lay::kTileBytes + c * Lay::kChunkBytes, &tmV, c * 64,
                      (j0 + j) * kTile, hh, bb, bar(kDbVFull + vs));
      }
    }
  } else if (warp == kDqMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0 && nkv > 0) {
      constexpr uint32_t id_sq = idesc_f16_f32(kTile, kTile, BF16, false, false);  // S, dP
      constexpr uint32_t id_dq = idesc_f16_f32(kTile, D, BF16, false, true);       // dQ
      const uint64_t dq_k = sdesc_sw128(sbase + Lay::kQ, 16, 1024);
      const uint64_t ddo_k = sdesc_sw128(sbase + Lay::kDO, 16, 1024);
      auto issue_s = [&](int j) -> bool {  // S_j = Q K_j^T into buffer j & 1
        const int ks = j % kDqKStages;
        if (!mbar_wait(bar(kDbKFull + ks), static_cast<uint32_t>(j / kDqKStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t dk = sdesc_sw128(sbase + Lay::kK + ks * Lay::kTileBytes, 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t koff = (k >> 2) * Lay::kChunkBytes + (k & 3) * 32;
          mma_ss(tmem + Lay::tS + (j & 1) * 128, sdesc_step(dq_k, koff), sdesc_step(dk, koff),
                 id_sq, k > 0 ? 1u : 0u);
        }
        mma_commit(bar(kDbSFull + (j & 1)));
        return true;
      };
      auto issue_dp = [&](int j) -> bool {  // dP_j = dO V_j^T
        const int vs = j % kDqVStages;
        if (!mbar_wait(bar(kDbVFull + vs), static_cast<uint32_t>(j / kDqVStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t dv = sdesc_sw128(sbase + Lay::kV + vs * Lay::kTileBytes, 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t koff = (k >> 2) * Lay::kChunkBytes + (k & 3) * 32;
          mma_ss(tmem + Lay::tDP, sdesc_step(ddo_k, koff), sdesc_step(dv, koff), id_sq,
                 k > 0 ? 1u : 0u);
        }
        mma_commit(bar(kDbVEmpty + vs));
        mma_commit(bar(kDbDPFull));
        return true;
      };
      bool ok = mbar_wait(bar(kDbQFull), 0, abort_flag) && issue_s(0) && issue_dp(0);
      for (int j = 0; ok && j < nkv; ++j) {
        // S_{j+1} overwrites the buffer of dS_{j-1} only after the dQ MMA that reads it
        // (issued in iteration j - 1; MMAs of one thread run in issue order).
        if (j + 1 < nkv && !issue_s(j + 1)) break;
        if (!mbar_wait(bar(kDbDSReady + (j & 1)), static_cast<uint32_t>(j >> 1) & 1, abort_flag))
          break;
        tc_fence_after();
        const int ks = j % kDqKStages;
        const uint64_t dk_mn =
            sdesc_sw128(sbase + Lay::kK + ks * Lay::kTileBytes, Lay::kChunkBytes, 1024);
        const uint32_t a_ds = tmem + Lay::tS + (j & 1) * 128;  // dS packed in 64 columns
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)
          mma_ts(tmem + Lay::tDQ, a_ds + k * 8, sdesc_step(dk_mn, k * 2048), id_dq,
                 (j > 0 || k > 0) ? 1u : 0u);
        mma_commit(bar(kDbKEmpty + ks));
        // dP_{j+1}: the compute warps have read dP_j (dS_j is ready)
        if (j + 1 < nkv && !issue_dp(j + 1)) break;
      }
      mma_commit(bar(kDbDone));
    }
  } else {
    // ----------------------------------------------------------------- compute
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int r = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const long prow = static_cast<long>(bh) * ntq * kTile + t * kTile + r;  // padded row
    const float nls = Ls[prow];  // -L log2(e) (-inf for padded rows and rows with no key)
    const float nd = Dv[prow];   // -D
    const uint64_t c2 = f2_pack(scale_log2, scale_log2);
    const uint64_t nls2 = f2_pack(nls, nls);
    const uint64_t nd2 = f2_pack(nd, nd);
    // The two warps of a pair meet at one named barrier per tile, and leave the loop
    // together: a failed wait is carried to the next meeting, where bar.red.and makes
    // both warps see it, so that neither is ever left waiting at the barrier alone.
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int b = j & 1;
      const bool got = __all_sync(0xffffffffu, ok && mbar_wait(bar(kDbSFull + b),
                                                               static_cast<uint32_t>(j >> 1) & 1,
                                                               abort_flag));
      float p[64];
      if (got) {
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(lane_base + Lay::tS + b * 128 + half * 64, sr);
        tmem_ld32(lane_base + Lay::tS + b * 128 + half * 64 + 32, sr + 32);
        tmem_wait_ld();
        reg_fence32(sr);
        reg_fence32(sr + 32);
#pragma unroll
        for (int c = 0; c < 64; ++c) p[c] = __uint_as_float(sr[c]);
      }
      // both halves have read their S columns before either writes dS over them
      ok = named_bar_and(1 + quarter, 64, got);
      if (!ok) break;
      // band and ragged-tile masks, as in the forward
      const int jt = j0 + j;
      const int delta = t * kTile + off - jt * kTile;
      const bool hmask = BAND && delta + wr < kTile - 1;
      const bool lmask = BAND && delta - wl > -(kTile - 1);
      const bool kmask = jt == ntk - 1 && last_keys < kTile;
      if (hmask || lmask || kmask) {
        int hi = kmask ? last_keys - 1 : kTile - 1;
        if (hmask) hi = min(hi, r + delta + wr);
        const int lo = (lmask ? r + delta - wl : 0) - half * 64;
        hi -= half * 64;
#pragma unroll
        for (int c = 0; c < 64; ++c) p[c] = (c > hi || c < lo) ? -INFINITY : p[c];
      }
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(p[c], p[c + 1]), c2, nls2), x0, x1);
        p[c] = ex2_approx(x0);
        p[c + 1] = ex2_approx(x1);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kDbDPFull), static_cast<uint32_t>(j & 1),
                                             abort_flag));
      if (!ok) continue;  // the pair agrees at the next meeting (or after the loop)
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dr[32];
        tmem_ld32(lane_base + Lay::tDP + half * 64 + c * 32, dr);
        tmem_wait_ld();
        reg_fence32(dr);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int q = c * 32 + 2 * e;
          float a0, a1;
          f2_unpack(f2_mul(f2_pack(p[q], p[q + 1]),
                           f2_add(f2_pack(__uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1])),
                                  nd2)),
                    a0, a1);
          pk[e] = pack2<BF16>(a0, a1);
        }
        tmem_st16(lane_base + Lay::tS + b * 128 + half * 32 + c * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kDbDSReady + b));
    }
    ok = __all_sync(0xffffffffu, ok && (nkv == 0 || mbar_wait(bar(kDbDone), 0, abort_flag)));
    // dQ = dtype(scale * accumulator), staged in the K ring (free once the last MMA is
    // done) in the tensor map's 128-byte-swizzled layout, then TMA-stored; a tile that
    // visits no key stores zeros.
    if (ok) {
      tc_fence_after();
      const uint32_t st = sbase + Lay::kK;
      const int sw = r & 7;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t v[32];
        if (nkv > 0) {
          tmem_ld32(lane_base + Lay::tDQ + half * (D / 2) + c * 32, v);
          tmem_wait_ld();
          reg_fence32(v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        uint32_t hw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          hw[e] = pack2<BF16>(__uint_as_float(v[2 * e]) * scale,
                              __uint_as_float(v[2 * e + 1]) * scale);
        const int col = half * (D / 2) + c * 32;
        const uint32_t chunk = static_cast<uint32_t>(col / 64) * Lay::kChunkBytes + r * 128;
        const int u0 = (col % 64) / 8;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           st + chunk + static_cast<uint32_t>(((u0 + u) ^ sw) * 16)),
                       "r"(hw[4 * u]), "r"(hw[4 * u + 1]), "r"(hw[4 * u + 2]), "r"(hw[4 * u + 3])
                       : "memory");
      }
      fence_async_smem();
    }
    if (named_bar_and(5, 256, ok) && threadIdx.x == 0) {
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_store_4d(&tmDQ, sbase + Lay::kK + c * Lay::kChunkBytes, c * 64, t * kTile, hh, bb);
      bulk_commit();
      bulk_wait_read_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDqMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
