// fa_decode_tc.cuh -- the decode form (a few query rows against a long key sequence,
// split across CTAs along the keys, merged by log-sum-exp) with its two products on
// the tensor cores, for 2-16 query rows per head at d = 128.
//
// With N_q rows the CUDA-core form (fa_decode.cuh) spends N_q dot products of length d
// on every key, and at 16 rows that arithmetic, not the K/V stream, sets its pace. Here
// both products are tcgen05 MMAs with the keys on the M side, where a 128-row MMA needs
// them:
//   S^T_j = K_j Q^T            M = 128 keys, N = 16 query columns (rows >= N_q are 0),
//                              K = d; A = the K tile as TMA lands it, B = Q (16 rows)
//   O^T  += V_j^T P_j^T        M = d = 128, N = 16, K = 128 keys; A = the V tile read
//                              M-major, B = P_j^T written to shared memory by the
//                              softmax warps (16 rows x 128 keys, 16-bit)
// S^T and O^T sit in tensor memory, lane = key (S^T) or lane = column of d (O^T). The
// online softmax of josueisai.com "flash-attention", section "El truco: trocear y
// llevar la cuenta del softmax", then runs down the lanes: thread r of the 128 softmax
// threads owns key r of the tile and holds its 16 scores; each query column's maximum
// is reduced over the warp with shuffles and over the four warps through shared memory
// once per tile. The reference of a column moves lazily (only past 2^8, as in the
// forward kernels), and then the O^T column is rescaled in tensor memory. P is rounded
// to 16 bits for the MMA; the sum of the rounded P normalises O and the sum of the
// unrounded P gives L, as in the forward.
//
// CTA (192 threads): warps 0-3 softmax (TMEM lane quarter w, keys 32 w .. 32 w + 31),
// warp 4 TMA producer (K_j and V_j of each key tile into a 3-stage ring), warp 5 MMA
// issuer and TMEM owner, in the order S_0 | S_1 PV_0 | S_2 PV_1 | ... (P V one tile
// behind, so that the softmax of tile j overlaps S_j+1).
#pragma once

#include "fa_band.cuh"
#include "fa_decode.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kDtcThreads = 192;
constexpr int kDtcProducerWarp = 4;
constexpr int kDtcMmaWarp = 5;
constexpr int kDtcN = 16;  // query columns of the MMAs (N_q <= 16, zero-padded)
constexpr int kDtcD = 128;
constexpr int kDtcStages = 3;
constexpr float kDtcRescaleSlack = 8.0f;

struct DtcLayout {
  static constexpr uint32_t kTileBytes = kTile * kDtcD * 2;  // 32 KB
  static constexpr uint32_t kChunkBytes = kTile * 128;       // 128 rows x 64 values
  static constexpr uint32_t kStageBytes = 2 * kTileBytes;    // K tile, then V tile
  static constexpr uint32_t kSmallChunk = kDtcN * 128;       // 16 rows x 64 values (2 KB)
  static constexpr uint32_t kSmallBytes = 2 * kSmallChunk;   // 16 rows x 128 values
  static constexpr uint32_t kQ = kDtcStages * kStageBytes;   // Q, 16 rows (B of S^T)
  static constexpr uint32_t kP = kQ + kSmallBytes;           // P^T, 2 buffers (B of O^T)
  static constexpr uint32_t kRed = kP + 2 * kSmallBytes;     // [2 parity][4 warps][16] fp32
  static constexpr uint32_t kBar = kRed + 2 * 4 * kDtcN * 4;
  static constexpr int kNumBars = 16;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 8;
  static constexpr uint32_t kBytes = kAbort + 8 + 1024;
  // TMEM columns (64 allocated): S^T buffers 0 and 16, O^T 32
  static constexpr uint32_t tS = 0;
  static constexpr uint32_t tO = 2 * kDtcN;
};

enum : int {
  kDtFull = 0,                      // + stage: K_j and V_j landed
  kDtEmpty = kDtFull + kDtcStages,  // + stage: P_j V_j (the stage's last reader) done
  kDtSFull = kDtEmpty + kDtcStages,  // + buffer
  kDtPFull = kDtSFull + 2,          // + buffer (128 arrivals)
  kDtPFree = kDtPFull + 2,          // + buffer: the P V that read it has completed
  kDtODone = kDtPFree + 2,          // + buffer of the P that the P V read
  kDtcNumBars = kDtODone + 2,
};
static_assert(kDtcNumBars <= 16, "barrier area");

// Offset within a 16-row, 128-byte-swizzled 16-bit tile (two 64-column chunks of
// 16 rows x 128 bytes) of element (row, col).
__device__ __forceinline__ uint32_t small_swz(int row, int col) {
  const int chunk = col >> 6;
  const int byte = (col & 63) * 2;
  return static_cast<uint32_t>(chunk * kDtcN * 128 + row * 128 +
                               ((((byte >> 4) ^ (row & 7)) << 4) | (byte & 15)));
}

// One CTA per (head bh, split s); the split covers key tiles [tile0 + s*tps,
// min(tile0 + ntiles, tile0 + (s+1)*tps)). Outputs as fa_decode_kernel: with one split
// O (16-bit, strides so) and L; otherwise the split's normalised O and its log-sum-exp
// into Opart [BH][splits][Nq][D] and Lpart [BH][splits][Nq] for fa_decode_merge_kernel.
template <bool BAND, bool BF16>
__global__ void __launch_bounds__(kDtcThreads, 1)
    fa_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const uint16_t* __restrict__ Q,
                        Strides sq, uint16_t* __restrict__ O, Strides so, float* __restrict__ Lse,
                        float* __restrict__ Opart, float* __restrict__ Lpart, int Nq, int Nk,
                        int H, int wl, int wr, int tile0, int ntiles, int tps, int splits,
                        float scale_log2) {
  constexpr int D = kDtcD;
  constexpr int S = kDtcStages;
  using Lay = DtcLayout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / splits;
  const int sp = blockIdx.x - bh * splits;
  const int hh = bh % H;
  const int bb = bh / H;
  const int t_begin = tile0 + sp * tps;
  const int t_end = min(tile0 + ntiles, t_begin + tps);
  const int nt = t_end > t_begin ? t_end - t_begin : 0;

  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kAbort);
  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) {
      mbar_init(bar(kDtFull + st), 1);
      mbar_init(bar(kDtEmpty + st), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kDtSFull + b), 1);
      mbar_init(bar(kDtPFull + b), 128);
      mbar_init(bar(kDtPFree + b), 1);
      mbar_init(bar(kDtODone + b), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kDtcMmaWarp) {
    tmem_alloc(sbase + Lay::kTmemSlot, 64);
    tmem_relinquish();
  }
  // Q (rows >= Nq as zeros) into its swizzled 16-row tile by the softmax threads: 256
  // units of 16 bytes, two per thread
  if (threadIdx.x < 128) {
#pragma unroll
    for (int u2 = 0; u2 < 2; ++u2) {
      const int unit = threadIdx.x * 2 + u2;  // 0 .. 255
      const int row = unit >> 4;              // 16 units per row
      const int col = (unit & 15) * 8;        // 8 values per unit
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row < Nq)
        v = *reinterpret_cast<const uint4*>(Q + bb * sq.sb + hh * sq.sh +
                                            static_cast<long>(row) * sq.sn + col);
      *reinterpret_cast<uint4*>(smem + Lay::kQ + small_swz(row, col)) = v;
    }
    fence_async_smem();  // generic-proxy stores, read by the tensor core's async proxy
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Lay::kTmemSlot);

  if (warp == kDtcProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      for (int i = 0; i < nt; ++i) {
        const int st = i % S;
        if (i >= S && !mbar_wait(bar(kDtEmpty + st), static_cast<uint32_t>(i / S - 1) & 1,
                                 abort_flag))
          break;
        const uint32_t dst = sbase + st * Lay::kStageBytes;
        mbar_expect_tx(bar(kDtFull + st), Lay::kStageBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(dst + c * Lay::kChunkBytes, &tmK, c * 64, (t_begin + i) * kTile, hh, bb,
                      bar(kDtFull + st));
          tma_load_4d(dst + Lay::kTileBytes + c * Lay::kChunkBytes, &tmV, c * 64,
                      (t_begin + i) * kTile, hh, bb, bar(kDtFull + st));
        }
      }
    }
  } else if (warp == kDtcMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16_f32(kTile, kDtcN, BF16, false, false);
      constexpr uint32_t id_o = idesc_f16_f32(D, kDtcN, BF16, true, false);
      const uint64_t dq = sdesc_sw128(sbase + Lay::kQ, 16, 1024);
      bool ok = true;
      for (int j = 0; ok && j < nt + 1; ++j) {
        if (j < nt) {  // S^T_j = K_j Q^T into buffer j & 1 (its P V, j - 2, went before)
          const int st = j % S;
          if (!mbar_wait(bar(kDtFull + st), static_cast<uint32_t>(j / S) & 1, abort_flag)) break;
          tc_fence_after();
          const uint64_t dk = sdesc_sw128(sbase + st * Lay::kStageBytes, 16, 1024);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t koff = (k >> 2) * Lay::kChunkBytes + (k & 3) * 32;
            const uint32_t qoff = (k >> 2) * Lay::kSmallChunk + (k & 3) * 32;
            mma_ss(tmem + Lay::tS + (j & 1) * kDtcN, sdesc_advance(dk, koff),
                   sdesc_advance(dq, qoff), id_s, k > 0 ? 1u : 0u);
          }
          mma_commit(bar(kDtSFull + (j & 1)));
        }
        if (j >= 1) {  // O^T += V_jj^T P_jj^T
          const int jj = j - 1;
          const int st = jj % S;
          const int pb = jj & 1;
          if (!mbar_wait(bar(kDtPFull + pb), static_cast<uint32_t>(jj >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          const uint64_t dv = sdesc_sw128(sbase + st * Lay::kStageBytes + Lay::kTileBytes,
                                          Lay::kChunkBytes, 1024);
          const uint64_t dp = sdesc_sw128(sbase + Lay::kP + pb * Lay::kSmallBytes, 16, 1024);
#pragma unroll
          for (int k = 0; k < kTile / 16; ++k) {
            const uint32_t poff = (k >> 2) * Lay::kSmallChunk + (k & 3) * 32;
            mma_ss(tmem + Lay::tO, sdesc_advance(dv, k * 2048), sdesc_advance(dp, poff), id_o,
                   (jj > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(bar(kDtEmpty + st));
          mma_commit(bar(kDtPFree + pb));
          mma_commit(bar(kDtODone + pb));
        }
      }
    }
  } else {
    // ----------------------------------------------------------------- softmax
    const int r = threadIdx.x;  // key row of the tile = TMEM lane (warp w: lanes 32 w ..)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float* red = reinterpret_cast<float*>(smem + Lay::kRed);  // [parity][warp][query]
    const int off = Nk - Nq;
    float m[kDtcN], l[kDtcN], l_o[kDtcN];
#pragma unroll
    for (int q = 0; q < kDtcN; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.f;  // this thread's (key's) share of the row sums
      l_o[q] = 0.f;
    }
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(kDtSFull + b),
                                                   static_cast<uint32_t>(j >> 1) & 1, abort_flag));
      float s[kDtcN];
      float mw[kDtcN];
      if (ok) {
        tc_fence_after();
        uint32_t sr[kDtcN];
        tmem_ld16(lane_base + Lay::tS + b * kDtcN, sr);
        tmem_wait_ld();
        reg_fence16(sr);
        const int key = (t_begin + j) * kTile + r;
#pragma unroll
        for (int q = 0; q < kDtcN; ++q) {
          const bool visible = key < Nk && q < Nq &&
                               (!BAND || (key >= q + off - wl && key <= q + off + wr));
          s[q] = visible ? __uint_as_float(sr[q]) * scale_log2 : -INFINITY;
          mw[q] = warp_max(s[q]);
        }
        if (lane == 0) {
#pragma unroll
          for (int q = 0; q < kDtcN; ++q) red[((j & 1) * 4 + warp) * kDtcN + q] = mw[q];
        }
      }
      // every column's maximum over the tile's 128 keys (the four warps' maxima)
      ok = named_bar_and(1, 128, ok);
      if (!ok) break;
      float alpha[kDtcN];
      bool moved = false;
#pragma unroll
      for (int q = 0; q < kDtcN; ++q) {
        const float* rq = red + (j & 1) * 4 * kDtcN + q;
        const float tmax = fmaxf(fmaxf(rq[0], rq[kDtcN]), fmaxf(rq[2 * kDtcN], rq[3 * kDtcN]));
        const float m_new = tmax > m[q] + kDtcRescaleSlack ? tmax : m[q];
        alpha[q] = m_new == -INFINITY ? 1.f : ex2_approx(m[q] - m_new);  // 0 on the first
        moved = moved || alpha[q] != 1.f;
        m[q] = m_new;
      }
      // P_j^T into shared-memory buffer b, once P_j-2 V_j-2 has read it
      if (j >= 2)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kDtPFree + b),
                                               static_cast<uint32_t>((j - 2) >> 1) & 1, abort_flag));
      uint8_t* pt = smem + Lay::kP + b * Lay::kSmallBytes;
#pragma unroll
      for (int q = 0; q < kDtcN; ++q) {
        // a column with no visible key so far keeps m = -inf and gets p = 0
        const float p = m[q] == -INFINITY ? 0.f : ex2_approx(s[q] - m[q]);
        const uint32_t pk = pack2<BF16>(p, 0.f);
        float pr, unused;
        unpack2<BF16>(pk, pr, unused);
        l[q] = l[q] * alpha[q] + p;
        l_o[q] = l_o[q] * alpha[q] + pr;
        *reinterpret_cast<uint16_t*>(pt + small_swz(q, r)) = static_cast<uint16_t>(pk & 0xFFFFu);
      }
      // O^T columns whose reference moved (the first tile, then rarely): rescale them
      // once P_j-1 V_j-1 has landed. Two barriers by parity make the skipped waits
      // safe: S_j, complete by now, was issued after P_j-2 V_j-2.
      if (ok && j > 0 && __any_sync(0xffffffffu, moved)) {
        const int pj = j - 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kDtODone + (pj & 1)),
                                               static_cast<uint32_t>(pj >> 1) & 1, abort_flag));
        if (ok) {
          tc_fence_after();
          uint32_t o[kDtcN];
          tmem_ld16(lane_base + Lay::tO, o);
          tmem_wait_ld();
          reg_fence16(o);
#pragma unroll
          for (int q = 0; q < kDtcN; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha[q]);
          tmem_st16(lane_base + Lay::tO, o);
          tmem_wait_st();
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(kDtPFull + b));
      // a wait that gave up in one warp reaches the others at the next tile's
      // named_bar_and, where all four leave the loop together
    }
    // the last P V, then the row sums over the 128 keys
    ok = __all_sync(0xffffffffu, ok && (nt == 0 || mbar_wait(bar(kDtODone + ((nt - 1) & 1)),
                                                            static_cast<uint32_t>((nt - 1) >> 1) & 1,
                                                            abort_flag)));
    float* sums = reinterpret_cast<float*>(smem);  // the ring is free now: [warp][2][query]
    named_bar_sync(1, 128);
#pragma unroll
    for (int q = 0; q < kDtcN; ++q) {
      const float a = warp_sum(l[q]), c = warp_sum(l_o[q]);
      if (lane == 0) {
        sums[(warp * 2 + 0) * kDtcN + q] = a;
        sums[(warp * 2 + 1) * kDtcN + q] = c;
      }
    }
    ok = named_bar_and(1, 128, ok);
    if (ok) {
      uint32_t o[kDtcN];
      if (nt > 0) {
        tc_fence_after();
        tmem_ld16(lane_base + Lay::tO, o);
        tmem_wait_ld();
        reg_fence16(o);
      } else {
#pragma unroll
        for (int q = 0; q < kDtcN; ++q) o[q] = 0u;
      }
      // thread r holds column r of d for every query row
      for (int q = 0; q < Nq; ++q) {
        float lq = 0.f, loq = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          lq += sums[(w * 2 + 0) * kDtcN + q];
          loq += sums[(w * 2 + 1) * kDtcN + q];
        }
        const float val = loq > 0.f ? __uint_as_float(o[q]) / loq : 0.f;  // no key: O = 0
        const float Lrow = lq > 0.f ? (m[q] + log2f(lq)) * 0.69314718055994530942f : -INFINITY;
        if (splits == 1) {
          O[bb * so.sb + hh * so.sh + static_cast<long>(q) * so.sn + r] =
              static_cast<uint16_t>(pack2<BF16>(val, 0.f) & 0xFFFFu);
          if (r == 0) Lse[static_cast<long>(bh) * Nq + q] = Lrow;
        } else {
          const long prow = (static_cast<long>(bh) * splits + sp) * Nq + q;
          Opart[prow * D + r] = val;
          if (r == 0) Lpart[prow] = Lrow;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDtcMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace fa
