// fa_bwd.cuh -- exact attention backward for sm_100a.
//
// The backward keeps no N x N matrix: the forward left only the per-row log-sum-exp
// L, and the scores are recomputed here from Q, K and V (josueisai.com
// "flash-attention", section "Recomputar sale mas barato que recordar"). With
// P = exp(scale * Q K^T - L) the gradients are the standard ones:
//
//   dV = P^T dO,   dP = dO V^T,   D_i = sum_t dO_it O_it,   dS = P * (dP - D),
//   dQ = scale * dS K,   dK = scale * dS^T Q.
//
// Three kernels:
//   fa_bwd_pre_kernel   -D with D = rowsum(dO * (O + O_res)) (fp32; O_res is the
//                       forward's rounding residual of O, optional), -L * log2(e),
//                       dQacc = 0. The two row vectors are stored negated so that the
//                       main kernel forms s * c - L log2(e) and dP - D with packed
//                       fp32x2 FMA/add and no extra negation.
//   fa_bwd_main_kernel  one CTA per 128-key tile j of one head: K_j, V_j stay in
//                       shared memory, the CTA walks the query tiles i that see
//                       them, accumulates dK_j and dV_j in TMEM, and adds each
//                       dQ_i partial into the fp32 accumulator with TMA reduce-adds.
//   fa_bwd_dq_kernel    dQ = dtype(scale * dQacc).
//
// Main-kernel warp roles (512 threads = 4 warpgroups; at launch every thread may
// hold 128 registers, then warpgroup 3 hands registers to warpgroup 2 with setmaxnreg):
//   warps 0-7  compute, in pairs: warps w and w+4 share TMEM lane quarter w % 4, so
//              thread r of the pair owns key row r = 32 (w % 4) + lane; warp w < 4
//              takes query columns 0-63, warp w+4 columns 64-127 (no row reduction
//              is needed here: L and D are per query column). P^T from S^T and L,
//              dS^T from dP^T and D; P^T goes back to TMEM (16-bit), dS^T to shared
//              memory (16-bit, 128-byte swizzle; the dQ MMA's A, read M-major, which
//              TMEM cannot give) and at d = 128 also to TMEM (16-bit, over dP^T
//              columns already read; the dK MMA's A); at the end the
//              dK_j / dV_j epilogue, each warp of the pair writing half the columns.
//   warps 8-11 dQ drain (200 registers each): thread owns query row (warp % 4) * 32 +
//              lane; takes the whole dQ_i row out of TMEM at once, so that the
//              columns are free again after one round of loads, then stages it in
//              shared memory and has the TMA unit add it into the fp32 accumulator
//              (cp.reduce.async.bulk.tensor).
//   warp 12    TMA producer: K_j, V_j once; Q_i, Ls_i, D_i into a 2-stage ring; dO_i
//              into a single buffer (its last reader, the dV MMA, finishes well
//              before the next dP^T MMA needs the next tile).
//   warp 13    MMA issuer (and TMEM owner), per query tile:
//                S^T = K_j Q_i^T, dP^T = V_j dO_i^T           (SMEM x SMEM)
//                dV += P^T dO_i                              (P^T from TMEM)
//                dK += dS^T Q_i                   (dS^T from TMEM at d = 128)
//                dQ_i = dS K_j                               (dS from SMEM)
//   warps 14-15 idle (they complete warpgroup 3, which runs on 56 registers).
#pragma once

#include "fa_band.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kBwdThreads = 512;
constexpr int kBwdDrainWarp0 = 8;  // warpgroup 2
constexpr int kBwdProducerWarp = 12;
constexpr int kBwdMmaWarp = 13;
// Registers per thread after the split: 2 x 128 (compute) + 200 (drain) + 56 = 4 x 128,
// the budget of one sub-partition (one warp of each warpgroup) at launch, when every
// thread holds kBwdLaunchRegs (the most 512 threads can have; the host checks that
// the compiled kernel uses exactly that many).
constexpr int kBwdLaunchRegs = 128;
constexpr int kBwdDrainRegs = 200;
constexpr int kBwdSmallRegs = 56;
static_assert(kBwdThreads * kBwdLaunchRegs == 65536, "launch register budget");
static_assert(2 * kBwdLaunchRegs + kBwdDrainRegs + kBwdSmallRegs == 4 * kBwdLaunchRegs,
              "register split");

template <int D>
struct BwdLayout {
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr uint32_t kChunkBytes = kTile * 128;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kTileBytes;
  static constexpr uint32_t kQ = kV + kTileBytes;       // 2 stages
  static constexpr uint32_t kDO = kQ + 2 * kTileBytes;  // 1 stage
  static constexpr uint32_t kDS = kDO + kTileBytes;     // 128 keys x 128 queries, 16-bit
  static constexpr uint32_t kDSBytes = kTile * kTile * 2;
  static constexpr uint32_t kStage = kDS + kDSBytes;    // dQ staging: two 128 x 32 fp32 boxes
  static constexpr uint32_t kStageBytes = 2 * kTile * 128;
  static constexpr uint32_t kL = kStage + kStageBytes;  // 2 stages x 128 fp32
  static constexpr uint32_t kDv = kL + 2 * 512;         // 2 stages x 128 fp32
  static constexpr uint32_t kBar = kDv + 2 * 512;
  static constexpr int kNumBars = 16;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 8;
  static constexpr uint32_t kNeeded = kAbort + 8;
  // TMEM columns
  static constexpr uint32_t tDV = 0;
  static constexpr uint32_t tDK = D;
  static constexpr uint32_t tS = 2 * D;
  static constexpr uint32_t tDP = 2 * D + 128;
  static constexpr uint32_t tDQ = (D == 128) ? tDP : 2 * D + 256;  // d=128: dQ reuses dP^T
};

enum : int {
  kBbKVFull = 0,
  kBbQFull = 1,   // +stage (Q_i, Ls_i, D_i)
  kBbQEmpty = 3,  // +stage
  kBbSFull = 5,
  kBbDPFull = 6,
  kBbPReady = 7,
  kBbDSFree = 8,
  kBbDQFull = 9,
  kBbDQEmpty = 10,
  kBbDone = 11,
  kBbDOFull = 12,
  kBbDOEmpty = 13,
  kBbDSReady = 14,
};

// ------------------------------------------------------------------ preprocess
// One group of D/8 threads per row: 8 elements (16 bytes) per thread. Rows are walked
// in the padded per-head layout of Dv and Ls (n_pad = 128 * ceil(N / 128) rows per
// head); a padded row gets D = 0 and -L log2(e) = -inf, so that its p is exactly 0.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
    fa_bwd_pre_kernel(const uint16_t* __restrict__ O, const uint16_t* __restrict__ O_res,
                      const uint16_t* __restrict__ dO, const float* __restrict__ L,
                      float* __restrict__ Dv, float* __restrict__ Ls,
                      float* __restrict__ dq_acc, int N, int n_pad, long padded_rows, int H,
                      Strides st) {
  constexpr int kTpr = D / 8;  // threads per row
  const long gid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long prow = gid / kTpr;  // row in the padded layout
  const int part = static_cast<int>(gid % kTpr);
  const long bh = prow / n_pad;
  const int n = static_cast<int>(prow - bh * n_pad);
  const bool real = prow < padded_rows && n < N;
  const long row = bh * N + n;  // row of L and of the dQ accumulator ([B][H][N] order)
  const int bhi = static_cast<int>(bh);  // < 2^31 (checked on the host)
  const long el = (bhi / H) * st.sb + (bhi % H) * st.sh + n * st.sn + part * 8;  // O, dO
  float acc = 0.f;
  if (real) {
    const uint4 o = *reinterpret_cast<const uint4*>(O + el);
    const uint4 g = *reinterpret_cast<const uint4*>(dO + el);
    const uint4 res = O_res != nullptr ? *reinterpret_cast<const uint4*>(O_res + el)
                                       : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t* ow = reinterpret_cast<const uint32_t*>(&o);
    const uint32_t* rw = reinterpret_cast<const uint32_t*>(&res);
    const uint32_t* gw = reinterpret_cast<const uint32_t*>(&g);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float o0, o1, r0, r1, g0, g1;
      unpack2<BF16>(ow[e], o0, o1);
      unpack2<BF16>(rw[e], r0, r1);
      unpack2<BF16>(gw[e], g0, g1);
      acc = fmaf(o0 + r0, g0, acc);
      acc = fmaf(o1 + r1, g1, acc);
    }
    if (dq_acc != nullptr) {
      float4* z = reinterpret_cast<float4*>(dq_acc + row * D + part * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (prow < padded_rows && part == 0) {
    Dv[prow] = real ? -acc : 0.f;
    // -L log2(e); a row that sees no key (L = -inf) gets -inf too, so that its p is 0
    Ls[prow] = (real && L[row] != -INFINITY) ? L[row] * -1.4426950408889634074f : -INFINITY;
  }
}

// ------------------------------------------------------------------ dQ convert
// dQ = dtype(scale * dQacc); the accumulator is [B*H][N][D] fp32, dQ has strides `st`.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
    fa_bwd_dq_kernel(const float* __restrict__ dq_acc, uint16_t* __restrict__ dQ, float scale,
                     long n8, int N, int H, Strides st) {
  const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(dq_acc)[2 * i + 1];
  uint4 out;
  out.x = pack2<BF16>(a.x * scale, a.y * scale);
  out.y = pack2<BF16>(a.z * scale, a.w * scale);
  out.z = pack2<BF16>(b.x * scale, b.y * scale);
  out.w = pack2<BF16>(b.z * scale, b.w * scale);
  const long row = i / (D / 8);
  const int part = static_cast<int>(i - row * (D / 8));
  const int bh = static_cast<int>(row / N);  // < 2^31 (checked on the host)
  const long n = row - static_cast<long>(bh) * N;
  *reinterpret_cast<uint4*>(dQ + (bh / H) * st.sb + (bh % H) * st.sh + n * st.sn + part * 8) =
      out;
}

// --------------------------------------------------------------- main dK/dV
// BAND as in the forward: false = every key visible, true = the key window [wl, wr]
// (causal: wl = kUnbounded, wr = 0). dK and dV are written with element strides `kv`.
// DQ = false leaves dQ to the separate pass of fa_bwd_dq.cuh: no dQ MMA, no drain.
template <int D, bool BAND, bool BF16, bool DQ>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmDQ, const float* __restrict__ Ls,
                       const float* __restrict__ Dv, float* __restrict__ dq_acc,
                       uint16_t* __restrict__ dK, uint16_t* __restrict__ dV, int Nq, int Nk,
                       int H, int wl, int wr, Strides kv, float scale, float scale_log2,
                       uint32_t smem_alloc, int group) {
  // dS^T for the dK MMA: from TMEM at d = 128, from shared memory at d = 64
  constexpr bool kDsInTmem = D == 128;
  using Lay = BwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  if (pad + Lay::kNeeded > smem_alloc) {
    // Shared memory is not placed as this kernel needs; report and do nothing.
    if (threadIdx.x == 0) atomicExch(&g_fa_status, -3);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;

  FA_TRACE_CTA(0);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntq = (Nq + kTile - 1) / kTile;  // query tiles per head
  const int ntk = (Nk + kTile - 1) / kTile;  // key tiles per head (one CTA each)
  // band: heads in groups, each group's key tiles rank-major (band_order; under the
  // causal mask key tile 0 has the most work); otherwise head-major
  int bh, j;  // j: key tile
  if (BAND) {
    band_order(blockIdx.x, ntk, gridDim.x / ntk, group, &bh, &j);
  } else {
    bh = blockIdx.x / ntk;
    j = blockIdx.x - bh * ntk;
  }
  const int hh = bh % H;  // head
  const int bb = bh / H;  // batch
  // Rows past Nq / Nk arrive as zeros through the tensor maps. Padded queries, and
  // queries that see no key, have Ls = -inf, so their P is 0. Padded keys of the last
  // key tile need no mask: their dK and dV rows are not stored, and their dS meets
  // zero rows of K in dQ = dS K. Ls and Dv are laid out per head with ntq * 128 rows.
  // The query tiles walked are those with a row that sees a key of this tile (under
  // the causal mask there is at least one, because the last query sees every key; a
  // sliding window may leave a key tile unseen, and its dK, dV are then zero).
  const TileRange qr = BAND ? query_tiles_of_kv_tile(j, kTile, Nq, Nk, wl, wr)
                            : TileRange{0, ntq};
  const int i_begin = qr.first;
  const int niter = qr.count;
  const int off = Nk - Nq;

  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar(kBbKVFull), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBbQFull + s), 1);
      mbar_init(bar(kBbQEmpty + s), 1);
    }
    mbar_init(bar(kBbSFull), 1);
    mbar_init(bar(kBbDPFull), 1);
    mbar_init(bar(kBbPReady), 256);
    mbar_init(bar(kBbDSReady), 256);
    mbar_init(bar(kBbDSFree), 1);
    mbar_init(bar(kBbDQFull), 1);
    mbar_init(bar(kBbDQEmpty), 128);
    mbar_init(bar(kBbDone), 1);
    mbar_init(bar(kBbDOFull), 1);
    mbar_init(bar(kBbDOEmpty), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(sbase + Lay::kTmemSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  FA_TRACE_BEGIN();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Lay::kTmemSlot);

  if (warp == kBwdProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    setmaxnreg_dec<kBwdSmallRegs>();  // each role of warpgroup 3 gives registers back
    if (lane == 0 && niter > 0) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      tma_prefetch(&tmDO);
      tma_prefetch(&tmDQ);

      mbar_expect_tx(bar(kBbKVFull), 2 * Lay::kTileBytes);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_4d(sbase + Lay::kK + c * Lay::kChunkBytes, &tmK, c * 64, j * kTile, hh, bb,
                    bar(kBbKVFull));
        tma_load_4d(sbase + Lay::kV + c * Lay::kChunkBytes, &tmV, c * 64, j * kTile, hh, bb,
                    bar(kBbKVFull));
      }
      for (int it = 0; it < niter; ++it) {
        const int st = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        const int qtile = (i_begin + it) * kTile;  // first query row within the head
        const long head_pad = static_cast<long>(bh) * ntq * kTile;  // Ls / Dv rows
        if (it >= 2 && !mbar_wait(bar(kBbQEmpty + st), (use - 1) & 1, abort_flag)) break;
        const uint32_t full = bar(kBbQFull + st);
        mbar_expect_tx(full, Lay::kTileBytes + 2 * 512);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Lay::kQ + st * Lay::kTileBytes + c * Lay::kChunkBytes, &tmQ, c * 64,
                      qtile, hh, bb, full);
        bulk_load(sbase + Lay::kL + st * 512, Ls + head_pad + qtile, 512, full);
        bulk_load(sbase + Lay::kDv + st * 512, Dv + head_pad + qtile, 512, full);
        if (it >= 1 &&
            !mbar_wait(bar(kBbDOEmpty), static_cast<uint32_t>((it - 1) & 1), abort_flag))
          break;
        mbar_expect_tx(bar(kBbDOFull), Lay::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Lay::kDO + c * Lay::kChunkBytes, &tmDO, c * 64, qtile, hh, bb,
                      bar(kBbDOFull));
        FA_TRACE_EVENT(it, 0);
      }
    }
  } else if (warp == kBwdMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    setmaxnreg_dec<kBwdSmallRegs>();
    // Software-pipelined over the query tiles: with G1 = S^T, G2 = dP^T, G3 = dV,
    // G4 = dK, G5 = dQ, the issue order is
    //   G1(0) G2(0) | G3(0) G1(1) G4(0) G5(0) G2(1) | G3(1) G1(2) G4(1) G5(1) G2(2) | ...
    // so that S^T of the next tile is computed while the compute warps form dS of the
    // current one, and dK/dQ of the current tile while they exponentiate the next.
    // G1(i+1) overwrites the S^T/P^T columns only after G3(i), which reads P^T, has
    // been issued (MMAs from one thread execute in issue order).
    if (lane == 0 && niter > 0) {
      constexpr uint32_t id_sq = idesc_f16_f32(kTile, kTile, BF16, false, false);  // S^T, dP^T
      constexpr uint32_t id_acc = idesc_f16_f32(kTile, D, BF16, false, true);      // dV, dK
      constexpr uint32_t id_dq = idesc_f16_f32(kTile, D, BF16, true, true);        // dQ
      // operand descriptors, built once: K-major views for S^T/dP^T/dK's A, MN-major
      // views for the B operands of dV/dK/dQ and dQ's A
      const uint64_t dk_k = sdesc_sw128(sbase + Lay::kK, 16, 1024);
      const uint64_t dv_k = sdesc_sw128(sbase + Lay::kV, 16, 1024);
      const uint64_t ddo_k = sdesc_sw128(sbase + Lay::kDO, 16, 1024);
      const uint64_t dds_k = sdesc_sw128(sbase + Lay::kDS, 16, 1024);
      const uint64_t dk_mn = sdesc_sw128(sbase + Lay::kK, Lay::kChunkBytes, 1024);
      const uint64_t ddo_mn = sdesc_sw128(sbase + Lay::kDO, Lay::kChunkBytes, 1024);
      const uint64_t dds_mn = sdesc_sw128(sbase + Lay::kDS, Lay::kChunkBytes, 1024);
      auto issue_s = [&](int it) -> bool {  // G1: S^T = K_j Q_i^T
        const int st = it & 1;
        if (!mbar_wait(bar(kBbQFull + st), static_cast<uint32_t>(it >> 1) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t dq = sdesc_sw128(sbase + Lay::kQ + st * Lay::kTileBytes, 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t koff = (k >> 2) * Lay::kChunkBytes + (k & 3) * 32;
          mma_ss(tmem + Lay::tS, sdesc_step(dk_k, koff), sdesc_step(dq, koff), id_sq,
                 k > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBbSFull));
        FA_TRACE_EVENT(it, 2);
        return true;
      };
      auto issue_dp = [&](int it) -> bool {  // G2: dP^T = V_j dO_i^T
        if (!mbar_wait(bar(kBbDOFull), static_cast<uint32_t>(it & 1), abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t koff = (k >> 2) * Lay::kChunkBytes + (k & 3) * 32;
          mma_ss(tmem + Lay::tDP, sdesc_step(dv_k, koff), sdesc_step(ddo_k, koff), id_sq,
                 k > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBbDPFull));
        FA_TRACE_EVENT(it, 4);
        return true;
      };
      bool ok = mbar_wait(bar(kBbKVFull), 0, abort_flag) && issue_s(0) && issue_dp(0);
      for (int it = 0; ok && it < niter; ++it) {
        const int st = it & 1;
        const uint32_t ph = static_cast<uint32_t>(it & 1);
        const uint32_t sq = sbase + Lay::kQ + st * Lay::kTileBytes;
        // G3: dV += P^T dO_i (K = the 128 queries of tile i), P^T from TMEM
        if (!mbar_wait(bar(kBbPReady), ph, abort_flag)) break;
        FA_TRACE_EVENT(it, 5);
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)
          mma_ts(tmem + Lay::tDV, tmem + Lay::tS + k * 8, sdesc_step(ddo_mn, k * 2048), id_acc,
                 (it > 0 || k > 0) ? 1u : 0u);
        mma_commit(bar(kBbDOEmpty));  // dO_i has been read for the last time
        FA_TRACE_EVENT(it, 3);
        if (it + 1 < niter && !issue_s(it + 1)) break;
        // G4, G5 once dS_i is in shared memory
        if (!mbar_wait(bar(kBbDSReady), ph, abort_flag)) break;
        FA_TRACE_EVENT(it, 1);
        if (DQ && D != 128 && it > 0 && !mbar_wait(bar(kBbDQEmpty), ph ^ 1u, abort_flag)) break;
        tc_fence_after();
        // dK += dS^T Q_i. At d = 128 dS^T comes from TMEM: query columns 16k .. 16k + 15
        // are packed in the dP^T columns of the compute warp that owns them (64 per half,
        // the first 32 used); at d = 64 from shared memory.
        const uint64_t dq_mn = sdesc_sw128(sq, Lay::kChunkBytes, 1024);
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
          if constexpr (kDsInTmem) {
            mma_ts(tmem + Lay::tDK, tmem + Lay::tDP + (k >> 2) * 64 + (k & 3) * 8,
                   sdesc_step(dq_mn, k * 2048), id_acc, (it > 0 || k > 0) ? 1u : 0u);
          } else {
            const uint32_t koff = (k >> 2) * Lay::kChunkBytes + (k & 3) * 32;
            mma_ss(tmem + Lay::tDK, sdesc_step(dds_k, koff), sdesc_step(dq_mn, k * 2048), id_acc,
                   (it > 0 || k > 0) ? 1u : 0u);
          }
        }
        if constexpr (DQ) {
          // dQ_i = dS K_j   (dS read M-major from the same shared tile)
#pragma unroll
          for (int k = 0; k < kTile / 16; ++k)
            mma_ss(tmem + Lay::tDQ, sdesc_step(dds_mn, k * 2048), sdesc_step(dk_mn, k * 2048),
                   id_dq, k > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBbQEmpty + st));
        mma_commit(bar(kBbDSFree));
        if constexpr (DQ) mma_commit(bar(kBbDQFull));
        FA_TRACE_EVENT(it, 6);
        if (it + 1 < niter) {
          // G2 of the next tile. At d = 128 its columns hold dQ_i until the drain has
          // copied it out.
          if (DQ && D == 128 && !mbar_wait(bar(kBbDQEmpty), ph, abort_flag)) break;
          if (!issue_dp(it + 1)) break;
        }
      }
      mma_commit(bar(kBbDone));
    }
  } else if (warp < 8) {
    // ----------------------------------------------------------------- compute
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int r = quarter * 32 + lane;  // key row within the tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint8_t* sds_row = smem + Lay::kDS + half * Lay::kChunkBytes + r * 128;
    const int sw = r & 7;
    // The two warps of a pair meet at one named barrier per query tile and leave the
    // loop together: a failed wait is carried to the next meeting, where bar.red.and
    // makes both warps see it, so that neither is ever left waiting there alone.
    bool ok = true;
    for (int it = 0; it < niter; ++it) {
      const int st = it & 1;
      const uint32_t ph = static_cast<uint32_t>(it & 1);
      // band: query column qc of tile i sees key row r when r - dl - wr <= qc <= r - dl + wl
      const int dl = (i_begin + it) * kTile + off - j * kTile;
      const bool lo_edge = BAND && dl + wr < kTile - 1;     // some columns below the band
      const bool hi_edge = BAND && dl - wl > -(kTile - 1);  // some columns above it
      const bool got = __all_sync(
          0xffffffffu,
          ok && mbar_wait(bar(kBbQFull + st), static_cast<uint32_t>(it >> 1) & 1, abort_flag) &&
              mbar_wait(bar(kBbSFull), ph, abort_flag));
      if (got && threadIdx.x == 0) FA_TRACE_EVENT(it, 7);
      const float* sL = reinterpret_cast<const float*>(smem + Lay::kL + st * 512) + half * 64;
      const float* sD = reinterpret_cast<const float*>(smem + Lay::kDv + st * 512) + half * 64;
      // Both halves load their S^T columns before either writes P^T: the packed P^T
      // of the upper half (columns 32-63) lands on S^T columns of the lower half.
      float p[64];
      if (got) {
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(lane_base + Lay::tS + half * 64, sr);
        tmem_ld32(lane_base + Lay::tS + half * 64 + 32, sr + 32);
        tmem_wait_ld();
        reg_fence32(sr);
        reg_fence32(sr + 32);
#pragma unroll
        for (int q = 0; q < 64; ++q) p[q] = __uint_as_float(sr[q]);
      }
      ok = named_bar_and(1 + quarter, 64, got);
      if (!ok) break;
      if (threadIdx.x == 0) FA_TRACE_EVENT(it, 8);
      const uint64_t c2 = f2_pack(scale_log2, scale_log2);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const int q = c * 32 + e4 * 4;  // query column within this half
          // -L log2(e) of four query columns (a broadcast read)
          const float4 nl = *reinterpret_cast<const float4*>(sL + q);
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(p[q], p[q + 1]), c2, f2_pack(nl.x, nl.y)), x0, x1);
          f2_unpack(f2_fma(f2_pack(p[q + 2], p[q + 3]), c2, f2_pack(nl.z, nl.w)), x2, x3);
          p[q] = ex2_approx(x0);
          p[q + 1] = ex2_approx(x1);
          p[q + 2] = ex2_approx(x2);
          p[q + 3] = ex2_approx(x3);
          if (lo_edge || hi_edge) {
            // this half's first and last visible column
            const int qmin = (lo_edge ? r - dl - wr : 0) - half * 64;
            const int qmax = (hi_edge ? r - dl + wl : kTile - 1) - half * 64;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (q + e < qmin || q + e > qmax) p[q + e] = 0.f;
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack2<BF16>(p[c * 32 + 2 * e], p[c * 32 + 2 * e + 1]);
        tmem_st16(lane_base + Lay::tS + half * 32 + c * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBbPReady));  // P^T is in TMEM: the dV MMA may go
      if (threadIdx.x == 0) FA_TRACE_EVENT(it, 9);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kBbDPFull), ph, abort_flag) &&
                                       (it == 0 || mbar_wait(bar(kBbDSFree), ph ^ 1u, abort_flag)));
      if (!ok) continue;  // the pair agrees at the next meeting (or after the loop)
      if (threadIdx.x == 0) FA_TRACE_EVENT(it, 10);
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dr[32];
        tmem_ld32(lane_base + Lay::tDP + half * 64 + c * 32, dr);
        tmem_wait_ld();
        reg_fence32(dr);
        // queries half*64 + c*32 .. +31 = 16-byte units c*4 .. c*4+3 of swizzle column `half`
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t ds[4];
          // -D of eight query columns (broadcast reads)
          const float4 nd0 = *reinterpret_cast<const float4*>(sD + c * 32 + 8 * u);
          const float4 nd1 = *reinterpret_cast<const float4*>(sD + c * 32 + 8 * u + 4);
          const float ndv[8] = {nd0.x, nd0.y, nd0.z, nd0.w, nd1.x, nd1.y, nd1.z, nd1.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k = 8 * u + 2 * e;  // column within this 32-column chunk
            const int q = c * 32 + k;
            // dS = P (dP - D), two columns per packed fp32x2 add and multiply
            float a, b;
            f2_unpack(f2_mul(f2_pack(p[q], p[q + 1]),
                             f2_add(f2_pack(__uint_as_float(dr[k]), __uint_as_float(dr[k + 1])),
                                    f2_pack(ndv[2 * e], ndv[2 * e + 1]))),
                      a, b);
            ds[e] = pack2<BF16>(a, b);
          }
          const int unit = (c * 4 + u) ^ sw;
          *reinterpret_cast<uint4*>(sds_row + unit * 16) = make_uint4(ds[0], ds[1], ds[2], ds[3]);
          // at d = 128 the same 8 query columns also go to tensor memory, packed over
          // dP^T columns this warp has loaded already (the first 32 of its 64): the dK
          // MMA takes its A operand from there and reads no shared memory for it (at
          // d = 64 the kernel has shared-memory bandwidth to spare, and the extra live
          // values would spill in its band variants)
          if constexpr (kDsInTmem)
            tmem_st4(lane_base + Lay::tDP + half * 64 + c * 16 + 4 * u, ds[0], ds[1], ds[2],
                     ds[3]);
        }
      }
      fence_async_smem();
      if constexpr (kDsInTmem) tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBbDSReady));  // dS^T is in place: dK and dQ may go
      if (threadIdx.x == 0) FA_TRACE_EVENT(it, 11);
    }
    // A key tile that no query sees (possible under a sliding window) ran no MMA: its
    // dK and dV rows are zero.
    const bool seen = niter > 0;
    ok = __all_sync(0xffffffffu, ok && (!seen || mbar_wait(bar(kBbDone), 0, abort_flag)));
    if (ok) {
      if (seen) tc_fence_after();
      const int key = j * kTile + r;
      const bool live_row = key < Nk;  // padded keys of the last tile are not stored
      const long el = bb * kv.sb + hh * kv.sh + static_cast<long>(key) * kv.sn + half * (D / 2);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = (which == 0 ? Lay::tDV : Lay::tDK) + half * (D / 2);
        const float mul = which == 0 ? 1.f : scale;
        uint16_t* dst_row = (which == 0 ? dV : dK) + el;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t v[32];
          if (seen) {
            tmem_ld32(lane_base + col + c * 32, v);
            tmem_wait_ld();
            reg_fence32(v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          uint4 pk[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pw[e] = pack2<BF16>(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
          uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
          if (live_row) {
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = pk[e];
          }
        }
      }
    }
  } else if (warp < kBwdDrainWarp0 + 4) {
    // ---------------------------------------------------------------- dQ drain
    setmaxnreg_inc<kBwdDrainRegs>();
    // dQ_i leaves TMEM into registers (then the MMA warp may reuse the columns), is
    // staged in shared memory in the 128-byte-swizzled layout of a 128-row x 32-column
    // fp32 box, and is added into the fp32 accumulator by TMA reduce-adds that one
    // thread issues. Before a round overwrites the staging buffer, that thread waits
    // until the TMA unit has read the previous round.
    const int quarter = warp & 3;
    const int qr = quarter * 32 + lane;  // query row within tile i
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool leader = (warp == kBwdDrainWarp0 && lane == 0);
    const uint32_t stage = sbase + Lay::kStage;
    uint8_t* stage_row = smem + Lay::kStage + qr * 128;
    const int sw = qr & 7;
    for (int it = 0; it < (DQ ? niter : 0); ++it) {
      // Each warp frees its TMEM lanes as soon as dQ_i is there (the next dP^T MMA
      // waits for that); the four warps agree before touching the shared staging
      // buffer, so that all of them meet every named barrier below.
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar(kBbDQFull),
                                                         static_cast<uint32_t>(it & 1), abort_flag));
      uint32_t v[D];
      if (got) {
        if (leader) FA_TRACE_EVENT(it, 12);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(lane_base + Lay::tDQ + c * 32, v + c * 32);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) reg_fence32(v + c * 32);
        tc_fence_before();
        mbar_arrive(bar(kBbDQEmpty));
        if (leader) FA_TRACE_EVENT(it, 13);
      }
      if (!named_bar_and(5, 128, got)) break;
      const int qtile = (i_begin + it) * kTile;
#pragma unroll
      for (int rnd = 0; rnd < D / 64; ++rnd) {
        if (leader) bulk_wait_read_all();  // previous round's boxes have been read
        named_bar_sync(5, 128);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int box = 2 * rnd + h;  // columns 32 box .. 32 box + 31
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(stage_row + h * Lay::kChunkBytes + ((u ^ sw) * 16)) =
                make_uint4(v[32 * box + 4 * u], v[32 * box + 4 * u + 1],
                           v[32 * box + 4 * u + 2], v[32 * box + 4 * u + 3]);
        }
        fence_async_smem();
        named_bar_sync(5, 128);
        if (leader) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_reduce_add_4d(&tmDQ, stage + h * Lay::kChunkBytes, 32 * (2 * rnd + h), qtile, hh,
                              bb);
          bulk_commit();
        }
      }
      if (leader) FA_TRACE_EVENT(it, 14);
    }
    if (leader) bulk_wait_all();  // every reduce-add has landed before the CTA exits
  } else {
    setmaxnreg_dec<kBwdSmallRegs>();  // warps 14-15: no role
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  FA_TRACE_CTA(1);
}

}  // namespace fa
