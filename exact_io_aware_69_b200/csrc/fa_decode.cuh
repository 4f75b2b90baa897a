// fa_decode.cuh -- a few query rows (decode) against a long key sequence, split
// across CTAs along the keys and merged by log-sum-exp.
//
// With N_q <= 16 rows per head there is too little work per head for one CTA per
// query tile, and every K and V element is used by at most 16 dot products: the pass
// is bound by reading K and V from HBM, not by arithmetic. So the keys of each head
// are cut into splits of consecutive 128-key tiles, one CTA per (head, split), each
// streaming its tiles through shared memory once and running the online softmax of
// josueisai.com "flash-attention", section "El truco: trocear y llevar la cuenta del
// softmax" (running max m, running sum l, rescaled partial output) over them on CUDA
// cores. A second kernel merges the splits' (O_s, L_s) the same way the recurrence
// merges blocks: L = ln sum_s exp(L_s), O = sum_s exp(L_s - L) O_s. (kerneldigest.dev
// "FlashAttention" names inference serving as a user of the method; foqum.io
// "FlashAttention", Q3, the long contexts it makes affordable.)
//
// CTA: 4 compute warps and 1 TMA producer warp, for up to 8 query rows (rows 9-16 of a
// head go to a second CTA over the same keys, whose tiles then mostly come from L2).
// Warp w takes keys 32 w .. 32 w + 31 of every tile. For the scores each lane owns d/32 columns: it forms 32 partial dot
// products (one per key of the warp's group) and a butterfly reduce-scatter over the
// lanes leaves lane k with the full score of key k. For P V each lane owns the same
// d/32 columns of O and takes the probabilities from the key lanes by shuffle. Each
// warp keeps its own (m, l, O) per query row; at the end of the split the four are
// merged through shared memory. P stays fp32 (no 16-bit rounding on this path).
#pragma once

#include "fa_band.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kDecWarps = 4;     // compute warps (one per 32 keys of a tile)
constexpr int kDecThreads = (kDecWarps + 1) * 32;  // + the TMA producer warp
constexpr int kDecMaxQ = 16;
constexpr int kDecQPerCta = 8;   // query rows one CTA carries; 9-16 rows take two CTAs

template <int D>
struct DecLayout {
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr uint32_t kChunkBytes = kTile * 128;
  static constexpr int kStages = D == 128 ? 3 : 6;
  static constexpr uint32_t kStageBytes = 2 * kTileBytes;  // K tile, then V tile
  static constexpr uint32_t kBar = kStages * kStageBytes;
  static constexpr int kNumBars = 2 * kStages;  // full, empty per stage (empty counts warps)
  static constexpr uint32_t kAbort = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kAbort + 8 + 1024;
  // per-warp (m, l, O) for the merge of the four warps, over the ring once it is done
  static constexpr uint32_t kMergeBytes = kDecWarps * kDecMaxQ * (2 + D) * 4;
  static_assert(kMergeBytes <= kBar, "merge scratch fits in the ring");
};

// Byte offset, within a 128-byte-swizzled [128 rows][D] 16-bit tile (64-column chunks
// of 128 rows x 128 bytes), of the `bytes`-wide piece of row `row` that starts at
// column `col`.
template <int D>
__device__ __forceinline__ uint32_t swz_offset(int row, int col) {
  const int chunk = col / 64;
  const int byte = (col % 64) * 2;
  return static_cast<uint32_t>(chunk * kTile * 128 + row * 128 +
                               ((((byte >> 4) ^ (row & 7)) << 4) | (byte & 15)));
}

// Loads this lane's d/32 columns of row `row` of a swizzled 16-bit tile as floats.
template <int D, bool BF16>
__device__ __forceinline__ void load_row_cols(uint32_t tile, int row, int lane, float* out) {
  constexpr int CPL = D / 32;
  const uint32_t addr = tile + swz_offset<D>(row, lane * CPL);
  if constexpr (CPL == 4) {
    uint32_t a, b;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "r"(addr));
    unpack2<BF16>(a, out[0], out[1]);
    unpack2<BF16>(b, out[2], out[3]);
  } else {
    uint32_t a;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(a) : "r"(addr));
    unpack2<BF16>(a, out[0], out[1]);
  }
}

// v[k] holds this lane's part of the sum for item k (k < 32); afterwards lane i holds
// the full sum over the 32 lanes of item i. Each round halves the items a lane keeps,
// choosing the half by one bit of its lane index, highest bit first.
__device__ __forceinline__ float reduce_scatter32(float* v, int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, s));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) x += __shfl_xor_sync(0xffffffffu, x, s);
  return x;
}

// One CTA per (head bh, split s, query group); the split covers key tiles
// [tile0 + s*tps, min(tile0 + ntiles, tile0 + (s+1)*tps)), the group query rows
// [8 group, 8 group + QW). With splits == 1 the CTA writes O (16-bit, strides so) and L
// itself; otherwise its normalised partial output and log-sum-exp go to Opart
// [BH][splits][Nq][D] and Lpart [BH][splits][Nq] (fp32) for the merge.
template <int D, int QW, bool BAND, bool BF16>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const uint16_t* __restrict__ Q,
                     Strides sq, uint16_t* __restrict__ O, Strides so, float* __restrict__ Lse,
                     float* __restrict__ Opart, float* __restrict__ Lpart, int Nq, int Nk, int H,
                     int wl, int wr, int tile0, int ntiles, int tps, int splits,
                     float scale_log2) {
  using Lay = DecLayout<D>;
  constexpr int CPL = D / 32;  // columns per lane
  constexpr int S = Lay::kStages;
  constexpr int kCompute = kDecWarps;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int groups = (Nq + kDecQPerCta - 1) / kDecQPerCta;
  const int cta = blockIdx.x / groups;  // (head, split)
  const int grp = blockIdx.x - cta * groups;
  const int bh = cta / splits;
  const int sp = cta - bh * splits;
  const int hh = bh % H;
  const int bb = bh / H;
  const int t_begin = tile0 + sp * tps;
  const int t_end = min(tile0 + ntiles, t_begin + tps);
  const int nt = t_end > t_begin ? t_end - t_begin : 0;

  auto full = [&](int st) -> uint32_t { return sbase + Lay::kBar + 8u * st; };
  auto empty = [&](int st) -> uint32_t { return sbase + Lay::kBar + 8u * (S + st); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kAbort);
  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), kCompute);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCompute) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      for (int i = 0; i < nt; ++i) {
        const int st = i % S;
        if (i >= S &&
            !mbar_wait(empty(st), static_cast<uint32_t>(i / S - 1) & 1, abort_flag))
          break;
        const uint32_t dst = sbase + st * Lay::kStageBytes;
        mbar_expect_tx(full(st), Lay::kStageBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(dst + c * Lay::kChunkBytes, &tmK, c * 64, (t_begin + i) * kTile, hh, bb,
                      full(st));
          tma_load_4d(dst + Lay::kTileBytes + c * Lay::kChunkBytes, &tmV, c * 64,
                      (t_begin + i) * kTile, hh, bb, full(st));
        }
      }
    }
    return;  // the producer takes no part in the merge below
  }

  // ------------------------------------------------------------------- compute
  const int kw = warp;            // key group: rows 32 kw .. 32 kw + 31 of every tile
  const int q0 = grp * kDecQPerCta;  // first query row of this CTA
  // this lane's columns of the group's query rows, times scale * log2(e): scores come
  // out in base-2 units
  float qr[QW][CPL];
#pragma unroll
  for (int qi = 0; qi < QW; ++qi) {
    const int q = q0 + qi;
    if (q < Nq) {
      const uint16_t* src = Q + bb * sq.sb + hh * sq.sh + static_cast<long>(q) * sq.sn + lane * CPL;
      float f[4];
      if constexpr (CPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(src);
        unpack2<BF16>(u.x, f[0], f[1]);
        unpack2<BF16>(u.y, f[2], f[3]);
      } else {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(src);
        unpack2<BF16>(u, f[0], f[1]);
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) qr[qi][c] = f[c] * scale_log2;
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) qr[qi][c] = 0.f;
    }
  }
  float m[QW], lp[QW], o[QW][CPL];
#pragma unroll
  for (int qi = 0; qi < QW; ++qi) {
    m[qi] = -INFINITY;
    lp[qi] = 0.f;  // this lane's share of the row sum
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[qi][c] = 0.f;
  }
  const int off = Nk - Nq;
  bool ok = true;
  for (int i = 0; i < nt && ok; ++i) {
    const int st = i % S;
    ok = __all_sync(0xffffffffu, mbar_wait(full(st), static_cast<uint32_t>(i / S) & 1, abort_flag));
    if (!ok) break;
    const uint32_t tk = sbase + st * Lay::kStageBytes;
    const uint32_t tv = tk + Lay::kTileBytes;
    const int row0 = kw * 32;                               // this warp's rows of the tile
    const int key = (t_begin + i) * kTile + row0 + lane;    // the key this lane scores
    float p[QW];
#pragma unroll
    for (int qi = 0; qi < QW; ++qi) {
      const int q = q0 + qi;
      float part[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        float kv[CPL];
        load_row_cols<D, BF16>(tk, row0 + k, lane, kv);
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc = fmaf(qr[qi][c], kv[c], acc);
        part[k] = acc;
      }
      float sc = reduce_scatter32(part, lane);
      const bool visible = key < Nk && q < Nq &&
                           (!BAND || (key >= q + off - wl && key <= q + off + wr));
      sc = visible ? sc : -INFINITY;
      const float m_new = fmaxf(m[qi], warp_max(sc));
      // a row with no visible key so far keeps m = -inf, alpha = 1, p = 0
      const float alpha = m_new == -INFINITY ? 1.f : ex2_approx(m[qi] - m_new);
      p[qi] = m_new == -INFINITY ? 0.f : ex2_approx(sc - m_new);
      lp[qi] = lp[qi] * alpha + p[qi];
#pragma unroll
      for (int c = 0; c < CPL; ++c) o[qi][c] *= alpha;
      m[qi] = m_new;
    }
#pragma unroll 4
    for (int k = 0; k < 32; ++k) {
      float vv[CPL];
      load_row_cols<D, BF16>(tv, row0 + k, lane, vv);
#pragma unroll
      for (int qi = 0; qi < QW; ++qi) {
        const float pk = __shfl_sync(0xffffffffu, p[qi], k);
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[qi][c] = fmaf(pk, vv[c], o[qi][c]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(st));
  }

  // merge the four key groups' (m, l, O) of every row of this CTA, in the ring (every
  // warp is past its last tile)
  const bool all_ok = named_bar_and(1, kCompute * 32, ok);
  float* wm = reinterpret_cast<float*>(smem);           // [key group][row]
  float* wsum = wm + kDecWarps * kDecMaxQ;               // [key group][row]
  float* wo = wsum + kDecWarps * kDecMaxQ;               // [key group][row][D]
  if (all_ok) {
#pragma unroll
    for (int qi = 0; qi < QW; ++qi) {
      const int q = q0 + qi;
      const float l = warp_sum(lp[qi]);
      if (lane == 0) {
        wm[kw * kDecMaxQ + q] = m[qi];
        wsum[kw * kDecMaxQ + q] = l;
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) wo[(kw * kDecMaxQ + q) * D + lane * CPL + c] = o[qi][c];
    }
  }
  named_bar_sync(1, kCompute * 32);
  if (!all_ok) return;
  const int q_end = min(Nq, q0 + QW);
  for (int q = q0 + warp; q < q_end; q += kCompute) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wm[w * kDecMaxQ + q]);
    float l = 0.f, oc[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) oc[c] = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = wm[w * kDecMaxQ + q];
        const float f = mw == -INFINITY ? 0.f : ex2_approx(mw - M);
        l += f * wsum[w * kDecMaxQ + q];
#pragma unroll
        for (int c = 0; c < CPL; ++c) oc[c] += f * wo[(w * kDecMaxQ + q) * D + lane * CPL + c];
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;  // a row with no visible key: O = 0
    const float Lrow = l > 0.f ? (M + log2f(l)) * 0.69314718055994530942f : -INFINITY;
    if (splits == 1) {
      uint16_t* dst = O + bb * so.sb + hh * so.sh + static_cast<long>(q) * so.sn + lane * CPL;
      if constexpr (CPL == 4) {
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(pack2<BF16>(oc[0] * inv, oc[1] * inv), pack2<BF16>(oc[2] * inv, oc[3] * inv));
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pack2<BF16>(oc[0] * inv, oc[1] * inv);
      }
      if (lane == 0) Lse[static_cast<long>(bh) * Nq + q] = Lrow;
    } else {
      const long prow = (static_cast<long>(bh) * splits + sp) * Nq + q;
#pragma unroll
      for (int c = 0; c < CPL; ++c) Opart[prow * D + lane * CPL + c] = oc[c] * inv;
      if (lane == 0) Lpart[prow] = Lrow;
    }
  }
}

// One warp per (head, query row): O = sum_s exp(L_s - L) O_s with L = ln sum_s exp(L_s);
// splits whose row saw no key (L_s = -inf) drop out; a row that saw none at all gets
// O = 0, L = -inf.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
    fa_decode_merge_kernel(const float* __restrict__ Opart, const float* __restrict__ Lpart,
                           uint16_t* __restrict__ O, Strides so, float* __restrict__ Lse, int Nq,
                           int H, int splits, long rows) {
  constexpr int CPL = D / 32;
  const long row = static_cast<long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int bh = static_cast<int>(row / Nq);
  const int q = static_cast<int>(row - static_cast<long>(bh) * Nq);
  const long base = static_cast<long>(bh) * splits * Nq + q;  // (bh, s = 0, q)
  float M = -INFINITY;
  for (int s = lane; s < splits; s += 32) M = fmaxf(M, Lpart[base + static_cast<long>(s) * Nq]);
  M = warp_max(M);
  float tot = 0.f, oc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) oc[c] = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const long pr = base + static_cast<long>(s) * Nq;
      const float Ls = Lpart[pr];
      const float w = Ls == -INFINITY ? 0.f : ex2_approx((Ls - M) * 1.4426950408889634074f);
      tot += w;
#pragma unroll
      for (int c = 0; c < CPL; ++c) oc[c] = fmaf(w, Opart[pr * D + lane * CPL + c], oc[c]);
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  uint16_t* dst = O + (bh / H) * so.sb + (bh % H) * so.sh + static_cast<long>(q) * so.sn + lane * CPL;
  if constexpr (CPL == 4) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack2<BF16>(oc[0] * inv, oc[1] * inv), pack2<BF16>(oc[2] * inv, oc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack2<BF16>(oc[0] * inv, oc[1] * inv);
  }
  if (lane == 0) Lse[row] = tot > 0.f ? M + logf(tot) : -INFINITY;
}

}  // namespace fa
