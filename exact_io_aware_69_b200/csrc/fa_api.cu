// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, TMA tensor
// maps, and kernel launches. All device work is in the .cuh kernels beside it.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "fa.h"
#include "fa_band.cuh"
#include "fa_bwd.cuh"
#include "fa_bwd_dq.cuh"
#include "fa_decode.cuh"
#include "fa_decode_tc.cuh"
#include "fa_fwd_d256.cuh"
#include "fa_fwd_pp.cuh"

namespace fa {
// Self-test of the bounded waits: one thread waits on an mbarrier that nothing will
// ever arrive on, through the same routine every pipeline wait uses, with a short
// limit. The wait gives up, records FA_ERR_TIMEOUT in the status word and the kernel
// returns normally.
__global__ void fa_selftest_wait_kernel(long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(smem_u32(&bar), 1);
  fence_mbar_init();
  mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_cycles);
}

// Self-test of the forward's FMA-pipe exponential: y = ex2_poly_pair(x) elementwise
// (n even), so that it can be held against CUDA's exp2f.
__global__ void fa_selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y,
                                        int npairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= npairs) return;
  float y0, y1;
  ex2_poly_pair(x[2 * i], x[2 * i + 1], y0, y1);
  y[2 * i] = y0;
  y[2 * i + 1] = y1;
}
}  // namespace fa

namespace {

constexpr int kVersion = 2;
constexpr size_t kMaxDynSmem = 232448;  // 227 KB per block on sm_100
// Nq + Nk must stay below this so that no window arithmetic overflows 32 bits.
constexpr long long kMaxRowsPerHead = 1LL << 29;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Element strides (b, h, n) of a [B][H][N][d] or [B][N][H][d] tensor.
fa::Strides strides_of(int layout, int H, int N, int d) {
  const long D = d;
  if (layout == FA_LAYOUT_BNHD) return {static_cast<long>(N) * H * D, D, static_cast<long>(H) * D};
  return {static_cast<long>(H) * N * D, static_cast<long>(N) * D, D};
}

// A tensor seen in four dimensions (column, row within a head, head, batch) with the
// strides of its layout, so that a 128-row box reaching past a head's N reads zeros
// and writes nothing there. 16-bit: box of 64 columns x 128 rows; fp32 (the dQ
// accumulator, target of TMA reduce-adds): 32 columns (128 bytes) x 128 rows.
// 128-byte swizzle.
bool make_tmap4(CUtensorMap* map, const void* ptr, int B, int H, int N, int d, int layout,
                CUtensorMapDataType type, int esize) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const fa::Strides s = strides_of(layout, H, N, d);
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s.sn) * esize,
                           static_cast<cuuint64_t>(s.sh) * esize,
                           static_cast<cuuint64_t>(s.sb) * esize};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / esize), 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, type, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
bool make_tmap(CUtensorMap* map, const void* ptr, int B, int H, int N, int d, int layout,
               int dtype) {
  return make_tmap4(map, ptr, B, H, N, d, layout,
                    dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                    2);
}
// The dQ accumulator is the library's own [B][H][N][d] fp32 array.
bool make_tmap_f32(CUtensorMap* map, const void* ptr, int B, int H, int N, int d) {
  return make_tmap4(map, ptr, B, H, N, d, FA_LAYOUT_BHND, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p && aligned16(p); }

// Shape checks shared by every entry point. Returns FA_OK to proceed, or an error;
// *empty is set for a valid problem with no query rows (the backward then still owes
// dK = dV = 0 when Nk > 0). Keys are required when there are queries: a row with no
// key at all has no softmax.
int check_shape(int B, int H, int Nq, int Nk, int d, int layout, int dtype, float scale,
                bool* empty, bool d256_ok = false) {
  *empty = false;
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d < 0) return FA_ERR_INVALID;
  if (!(scale > 0.f) || !isfinite(scale)) return FA_ERR_INVALID;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BNHD) return FA_ERR_INVALID;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128 && !(d256_ok && d == 256)) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * Nq == 0) {
    *empty = true;
    return FA_OK;
  }
  if (Nk == 0) return FA_ERR_INVALID;
  if (static_cast<long long>(Nq) + Nk > kMaxRowsPerHead) return FA_ERR_UNSUPPORTED;
  // TMA coordinates and grid indices are 32-bit (rows counted with N padded to 128)
  const long long pq = (Nq + fa::kTile - 1) / fa::kTile * fa::kTile;
  const long long pk = (Nk + fa::kTile - 1) / fa::kTile * fa::kTile;
  if (static_cast<long long>(B) * H * (pq > pk ? pq : pk) >= (1LL << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// The key window in the kernels' form: an edge that bounds nothing becomes
// fa::kUnbounded; *band is false when no (query, key) pair is outside the window.
struct Window {
  int wl, wr;
  bool band;
};
Window window_of(int Nq, int Nk, int left, int right) {
  Window w;
  w.wl = (left < 0 || left >= fa::kUnbounded) ? fa::kUnbounded : left;
  w.wr = (right < 0 || right >= fa::kUnbounded) ? fa::kUnbounded : right;
  // every key is visible iff the left edge reaches key 0 from the last query and the
  // right edge reaches key Nk - 1 from the first
  w.band = !(static_cast<long long>(w.wl) >= Nk - 1 && static_cast<long long>(w.wr) >= Nq - 1);
  return w;
}

template <int D, bool BAND, bool BF16>
int launch_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
               const CUtensorMap& o, const CUtensorMap& o_res, bool has_res, float* L, int B,
               int H, int Nq, int Nk, Window w, float scale, cudaStream_t stream) {
  auto kern = fa::fa_fwd_pp_kernel<D, BAND, BF16>;
  // At least 120 KB so that one CTA -- and one 512-column TMEM allocation -- sits on
  // each SM (two CTAs would serialise on the tensor-memory allocation anyway).
  const int smem = fa::PpLayout<D>::kBytes > 120 * 1024 ? fa::PpLayout<D>::kBytes : 120 * 1024;
  if (static_cast<size_t>(smem) > kMaxDynSmem) return FA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  // The kernel moves registers between warpgroups (setmaxnreg); its split adds up to
  // exactly 168 registers per thread at launch (the build fails otherwise too).
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return FA_ERR_CUDA;
  if (attr.numRegs != fa::kPpLaunchRegs) return FA_ERR_UNSUPPORTED;
  const unsigned pairs = static_cast<unsigned>(((Nq + fa::kTile - 1) / fa::kTile + 1) / 2);
  const unsigned grid = static_cast<unsigned>(B) * static_cast<unsigned>(H) * pairs;
  // band: heaviest pairs first within groups of heads that share L2 (K and V streamed)
  const int group = w.band ? fa::band_group(static_cast<long>(B) * H, 4L * Nk * D,
                                            fa::kFwdGroupMin, fa::kFwdGroupBytes)
                           : 1;
  kern<<<grid, fa::kPpThreads, smem, stream>>>(q, k, v, o, o_res, has_res, L, Nq, Nk, H, w.wl,
                                                w.wr, scale * 1.4426950408889634074f, group);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// d = 256: one query tile per CTA (fa_fwd_d256.cuh).
template <bool BAND, bool BF16>
int launch_fwd_d256(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                    const CUtensorMap& o, const CUtensorMap& o_res, bool has_res, float* L, int B,
                    int H, int Nq, int Nk, Window w, float scale, cudaStream_t stream) {
  auto kern = fa::fa_fwd_d256_kernel<BAND, BF16>;
  const int smem = static_cast<int>(fa::WideLayout::kBytes);
  if (static_cast<size_t>(smem) > kMaxDynSmem) return FA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  const unsigned tiles = static_cast<unsigned>((Nq + fa::kTile - 1) / fa::kTile);
  const unsigned grid = static_cast<unsigned>(B) * static_cast<unsigned>(H) * tiles;
  const int group = w.band ? fa::band_group(static_cast<long>(B) * H, 4L * Nk * 256,
                                            fa::kFwdGroupMin, fa::kFwdGroupBytes)
                           : 1;
  kern<<<grid, fa::kWThreads, smem, stream>>>(q, k, v, o, o_res, has_res, L, Nq, Nk, H, w.wl,
                                              w.wr, scale * 1.4426950408889634074f, group);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

struct BwdArgs {
  const CUtensorMap* q;
  const CUtensorMap* k;
  const CUtensorMap* v;
  const CUtensorMap* dO_map;
  const CUtensorMap* dq_map;   // the fp32 dQ accumulator (reduce-add target)
  const CUtensorMap* dq_out;   // dQ itself (deterministic mode: the dQ pass stores it)
  const void* O;
  const void* O_res;
  const void* dO;
  const float* L;
  void* dQ;
  void* dK;
  void* dV;
  int B;
  int H;
  int Nq;  // query rows (Q, O, dO, dQ, L, the workspace)
  int Nk;  // key rows (K, V, dK, dV)
  int layout;
  Window w;
  bool det;  // deterministic: dQ by its own pass, no accumulator
  float scale;
  void* workspace;
  cudaStream_t stream;
};

// Workspace: D and Ls as [B*H][n_pad] fp32 (n_pad = Nq rounded up to 128, so that every
// query tile reads whole 512-byte rows), then (not in deterministic mode) the dQ
// accumulator [B*H][Nq][d] fp32.
template <int D, bool BAND, bool BF16>
int launch_bwd(const BwdArgs& a, int stages) {
  const int BH = a.B * a.H;
  const long rows = static_cast<long>(BH) * a.Nq;
  const int n_pad = (a.Nq + fa::kTile - 1) / fa::kTile * fa::kTile;
  const long prows = static_cast<long>(BH) * n_pad;
  float* Dv = static_cast<float*>(a.workspace);
  float* Ls = Dv + prows;
  float* dq_acc = a.det ? nullptr : Ls + prows;
  const fa::Strides sq = strides_of(a.layout, a.H, a.Nq, D);
  const fa::Strides sk = strides_of(a.layout, a.H, a.Nk, D);
  const float scale_log2 = a.scale * 1.4426950408889634074f;
  if (stages & FA_STAGE_PREPROCESS) {
    const long threads = prows * (D / 8);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    fa::fa_bwd_pre_kernel<D, BF16><<<blocks, 256, 0, a.stream>>>(
        static_cast<const uint16_t*>(a.O), static_cast<const uint16_t*>(a.O_res),
        static_cast<const uint16_t*>(a.dO), a.L, Dv, Ls, dq_acc, a.Nq, n_pad, prows, a.H, sq);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (stages & FA_STAGE_DKDV) {
    auto kern = a.det ? fa::fa_bwd_main_kernel<D, BAND, BF16, false>
                      : fa::fa_bwd_main_kernel<D, BAND, BF16, true>;
    const size_t need = fa::BwdLayout<D>::kNeeded;
    if (need > kMaxDynSmem) return FA_ERR_UNSUPPORTED;
    const size_t smem = need + 1024 <= kMaxDynSmem ? need + 1024 : kMaxDynSmem;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return FA_ERR_CUDA;
    // The kernel moves registers between warpgroups (setmaxnreg); its split adds up to
    // exactly 128 registers per thread at launch. Launched with fewer, the increase
    // would wait for registers that never come back, so refuse instead (the build
    // also fails for such a kernel).
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return FA_ERR_CUDA;
    if (attr.numRegs != fa::kBwdLaunchRegs) return FA_ERR_UNSUPPORTED;
    const unsigned grid = static_cast<unsigned>(BH) *  // one CTA per key tile
                          static_cast<unsigned>((a.Nk + fa::kTile - 1) / fa::kTile);
    kern<<<grid, fa::kBwdThreads, smem, a.stream>>>(
        *a.q, *a.k, *a.v, *a.dO_map, *a.dq_map, Ls, Dv, dq_acc, static_cast<uint16_t*>(a.dK),
        static_cast<uint16_t*>(a.dV), a.Nq, a.Nk, a.H, a.w.wl, a.w.wr, sk, a.scale, scale_log2,
        static_cast<uint32_t>(smem),
        // Q and dO streamed per key tile, and the fp32 dQ accumulator added into
        a.w.band ? fa::band_group(BH, 8L * a.Nq * D, fa::kBwdGroupMin, fa::kBwdGroupBytes) : 1);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if ((stages & FA_STAGE_DQ) && a.det) {
    auto kern = fa::fa_bwd_dq_pass_kernel<D, BAND, BF16>;
    const int smem = fa::DqLayout<D>::kBytes > 120 * 1024 ? fa::DqLayout<D>::kBytes : 120 * 1024;
    if (static_cast<size_t>(smem) > kMaxDynSmem) return FA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return FA_ERR_CUDA;
    const unsigned grid = static_cast<unsigned>(BH) *  // one CTA per query tile
                          static_cast<unsigned>((a.Nq + fa::kTile - 1) / fa::kTile);
    kern<<<grid, fa::kDqThreads, smem, a.stream>>>(*a.q, *a.k, *a.v, *a.dO_map, *a.dq_out, Ls,
                                                   Dv, a.Nq, a.Nk, a.H, a.w.wl, a.w.wr, a.scale,
                                                   scale_log2,
                                                   a.w.band ? fa::band_group(BH, 4L * a.Nk * D,
                                                                             fa::kFwdGroupMin,
                                                                             fa::kFwdGroupBytes)
                                                            : 1);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  } else if (stages & FA_STAGE_DQ) {
    const long n8 = rows * D / 8;
    const unsigned blocks = static_cast<unsigned>((n8 + 255) / 256);
    fa::fa_bwd_dq_kernel<D, BF16><<<blocks, 256, 0, a.stream>>>(
        dq_acc, static_cast<uint16_t*>(a.dQ), a.scale, n8, a.Nq, a.H, sq);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Compile-time dispatch over (d, band, dtype).
template <template <int, bool, bool> class F, typename... Args>
int dispatch(int d, bool band, int dtype, Args&&... args) {
  const bool bf = dtype == FA_BF16;
  if (d == 64) {
    if (band) return bf ? F<64, true, true>::run(args...) : F<64, true, false>::run(args...);
    return bf ? F<64, false, true>::run(args...) : F<64, false, false>::run(args...);
  }
  if (band) return bf ? F<128, true, true>::run(args...) : F<128, true, false>::run(args...);
  return bf ? F<128, false, true>::run(args...) : F<128, false, false>::run(args...);
}

template <int D, bool C, bool B>
struct FwdRun {
  template <typename... A>
  static int run(A&&... a) { return launch_fwd<D, C, B>(a...); }
};
template <int D, bool C, bool B>
struct BwdRun {
  template <typename... A>
  static int run(A&&... a) { return launch_bwd<D, C, B>(a...); }
};

size_t workspace_bytes_for(int B, int H, int Nq, int d, bool det) {
  const size_t rows = static_cast<size_t>(B) * H * Nq;
  if (rows == 0) return 0;
  // D and Ls (fp32 per row, Nq padded to a multiple of 128 per head), then the fp32 dQ
  // accumulator; its start is 1024-byte aligned because the padded row count is a
  // multiple of 128. The deterministic mode forms dQ in its own pass and keeps no
  // accumulator.
  const size_t n_pad = (static_cast<size_t>(Nq) + 127) / 128 * 128;
  const size_t stats = static_cast<size_t>(B) * H * n_pad * 4 * 2;
  return det ? stats : stats + rows * static_cast<size_t>(d) * 4;
}

// The backward (all stages, or the ones in `stages`), checked like fa_bwd_ex. Pointers
// a stage does not use may be NULL when only that stage runs.
int bwd_checked(const void* Q, const void* K, const void* V, const void* O, const void* O_res,
                const void* dO, const float* L, void* dQ, void* dK, void* dV, int B, int H,
                int Nq, int Nk, int d, int layout, int window_left, int window_right,
                int deterministic, float scale, int dtype, void* workspace,
                size_t workspace_bytes, void* stream, int stages) {
  bool empty;
  int st = check_shape(B, H, Nq, Nk, d, layout, dtype, scale, &empty);
  if (st != FA_OK) return st;
  if (deterministic != 0 && deterministic != 1) return FA_ERR_INVALID;
  if (stages <= 0 || stages > FA_STAGE_ALL) return FA_ERR_INVALID;
  const bool det = deterministic != 0;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (empty) {
    // no query rows: every key's gradient is an empty sum
    if (!(stages & FA_STAGE_DKDV)) return FA_OK;
    const size_t bytes = static_cast<size_t>(B) * H * Nk * d * 2;
    if (bytes == 0) return FA_OK;
    if (!ok_ptr(dK) || !ok_ptr(dV)) return FA_ERR_INVALID;
    return cudaMemsetAsync(dK, 0, bytes, s) == cudaSuccess &&
                   cudaMemsetAsync(dV, 0, bytes, s) == cudaSuccess
               ? FA_OK
               : FA_ERR_CUDA;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID;
  if (workspace_bytes < workspace_bytes_for(B, H, Nq, d, det)) return FA_ERR_INVALID;
  if (!aligned16(O_res)) return FA_ERR_INVALID;
  if ((stages & FA_STAGE_PREPROCESS) && (!ok_ptr(O) || !ok_ptr(dO) || !ok_ptr(L)))
    return FA_ERR_INVALID;
  if ((stages & FA_STAGE_DKDV) &&
      (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(dO) || !ok_ptr(dK) || !ok_ptr(dV)))
    return FA_ERR_INVALID;
  if ((stages & FA_STAGE_DQ) && !ok_ptr(dQ)) return FA_ERR_INVALID;
  if (det && (stages & FA_STAGE_DQ) &&
      (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(dO)))  // the dQ pass reads them
    return FA_ERR_INVALID;
  const Window w = window_of(Nq, Nk, window_left, window_right);
  const int BH = B * H;
  const long prows = static_cast<long>(BH) * ((Nq + fa::kTile - 1) / fa::kTile * fa::kTile);
  CUtensorMap tq, tk, tv, tdo, tdq, tdqo;
  if ((stages & FA_STAGE_DKDV) || (det && (stages & FA_STAGE_DQ))) {
    if (!make_tmap(&tq, Q, B, H, Nq, d, layout, dtype) ||
        !make_tmap(&tk, K, B, H, Nk, d, layout, dtype) ||
        !make_tmap(&tv, V, B, H, Nk, d, layout, dtype) ||
        !make_tmap(&tdo, dO, B, H, Nq, d, layout, dtype))
      return FA_ERR_CUDA;
  }
  // the accumulator's map (a deterministic run never touches it, so any valid base works)
  const float* dq_acc = static_cast<const float*>(workspace) + (det ? 0 : 2 * prows);
  if ((stages & FA_STAGE_DKDV) && !make_tmap_f32(&tdq, dq_acc, B, H, Nq, d)) return FA_ERR_CUDA;
  if (det && (stages & FA_STAGE_DQ) && !make_tmap(&tdqo, dQ, B, H, Nq, d, layout, dtype))
    return FA_ERR_CUDA;
  BwdArgs a{&tq,  &tk, &tv, &tdo, &tdq,   &tdqo, O,   O_res, dO,    L,         dQ,
            dK,   dV,  B,   H,    Nq,     Nk,    layout, w,  det,   scale,     workspace, s};
  return dispatch<BwdRun>(d, w.band, dtype, a, stages);
}

// ------------------------------------------------------------------- decode
// Key tiles that the decode rows (Nq <= 16, all in query tile 0) visit together.
fa::TileRange decode_tiles(int Nq, int Nk, const Window& w) {
  const int ntk = (Nk + fa::kTile - 1) / fa::kTile;
  return w.band ? fa::kv_tiles_of_query_tile(0, fa::kTile, Nq, Nk, w.wl, w.wr)
                : fa::TileRange{0, ntk};
}

// Splits per head: the count that minimises the estimated time, (waves of 148 CTAs,
// one CTA per SM) x (tiles per split + a fixed cost of about two tiles per CTA). A
// fixed SM count keeps the split -- and so the rounding of the merge -- the same on
// every B200.
int decode_splits(long BH, int ntiles) {
  if (ntiles <= 1) return 1;
  constexpr long kSms = 148;
  int best = 1;
  long best_cost = -1;
  const int max_s = ntiles < 1024 ? ntiles : 1024;
  for (int s = 1; s <= max_s; ++s) {
    const int tps = (ntiles + s - 1) / s;
    if ((ntiles + tps - 1) / tps != s) continue;  // every split gets at least one tile
    const long waves = (BH * s + kSms - 1) / kSms;
    const long cost = waves * (tps + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

size_t decode_workspace(long BH, int Nq, int d, int splits) {
  return splits <= 1 ? 0 : static_cast<size_t>(BH) * splits * Nq * (static_cast<size_t>(d) + 1) * 4;
}

template <int D, int QW, bool BAND, bool BF16>
int launch_decode_nq(const CUtensorMap& k, const CUtensorMap& v, const void* Q,
                     const fa::Strides& sq, void* O, float* L, float* opart, float* lpart, int B,
                     int H, int Nq, int Nk, const Window& w, fa::TileRange tiles, int splits,
                     float scale, cudaStream_t stream) {
  auto kern = fa::fa_decode_kernel<D, QW, BAND, BF16>;
  const int smem = fa::DecLayout<D>::kBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  const long BH = static_cast<long>(B) * H;
  const int tps = tiles.count > 0 ? (tiles.count + splits - 1) / splits : 0;
  const long groups = (Nq + fa::kDecQPerCta - 1) / fa::kDecQPerCta;
  kern<<<static_cast<unsigned>(BH * splits * groups), fa::kDecThreads, smem, stream>>>(
      k, v, static_cast<const uint16_t*>(Q), sq, static_cast<uint16_t*>(O), sq, L, opart, lpart,
      Nq, Nk, H, w.wl, w.wr, tiles.first, tiles.count, tps, splits,
      scale * 1.4426950408889634074f);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (splits > 1) {
    const long rows = BH * Nq;
    fa::fa_decode_merge_kernel<D, BF16><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
        opart, lpart, static_cast<uint16_t*>(O), sq, L, Nq, H, splits, rows);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// The tensor-core form (fa_decode_tc.cuh), d = 128 and kDecTcMinQ..16 rows per head:
// one CTA per (head, split) whatever the row count.
template <bool BAND, bool BF16>
int launch_decode_tc(const CUtensorMap& k, const CUtensorMap& v, const void* Q,
                     const fa::Strides& sq, void* O, float* L, float* opart, float* lpart, int B,
                     int H, int Nq, int Nk, const Window& w, fa::TileRange tiles, int splits,
                     float scale, cudaStream_t stream) {
  auto kern = fa::fa_decode_tc_kernel<BAND, BF16>;
  const int smem = static_cast<int>(fa::DtcLayout::kBytes);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  const long BH = static_cast<long>(B) * H;
  const int tps = tiles.count > 0 ? (tiles.count + splits - 1) / splits : 0;
  kern<<<static_cast<unsigned>(BH * splits), fa::kDtcThreads, smem, stream>>>(
      k, v, static_cast<const uint16_t*>(Q), sq, static_cast<uint16_t*>(O), sq, L, opart, lpart,
      Nq, Nk, H, w.wl, w.wr, tiles.first, tiles.count, tps, splits,
      scale * 1.4426950408889634074f);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (splits > 1) {
    const long rows = BH * Nq;
    fa::fa_decode_merge_kernel<128, BF16><<<static_cast<unsigned>((rows + 7) / 8), 256, 0,
                                             stream>>>(opart, lpart, static_cast<uint16_t*>(O),
                                                       sq, L, Nq, H, splits, rows);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Rows per head from which d = 128 decode takes the tensor-core form.
constexpr int kDecTcMinQ = 2;

template <int D, bool BAND, bool BF16>
struct DecodeRun {
  template <typename... A>
  static int run(int Nq, A&&... a) {
    if constexpr (D == 128) {
      if (Nq >= kDecTcMinQ) return launch_decode_tc<BAND, BF16>(a...);
    }
    if (Nq <= 1) return launch_decode_nq<D, 1, BAND, BF16>(a...);
    if (Nq <= 4) return launch_decode_nq<D, 4, BAND, BF16>(a...);
    return launch_decode_nq<D, 8, BAND, BF16>(a...);  // 8 rows per CTA
  }
};

// ------------------------------------------------ backward without allocation
// Scratch of fa_bwd_noalloc: a fixed device array that every CUDA context using this
// library holds until the context is destroyed. 32 MiB covers the backward workspace
// of B*H*N up to 64,527 rows at d = 128 (127,100 rows at d = 64).
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch in the calling thread's current context. In
// host code the array's name is only a host-side stand-in, and every context (the
// primary one of each device, or one a host application created itself) holds its
// own copy of the array at its own address, which also changes when a context is
// destroyed and created again. So the address is looked up on every call, in the
// context the work is enqueued in; the lookup is a host-side table query.
void* noalloc_scratch_address(int* status) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
    *status = FA_ERR_CUDA;
    return nullptr;
  }
  *status = FA_OK;
  return p;
}

}  // namespace

extern "C" {

int fa_version(void) { return kVersion; }

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID: return "FA_ERR_INVALID";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    default: return "FA_ERR_UNKNOWN";
  }
}

int fa_fwd_ex(const void* Q, const void* K, const void* V, void* O, void* O_res, float* L,
              int B, int H, int Nq, int Nk, int d, int layout, int window_left,
              int window_right, float scale, int dtype, void* stream) {
  bool empty;
  int st = check_shape(B, H, Nq, Nk, d, layout, dtype, scale, &empty, /*d256_ok=*/true);
  if (st != FA_OK || empty) return st;
  if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(O) || !ok_ptr(L) || !aligned16(O_res))
    return FA_ERR_INVALID;
  CUtensorMap tq, tk, tv, to, tr;
  if (!make_tmap(&tq, Q, B, H, Nq, d, layout, dtype) ||
      !make_tmap(&tk, K, B, H, Nk, d, layout, dtype) ||
      !make_tmap(&tv, V, B, H, Nk, d, layout, dtype) ||
      !make_tmap(&to, O, B, H, Nq, d, layout, dtype) ||
      !make_tmap(&tr, O_res != nullptr ? O_res : O, B, H, Nq, d, layout, dtype))
    return FA_ERR_CUDA;
  const Window w = window_of(Nq, Nk, window_left, window_right);
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (d == 256) {
    const bool bf = dtype == FA_BF16;
    if (w.band)
      return bf ? launch_fwd_d256<true, true>(tq, tk, tv, to, tr, O_res != nullptr, L, B, H, Nq,
                                              Nk, w, scale, cs)
                : launch_fwd_d256<true, false>(tq, tk, tv, to, tr, O_res != nullptr, L, B, H, Nq,
                                               Nk, w, scale, cs);
    return bf ? launch_fwd_d256<false, true>(tq, tk, tv, to, tr, O_res != nullptr, L, B, H, Nq,
                                             Nk, w, scale, cs)
              : launch_fwd_d256<false, false>(tq, tk, tv, to, tr, O_res != nullptr, L, B, H, Nq,
                                              Nk, w, scale, cs);
  }
  return dispatch<FwdRun>(d, w.band, dtype, tq, tk, tv, to, tr, O_res != nullptr, L, B, H, Nq,
                          Nk, w, scale, cs);
}

int fa_fwd_qk(const void* Q, const void* K, const void* V, void* O, void* O_res, float* L,
              int B, int H, int Nq, int Nk, int d, int causal, float scale, int dtype,
              void* stream) {
  return fa_fwd_ex(Q, K, V, O, O_res, L, B, H, Nq, Nk, d, FA_LAYOUT_BHND, -1, causal ? 0 : -1,
                   scale, dtype, stream);
}

int fa_fwd(const void* Q, const void* K, const void* V, void* O, void* O_res, float* L, int B,
           int H, int N, int d, int causal, float scale, int dtype, void* stream) {
  return fa_fwd_qk(Q, K, V, O, O_res, L, B, H, N, N, d, causal, scale, dtype, stream);
}

size_t fa_bwd_ex_workspace_size(int B, int H, int Nq, int Nk, int d, int deterministic) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d < 0) return static_cast<size_t>(-1);
  return workspace_bytes_for(B, H, Nq, d, deterministic != 0);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  return fa_bwd_ex_workspace_size(B, H, N, N, d, 0);
}

int fa_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* O_res,
              const void* dO, const float* L, void* dQ, void* dK, void* dV, int B, int H, int Nq,
              int Nk, int d, int layout, int window_left, int window_right, int deterministic,
              float scale, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_checked(Q, K, V, O, O_res, dO, L, dQ, dK, dV, B, H, Nq, Nk, d, layout, window_left,
                     window_right, deterministic, scale, dtype, workspace, workspace_bytes,
                     stream, FA_STAGE_ALL);
}

int fa_bwd_ex_stage(int stages, const void* Q, const void* K, const void* V, const void* O,
                    const void* O_res, const void* dO, const float* L, void* dQ, void* dK,
                    void* dV, int B, int H, int Nq, int Nk, int d, int layout, int window_left,
                    int window_right, int deterministic, float scale, int dtype, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return bwd_checked(Q, K, V, O, O_res, dO, L, dQ, dK, dV, B, H, Nq, Nk, d, layout, window_left,
                     window_right, deterministic, scale, dtype, workspace, workspace_bytes,
                     stream, stages);
}

int fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* O_res,
              const void* dO, const float* L, void* dQ, void* dK, void* dV, int B, int H, int Nq,
              int Nk, int d, int causal, float scale, int dtype, void* workspace,
              size_t workspace_bytes, void* stream) {
  return fa_bwd_ex(Q, K, V, O, O_res, dO, L, dQ, dK, dV, B, H, Nq, Nk, d, FA_LAYOUT_BHND, -1,
                   causal ? 0 : -1, 0, scale, dtype, workspace, workspace_bytes, stream);
}

int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* O_res,
           const void* dO, const float* L, void* dQ, void* dK, void* dV, int B, int H, int N,
           int d, int causal, float scale, int dtype, void* workspace, size_t workspace_bytes,
           void* stream) {
  return fa_bwd_qk(Q, K, V, O, O_res, dO, L, dQ, dK, dV, B, H, N, N, d, causal, scale, dtype,
                   workspace, workspace_bytes, stream);
}

int fa_bwd_preprocess(const void* O, const void* O_res, const void* dO, const float* L, int B,
                      int H, int N, int d, int dtype, void* workspace, size_t workspace_bytes,
                      void* stream) {
  return bwd_checked(nullptr, nullptr, nullptr, O, O_res, dO, L, nullptr, nullptr, nullptr, B, H,
                     N, N, d, FA_LAYOUT_BHND, -1, -1, 0, 1.f, dtype, workspace, workspace_bytes,
                     stream, FA_STAGE_PREPROCESS);
}

int fa_bwd_dkdv(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV,
                int B, int H, int N, int d, int causal, float scale, int dtype, void* workspace,
                size_t workspace_bytes, void* stream) {
  return bwd_checked(Q, K, V, nullptr, nullptr, dO, nullptr, nullptr, dK, dV, B, H, N, N, d,
                     FA_LAYOUT_BHND, -1, causal ? 0 : -1, 0, scale, dtype, workspace,
                     workspace_bytes, stream, FA_STAGE_DKDV);
}

int fa_bwd_dq_convert(void* dQ, int B, int H, int N, int d, float scale, int dtype,
                      void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_checked(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dQ, nullptr,
                     nullptr, B, H, N, N, d, FA_LAYOUT_BHND, -1, -1, 0, scale, dtype, workspace,
                     workspace_bytes, stream, FA_STAGE_DQ);
}

int fa_tile_range(int query_side, int tile, int Nq, int Nk, int window_left, int window_right,
                  int* first, int* count) {
  if (!first || !count || Nq <= 0 || Nk <= 0 || tile < 0 ||
      static_cast<long long>(Nq) + Nk > kMaxRowsPerHead)
    return FA_ERR_INVALID;
  const Window w = window_of(Nq, Nk, window_left, window_right);
  const int ntq = (Nq + fa::kTile - 1) / fa::kTile;
  const int ntk = (Nk + fa::kTile - 1) / fa::kTile;
  fa::TileRange r;
  if (query_side) {
    if (tile >= ntq) return FA_ERR_INVALID;
    r = w.band ? fa::kv_tiles_of_query_tile(tile, fa::kTile, Nq, Nk, w.wl, w.wr)
               : fa::TileRange{0, ntk};
  } else {
    if (tile >= ntk) return FA_ERR_INVALID;
    r = w.band ? fa::query_tiles_of_kv_tile(tile, fa::kTile, Nq, Nk, w.wl, w.wr)
               : fa::TileRange{0, ntq};
  }
  *first = r.first;
  *count = r.count;
  return FA_OK;
}

size_t fa_decode_workspace_size(int B, int H, int Nq, int Nk, int d, int window_left,
                                int window_right) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d < 0) return static_cast<size_t>(-1);
  if (static_cast<long long>(B) * H * Nq == 0 || Nk == 0 || Nq > fa::kDecMaxQ ||
      static_cast<long long>(Nq) + Nk > kMaxRowsPerHead)
    return 0;
  const Window w = window_of(Nq, Nk, window_left, window_right);
  const long BH = static_cast<long>(B) * H;
  return decode_workspace(BH, Nq, d, decode_splits(BH, decode_tiles(Nq, Nk, w).count));
}

int fa_decode(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H,
              int Nq, int Nk, int d, int layout, int window_left, int window_right, float scale,
              int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  bool empty;
  int st = check_shape(B, H, Nq, Nk, d, layout, dtype, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (Nq > fa::kDecMaxQ) return FA_ERR_UNSUPPORTED;
  if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(O) || !ok_ptr(L)) return FA_ERR_INVALID;
  const Window w = window_of(Nq, Nk, window_left, window_right);
  const long BH = static_cast<long>(B) * H;
  const fa::TileRange tiles = decode_tiles(Nq, Nk, w);
  const int splits = decode_splits(BH, tiles.count);
  const size_t need = decode_workspace(BH, Nq, d, splits);
  if (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
                   workspace_bytes < need))
    return FA_ERR_INVALID;
  if (BH * splits * 2 >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
  CUtensorMap tk, tv;
  if (!make_tmap(&tk, K, B, H, Nk, d, layout, dtype) ||
      !make_tmap(&tv, V, B, H, Nk, d, layout, dtype))
    return FA_ERR_CUDA;
  float* opart = static_cast<float*>(workspace);
  float* lpart = splits > 1 ? opart + BH * splits * Nq * d : nullptr;
  const fa::Strides sq = strides_of(layout, H, Nq, d);
  return dispatch<DecodeRun>(d, w.band, dtype, Nq, tk, tv, Q, sq, O, L, opart, lpart, B, H, Nq,
                             Nk, w, tiles, splits, scale, static_cast<cudaStream_t>(stream));
}

int fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O,
                   const void* O_res, const void* dO, const float* L, void* dQ, void* dK,
                   void* dV, int B, int H, int N, int d, int causal, float scale, int dtype,
                   void* stream) {
  // Same checks as fa_bwd, and the size limit first: nothing touches the device for
  // a problem that does not fit.
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == static_cast<size_t>(-1)) return FA_ERR_INVALID;
  if (need > kNoAllocScratchBytes) return FA_ERR_UNSUPPORTED;
  bool empty;
  int st = check_shape(B, H, N, N, d, FA_LAYOUT_BHND, dtype, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(O) || !ok_ptr(dO) || !ok_ptr(L) ||
      !ok_ptr(dQ) || !ok_ptr(dK) || !ok_ptr(dV) || !aligned16(O_res))
    return FA_ERR_INVALID;
  void* scratch = noalloc_scratch_address(&st);
  if (st != FA_OK) return st;
  return fa_bwd(Q, K, V, O, O_res, dO, L, dQ, dK, dV, B, H, N, d, causal, scale, dtype, scratch,
                kNoAllocScratchBytes, stream);
}

int fa_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles <= 0 || limit_cycles > fa::kWaitLimitCycles) return FA_ERR_INVALID;
  fa::fa_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_selftest_exp2(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n & 1)) return FA_ERR_INVALID;
  if (n == 0) return FA_OK;
  if (x == nullptr || y == nullptr || (reinterpret_cast<uintptr_t>(x) & 7) ||
      (reinterpret_cast<uintptr_t>(y) & 7))
    return FA_ERR_INVALID;
  const int npairs = n / 2;
  fa::fa_selftest_exp2_kernel<<<(npairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y, npairs);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

#ifdef FA_TRACE
// Trace builds only: point the kernels at a device buffer of
// kTraceSlots * kTraceIters * kTraceEvents uint64 and choose the CTAs to record.
int fa_trace_attach(void* buf, const int* ctas) {
  if (cudaMemcpyToSymbol(fa::g_fa_trace, &buf, sizeof(void*)) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaMemcpyToSymbol(fa::g_fa_trace_cta, ctas, sizeof(int) * fa::kTraceSlots) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}
// Trace builds only: a device buffer of 8 uint64 per CTA for the per-CTA life log.
int fa_trace_cta_log(void* buf) {
  return cudaMemcpyToSymbol(fa::g_fa_cta_log, &buf, sizeof(void*)) == cudaSuccess ? FA_OK
                                                                                : FA_ERR_CUDA;
}
#endif

int fa_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_fa_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(int)) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  return v;
}

}  // extern "C"
