// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, TMA tensor
// maps, and kernel launches. All device work is in fa_fwd.cuh / fa_bwd.cuh.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_fwd.cuh"

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
}  // namespace fa

namespace {

constexpr int kVersion = 1;
constexpr size_t kMaxDynSmem = 232448;  // 227 KB per block on sm_100

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

// [BH][N][d] row-major tensor seen in three dimensions (column, row within a head,
// head), so that a 128-row box reaching past a head's N reads zeros and writes
// nothing there. 16-bit: box of 64 columns x 128 rows; fp32 (the dQ accumulator,
// target of TMA reduce-adds): 32 columns (128 bytes) x 128 rows. 128-byte swizzle.
bool make_tmap3(CUtensorMap* map, const void* ptr, int BH, int N, int d,
                CUtensorMapDataType type, int esize) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esize,
                           static_cast<cuuint64_t>(N) * d * esize};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esize), 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, type, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
bool make_tmap(CUtensorMap* map, const void* ptr, int BH, int N, int d, int dtype) {
  return make_tmap3(map, ptr, BH, N, d,
                    dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                    2);
}
bool make_tmap_f32(CUtensorMap* map, const void* ptr, int BH, int N, int d) {
  return make_tmap3(map, ptr, BH, N, d, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by the forward and backward entry points. Returns FA_OK to
// proceed, or an error; *empty is set for a valid problem with no query rows (the
// backward then still owes dK = dV = 0 when Nk > 0). Keys are required when there are
// queries: a row with no key at all has no softmax.
int check_shape_qk(int B, int H, int Nq, int Nk, int d, int dtype, float scale, bool* empty) {
  *empty = false;
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d < 0) return FA_ERR_INVALID;
  if (!(scale > 0.f) || !isfinite(scale)) return FA_ERR_INVALID;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * Nq == 0) {
    *empty = true;
    return FA_OK;
  }
  if (Nk == 0) return FA_ERR_INVALID;
  // TMA coordinates and grid indices are 32-bit (rows counted with N padded to 128)
  const long long pq = (Nq + fa::kTile - 1) / fa::kTile * fa::kTile;
  const long long pk = (Nk + fa::kTile - 1) / fa::kTile * fa::kTile;
  if (static_cast<long long>(B) * H * (pq > pk ? pq : pk) >= (1LL << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}
int check_shape(int B, int H, int N, int d, int dtype, float scale, bool* empty) {
  return check_shape_qk(B, H, N, N, d, dtype, scale, empty);
}

template <int D, bool CAUSAL, bool BF16>
int launch_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
               const CUtensorMap& o, const CUtensorMap& o_res, bool has_res, float* L, int BH,
               int Nq, int Nk, float scale, cudaStream_t stream) {
  auto kern = fa::fa_fwd_kernel<D, CAUSAL, BF16>;
  // At least 120 KB so that one CTA -- and one 512-column TMEM allocation -- sits on
  // each SM (two CTAs would serialise on the tensor-memory allocation anyway).
  const int smem = fa::FwdLayout<D>::kBytes > 120 * 1024 ? fa::FwdLayout<D>::kBytes : 120 * 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  const unsigned grid =
      static_cast<unsigned>(BH) * static_cast<unsigned>((Nq + fa::kTile - 1) / fa::kTile);
  kern<<<grid, fa::kFwdThreads, smem, stream>>>(q, k, v, o, o_res, has_res, L, Nq, Nk,
                                                 scale * 1.4426950408889634074f);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

struct BwdArgs {
  const CUtensorMap* q;
  const CUtensorMap* k;
  const CUtensorMap* v;
  const CUtensorMap* dO_map;
  const CUtensorMap* dq_map;
  const void* O;
  const void* O_res;
  const void* dO;
  const float* L;
  void* dQ;
  void* dK;
  void* dV;
  int BH;
  int Nq;  // query rows (Q, O, dO, dQ, L, the workspace)
  int Nk;  // key rows (K, V, dK, dV)
  float scale;
  void* workspace;
  cudaStream_t stream;
};

enum { kStagePre = 1, kStageMain = 2, kStageDq = 4, kStageAll = 7 };

// Workspace: D and Ls as [BH][n_pad] fp32 (n_pad = Nq rounded up to 128, so that every
// query tile reads whole 512-byte rows), then the dQ accumulator [BH][Nq][d] fp32.
template <int D, bool CAUSAL, bool BF16>
int launch_bwd(const BwdArgs& a, int stages) {
  const long rows = static_cast<long>(a.BH) * a.Nq;
  const int n_pad = (a.Nq + fa::kTile - 1) / fa::kTile * fa::kTile;
  const long prows = static_cast<long>(a.BH) * n_pad;
  float* Dv = static_cast<float*>(a.workspace);
  float* Ls = Dv + prows;
  float* dq_acc = Ls + prows;
  if (stages & kStagePre) {
    const long threads = prows * (D / 8);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    fa::fa_bwd_pre_kernel<D, BF16><<<blocks, 256, 0, a.stream>>>(
        static_cast<const uint16_t*>(a.O), static_cast<const uint16_t*>(a.O_res),
        static_cast<const uint16_t*>(a.dO), a.L, Dv, Ls, dq_acc, a.Nq, n_pad, prows);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (stages & kStageMain) {
    auto kern = fa::fa_bwd_main_kernel<D, CAUSAL, BF16>;
    const size_t need = fa::BwdLayout<D>::kNeeded;
    if (need > kMaxDynSmem) return FA_ERR_UNSUPPORTED;
    const size_t smem = need + 1024 <= kMaxDynSmem ? need + 1024 : kMaxDynSmem;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return FA_ERR_CUDA;
    // The kernel moves registers between warpgroups (setmaxnreg); its split adds up to
    // exactly 128 registers per thread at launch. Launched with fewer, the increase
    // would wait for registers that never come back, so refuse instead.
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return FA_ERR_CUDA;
    if (attr.numRegs != fa::kBwdLaunchRegs) return FA_ERR_UNSUPPORTED;
    const unsigned grid =  // one CTA per key tile
        static_cast<unsigned>(a.BH) * static_cast<unsigned>((a.Nk + fa::kTile - 1) / fa::kTile);
    kern<<<grid, fa::kBwdThreads, smem, a.stream>>>(
        *a.q, *a.k, *a.v, *a.dO_map, *a.dq_map, Ls, Dv, dq_acc, static_cast<uint16_t*>(a.dK),
        static_cast<uint16_t*>(a.dV), a.Nq, a.Nk, a.scale, a.scale * 1.4426950408889634074f,
        static_cast<uint32_t>(smem));
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (stages & kStageDq) {
    const long n8 = rows * D / 8;
    const unsigned blocks = static_cast<unsigned>((n8 + 255) / 256);
    fa::fa_bwd_dq_kernel<D, BF16><<<blocks, 256, 0, a.stream>>>(
        dq_acc, static_cast<uint16_t*>(a.dQ), a.scale, n8);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Compile-time dispatch over (d, causal, dtype).
template <template <int, bool, bool> class F, typename... Args>
int dispatch(int d, int causal, int dtype, Args&&... args) {
  const bool bf = dtype == FA_BF16;
  if (d == 64) {
    if (causal) return bf ? F<64, true, true>::run(args...) : F<64, true, false>::run(args...);
    return bf ? F<64, false, true>::run(args...) : F<64, false, false>::run(args...);
  }
  if (causal) return bf ? F<128, true, true>::run(args...) : F<128, true, false>::run(args...);
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

int fa_fwd_qk(const void* Q, const void* K, const void* V, void* O, void* O_res, float* L,
              int B, int H, int Nq, int Nk, int d, int causal, float scale, int dtype,
              void* stream) {
  bool empty;
  int st = check_shape_qk(B, H, Nq, Nk, d, dtype, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (!Q || !K || !V || !O || !L) return FA_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(L) ||
      !aligned16(O_res))
    return FA_ERR_INVALID;
  const int BH = B * H;
  CUtensorMap tq, tk, tv, to, tr;
  if (!make_tmap(&tq, Q, BH, Nq, d, dtype) || !make_tmap(&tk, K, BH, Nk, d, dtype) ||
      !make_tmap(&tv, V, BH, Nk, d, dtype) || !make_tmap(&to, O, BH, Nq, d, dtype) ||
      !make_tmap(&tr, O_res != nullptr ? O_res : O, BH, Nq, d, dtype))
    return FA_ERR_CUDA;
  return dispatch<FwdRun>(d, causal, dtype, tq, tk, tv, to, tr, O_res != nullptr, L, BH, Nq, Nk,
                          scale, static_cast<cudaStream_t>(stream));
}

int fa_fwd(const void* Q, const void* K, const void* V, void* O, void* O_res, float* L, int B,
           int H, int N, int d, int causal, float scale, int dtype, void* stream) {
  return fa_fwd_qk(Q, K, V, O, O_res, L, B, H, N, N, d, causal, scale, dtype, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0 || d < 0) return static_cast<size_t>(-1);
  const size_t rows = static_cast<size_t>(B) * H * N;
  if (rows == 0) return 0;
  // D and Ls (fp32 per row, N padded to a multiple of 128 per head), then the fp32 dQ
  // accumulator; its start is 1024-byte aligned because the padded row count is a
  // multiple of 128.
  const size_t n_pad = (static_cast<size_t>(N) + 127) / 128 * 128;
  return static_cast<size_t>(B) * H * n_pad * 4 * 2 + rows * static_cast<size_t>(d) * 4;
}

// Validation shared by fa_bwd and its stages; the pointers a stage does not use may
// be NULL (checked by the caller).
static int bwd_common_qk(int B, int H, int Nq, int Nk, int d, int dtype, float scale,
                         void* workspace, size_t workspace_bytes, bool* empty) {
  int st = check_shape_qk(B, H, Nq, Nk, d, dtype, scale, empty);
  if (st != FA_OK || *empty) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID;
  if (workspace_bytes < fa_bwd_workspace_size(B, H, Nq, d)) return FA_ERR_INVALID;
  return FA_OK;
}
static int bwd_common(int B, int H, int N, int d, int dtype, float scale, void* workspace,
                      size_t workspace_bytes, bool* empty) {
  return bwd_common_qk(B, H, N, N, d, dtype, scale, workspace, workspace_bytes, empty);
}

static int bwd_run(const void* Q, const void* K, const void* V, const void* O, const void* O_res,
                   const void* dO, const float* L, void* dQ, void* dK, void* dV, int B, int H,
                   int Nq, int Nk, int d, int causal, float scale, int dtype, void* workspace,
                   void* stream, int stages) {
  const int BH = B * H;
  const long prows = static_cast<long>(BH) * ((Nq + fa::kTile - 1) / fa::kTile * fa::kTile);
  CUtensorMap tq, tk, tv, tdo, tdq;
  if (stages & kStageMain) {
    const float* dq_acc = static_cast<const float*>(workspace) + 2 * prows;
    if (!make_tmap(&tq, Q, BH, Nq, d, dtype) || !make_tmap(&tk, K, BH, Nk, d, dtype) ||
        !make_tmap(&tv, V, BH, Nk, d, dtype) || !make_tmap(&tdo, dO, BH, Nq, d, dtype) ||
        !make_tmap_f32(&tdq, dq_acc, BH, Nq, d))
      return FA_ERR_CUDA;
  }
  BwdArgs a{&tq, &tk, &tv, &tdo, &tdq, O, O_res, dO, L, dQ, dK, dV, BH, Nq, Nk, scale, workspace,
            static_cast<cudaStream_t>(stream)};
  return dispatch<BwdRun>(d, causal, dtype, a, stages);
}

static bool ok_ptr(const void* p) { return p && aligned16(p); }

int fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* O_res,
              const void* dO, const float* L, void* dQ, void* dK, void* dV, int B, int H, int Nq,
              int Nk, int d, int causal, float scale, int dtype, void* workspace,
              size_t workspace_bytes, void* stream) {
  bool empty;
  int st = bwd_common_qk(B, H, Nq, Nk, d, dtype, scale, workspace, workspace_bytes, &empty);
  if (st != FA_OK) return st;
  if (empty) {
    // no query rows: every key's gradient is an empty sum
    const size_t bytes = static_cast<size_t>(B) * H * Nk * d * 2;
    if (bytes == 0) return FA_OK;
    if (!ok_ptr(dK) || !ok_ptr(dV)) return FA_ERR_INVALID;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return cudaMemsetAsync(dK, 0, bytes, s) == cudaSuccess &&
                   cudaMemsetAsync(dV, 0, bytes, s) == cudaSuccess
               ? FA_OK
               : FA_ERR_CUDA;
  }
  if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(O) || !ok_ptr(dO) || !ok_ptr(L) ||
      !ok_ptr(dQ) || !ok_ptr(dK) || !ok_ptr(dV) || !aligned16(O_res))
    return FA_ERR_INVALID;
  return bwd_run(Q, K, V, O, O_res, dO, L, dQ, dK, dV, B, H, Nq, Nk, d, causal, scale, dtype,
                 workspace, stream, kStageAll);
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
  bool empty;
  int st = bwd_common(B, H, N, d, dtype, 1.f, workspace, workspace_bytes, &empty);
  if (st != FA_OK || empty) return st;
  if (!ok_ptr(O) || !ok_ptr(dO) || !ok_ptr(L) || !aligned16(O_res)) return FA_ERR_INVALID;
  return bwd_run(nullptr, nullptr, nullptr, O, O_res, dO, L, nullptr, nullptr, nullptr, B, H, N,
                 N, d, 0, 1.f, dtype, workspace, stream, kStagePre);
}

int fa_bwd_dkdv(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV,
                int B, int H, int N, int d, int causal, float scale, int dtype, void* workspace,
                size_t workspace_bytes, void* stream) {
  bool empty;
  int st = bwd_common(B, H, N, d, dtype, scale, workspace, workspace_bytes, &empty);
  if (st != FA_OK || empty) return st;
  if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(dO) || !ok_ptr(dK) || !ok_ptr(dV))
    return FA_ERR_INVALID;
  return bwd_run(Q, K, V, nullptr, nullptr, dO, nullptr, nullptr, dK, dV, B, H, N, N, d, causal,
                 scale, dtype, workspace, stream, kStageMain);
}

int fa_bwd_dq_convert(void* dQ, int B, int H, int N, int d, float scale, int dtype,
                      void* workspace, size_t workspace_bytes, void* stream) {
  bool empty;
  int st = bwd_common(B, H, N, d, dtype, scale, workspace, workspace_bytes, &empty);
  if (st != FA_OK || empty) return st;
  if (!ok_ptr(dQ)) return FA_ERR_INVALID;
  return bwd_run(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dQ, nullptr,
                 nullptr, B, H, N, N, d, 0, scale, dtype, workspace, stream, kStageDq);
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
  int st = check_shape(B, H, N, d, dtype, scale, &empty);
  if (st != FA_OK || empty) return st;
  if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(O) || !ok_ptr(dO) || !ok_ptr(L) ||
      !ok_ptr(dQ) || !ok_ptr(dK) || !ok_ptr(dV) || !aligned16(O_res))
    return FA_ERR_INVALID;
  void* scratch = noalloc_scratch_address(&st);
  if (st != FA_OK) return st;
  return bwd_run(Q, K, V, O, O_res, dO, L, dQ, dK, dV, B, H, N, N, d, causal, scale, dtype,
                 scratch, stream, kStageAll);
}

int fa_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles <= 0 || limit_cycles > fa::kWaitLimitCycles) return FA_ERR_INVALID;
  fa::fa_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
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
