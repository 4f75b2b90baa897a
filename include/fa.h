/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library, libfa.so.
 *
 * Operation. Exact scaled-dot-product attention, per batch b and head h:
 *
 *   S = scale * Q K^T          (N x N, never stored)
 *   P = softmax(S) by rows     (N x N, never stored)
 *   O = P V
 *
 * the three steps of josueisai.com "flash-attention", section "La matriz que nunca
 * deberias guardar", computed tile by tile with the online softmax of section "El
 * truco: trocear y llevar la cuenta del softmax" so that S and P stay on chip. The
 * forward also writes the per-row log-sum-exp L (kerneldigest.dev "FlashAttention",
 * first paragraph: online log-sum-exp scaling). The backward keeps no P: it
 * recomputes the scores from Q, K, V and uses L (josueisai.com, section "Recomputar
 * sale mas barato que recordar").
 *
 * Masks (not on the pages). Every mask is a key window around the bottom-right
 * diagonal: with off = N_k - N_q, query i sees key j iff
 *     i + off - window_left <= j <= i + off + window_right,
 * a negative edge bounding nothing. (-1, -1) is unmasked attention, (-1, 0) the causal
 * mask (with N_q = N_k: j <= i), and bounded edges a sliding window, the combination
 * josueisai.com "flash-attention", section "Que ganas y que no", names for very long
 * sequences. The basic calls' `causal` flag is (-1, 0) when set, (-1, -1) otherwise.
 * A query row that sees no key gets O = 0 and L = -inf and contributes nothing to
 * the gradients.
 *
 * Layout. Every 16-bit tensor (Q, K, V, O, dO, dQ, dK, dV) is a dense row-major array
 * of one element type (bf16 or fp16, the `dtype` argument), either [B][H][N][d]
 * (FA_LAYOUT_BHND, the basic calls' layout: element (b, h, n, t) at
 * ((b*H + h)*N + n)*d + t) or [B][N][H][d] (FA_LAYOUT_BNHD: ((b*N + n)*H + h)*d + t).
 * L is fp32 [B][H][N] in both, in natural-log units of the scaled score:
 * L_i = m_i + ln(sum_j exp(s_ij - m_i)).
 * Arithmetic is fp32 with 16-bit MMA operands (P and dS are rounded to `dtype`
 * before their products).
 *
 * Pointers are DEVICE pointers and must be 16-byte aligned. `stream` is a
 * cudaStream_t (NULL = legacy default stream). Every call only enqueues work on
 * `stream` and returns; outputs are valid once the stream has reached that point.
 *
 * Ownership. The caller allocates and owns every buffer, including the backward
 * workspace sized by fa_bwd_workspace_size(). The library allocates no device
 * memory in these calls; its only state is one device-side error word per device.
 *
 * Supported now: d in {64, 128} for every call, and d = 256 for the forward calls
 * (fa_fwd, fa_fwd_qk, fa_fwd_ex: one query tile per CTA, its score buffers and O
 * filling the 512 tensor-memory columns); any N >= 1 (the last 128-row tile of a head
 * may be partial); dtype bf16 or fp16; B*H*N with N rounded up to 128 below 2^31, and
 * N_q + N_k <= 2^29.
 *
 * Errors are checked on the host before anything is enqueued and are returned as
 * codes (no exception, no abort, no fallback to another implementation):
 *   FA_ERR_INVALID      null pointer, negative size, misaligned pointer, a workspace
 *                       that is too small, a non-finite / non-positive scale, or an
 *                       unknown layout or stage;
 *   FA_ERR_UNSUPPORTED  d not in {64, 128} (forward calls: {64, 128, 256}), dtype not
 *                       bf16/fp16, B*H*roundup(N,128)
 *                       >= 2^31 (32-bit TMA coordinates and grid indices), or
 *                       N_q + N_k > 2^29;
 *   FA_ERR_CUDA         a CUDA runtime/driver call or a launch failed;
 *   FA_ERR_TIMEOUT      (from fa_get_device_status only) a kernel gave up a bounded
 *                       wait on the device and returned without finishing.
 * B*H*N == 0 is a valid empty problem: FA_OK, nothing is enqueued.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID = -1,
    FA_ERR_UNSUPPORTED = -2,
    FA_ERR_CUDA = -3,
    FA_ERR_TIMEOUT = -4
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

typedef enum { FA_LAYOUT_BHND = 0, FA_LAYOUT_BNHD = 1 } fa_layout;

/* Stages of the backward, for fa_bwd_ex_stage (bit flags; FA_STAGE_ALL = fa_bwd_ex). */
typedef enum {
    FA_STAGE_PREPROCESS = 1,
    FA_STAGE_DKDV = 2,
    FA_STAGE_DQ = 4,
    FA_STAGE_ALL = 7
} fa_stage;

/*
 * Forward. Reads Q, K, V [B][H][N][d]; writes O [B][H][N][d] (dtype) and
 * L [B][H][N] (fp32). One kernel launch.
 *
 * O_res (optional, may be NULL; otherwise [B][H][N][d] dtype, 16-byte aligned)
 * receives the rounding residual of O: O_res = dtype(O_exact_fp32 - O), so that
 * O + O_res holds the output to about 2^-17 relative. fa_bwd uses it for
 * D_i = sum_t dO_it O_it; without it D carries the 16-bit rounding of O, which for
 * rows dominated by one key (large logits) moves dK by several 1e-2.
 */
int fa_fwd(const void *Q, const void *K, const void *V, void *O, void *O_res, float *L, int B,
           int H, int N, int d, int causal, float scale, int dtype, void *stream);

/*
 * Forward with separate query and key lengths: Q, O, O_res [B][H][Nq][d], K, V
 * [B][H][Nk][d], L [B][H][Nq]. Causal masking is bottom-right aligned: query i sees
 * keys j <= i + Nk - Nq, so the last query sees every key (with Nq = Nk this is
 * j <= i). With Nq > Nk the first Nq - Nk queries see no key; their O rows are 0
 * and their L is -inf. Nk = 0 with Nq > 0 is FA_ERR_INVALID. fa_fwd is
 * fa_fwd_qk(..., N, N, ...).
 */
int fa_fwd_qk(const void *Q, const void *K, const void *V, void *O, void *O_res, float *L, int B,
              int H, int Nq, int Nk, int d, int causal, float scale, int dtype, void *stream);

/*
 * Forward, general form: Q, O, O_res [.., Nq, ..], K, V [.., Nk, ..] in `layout`
 * (FA_LAYOUT_BHND or FA_LAYOUT_BNHD), L [B][H][Nq] fp32, the key window
 * [window_left, window_right] described at the top of this file (negative = that side
 * unbounded). Key tiles outside every row's window are neither loaded nor multiplied.
 * fa_fwd_qk(..., causal, ...) is fa_fwd_ex(..., FA_LAYOUT_BHND, -1, causal ? 0 : -1,
 * ...). One kernel launch.
 */
int fa_fwd_ex(const void *Q, const void *K, const void *V, void *O, void *O_res, float *L,
              int B, int H, int Nq, int Nk, int d, int layout, int window_left,
              int window_right, float scale, int dtype, void *stream);

/*
 * Bytes of device workspace that fa_bwd needs for this shape: fp32 D and scaled L
 * ([B][H][Np] each, Np = N rounded up to a multiple of 128) plus an fp32 dQ
 * accumulator [B][H][N][d]: B*H*Np*8 + B*H*N*d*4. 0 for an empty problem;
 * (size_t)-1 for sizes that fa_bwd rejects as invalid.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward. Given Q, K, V, the forward's O, O_res (NULL allowed: D then uses O
 * alone) and L, and dO, writes dQ, dK, dV ([B][H][N][d], dtype). `workspace` is a caller-owned device buffer of at least
 * fa_bwd_workspace_size(B, H, N, d) bytes, 256-byte aligned; its contents on entry
 * do not matter and on return are scratch. Three kernel launches: D = rowsum(dO * O)
 * and zeroing of the dQ accumulator; the dK/dV pass that recomputes P from L and
 * adds dQ partials atomically; the conversion of dQ to dtype.
 */
int fa_bwd(const void *Q, const void *K, const void *V, const void *O, const void *O_res,
           const void *dO, const float *L, void *dQ, void *dK, void *dV, int B, int H, int N,
           int d, int causal, float scale, int dtype, void *workspace, size_t workspace_bytes,
           void *stream);

/*
 * Backward with separate query and key lengths (shapes and masking as fa_fwd_qk; dQ
 * and dO [B][H][Nq][d], dK and dV [B][H][Nk][d]). The workspace is sized by
 * fa_bwd_workspace_size(B, H, Nq, d). Queries that see no key contribute nothing.
 * With B*H*Nq == 0 and Nk > 0, dK and dV are set to zero (only they are touched).
 * fa_bwd is fa_bwd_qk(..., N, N, ...).
 */
int fa_bwd_qk(const void *Q, const void *K, const void *V, const void *O, const void *O_res,
              const void *dO, const float *L, void *dQ, void *dK, void *dV, int B, int H, int Nq,
              int Nk, int d, int causal, float scale, int dtype, void *workspace,
              size_t workspace_bytes, void *stream);

/*
 * Backward, general form (shapes, layout and window as fa_fwd_ex; dQ and dO are
 * [.., Nq, ..], dK and dV [.., Nk, ..]). With B*H*Nq == 0 and Nk > 0, dK and dV are set
 * to zero. The workspace is sized by fa_bwd_ex_workspace_size with the same arguments.
 *
 * `deterministic` = 0: dQ partial sums of the key tiles are added into an fp32
 * accumulator in the workspace by the dK/dV kernel, in whatever order its CTAs finish,
 * so dQ may differ in its last bits between calls (dK, dV, O, L never do).
 * `deterministic` = 1: dQ is formed by a separate pass over the keys (one CTA per query
 * tile summing the key tiles of its band in increasing order, accumulating in tensor
 * memory), so every result is identical on every call; the dK/dV kernel then skips its
 * dQ work and the workspace holds only the row statistics (B*H*Np*8 bytes). It costs
 * the recomputation of S and dP in the dQ pass. Other values: FA_ERR_INVALID.
 */
size_t fa_bwd_ex_workspace_size(int B, int H, int Nq, int Nk, int d, int deterministic);
int fa_bwd_ex(const void *Q, const void *K, const void *V, const void *O, const void *O_res,
              const void *dO, const float *L, void *dQ, void *dK, void *dV, int B, int H, int Nq,
              int Nk, int d, int layout, int window_left, int window_right, int deterministic,
              float scale, int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The stages of fa_bwd_ex selected by the bit set `stages` (fa_stage), with the same
 * arguments and checks; pointers that the selected stages do not read or write may be
 * NULL. Running FA_STAGE_PREPROCESS, FA_STAGE_DKDV and FA_STAGE_DQ in this order on one
 * stream is fa_bwd_ex; each stage is one kernel launch (bench.py times them one by
 * one).
 *   FA_STAGE_PREPROCESS  D_i = sum_t dO_it (O_it + O_res_it) and -L * log2(e) into the
 *                        workspace, and zeroes its fp32 dQ accumulator (if any);
 *   FA_STAGE_DKDV        recomputes P from Q, K and the workspace's scaled L, writes
 *                        dK and dV, and adds the dQ partials into the accumulator;
 *   FA_STAGE_DQ          dQ = dtype(scale * accumulator); in deterministic mode the
 *                        separate dQ pass, which reads Q, K, V, dO and the workspace's
 *                        row statistics.
 */
int fa_bwd_ex_stage(int stages, const void *Q, const void *K, const void *V, const void *O,
                    const void *O_res, const void *dO, const float *L, void *dQ, void *dK,
                    void *dV, int B, int H, int Nq, int Nk, int d, int layout, int window_left,
                    int window_right, int deterministic, float scale, int dtype, void *workspace,
                    size_t workspace_bytes, void *stream);

/*
 * The tile schedule of a key window, for callers that size or account for the work:
 * with query_side = 1, the key/value tiles (of 128 keys) that query tile `tile` (rows
 * 128*tile .. 128*tile + 127) visits in the forward; with query_side = 0, the query
 * tiles that key tile `tile` visits in the dK/dV pass. Writes the first tile and the
 * count (0: none) of a consecutive range. FA_ERR_INVALID for a tile out of range,
 * non-positive lengths or a NULL output. Touches no device.
 */
int fa_tile_range(int query_side, int tile, int Nq, int Nk, int window_left, int window_right,
                  int *first, int *count);

/*
 * The three stages of fa_bwd, callable one by one (same arguments, same checks, same
 * workspace; fa_bwd is exactly these three in this order on one stream). Each is one
 * kernel launch.
 *   fa_bwd_preprocess  D_i = sum_t dO_it (O_it + O_res_it) and L * log2(e) into the
 *                      workspace, and zeroes its fp32 dQ accumulator.
 *   fa_bwd_dkdv        recomputes P from Q, K and the workspace's scaled L, writes
 *                      dK and dV, and adds the dQ partials into the accumulator.
 *                      Needs fa_bwd_preprocess to have run on this workspace.
 *   fa_bwd_dq_convert  dQ = dtype(scale * accumulator).
 */
int fa_bwd_preprocess(const void *O, const void *O_res, const void *dO, const float *L, int B,
                      int H, int N, int d, int dtype, void *workspace, size_t workspace_bytes,
                      void *stream);
int fa_bwd_dkdv(const void *Q, const void *K, const void *V, const void *dO, void *dK, void *dV,
                int B, int H, int N, int d, int causal, float scale, int dtype, void *workspace,
                size_t workspace_bytes, void *stream);
int fa_bwd_dq_convert(void *dQ, int B, int H, int N, int d, float scale, int dtype,
                      void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward without any device allocation. (The pages have no counterpart to this
 * call: it is an interface convenience.) Some callers cannot allocate device memory
 * at the point where they run the backward -- for instance a plugin inside a host
 * application whose allocator owns the whole device, or a service that must not
 * block or fail on an allocation in its steady state -- and so cannot provide the
 * workspace fa_bwd wants. This variant takes the same arguments as fa_bwd minus the
 * workspace and uses a fixed scratch array that is part of the library instead:
 * 32 MiB, held on every GPU that loads the library until the process exits. It
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Limit: fa_bwd_workspace_size(B, H, N, d) <= 32 MiB, i.e. (for N a multiple of 128)
 * B*H*N <= 64,527 at d = 128 and <= 127,100 at d = 64 (each row takes 8 bytes of
 * row statistics and 4*d bytes of dQ accumulator); larger problems return
 * FA_ERR_UNSUPPORTED before anything touches the device. Other checks and results
 * are those of fa_bwd.
 *
 * The array is per CUDA context: each context that runs this call (the primary
 * context of a device, or one the host application created) holds its own copy.
 * Every call looks up the array's address in the calling thread's current context
 * (cudaGetSymbolAddress); the first call in a context may also load the library's
 * device code there, so make that first call before any stream capture. All calls
 * in one context share the one array: the part that must start at zero (the dQ
 * accumulator) is cleared by every call, but two calls whose work overlaps on the
 * GPU (different streams, no ordering between them) race on it and give wrong
 * gradients. Order such calls on one stream.
 */
int fa_bwd_noalloc(const void *Q, const void *K, const void *V, const void *O, const void *O_res,
                   const void *dO, const float *L, void *dQ, void *dK, void *dV, int B, int H,
                   int N, int d, int causal, float scale, int dtype, void *stream);

/*
 * Decode: a few query rows (1 <= Nq <= 16 per head) against a long key sequence,
 * forward only. Same operation, shapes, layouts and key window as fa_fwd_ex (with
 * Nq <= 16 the bottom-right-aligned causal mask lets query i see keys j <= i + Nk - Nq);
 * writes O and L. The keys of each head are cut into splits of 128-key tiles, one CTA
 * per (head, split), each running the online softmax over its tiles; a second kernel
 * merges the splits' partial outputs by their log-sum-exps (L = ln sum_s exp(L_s),
 * O = sum_s exp(L_s - L) O_s), the recurrence of josueisai.com "flash-attention",
 * section "El truco", applied to whole splits. The pass reads K and V once and is
 * bound by HBM, so it runs on CUDA cores; P is not rounded to 16 bits.
 *
 * The split count depends only on B*H, Nq, Nk and the window (it is chosen for 148
 * SMs), so results are the same bits on every call. `workspace` (device, 256-byte
 * aligned, caller-owned) holds the splits' partial results: at least
 * fa_decode_workspace_size(B, H, Nq, Nk, d, window_left, window_right) bytes, which
 * is 0 when one split suffices (workspace may then be NULL). Nq > 16:
 * FA_ERR_UNSUPPORTED (use fa_fwd_ex).
 */
size_t fa_decode_workspace_size(int B, int H, int Nq, int Nk, int d, int window_left,
                                int window_right);
int fa_decode(const void *Q, const void *K, const void *V, void *O, float *L, int B, int H,
              int Nq, int Nk, int d, int layout, int window_left, int window_right, float scale,
              int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Synchronises `stream`, then returns and clears the device error word of the
 * current device: FA_OK; FA_ERR_TIMEOUT if a kernel abandoned a bounded wait;
 * FA_ERR_CUDA if the synchronisation failed or a kernel found its shared memory
 * placed differently than it needs (it then returned without doing anything).
 */
int fa_get_device_status(void *stream);

/*
 * Self-test of the device-side failure detection: launches one tiny kernel that waits
 * on a barrier nothing will complete, with the bounded-wait routine every kernel of
 * this library uses and a limit of `limit_cycles` SM clock cycles (1 .. 4e9). The
 * wait gives up and records FA_ERR_TIMEOUT, so the next fa_get_device_status(stream)
 * returns FA_ERR_TIMEOUT (and clears it); the context stays usable. FA_ERR_INVALID
 * for a limit out of range.
 */
int fa_selftest_wait_timeout(long long limit_cycles, void *stream);

/*
 * Self-test of the forward kernel's exponential on the FMA pipe (part of each softmax
 * thread's 2^x is computed without the MUFU unit: a Cody-Waite style split x = i + f
 * and a minimax polynomial for 2^f on [-1/2, 1/2]). Writes y[k] = that 2^x[k] for
 * k < n, asynchronously on `stream`. x and y: device float arrays of n elements,
 * 8-byte aligned, owned by the caller. n must be even; n = 0 returns FA_OK without a
 * launch. FA_ERR_INVALID for a negative or odd n, a null or misaligned pointer.
 * Inputs below -125 give 2^-125 (the kernel keeps masked scores off this path).
 */
int fa_selftest_exp2(const float *x, float *y, int n, void *stream);

/* Static, human-readable name of a status code. */
const char *fa_status_string(int status);

/* Library version, for the binding's load check. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
