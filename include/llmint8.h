/*
 * llmint8.h -- C ABI of the B200 (sm_100a) LLM.int8() mixed-precision
 * decomposition matmul  Y[M,N] = X[M,K] . W[K,N].
 *
 * The method (page titles and sections it is taken from):
 *  - "LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale",
 *    arXiv abstract: weights are loaded, converted to int8 and used at once;
 *    vector-wise quantization with one normalization constant per inner
 *    product; the emergent outlier feature dimensions go to a 16-bit matmul
 *    while more than 99.9 % of the values are multiplied in 8-bit.
 *  - "Compress your LLMs", bullets "Vector-wise quantization" and
 *    "Mixed-precision decomposition": one scaling constant per row of the
 *    input X and one per column of the weight W; outlier dimensions (~0.1 %)
 *    in 16-bit, the rest in 8-bit.
 *  - "8-bit Matrix Multiplication for Large Language Models", Summary &
 *    Methodology Analysis: the int8 product is dequantized by the outer
 *    product of the row and column constants and added to the outlier product
 *    in 16-bit floating point.
 *  - "What is 8-bit LLM quantization?", How does INT8 quantization work?:
 *    q = round(value / step), value ~ q * step.
 *
 * Definitions used by every entry point (tau = threshold):
 *   O      = ascending { k : |X[i,k]| >= tau for some row i of this call }
 *   rs[i]  = max over k not in O of |X[i,k]|           (row absmax, fp32)
 *   Xq[i,k]= k in O or rs[i]==0 ? 0 : rha(127 * X[i,k] / rs[i])
 *   cs[j]  = max over all k of |W[k,j]|                 (column absmax, fp32)
 *   Wq[j,k]= cs[j]==0 ? 0 : rha(127 * W[k,j] / cs[j])
 *   acc    = Xq . Wq^T (exact, int32; needs K <= 133143)
 *   Y[i,j] = fp16_RNE( acc[i,j] * rs[i] * cs[j] / 127^2
 *                      + sum over k in O of X[i,k] * W[k,j] )
 * rha = round half away from zero; every code is exact (no approximate
 * division), so Xq, Wq, rs, cs, O and acc are unique.  The outlier product is
 * accumulated in fp32 and Y is rounded once to fp16.
 *
 * Conventions.  Every pointer argument except host-only ones is a DEVICE
 * pointer on the current CUDA device; the library allocates no memory and
 * keeps no per-call state.  `stream` is a cudaStream_t (NULL = legacy default
 * stream); every call only enqueues work on it and returns without waiting.
 * Leading dimensions are in ELEMENTS.  Arguments are validated on the host
 * before anything is launched; on an error nothing is launched.  Conditions
 * only the device can see (outlier overflow, a bounded wait that gave up) set
 * bits of a status word held in the workspace; llmint8_check_status() reads
 * and clears it.  Calls that share a workspace must be ordered on one stream.
 */
#ifndef LLMINT8_H
#define LLMINT8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum llmint8_status {
    LLMINT8_OK = 0,
    LLMINT8_ERR_INVALID_ARG = 1,      /* bad size, null or misaligned pointer, bad ld, NaN tau */
    LLMINT8_ERR_UNSUPPORTED = 2,      /* current device is not sm_100 (B200) */
    LLMINT8_ERR_WORKSPACE = 3,        /* workspace null, too small or not 256-byte aligned */
    LLMINT8_ERR_CUDA = 4,             /* a CUDA runtime or driver call failed */
    LLMINT8_ERR_OUTLIER_OVERFLOW = 5, /* device: n_o > outlier_cap (Y is NaN-filled) */
    LLMINT8_ERR_TIMEOUT = 6           /* device: a bounded wait inside a kernel gave up */
} llmint8_status;

/* Bits of the device status word (see llmint8_check_status). */
#define LLMINT8_STATUS_OUTLIER_OVERFLOW 0x1u
#define LLMINT8_STATUS_TIMEOUT 0x2u

/* Human-readable name of a status code (static string, never NULL). */
const char* llmint8_status_string(llmint8_status s);

/* Size in bytes of the workspace one call of llmint8_mixed_matmul or
 * llmint8_quantize_act_rowwise_outliers needs for these sizes.  The workspace
 * is caller-owned device memory, 256-byte aligned, zero-filled once before its
 * first use (llmint8_workspace_init or any memset); the library leaves the
 * parts that must start at zero back at zero.  It holds the status word, the
 * column maxima, the outlier set, the row scales, Xq, the gathered outlier
 * columns of X and, for M <= 32, the split-K sums of the decode GEMM, or, for
 * M > 32, the operands of the tensor-core outlier product (fp16 [M, 256] and
 * [N, 256], 512 * (M + N) bytes).  Returns 0 for invalid sizes. */
size_t llmint8_workspace_size(int64_t M, int64_t N, int64_t K, int64_t outlier_cap);

/* Zero-fill `ws` (cudaMemsetAsync on `stream`). */
llmint8_status llmint8_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Byte offsets of the intermediates inside a workspace sized by
 * llmint8_workspace_size (for inspection by tests and tools). */
typedef struct llmint8_ws_layout {
    size_t status;      /* uint32 status word */
    size_t n_outlier;   /* int32 n_o (true count, may exceed outlier_cap) */
    size_t outlier_idx; /* int32 [outlier_cap], ascending O */
    size_t row_scale;   /* fp32 [M] */
    size_t xq;          /* int8 [M, ldq], ldq = round_up(K, 16) */
    size_t xo;          /* fp16 [M, ldo], ldo = round_up(max(outlier_cap,1), 8): X[:, O] */
    int64_t ldq;
    int64_t ldo;
    size_t total;
} llmint8_ws_layout;
llmint8_status llmint8_workspace_layout(int64_t M, int64_t N, int64_t K, int64_t outlier_cap,
                                        llmint8_ws_layout* out /* host */);

/* Step a0, offline: column-wise int8 quantization of the weight ("Compress
 * your LLMs", Vector-wise quantization: one constant per column of W; arXiv
 * abstract: a 16-bit checkpoint is converted to int8 at load time).
 *   W         fp16 [K, N], row stride ldw >= N (row-major, as stored in a
 *             checkpoint).  Read only.
 *   Wq        int8 [N, ldk] written: Wq[j*ldk + k] = code of W[k,j] (the
 *             transpose, K contiguous, the layout the int8 tensor-core GEMM
 *             reads); ldk >= K, ldk % 16 == 0, Wq 16-byte aligned; entries
 *             k in [K, ldk) are written 0.
 *   col_scale fp32 [N] written: cs[j] (the absmax, exact fp16 value).
 * Errors: INVALID_ARG for K < 1, N < 1, ldw < N, bad ldk or alignment, null
 * pointers; UNSUPPORTED off sm_100; CUDA on a launch failure. */
llmint8_status llmint8_quantize_weight_colwise(const void* W, int64_t K, int64_t N, int64_t ldw,
                                               int8_t* Wq, int64_t ldk, float* col_scale,
                                               void* stream);

/* Steps a1-a4 on the activation: outlier-column scan, row absmax over the
 * non-outlier columns, row-wise int8 quantization and gather of the outlier
 * columns ("Compress your LLMs", both bullets; arXiv abstract).
 *   X           fp16 [M, K], row stride ldx >= K.  Read only.
 *   tau         threshold, >= 0 or +inf (NaN rejected).  |x| >= tau marks x's
 *               column an outlier over all M rows of this call.
 *   Xq          int8 [M, ldq] written; ldq >= K, ldq % 16 == 0, 16-byte
 *               aligned; outlier columns and columns [K, ldq) are 0.
 *   row_scale   fp32 [M] written.
 *   outlier_idx int32 [outlier_cap] written: the first min(n_o, cap) entries
 *               of O, ascending.
 *   n_outlier   int32 [1] written: n_o (may exceed outlier_cap; then the
 *               status word gets LLMINT8_STATUS_OUTLIER_OVERFLOW).
 *   Xo          optional fp16 [M, ldo] (NULL to skip): Xo[i,t] = X[i,O[t]]
 *               for t < min(n_o, cap); ldo >= outlier_cap.
 *   ws          workspace (see llmint8_workspace_size).
 * All outputs are device-side; nothing is copied to the host.  When X's rows
 * are 16-byte aligned (ldx % 8 == 0, K % 8 == 0) and X fits in shared memory
 * spread over the SMs (at most 16 rows and 200 KB per SM), the step is one
 * cooperative kernel (the driver guarantees its CTAs are resident together):
 * X is read once, and the CTAs meet at a grid barrier between the column scan
 * and the row quantization (bounded: after 2 s it sets
 * LLMINT8_STATUS_TIMEOUT, and the workspace must be zero-filled again before
 * reuse).  Otherwise two kernels: for many such rows with 2048 <= K <= 16384
 * a column scan and a row pass that stream whole rows through shared memory,
 * else a column scan and a per-row kernel. */
llmint8_status llmint8_quantize_act_rowwise_outliers(const void* X, int64_t M, int64_t K, int64_t ldx,
                                                     float tau, int8_t* Xq, int64_t ldq, float* row_scale,
                                                     int32_t* outlier_idx, int64_t outlier_cap,
                                                     int32_t* n_outlier, void* Xo, int64_t ldo, void* ws,
                                                     size_t ws_bytes, void* stream);

/* The whole forward path a1-a7: Y = X . W by the mixed-precision
 * decomposition ("8-bit Matrix Multiplication for Large Language Models",
 * Summary & Methodology Analysis; arXiv abstract).
 *   X          fp16 [M, K], row stride ldx >= K.
 *   Wq, ldk    int8 [N, ldk] and
 *   col_scale  fp32 [N] from llmint8_quantize_weight_colwise.
 *   W, ldw     fp16 [K, N] row-major, row stride ldw >= N: only the rows in O
 *              are read (the 16-bit outlier product).  W may be NULL (ldw
 *              ignored) when no fp16 copy of the weight is kept: the outlier
 *              rows are then recovered from Wq, W~[k, j] = fp16_RNE(Wq[j, k]
 *              * cs[j] / 127), so the weight lives in memory as int8 only
 *              ("LLM.int8()" arXiv abstract: inference memory halved).
 *   bias       optional fp16 [N] (NULL for none), 2-byte aligned: the linear
 *              layer's bias, added to every row after the outlier product and
 *              before the fp16 rounding (Y = X W + b).
 *   tau        threshold (>= 0 or +inf).
 *   outlier_cap  bound on n_o the workspace is sized for; outlier_cap = K is
 *              always enough.  If n_o > outlier_cap, Y is filled with NaN and
 *              LLMINT8_STATUS_OUTLIER_OVERFLOW is set.
 *   Y, ldy     fp16 [M, N] written, row stride ldy >= N.
 *   ws         workspace of at least llmint8_workspace_size(M, N, K, cap).
 * Runs three kernels on `stream` (scan/max, quantize/gather, int8 tcgen05
 * GEMM with the dequantize + outlier epilogue; for M <= 32 a split-K GEMM
 * that streams Wq on all SMs), or two when the activation step fits one
 * kernel.  Decode-shaped calls (ldx % 8 == 0, X 16-byte aligned) take one
 * kernel for all of it: for M <= 8 with K a multiple of 512 up to 4096 and at
 * most 64 Wq rows per SM, each CTA owns whole Wq rows; otherwise for M <= 32
 * with K % 8 == 0 and K <= 16384 (and N, K small enough that each CTA's share
 * of Xq fits in 32 KB of shared memory) CTA clusters split K, exchange outlier
 * flags and row maxima through distributed shared memory and reduce their
 * int32 partial sums there.  Both start reading Wq before the preceding
 * kernel on the stream has finished (programmatic dependent launch), so Wq
 * must not be written by a kernel that lets its dependents start early
 * (llmint8_quantize_weight_colwise's kernel does not).  The workspace then
 * receives the same Xq, row scales, O, n_o and Xo.
 * Where the 16-bit outlier product runs in the prefill GEMM's epilogue: for
 * n_o <= K / 256 on the CUDA cores (fp32 FMAs of the exact fp16 products);
 * with K / 256 < n_o <= 256 on the 5th-generation tensor cores: the epilogue
 * dequantizes the tile in TMEM, the MMA issuer accumulates Xo . W[O, :] onto
 * it (tcgen05.mma kind::f16, fp32) from operands the kernel gathers into the
 * workspace (Xo and W[O, :]^T, zero padded to whole 64-column blocks), and
 * the epilogue rounds the result; past 256 outliers by warp-level mma.sync.
 * All three accumulate the exact fp16 products in fp32.
 * llmint8_mixed_matmul_path names the kernels of a call.  No host
 * synchronisation. */
llmint8_status llmint8_mixed_matmul(const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* Wq,
                                    int64_t ldk, const float* col_scale, const void* W, int64_t ldw,
                                    const void* bias, int64_t N, float tau, int64_t outlier_cap, void* Y,
                                    int64_t ldy, void* ws, size_t ws_bytes, void* stream);

/* Outlier statistics of X for the threshold tau, the quantities the pages
 * report ("8-bit Matrix Multiplication for Large Language Models", Summary &
 * Methodology Analysis: at 6.7B, 150,000 outliers per sequence concentrated
 * in 6 feature dimensions):
 *   stats  int64 [3] (device, 8-byte aligned) written: the number of values
 *          with |x| >= tau, of columns holding one (n_o), of rows holding one.
 *          NaN never counts.
 *   ws     a workspace of llmint8_workspace_size(M', N', K, cap) bytes for
 *          any M', N', cap (the statistics use a K-sized part of it, left at
 *          zero); zero-filled once like every workspace.
 * One kernel on `stream`; no host synchronisation. */
llmint8_status llmint8_outlier_stats(const void* X, int64_t M, int64_t K, int64_t ldx, float tau, int64_t* stats,
                                     void* ws, size_t ws_bytes, void* stream);

/* Number of kernels llmint8_mixed_matmul launches on the current device for
 * these arguments, for a Wq with the packed leading dimension ldk =
 * round_up(K, 16): 1 on a one-kernel decode path, 2 when the activation step
 * is one kernel, else 3 (0 for invalid sizes or no supported device).
 * llmint8_mixed_matmul_path takes ldk.  Host-only query. */
int llmint8_mixed_matmul_kernels(int64_t M, int64_t N, int64_t K, int64_t ldx, const void* X);

/* The kernels llmint8_mixed_matmul launches for these arguments, by name, in
 * launch order and comma-separated: "decode_gemv_kernel" (M <= 8, whole Wq
 * rows per CTA), "decode_fused_kernel" (M <= 32, cluster split-K), or the
 * activation step ("act_fused_kernel"; "scan_stream_kernel" then
 * "quantize_stream_kernel" for many 16-byte aligned rows with 2048 <= K <=
 * 16384; else "scan_columns_kernel" then "quantize_rows_kernel" /
 * "quantize_rows_long_kernel") followed by the GEMM
 * ("gemm_i8_decode_kernel" for M <= 32, else "gemm_i8_kernel").  ldk is the
 * leading dimension of the Wq the call will get.  The string is static (do
 * not free it).  NULL for arguments the call rejects as invalid, or when no
 * CUDA device is current.  Launches nothing. */
const char* llmint8_mixed_matmul_path(int64_t M, int64_t N, int64_t K, int64_t ldx, int64_t ldk, const void* X);

/* Steps a5-a7 alone, on an activation already quantized by
 * llmint8_quantize_act_rowwise_outliers (so that one quantized X can feed
 * several weights, e.g. projections that share their input):
 *   Y = fp16( (Xq . Wq^T) * rs (x) cs / 127^2 + Xo . W[O, :] ).
 *   Xq, ldq          int8 [M, ldq] (ldq % 16 == 0, 16-byte aligned)
 *   row_scale        fp32 [M]
 *   outlier_idx      int32 [outlier_cap], n_outlier int32 [1] (device)
 *   Xo, ldo          fp16 [M, ldo], ldo >= outlier_cap
 *   Wq, ldk, col_scale, W, ldw, bias, Y, ldy  as for llmint8_mixed_matmul
 *   ws               at least 256 bytes (status word).  For M <= 32 the GEMM
 *                    splits K across CTAs when ws also holds its reduction
 *                    scratch (a workspace of llmint8_workspace_size(M, N, K,
 *                    outlier_cap) bytes, zero-filled once, does); the scratch is
 *                    the end of ws and is left at zero.  For M > 32 such a
 *                    workspace also holds the operands of the tensor-core
 *                    outlier product (see llmint8_mixed_matmul), at the same
 *                    place as for llmint8_mixed_matmul: past the activation
 *                    step's scratch, Xq and Xo, so the workspace of the
 *                    quantize call serves here too; a smaller one leaves the
 *                    product to the epilogue.
 * If n_outlier > outlier_cap, Y is NaN-filled (the status bit was set by the
 * quantize call).  One kernel launch (the tcgen05 GEMM). */
llmint8_status llmint8_mixed_gemm(const int8_t* Xq, int64_t ldq, const float* row_scale,
                                  const int32_t* outlier_idx, const int32_t* n_outlier, int64_t outlier_cap,
                                  const void* Xo, int64_t ldo, const int8_t* Wq, int64_t ldk,
                                  const float* col_scale, const void* W, int64_t ldw, const void* bias,
                                  int64_t M, int64_t N, int64_t K, void* Y, int64_t ldy, void* ws,
                                  size_t ws_bytes, void* stream);

/* Allocation-free variant of llmint8_quantize_act_rowwise_outliers (the
 * pages have no counterpart: this serves callers of this library that cannot
 * give it a device workspace -- an engine that plans all device memory up
 * front, or code that may not call cudaMalloc at call time because it would
 * synchronise the device or break a latency budget).  Same arguments and
 * outputs, minus the workspace; the scratch (status word, column maxima,
 * per-block counters, outlier bitmask) lives in a 256 KiB device array inside
 * the library, which every GPU it is used on keeps until the process exits.
 *   K <= LLMINT8_NOALLOC_MAX_K, otherwise LLMINT8_ERR_WORKSPACE and nothing
 *   runs.  This entry point calls no cudaMalloc, cudaFree or allocating
 *   library routine.  With lazy module loading (the CUDA 12 default) the
 *   first call on a device loads the library's device code, and the driver
 *   places the array in device memory at that moment: a caller that must not
 *   see any allocation at call time makes one call during its initialisation.
 *   Every call looks up the array's device address on the current device (so
 *   a device reset or a new primary context is picked up); the first call
 *   that sees a new address zero-fills the array on `stream`, so make that
 *   first call before any stream capture.  All calls share the array and it
 *   keeps the last call's contents (the kernels return the parts that must
 *   start at zero to zero): calls that overlap on the GPU (different streams
 *   or host threads) race and must be ordered by the caller.  The status word
 *   is not reported; an outlier overflow shows as *n_outlier > outlier_cap. */
#define LLMINT8_NOALLOC_MAX_K 61440
llmint8_status llmint8_quantize_act_rowwise_outliers_noalloc(const void* X, int64_t M, int64_t K, int64_t ldx,
                                                             float tau, int8_t* Xq, int64_t ldq, float* row_scale,
                                                             int32_t* outlier_idx, int64_t outlier_cap,
                                                             int32_t* n_outlier, void* Xo, int64_t ldo,
                                                             void* stream);

/* Reassembly of an output whose columns were computed on several GPUs
 * ("Compress your LLMs": the pages serve one model from 8 GPUs; the
 * column-parallel split needs no exchange before the matmul, since the outlier
 * set is a function of the replicated X, and one all-gather of Y after it).
 *   blocks   fp16 [world, M, ld_block] (device): block r holds Y[:, bounds[r]
 *            .. bounds[r+1]) in its first bounds[r+1] - bounds[r] <= ld_block
 *            columns (what an all-gather of each GPU's shard leaves behind).
 *   bounds   int64 [world + 1] (HOST), bounds[0] = 0, non-decreasing,
 *            bounds[world] = N >= 1.  world <= 64.
 *   Y, ldy   fp16 [M, N] written, row stride ldy >= N.
 * One copy kernel on `stream` (16-byte moves when the block starts and both
 * strides are multiples of 8 halves).  INVALID_ARG for bad sizes or bounds. */
llmint8_status llmint8_unshard_columns(const void* blocks, int64_t world, int64_t M, int64_t ld_block,
                                       const int64_t* bounds, void* Y, int64_t ldy, void* stream);

/* Synchronise `stream`, read the status word of `ws`, clear it, and return
 * LLMINT8_OK, LLMINT8_ERR_OUTLIER_OVERFLOW or LLMINT8_ERR_TIMEOUT (timeout
 * wins).  `flags_out` (host, may be NULL) receives the raw bits.  After a
 * timeout the workspace's internal counters may be left non-zero: zero it
 * (llmint8_workspace_init) before its next use. */
llmint8_status llmint8_check_status(void* ws, void* stream, uint32_t* flags_out);

/* Test hook for step a5 alone: C[i,j] = sum_k Xq[i,k] * Wq[j,k] as int32,
 * computed by the same tcgen05 kernel as llmint8_mixed_matmul (the epilogue
 * stores the raw accumulator instead of dequantizing).
 *   Xq int8 [M, ldq], Wq int8 [N, ldk] (ld % 16 == 0, 16-byte aligned),
 *   C int32 [M, ldc] written, ldc >= N.  `ws` supplies the status word (and,
 *   for M <= 32, the split-K scratch as for llmint8_mixed_gemm). */
llmint8_status llmint8_debug_int8_gemm_i32(const int8_t* Xq, int64_t ldq, const int8_t* Wq, int64_t ldk,
                                           int64_t M, int64_t N, int64_t K, int32_t* C, int64_t ldc,
                                           void* ws, size_t ws_bytes, void* stream);

/* Test hook for the whole path's step a5: runs exactly what
 * llmint8_mixed_matmul runs for these arguments (the same kernels, launch
 * plan and workspace outputs Xq, rs, O, n_o, Xo), except that every path's
 * epilogue stores the raw int32 accumulator
 *   C[i,j] = sum_k Xq[i,k] * Wq[j,k]      ("Compress your LLMs", Vector-wise
 * quantization: the int8 product before the outer-product dequantization)
 * into C int32 [M, ldc] (ldc >= N, 4-byte aligned) instead of Y, so that the
 * one-kernel decode paths' int32 sums can be compared exactly.  No fp16
 * weight or bias is read.  Same errors as llmint8_mixed_matmul. */
llmint8_status llmint8_debug_mixed_matmul_i32(const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* Wq,
                                              int64_t ldk, const float* col_scale, int64_t N, float tau,
                                              int64_t outlier_cap, int32_t* C, int64_t ldc, void* ws,
                                              size_t ws_bytes, void* stream);

/* Test hook for failure detection (the pages have no counterpart).  Sets, on
 * the current device, the bound after which every bounded wait inside the
 * kernels gives up (default 2 s) and a mask of waits that are made to wait
 * for an event that never comes, so that a test can watch a wait run out and
 * the kernel return with LLMINT8_STATUS_TIMEOUT set instead of hanging:
 *   0x1  the one-kernel activation step's grid barrier,
 *   0x2  the matrix-vector decode kernel's wait for its weight copy,
 *   0x4  the tcgen05 GEMM's MMA issuer, before its first operand stage.
 * The kernels still let every copy they issued land before they exit.  After
 * a stalled activation step the workspace must be zero-filled again.
 * limit_ns == 0 is rejected (INVALID_ARG).  Synchronous; call it with no work
 * of this library in flight, and call llmint8_debug_set_waits(2000000000, 0)
 * to restore the defaults. */
llmint8_status llmint8_debug_set_waits(uint64_t limit_ns, uint32_t stall_mask);

#ifdef __cplusplus
}
#endif

#endif /* LLMINT8_H */
