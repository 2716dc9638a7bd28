// kernels.cuh -- launch interfaces between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace llmint8 {

// Scratch the activation kernels keep in the caller's workspace.
struct ActWs {
  uint32_t* colmax;       // [K] fp16 bit patterns of the column maxima; zero between calls
  uint32_t* blk_counter;  // [ceil(K/256)] scan CTAs finished per column block; zero between calls
  uint32_t* bitmask;      // [ceil(K/32)] outlier flags of this call; zero between calls
  uint32_t* status;       // status word
  // One-kernel activation step (optional, nullptr: not used): a 64-bit grid
  // arrival counter followed by two outlier bitmasks of ceil(K/32) words each
  // (this call ORs into one, zeroes the other for the next call); zero-filled
  // once with the workspace.
  uint32_t* fused = nullptr;
  uint32_t stall = 0;  // test hook: stall mask (ptx.cuh), 0 in normal use
};

// Bytes of ActWs::fused for K columns (256-byte multiple).
inline size_t act_fused_bytes(int64_t K) { return (16 + 8 * size_t((K + 31) / 32) + 255) / 256 * 256; }

// Outlier statistics scratch (zero between calls): a column bitmask of
// ceil(K/32) words, then three 64-bit counters (values, rows, CTAs done).
inline size_t stats_scratch_bytes(int64_t K) {
  return (8 * size_t(((K + 31) / 32 + 1) / 2) + 24 + 255) / 256 * 256;
}
// stats: int64 [3] (device) <- values with |x| >= tau, their columns, their rows.
cudaError_t launch_outlier_stats(const void* X, int64_t M, int64_t K, int64_t ldx, float tau, uint32_t* scratch,
                                 int64_t* stats, int num_sms, cudaStream_t stream);

cudaError_t launch_quantize_weight_colwise(const void* W, int64_t K, int64_t N, int64_t ldw, int8_t* Wq,
                                           int64_t ldk, float* col_scale, cudaStream_t stream);

// Whether the activation step for these arguments runs as one kernel (X fits
// in shared memory spread over num_sms CTAs and its rows allow 16-byte loads).
bool act_fused_plan(int64_t M, int64_t K, int64_t ldx, const void* X, int num_sms);

// Whether the activation step for these arguments runs as the two streaming
// kernels (many rows, 16-byte aligned, K % 8 == 0, kStreamMinK <= K <= kStreamMaxK).
constexpr int64_t kStreamMinK = 2048;
constexpr int64_t kStreamMaxK = 16384;
bool act_stream_plan(int64_t M, int64_t K, int64_t ldx, const void* X, int num_sms);

// num_sms > 0 and ws.fused set: shapes whose X fits in shared memory across
// the SMs run as one persistent kernel (grid barrier between the column scan
// and the row quantization); otherwise two kernels (the streaming pair when
// act_stream_plan holds).
cudaError_t launch_quantize_act(const void* X, int64_t M, int64_t K, int64_t ldx, float tau, int8_t* Xq,
                                int64_t ldq, float* rs, int32_t* O, int64_t cap, int32_t* n_out, void* Xo,
                                int64_t ldo, ActWs ws, cudaStream_t stream, bool pdl, int num_sms = 0);

// Everything the GEMM epilogue needs besides the two tensor maps.
struct GemmArgs {
  int M, N, K;
  const float* rs;    // [M] row scales
  const float* cs;    // [N] column scales
  const void* Xo;     // fp16 [M, ldo] gathered outlier columns of X
  int64_t ldo;
  const int32_t* O;   // [cap] outlier columns (rows of W)
  const int32_t* n_o; // device count
  int cap;
  const void* W;      // fp16 [K, ldw]; nullptr: the outlier rows come from Wq
  int64_t ldw;
  const int8_t* Wq;   // int8 [N, ldk] (read for the outlier rows when W is nullptr)
  int64_t ldk;
  const void* bias;   // fp16 [N] added to every row, or nullptr
  void* Y;            // fp16 [M, ldy]
  int64_t ldy;
  int32_t* C;         // int32 [M, ldc] (raw accumulator output mode)
  int64_t ldc;
  uint32_t* status;
  bool y_tma;         // Y is written through the tmY tensor map (16-byte aligned rows)
  uint32_t stall;     // test hook: stall mask (ptx.cuh), 0 in normal use
  // The outlier product on the tensor cores (K/256 < n_o <= kOutlierMmaMax):
  // the kernel gathers Xo and the outlier rows of W, zero padded to a
  // multiple of 64 columns, into xo_p [M, kOutlierMmaMax] and wo_t
  // [N, kOutlierMmaMax] (fp16, K-major, read back through the tmXo / tmWo
  // tensor maps); om_sync holds two counters that are zero between calls.
  // om_ok false: never.
  bool om_ok;
  void* xo_p;
  void* wo_t;
  uint32_t* om_sync;
};

// Outlier columns the tensor-core outlier product takes at most (four blocks
// of 64 fp16 columns), and the workspace bytes it needs for M x N.
constexpr int kOutlierMmaMax = 256;
inline size_t outlier_mma_bytes(int64_t M, int64_t N) {
  return size_t(M) * 2 * kOutlierMmaMax + size_t(N) * 2 * kOutlierMmaMax;
}

// Whether the GEMM for M rows runs as CTA pairs (256 x 256 tiles, cta_group::2)
// rather than single CTAs (128 x 256 tiles).
bool gemm_uses_pair(int M);

// tmA: Xq [M rows, K cols] int8 in boxes of 128 rows, tmB: Wq [N rows, K cols]
// int8 in boxes of gemm_b_box_rows(M) rows, 128 bytes along K, 128-byte
// swizzle.  raw_i32 selects the accumulator-dump epilogue.
// tmY: Y [M rows, N cols] fp16 in boxes of 16 rows x 64 columns, 128-byte
// swizzle (used when a.y_tma).  tmXo / tmWo: a.xo_p [M rows, kOutlierMmaMax
// cols] and a.wo_t [N rows, kOutlierMmaMax cols] fp16 in boxes of 64 columns
// and 128 (Xo) / gemm_b_box_rows(M) (W) rows, 128-byte swizzle (used when
// a.om_ok).
cudaError_t launch_gemm_i8(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmY,
                           const CUtensorMap& tmXo, const CUtensorMap& tmWo, const GemmArgs& a, bool raw_i32,
                           int num_sms, cudaStream_t stream, bool pdl);

// Tile sizes of the GEMM per CTA (accumulator rows / columns, K bytes per stage).
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 128;

inline unsigned gemm_b_box_rows(int M) { return gemm_uses_pair(M) ? kGemmBN / 2 : kGemmBN; }

// ------------------------------------------------------------------ decode GEMM (M <= kDecodeMaxM)
constexpr int kDecodeMaxM = 32;

struct DecodeArgs {
  int M, N, K;
  int splits;        // K slices per 128-row tile of Wq
  int kb_per_split;  // 128-byte K blocks per slice
  const float* rs;
  const float* cs;
  const void* Xo;
  int64_t ldo;
  const int32_t* O;
  const int32_t* n_o;
  int cap;
  const void* W;       // nullptr: the outlier rows come from Wq
  int64_t ldw;
  const int8_t* Wq;    // int8 [N, ldk]
  int64_t ldk;
  const void* bias;    // fp16 [N] or nullptr
  void* Y;
  int64_t ldy;
  int32_t* C;  // raw int32 output mode
  int64_t ldc;
  int32_t* partial;         // int32 [N, NP] split-K sums, zero between calls (splits > 1)
  uint32_t* tile_counter;   // [ceil(N/128)] slices finished per tile, zero between calls
  uint32_t* status;
};

// Rows of X padded to the MMA's N (16 or 32).
int decode_rows_padded(int M);
// K slices per tile so that tiles x slices CTAs cover num_sms (1 if !can_split).
void decode_split(int M, int N, int K, int num_sms, bool can_split, int* splits, int* kb_per_split);
// Scratch bytes of the split-K reduction: partial sums + per-tile counters.
inline size_t decode_scratch_bytes(int M, int N) {
  const size_t partial = size_t(N) * size_t(M <= 16 ? 16 : 32) * 4;
  const size_t counters = size_t((N + 127) / 128) * 4;
  return ((partial + 255) / 256) * 256 + ((counters + 255) / 256) * 256;
}
// tmA: Wq [N rows, K cols] int8 in boxes of 128 rows x 128 bytes; tmB: Xq
// [M rows, K cols] in boxes of decode_rows_padded(M) rows x 128 bytes (both
// 128-byte swizzle).
cudaError_t launch_gemm_i8_decode(const CUtensorMap& tmA, const CUtensorMap& tmB, const DecodeArgs& a, bool raw_i32,
                                  cudaStream_t stream, bool pdl);

// ------------------------------------------------------------------ fused decode path (a1-a7, one kernel)
constexpr int kFusedMaxK = 16384;     // longest K the fused kernel takes
constexpr int kFusedXqBytes = 32768;  // quantized activation a CTA keeps in shared memory

struct FusedArgs {
  const void* X;  // fp16 [M, ldx], rows 16-byte aligned, K % 8 == 0
  int64_t ldx;
  int M, N, K;
  float tau;
  const float* cs;
  const void* W;  // fp16 [K, ldw]: outlier rows; nullptr: recovered from Wq
  int64_t ldw;
  const int8_t* Wq;  // int8 [N, ldk]
  int64_t ldk;
  const void* bias;  // fp16 [N] or nullptr
  void* Y;
  int64_t ldy;
  int8_t* Xq;  // workspace outputs, written by the first cluster
  int64_t ldq;
  float* rs;
  int32_t* O;
  int32_t* n_out;
  void* Xo;
  int64_t ldo;
  int cap;
  uint32_t* status;
  int splits;  // CTAs per tile (cluster size): 1, 2, 4 or 8
  int kb_per;  // 128-column K blocks per CTA (a power of two)
  int stages;  // Wq ring depth: 4 (two CTAs per SM) or 8
  int32_t* C;  // test hook: non-null stores the int32 accumulator [M, ldc] instead of Y
  int64_t ldc;
};

// ------------------------------------------------------------------ decode as a matrix-vector product (M <= 8)
struct GemvArgs {
  const void* X;  // fp16 [M, ldx], rows 16-byte aligned
  int64_t ldx;
  int M, N;
  int64_t K;      // K % 512 == 0, K <= 4096
  float tau;
  const float* cs;
  const void* W;  // fp16 [K, ldw] outlier rows, or nullptr (recovered from Wq)
  int64_t ldw;
  const int8_t* Wq;  // int8 [N, ldk]
  int64_t ldk;
  const void* bias;  // fp16 [N] or nullptr
  void* Y;
  int64_t ldy;
  int8_t* Xq;  // workspace outputs, written by the first CTA
  int64_t ldq;
  float* rs;
  int32_t* O;
  int32_t* n_out;
  void* Xo;
  int64_t ldo;
  int cap;
  uint32_t* status;
  int rows_per;  // Wq rows per CTA
  int tiles;     // 16-row MMA tiles covering rows_per (at most 4)
  int32_t* C;    // test hook: non-null stores the int32 accumulator [M, ldc] instead of Y
  int64_t ldc;
  uint32_t stall;  // test hook: stall mask (ptx.cuh), 0 in normal use
};
// Rows per CTA and tiles for a call; false if this kernel does not take the shape.
bool decode_gemv_plan(int M, int N, int K, int64_t ldk, int num_sms, int* rows_per, int* tiles);
cudaError_t launch_decode_gemv(const GemvArgs& a, cudaStream_t stream, bool pdl);

// Cluster size and K blocks per CTA for a decode call; false if the fused
// kernel does not take this shape (the caller then runs the three-kernel path).
bool decode_fused_plan(int M, int N, int K, int num_sms, int* splits, int* kb_per, int* stages);
// tmA: Wq [N rows, K cols] int8, boxes of 128 rows x 128 bytes, 128-byte swizzle.
cudaError_t launch_decode_fused(const CUtensorMap& tmA, const FusedArgs& a, cudaStream_t stream, bool pdl);

// ------------------------------------------------------------------ column-sharded output (several GPUs)
constexpr int kUnshardMaxWorld = 64;
struct UnshardBounds {
  int64_t bounds[kUnshardMaxWorld + 1];  // block r holds columns [bounds[r], bounds[r+1]) of Y
};
// blocks: fp16 [world, M, ld_block] -> Y fp16 [M, bounds[world]] (row stride ldy).
cudaError_t launch_unshard_columns(const void* blocks, int world, int64_t M, int64_t ld_block, const UnshardBounds& b,
                                   void* Y, int64_t ldy, int num_sms, cudaStream_t stream);

// ------------------------------------------------------------------ test hooks
// Each compiled file keeps its own copy of the wait bound (ptx.cuh); these
// set it, one per file.  The stall mask travels in the launch arguments.
cudaError_t set_debug_waits_decode_fused(uint64_t limit_ns);
cudaError_t set_debug_waits_decode_gemv(uint64_t limit_ns);
cudaError_t set_debug_waits_gemm_i8(uint64_t limit_ns);
cudaError_t set_debug_waits_gemm_i8_decode(uint64_t limit_ns);
cudaError_t set_debug_waits_quant_act(uint64_t limit_ns);

}  // namespace llmint8
