// capi.cu -- the extern "C" boundary declared in include/llmint8.h:
// argument validation, workspace layout, TMA tensor-map encoding and kernel
// launches.  No memory is allocated here; every buffer is the caller's.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "kernels.cuh"
#include "llmint8.h"

using namespace llmint8;

namespace {

// An NVTX range around each entry point's host work and launches, so that a
// profiler timeline shows which library call issued which kernels (the
// header-only NVTX calls cost nothing when no tool is attached).
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
};

constexpr int64_t kMaxK = 133143;  // 127^2 * K < 2^31: the int32 accumulator cannot overflow
constexpr int kMaxDevices = 64;

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
bool aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

// ------------------------------------------------------------------ devices
struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int num_sms = 0;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

llmint8_status current_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LLMINT8_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return LLMINT8_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);  // sm_100: the code is built for sm_100a only
    d.num_sms = sms;
    d.probed = true;
  }
  if (!d.supported) return LLMINT8_ERR_UNSUPPORTED;
  if (num_sms) *num_sms = d.num_sms;
  return LLMINT8_OK;
}

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A 2D tensor map with the 128-byte swizzle (out-of-range reads give 0).  A
// map depends only on its arguments, so the last kMapCache maps encoded on
// this thread are kept and handed out again for the same arguments: a call
// that repeats the previous calls' buffers and shapes encodes nothing.
constexpr int kMapCache = 64;
struct MapKey {
  CUtensorMapDataType type;
  const void* base;
  uint64_t cols, rows, stride;
  uint32_t box_cols, box_rows;
  bool operator==(const MapKey& o) const {
    return type == o.type && base == o.base && cols == o.cols && rows == o.rows && stride == o.stride &&
           box_cols == o.box_cols && box_rows == o.box_rows;
  }
};
struct MapCache {
  MapKey key[kMapCache];
  CUtensorMap map[kMapCache];
  int size = 0, next = 0;
};

bool encode_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, int64_t cols, int64_t rows,
               int64_t stride_bytes, uint32_t box_cols, uint32_t box_rows) {
  thread_local MapCache cache;
  const MapKey k = {type, base, static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                    static_cast<uint64_t>(stride_bytes), box_cols, box_rows};
  for (int i = 0; i < cache.size; ++i) {
    if (cache.key[i] == k) {
      *map = cache.map[i];
      return true;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride_bytes)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  cache.key[cache.next] = k;
  cache.map[cache.next] = *map;
  cache.next = (cache.next + 1) % kMapCache;
  if (cache.size < kMapCache) ++cache.size;
  return true;
}

// int8 matrix [rows, cols] with row stride ld (bytes), read in boxes of
// box_rows x 128 bytes with the 128-byte swizzle; out-of-range reads are 0.
bool encode_operand_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld,
                        uint32_t box_rows) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, cols, rows, ld, kGemmBK, box_rows);
}

// fp16 operand of the tensor-core outlier product: [rows, kOutlierMmaMax]
// contiguous, read in boxes of box_rows x 64 columns (128 bytes) with the
// 128-byte swizzle.
bool encode_outlier_map(CUtensorMap* map, const void* base, int64_t rows, uint32_t box_rows) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, kOutlierMmaMax, rows, 2 * kOutlierMmaMax, 64,
                   box_rows);
}

// The tensor-core outlier product of the prefill GEMM: its two counters sit in
// the workspace header (zero between calls), its gathered operands (Xo
// [M, kOutlierMmaMax] then W^T [N, kOutlierMmaMax], fp16) at `data`.  Leaves
// a.om_ok false (the epilogue computes the product) when the maps cannot be
// made.
void prepare_outlier_mma(GemmArgs& a, CUtensorMap* tmXo, CUtensorMap* tmWo, void* ws, uint8_t* data) {
  std::memset(tmXo, 0, sizeof(*tmXo));
  std::memset(tmWo, 0, sizeof(*tmWo));
  a.om_ok = false;
  if (data == nullptr) return;
  uint8_t* wo_t = data + size_t(a.M) * 2 * kOutlierMmaMax;
  if (!encode_outlier_map(tmXo, data, a.M, kGemmBM) ||
      !encode_outlier_map(tmWo, wo_t, a.N, gemm_b_box_rows(a.M)))
    return;
  a.xo_p = data;
  a.wo_t = wo_t;
  a.om_sync = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + 16);
  a.om_ok = true;
}

// fp16 output Y [rows, cols] with row stride ld (elements), written in boxes of
// 16 rows x 64 columns with the 128-byte swizzle.  Needs 16-byte aligned rows.
bool encode_output_map(CUtensorMap* map, void* base, int64_t rows, int64_t cols, int64_t ld) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, cols, rows, 2 * ld, 64, 16);
}

// Y through TMA stores when its rows are 16-byte aligned; direct stores otherwise.
bool prepare_output(CUtensorMap* map, void* Y, int64_t M, int64_t N, int64_t ldy) {
  std::memset(map, 0, sizeof(*map));
  if (ldy % 8 != 0 || !aligned(Y, 16)) return false;
  return encode_output_map(map, Y, M, N, ldy);
}

// ------------------------------------------------------------------ workspace
// [0, 256)        header: status u32 @0, n_o i32 @8, outlier-product counters u32 [2] @16 (zero between calls)
// colmax          u32 [K]                 zero between calls
// blk_counter     u32 [ceil(K/256)]       zero between calls
// bitmask         u32 [ceil(K/32)]
// outlier_idx     i32 [cap]
// row_scale       f32 [M]
// xq              i8  [M, ldq]
// xo              f16 [M, ldo]
// decode          (M <= kDecodeMaxM) split-K partial sums + tile counters, zero between calls
// outlier operands (M > 32) fp16 Xo [M, 256] + W^T [N, 256] of the tensor-core outlier product
bool make_layout(int64_t M, int64_t K, int64_t cap, llmint8_ws_layout* L, size_t* colmax, size_t* bitmask,
                 int64_t N = 0, size_t* decode = nullptr, size_t* outlier_ops = nullptr) {
  if (M < 1 || K < 1 || K > kMaxK || cap < 0 || cap > K) return false;
  size_t off = 256;
  *colmax = off;
  off = align_up(off + 4 * size_t(K), 256);
  off = align_up(off + 4 * size_t((K + 255) / 256), 256);  // block counters follow colmax
  *bitmask = off;
  off = align_up(off + 4 * size_t((K + 31) / 32), 256);
  off += act_fused_bytes(K);      // the one-kernel activation step's counters and bitmasks
  off += stats_scratch_bytes(K);  // the outlier statistics' bitmask and counters
  L->status = 0;
  L->n_outlier = 8;
  L->outlier_idx = off;
  off = align_up(off + 4 * size_t(cap > 0 ? cap : 1), 256);
  L->row_scale = off;
  off = align_up(off + 4 * size_t(M), 1024);
  L->ldq = round_up(K, 16);
  L->xq = off;
  off = align_up(off + size_t(M) * size_t(L->ldq), 256);
  L->ldo = round_up(cap > 0 ? cap : 1, 8);
  L->xo = off;
  off = align_up(off + 2 * size_t(M) * size_t(L->ldo), 256);
  if (decode) *decode = off;
  if (M <= kDecodeMaxM && N > 0) off += decode_scratch_bytes(static_cast<int>(M), static_cast<int>(N));
  if (N > 0 && M > kDecodeMaxM) {
    off = align_up(off, 256);
    if (outlier_ops) *outlier_ops = off;
    off += outlier_mma_bytes(M, N);
  }
  L->total = off;
  return true;
}

// Xq and Wq maps of the decode kernel: Wq is the MMA's A operand (128-row boxes),
// Xq its B operand (boxes of the padded row count).
bool encode_decode_maps(CUtensorMap* tmA, CUtensorMap* tmB, const int8_t* Wq, int64_t N, int64_t ldk,
                        const int8_t* Xq, int64_t M, int64_t ldq, int64_t K) {
  return encode_operand_map(tmA, Wq, N, K, ldk, 128) &&
         encode_operand_map(tmB, Xq, M, K, ldq, static_cast<uint32_t>(decode_rows_padded(static_cast<int>(M))));
}

// Test hook: the stall mask of llmint8_debug_set_waits, passed to the kernels
// in their launch arguments (0 in normal use).
std::atomic<uint32_t> g_stall_mask{0};
uint32_t stall_mask() { return g_stall_mask.load(std::memory_order_relaxed); }

ActWs act_ws(void* ws, size_t colmax_off, size_t bitmask_off, int64_t K) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  ActWs a;
  a.status = reinterpret_cast<uint32_t*>(b);
  a.colmax = reinterpret_cast<uint32_t*>(b + colmax_off);
  a.blk_counter = reinterpret_cast<uint32_t*>(b + align_up(colmax_off + 4 * size_t(K), 256));
  a.bitmask = reinterpret_cast<uint32_t*>(b + bitmask_off);
  a.fused = reinterpret_cast<uint32_t*>(b + align_up(bitmask_off + 4 * size_t((K + 31) / 32), 256));
  a.stall = stall_mask();
  return a;
}

llmint8_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA; }


bool valid_tau(float tau) { return !std::isnan(tau) && tau >= 0.0f; }

// Whether llmint8_mixed_matmul runs the matrix-vector decode kernel (M <= 8).
// Rows of X the matrix-vector kernel takes.  It needs K a multiple of 512 up
// to 4096 and at most 64 Wq rows per SM; other decode calls take the cluster
// kernel, which costs about the same at any row count up to 32.
constexpr int64_t kGemvMaxM = 8;

bool use_gemv_decode(int64_t M, int64_t N, int64_t K, int64_t ldx, int64_t ldk, const void* X, int num_sms,
                     int* rows_per, int* tiles) {
  return M <= kGemvMaxM && ldx % 8 == 0 && aligned(X, 16) && K <= kFusedMaxK &&
         decode_gemv_plan(static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), ldk, num_sms, rows_per,
                          tiles);
}

// Whether llmint8_mixed_matmul runs the one-kernel decode path for these
// arguments (then *splits, *kb_per receive its plan).
bool use_fused_decode(int64_t M, int64_t N, int64_t K, int64_t ldx, const void* X, int num_sms, int* splits,
                      int* kb_per, int* stages) {
  return M <= kDecodeMaxM && K % 8 == 0 && ldx % 8 == 0 && aligned(X, 16) &&
         decode_fused_plan(static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), num_sms, splits, kb_per,
                           stages);
}

}  // namespace

extern "C" {

const char* llmint8_status_string(llmint8_status s) {
  switch (s) {
    case LLMINT8_OK: return "LLMINT8_OK";
    case LLMINT8_ERR_INVALID_ARG: return "LLMINT8_ERR_INVALID_ARG";
    case LLMINT8_ERR_UNSUPPORTED: return "LLMINT8_ERR_UNSUPPORTED";
    case LLMINT8_ERR_WORKSPACE: return "LLMINT8_ERR_WORKSPACE";
    case LLMINT8_ERR_CUDA: return "LLMINT8_ERR_CUDA";
    case LLMINT8_ERR_OUTLIER_OVERFLOW: return "LLMINT8_ERR_OUTLIER_OVERFLOW";
    case LLMINT8_ERR_TIMEOUT: return "LLMINT8_ERR_TIMEOUT";
  }
  return "LLMINT8_UNKNOWN_STATUS";
}

llmint8_status llmint8_workspace_layout(int64_t M, int64_t N, int64_t K, int64_t outlier_cap,
                                        llmint8_ws_layout* out) {
  if (!out || N < 1) return LLMINT8_ERR_INVALID_ARG;
  size_t c, b, d;
  if (!make_layout(M, K, outlier_cap, out, &c, &b, N, &d)) return LLMINT8_ERR_INVALID_ARG;
  return LLMINT8_OK;
}

llmint8_status llmint8_outlier_stats(const void* X, int64_t M, int64_t K, int64_t ldx, float tau, int64_t* stats,
                                     void* ws, size_t ws_bytes, void* stream) {
  const Range range("llmint8_outlier_stats");
  if (!X || !stats) return LLMINT8_ERR_INVALID_ARG;
  if (M < 1 || K < 1 || K > kMaxK || M > (int64_t(1) << 31) - 1 || ldx < K || !valid_tau(tau))
    return LLMINT8_ERR_INVALID_ARG;
  if (!aligned(X, 2) || !aligned(stats, 8)) return LLMINT8_ERR_INVALID_ARG;
  llmint8_ws_layout L;
  size_t colmax, bitmask;
  if (!make_layout(1, K, 1, &L, &colmax, &bitmask)) return LLMINT8_ERR_INVALID_ARG;
  const size_t scratch_off = align_up(bitmask + 4 * size_t((K + 31) / 32), 256) + act_fused_bytes(K);
  if (!ws || !aligned(ws, 256) || ws_bytes < scratch_off + stats_scratch_bytes(K)) return LLMINT8_ERR_WORKSPACE;
  int num_sms = 0;
  llmint8_status st = current_device(&num_sms);
  if (st != LLMINT8_OK) return st;
  uint32_t* scratch = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + scratch_off);
  return cuda_status(launch_outlier_stats(X, M, K, ldx, tau, scratch, stats, num_sms, static_cast<cudaStream_t>(stream)));
}

int llmint8_mixed_matmul_kernels(int64_t M, int64_t N, int64_t K, int64_t ldx, const void* X) {
  if (!X || M < 1 || N < 1 || K < 1 || K > kMaxK || ldx < K || M > (int64_t(1) << 31) - 1 ||
      N > (int64_t(1) << 31) - 1)
    return 0;
  int num_sms = 0, s = 0, kb = 0, stages = 0;
  if (current_device(&num_sms) != LLMINT8_OK) return 0;
  if (use_gemv_decode(M, N, K, ldx, round_up(K, 16), X, num_sms, &s, &kb)) return 1;
  if (use_fused_decode(M, N, K, ldx, X, num_sms, &s, &kb, &stages)) return 1;
  return act_fused_plan(M, K, ldx, X, num_sms) ? 2 : 3;  // activation step in one or two kernels, then the GEMM
}

const char* llmint8_mixed_matmul_path(int64_t M, int64_t N, int64_t K, int64_t ldx, int64_t ldk, const void* X) {
  if (!X || M < 1 || N < 1 || K < 1 || K > kMaxK || ldx < K || ldk < K || ldk % 16 != 0 ||
      M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1)
    return nullptr;
  int num_sms = 0, s = 0, kb = 0, stages = 0;
  if (current_device(&num_sms) != LLMINT8_OK) return nullptr;
  if (use_gemv_decode(M, N, K, ldx, ldk, X, num_sms, &s, &kb)) return "decode_gemv_kernel";
  if (use_fused_decode(M, N, K, ldx, X, num_sms, &s, &kb, &stages)) return "decode_fused_kernel";
  const bool decode = M <= kDecodeMaxM;
  if (act_fused_plan(M, K, ldx, X, num_sms))
    return decode ? "act_fused_kernel,gemm_i8_decode_kernel" : "act_fused_kernel,gemm_i8_kernel";
  if (act_stream_plan(M, K, ldx, X, num_sms))
    return decode ? "scan_stream_kernel,quantize_stream_kernel,gemm_i8_decode_kernel"
                  : "scan_stream_kernel,quantize_stream_kernel,gemm_i8_kernel";
  // the row kernel takes rows of up to 2048 chunks of 8 columns; longer rows the long-row kernel
  if ((K + 7) / 8 > 2048)
    return decode ? "scan_columns_kernel,quantize_rows_long_kernel,gemm_i8_decode_kernel"
                  : "scan_columns_kernel,quantize_rows_long_kernel,gemm_i8_kernel";
  return decode ? "scan_columns_kernel,quantize_rows_kernel,gemm_i8_decode_kernel"
                : "scan_columns_kernel,quantize_rows_kernel,gemm_i8_kernel";
}

size_t llmint8_workspace_size(int64_t M, int64_t N, int64_t K, int64_t outlier_cap) {
  llmint8_ws_layout L;
  if (llmint8_workspace_layout(M, N, K, outlier_cap, &L) != LLMINT8_OK) return 0;
  return L.total;
}

llmint8_status llmint8_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256 || !aligned(ws, 256)) return LLMINT8_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

llmint8_status llmint8_quantize_weight_colwise(const void* W, int64_t K, int64_t N, int64_t ldw, int8_t* Wq,
                                               int64_t ldk, float* col_scale, void* stream) {
  const Range range("llmint8_quantize_weight_colwise");
  if (!W || !Wq || !col_scale) return LLMINT8_ERR_INVALID_ARG;
  if (K < 1 || N < 1 || K > kMaxK || N > (int64_t(1) << 31) - 1 || ldw < N) return LLMINT8_ERR_INVALID_ARG;
  if (ldk < K || ldk % 16 != 0 || !aligned(Wq, 16) || !aligned(W, 2) || !aligned(col_scale, 4))
    return LLMINT8_ERR_INVALID_ARG;
  llmint8_status st = current_device(nullptr);
  if (st != LLMINT8_OK) return st;
  return cuda_status(
      launch_quantize_weight_colwise(W, K, N, ldw, Wq, ldk, col_scale, static_cast<cudaStream_t>(stream)));
}

llmint8_status llmint8_quantize_act_rowwise_outliers(const void* X, int64_t M, int64_t K, int64_t ldx,
                                                     float tau, int8_t* Xq, int64_t ldq, float* row_scale,
                                                     int32_t* outlier_idx, int64_t outlier_cap,
                                                     int32_t* n_outlier, void* Xo, int64_t ldo, void* ws,
                                                     size_t ws_bytes, void* stream) {
  const Range range("llmint8_quantize_act_rowwise_outliers");
  if (!X || !Xq || !row_scale || !outlier_idx || !n_outlier) return LLMINT8_ERR_INVALID_ARG;
  if (M < 1 || K < 1 || K > kMaxK || M > (int64_t(1) << 31) - 1 || ldx < K || !valid_tau(tau))
    return LLMINT8_ERR_INVALID_ARG;
  if (outlier_cap < 1 || outlier_cap > K) return LLMINT8_ERR_INVALID_ARG;
  if (ldq < K || ldq % 16 != 0 || !aligned(Xq, 16) || !aligned(X, 2)) return LLMINT8_ERR_INVALID_ARG;
  if (Xo && (ldo < outlier_cap || !aligned(Xo, 2))) return LLMINT8_ERR_INVALID_ARG;
  llmint8_ws_layout L;
  size_t colmax, bitmask;
  if (!make_layout(M, K, outlier_cap, &L, &colmax, &bitmask)) return LLMINT8_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return LLMINT8_ERR_WORKSPACE;
  int num_sms = 0;
  llmint8_status st = current_device(&num_sms);
  if (st != LLMINT8_OK) return st;
  return cuda_status(launch_quantize_act(X, M, K, ldx, tau, Xq, ldq, row_scale, outlier_idx, outlier_cap,
                                         n_outlier, Xo, ldo, act_ws(ws, colmax, bitmask, K),
                                         static_cast<cudaStream_t>(stream), true, num_sms));
}

}  // extern "C"

namespace {

// llmint8_mixed_matmul, and its test hook: with C non-null every path stores
// the raw int32 accumulator [M, ldc] in place of Y (Y, W and bias unused),
// through the same kernels and launch plan.
llmint8_status mixed_matmul_impl(const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* Wq, int64_t ldk,
                                 const float* col_scale, const void* W, int64_t ldw, const void* bias, int64_t N,
                                 float tau, int64_t outlier_cap, void* Y, int64_t ldy, void* ws, size_t ws_bytes,
                                 void* stream, int32_t* C, int64_t ldc) {
  if (!X || !Wq || !col_scale || !Y) return LLMINT8_ERR_INVALID_ARG;  // W may be NULL: int8-only weight
  if (M < 1 || N < 1 || K < 1 || K > kMaxK || M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1)
    return LLMINT8_ERR_INVALID_ARG;
  if (ldx < K || (W && ldw < N) || ldy < N || ldk < K || ldk % 16 != 0 || !valid_tau(tau))
    return LLMINT8_ERR_INVALID_ARG;
  if (C && (ldc < N || !aligned(C, 4))) return LLMINT8_ERR_INVALID_ARG;
  if (outlier_cap < 1 || outlier_cap > K) return LLMINT8_ERR_INVALID_ARG;
  if (!aligned(Wq, 16) || !aligned(X, 2) || (W && !aligned(W, 2)) || !aligned(Y, 2) || !aligned(col_scale, 4) ||
      !aligned(bias, 2))
    return LLMINT8_ERR_INVALID_ARG;
  llmint8_ws_layout L;
  size_t colmax_off, bitmask_off, decode_off, om_off = 0;
  if (!make_layout(M, K, outlier_cap, &L, &colmax_off, &bitmask_off, N, &decode_off, &om_off))
    return LLMINT8_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return LLMINT8_ERR_WORKSPACE;
  int num_sms = 0;
  llmint8_status st = current_device(&num_sms);
  if (st != LLMINT8_OK) return st;

  uint8_t* b = static_cast<uint8_t*>(ws);
  int8_t* xq = reinterpret_cast<int8_t*>(b + L.xq);
  float* rs = reinterpret_cast<float*>(b + L.row_scale);
  int32_t* O = reinterpret_cast<int32_t*>(b + L.outlier_idx);
  int32_t* n_o = reinterpret_cast<int32_t*>(b + L.n_outlier);
  void* xo = b + L.xo;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool decode = M <= kDecodeMaxM;

  // Up to 8 rows of X with 16-byte aligned rows, K a multiple of 512 up to 4096:
  // one kernel, each CTA owning whole rows of Wq (no split of K).
  int g_rows = 0, g_tiles = 0;
  if (use_gemv_decode(M, N, K, ldx, ldk, X, num_sms, &g_rows, &g_tiles)) {
    GemvArgs g = {};
    g.X = X;
    g.ldx = ldx;
    g.M = static_cast<int>(M);
    g.N = static_cast<int>(N);
    g.K = K;
    g.tau = tau;
    g.cs = col_scale;
    g.W = W;
    g.ldw = ldw;
    g.Wq = Wq;
    g.ldk = ldk;
    g.bias = bias;
    g.Y = Y;
    g.ldy = ldy;
    g.Xq = xq;
    g.ldq = L.ldq;
    g.rs = rs;
    g.O = O;
    g.n_out = n_o;
    g.Xo = xo;
    g.ldo = L.ldo;
    g.cap = static_cast<int>(outlier_cap);
    g.status = reinterpret_cast<uint32_t*>(b + L.status);
    g.rows_per = g_rows;
    g.tiles = g_tiles;
    g.C = C;
    g.ldc = ldc;
    g.stall = stall_mask();
    return cuda_status(launch_decode_gemv(g, s, true));
  }

  // Decode calls whose X rows allow 16-byte loads: the whole path in one kernel.
  int f_splits = 0, f_kb = 0, f_stages = 0;
  if (use_fused_decode(M, N, K, ldx, X, num_sms, &f_splits, &f_kb, &f_stages)) {
    CUtensorMap tmW;
    if (!encode_operand_map(&tmW, Wq, N, K, ldk, 128)) return LLMINT8_ERR_CUDA;
    FusedArgs f = {};
    f.X = X;
    f.ldx = ldx;
    f.M = static_cast<int>(M);
    f.N = static_cast<int>(N);
    f.K = static_cast<int>(K);
    f.tau = tau;
    f.cs = col_scale;
    f.W = W;
    f.ldw = ldw;
    f.Wq = Wq;
    f.ldk = ldk;
    f.bias = bias;
    f.Y = Y;
    f.ldy = ldy;
    f.Xq = xq;
    f.ldq = L.ldq;
    f.rs = rs;
    f.O = O;
    f.n_out = n_o;
    f.Xo = xo;
    f.ldo = L.ldo;
    f.cap = static_cast<int>(outlier_cap);
    f.status = reinterpret_cast<uint32_t*>(b + L.status);
    f.splits = f_splits;
    f.kb_per = f_kb;
    f.stages = f_stages;
    f.C = C;
    f.ldc = ldc;
    return cuda_status(launch_decode_fused(tmW, f, s, true));
  }

  CUtensorMap tmA, tmB;
  if (decode) {
    if (!encode_decode_maps(&tmA, &tmB, Wq, N, ldk, xq, M, L.ldq, K)) return LLMINT8_ERR_CUDA;
  } else if (!encode_operand_map(&tmA, xq, M, K, L.ldq, kGemmBM) ||
             !encode_operand_map(&tmB, Wq, N, K, ldk, gemm_b_box_rows(static_cast<int>(M)))) {
    return LLMINT8_ERR_CUDA;
  }

  cudaError_t e = launch_quantize_act(X, M, K, ldx, tau, xq, L.ldq, rs, O, outlier_cap, n_o, xo, L.ldo,
                                      act_ws(ws, colmax_off, bitmask_off, K), s, true, num_sms);
  if (e != cudaSuccess) return LLMINT8_ERR_CUDA;

  if (decode) {
    DecodeArgs d = {};
    d.M = static_cast<int>(M);
    d.N = static_cast<int>(N);
    d.K = static_cast<int>(K);
    decode_split(d.M, d.N, d.K, num_sms, true, &d.splits, &d.kb_per_split);
    d.rs = rs;
    d.cs = col_scale;
    d.Xo = xo;
    d.ldo = L.ldo;
    d.O = O;
    d.n_o = n_o;
    d.cap = static_cast<int>(outlier_cap);
    d.W = W;
    d.ldw = ldw;
    d.Wq = Wq;
    d.ldk = ldk;
    d.bias = bias;
    d.Y = Y;
    d.ldy = ldy;
    d.partial = reinterpret_cast<int32_t*>(b + decode_off);
    d.tile_counter = reinterpret_cast<uint32_t*>(
        b + decode_off + align_up(size_t(N) * size_t(decode_rows_padded(d.M)) * 4, 256));
    d.status = reinterpret_cast<uint32_t*>(b + L.status);
    d.C = C;
    d.ldc = ldc;
    return cuda_status(launch_gemm_i8_decode(tmA, tmB, d, C != nullptr, s, true));
  }

  GemmArgs a = {};
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.rs = rs;
  a.cs = col_scale;
  a.Xo = xo;
  a.ldo = L.ldo;
  a.O = O;
  a.n_o = n_o;
  a.cap = static_cast<int>(outlier_cap);
  a.W = W;
  a.ldw = ldw;
  a.Wq = Wq;
  a.ldk = ldk;
  a.bias = bias;
  a.Y = Y;
  a.ldy = ldy;
  a.C = C;
  a.ldc = ldc;
  a.status = reinterpret_cast<uint32_t*>(b + L.status);
  a.stall = stall_mask();
  CUtensorMap tmY, tmXo, tmWo;
  if (C) {
    std::memset(&tmY, 0, sizeof(tmY));
    a.y_tma = false;
  } else {
    a.y_tma = prepare_output(&tmY, Y, M, N, ldy);
  }
  prepare_outlier_mma(a, &tmXo, &tmWo, ws, om_off ? b + om_off : nullptr);
  return cuda_status(launch_gemm_i8(tmA, tmB, tmY, tmXo, tmWo, a, C != nullptr, num_sms, s, true));
}

}  // namespace

extern "C" {

llmint8_status llmint8_mixed_matmul(const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* Wq,
                                    int64_t ldk, const float* col_scale, const void* W, int64_t ldw,
                                    const void* bias, int64_t N, float tau, int64_t outlier_cap, void* Y,
                                    int64_t ldy, void* ws, size_t ws_bytes, void* stream) {
  const Range range("llmint8_mixed_matmul");
  return mixed_matmul_impl(X, M, K, ldx, Wq, ldk, col_scale, W, ldw, bias, N, tau, outlier_cap, Y, ldy, ws, ws_bytes,
                           stream, nullptr, 0);
}

llmint8_status llmint8_debug_mixed_matmul_i32(const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* Wq,
                                              int64_t ldk, const float* col_scale, int64_t N, float tau,
                                              int64_t outlier_cap, int32_t* C, int64_t ldc, void* ws,
                                              size_t ws_bytes, void* stream) {
  const Range range("llmint8_debug_mixed_matmul_i32");
  if (!C) return LLMINT8_ERR_INVALID_ARG;
  // Y is not written on this path; C stands in for the pointer check only
  return mixed_matmul_impl(X, M, K, ldx, Wq, ldk, col_scale, nullptr, 0, nullptr, N, tau, outlier_cap, C, ldc, ws,
                           ws_bytes, stream, C, ldc);
}

llmint8_status llmint8_debug_set_waits(uint64_t limit_ns, uint32_t stall_mask) {
  if (limit_ns == 0) return LLMINT8_ERR_INVALID_ARG;
  if (current_device(nullptr) != LLMINT8_OK) return LLMINT8_ERR_CUDA;
  cudaError_t (*const setters[])(uint64_t) = {set_debug_waits_decode_fused, set_debug_waits_decode_gemv,
                                             set_debug_waits_gemm_i8, set_debug_waits_gemm_i8_decode,
                                             set_debug_waits_quant_act};
  for (auto fn : setters)
    if (fn(limit_ns) != cudaSuccess) return LLMINT8_ERR_CUDA;
  g_stall_mask.store(stall_mask, std::memory_order_relaxed);
  return LLMINT8_OK;
}

llmint8_status llmint8_mixed_gemm(const int8_t* Xq, int64_t ldq, const float* row_scale,
                                  const int32_t* outlier_idx, const int32_t* n_outlier, int64_t outlier_cap,
                                  const void* Xo, int64_t ldo, const int8_t* Wq, int64_t ldk,
                                  const float* col_scale, const void* W, int64_t ldw, const void* bias,
                                  int64_t M, int64_t N, int64_t K, void* Y, int64_t ldy, void* ws,
                                  size_t ws_bytes, void* stream) {
  const Range range("llmint8_mixed_gemm");
  if (!Xq || !row_scale || !outlier_idx || !n_outlier || !Xo || !Wq || !col_scale || !Y)
    return LLMINT8_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || K > kMaxK || M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1)
    return LLMINT8_ERR_INVALID_ARG;
  if (outlier_cap < 1 || outlier_cap > K || ldo < outlier_cap) return LLMINT8_ERR_INVALID_ARG;
  if (ldq < K || ldk < K || ldq % 16 != 0 || ldk % 16 != 0 || (W && ldw < N) || ldy < N)
    return LLMINT8_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Xo, 2) || (W && !aligned(W, 2)) || !aligned(Y, 2) ||
      !aligned(bias, 2) ||
      !aligned(row_scale, 4) || !aligned(col_scale, 4))
    return LLMINT8_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < 256) return LLMINT8_ERR_WORKSPACE;
  int num_sms = 0;
  llmint8_status st = current_device(&num_sms);
  if (st != LLMINT8_OK) return st;
  CUtensorMap tmA, tmB;
  if (M <= kDecodeMaxM) {
    if (!encode_decode_maps(&tmA, &tmB, Wq, N, ldk, Xq, M, ldq, K)) return LLMINT8_ERR_CUDA;
    DecodeArgs d = {};
    d.M = static_cast<int>(M);
    d.N = static_cast<int>(N);
    d.K = static_cast<int>(K);
    // split-K needs its scratch after the status block of the workspace
    const bool can_split = ws_bytes >= 256 + decode_scratch_bytes(d.M, d.N);
    decode_split(d.M, d.N, d.K, num_sms, can_split, &d.splits, &d.kb_per_split);
    d.rs = row_scale;
    d.cs = col_scale;
    d.Xo = Xo;
    d.ldo = ldo;
    d.O = outlier_idx;
    d.n_o = n_outlier;
    d.cap = static_cast<int>(outlier_cap);
    d.W = W;
    d.ldw = ldw;
    d.Wq = Wq;
    d.ldk = ldk;
    d.bias = bias;
    d.Y = Y;
    d.ldy = ldy;
    // the split-K scratch is the last decode_scratch_bytes of the workspace
    // (the decode region of a workspace sized by llmint8_workspace_size)
    uint8_t* b = static_cast<uint8_t*>(ws) + (can_split ? (ws_bytes - decode_scratch_bytes(d.M, d.N)) / 256 * 256 : 256);
    d.partial = reinterpret_cast<int32_t*>(b);
    d.tile_counter = reinterpret_cast<uint32_t*>(b + align_up(size_t(N) * size_t(decode_rows_padded(d.M)) * 4, 256));
    d.status = static_cast<uint32_t*>(ws);
    return cuda_status(launch_gemm_i8_decode(tmA, tmB, d, false, static_cast<cudaStream_t>(stream), true));
  }
  if (!encode_operand_map(&tmA, Xq, M, K, ldq, kGemmBM) || !encode_operand_map(&tmB, Wq, N, K, ldk, gemm_b_box_rows(static_cast<int>(M))))
    return LLMINT8_ERR_CUDA;
  GemmArgs a = {};
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.rs = row_scale;
  a.cs = col_scale;
  a.Xo = Xo;
  a.ldo = ldo;
  a.O = outlier_idx;
  a.n_o = n_outlier;
  a.cap = static_cast<int>(outlier_cap);
  a.W = W;
  a.ldw = ldw;
  a.Wq = Wq;
  a.ldk = ldk;
  a.bias = bias;
  a.Y = Y;
  a.ldy = ldy;
  a.status = static_cast<uint32_t*>(ws);
  a.stall = stall_mask();
  CUtensorMap tmY, tmXo, tmWo;
  a.y_tma = prepare_output(&tmY, Y, M, N, ldy);
  // The outlier operands where llmint8_mixed_matmul keeps them, when the
  // workspace is that large: past the activation step's scratch and its Xq
  // and Xo, so the same workspace serves both entry points.
  llmint8_ws_layout Lw;
  size_t colmax_off, bitmask_off, om_off = 0;
  const bool om_room = make_layout(M, K, outlier_cap, &Lw, &colmax_off, &bitmask_off, N, nullptr, &om_off) &&
                       om_off != 0 && ws_bytes >= Lw.total;
  prepare_outlier_mma(a, &tmXo, &tmWo, ws, om_room ? static_cast<uint8_t*>(ws) + om_off : nullptr);
  return cuda_status(
      launch_gemm_i8(tmA, tmB, tmY, tmXo, tmWo, a, false, num_sms, static_cast<cudaStream_t>(stream), true));
}

llmint8_status llmint8_debug_int8_gemm_i32(const int8_t* Xq, int64_t ldq, const int8_t* Wq, int64_t ldk,
                                           int64_t M, int64_t N, int64_t K, int32_t* C, int64_t ldc, void* ws,
                                           size_t ws_bytes, void* stream) {
  const Range range("llmint8_debug_int8_gemm_i32");
  if (!Xq || !Wq || !C) return LLMINT8_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || K > kMaxK || M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1)
    return LLMINT8_ERR_INVALID_ARG;
  if (ldq < K || ldk < K || ldq % 16 != 0 || ldk % 16 != 0 || ldc < N) return LLMINT8_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(C, 4)) return LLMINT8_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < 256) return LLMINT8_ERR_WORKSPACE;
  int num_sms = 0;
  llmint8_status st = current_device(&num_sms);
  if (st != LLMINT8_OK) return st;
  CUtensorMap tmA, tmB;
  if (M <= kDecodeMaxM) {
    if (!encode_decode_maps(&tmA, &tmB, Wq, N, ldk, Xq, M, ldq, K)) return LLMINT8_ERR_CUDA;
    DecodeArgs d = {};
    d.M = static_cast<int>(M);
    d.N = static_cast<int>(N);
    d.K = static_cast<int>(K);
    const bool can_split = ws_bytes >= 256 + decode_scratch_bytes(d.M, d.N);
    decode_split(d.M, d.N, d.K, num_sms, can_split, &d.splits, &d.kb_per_split);
    d.C = C;
    d.ldc = ldc;
    // the split-K scratch is the last decode_scratch_bytes of the workspace
    // (the decode region of a workspace sized by llmint8_workspace_size)
    uint8_t* b = static_cast<uint8_t*>(ws) + (can_split ? (ws_bytes - decode_scratch_bytes(d.M, d.N)) / 256 * 256 : 256);
    d.partial = reinterpret_cast<int32_t*>(b);
    d.tile_counter = reinterpret_cast<uint32_t*>(b + align_up(size_t(N) * size_t(decode_rows_padded(d.M)) * 4, 256));
    d.status = static_cast<uint32_t*>(ws);
    return cuda_status(launch_gemm_i8_decode(tmA, tmB, d, true, static_cast<cudaStream_t>(stream), false));
  }
  if (!encode_operand_map(&tmA, Xq, M, K, ldq, kGemmBM) || !encode_operand_map(&tmB, Wq, N, K, ldk, gemm_b_box_rows(static_cast<int>(M))))
    return LLMINT8_ERR_CUDA;
  GemmArgs a = {};
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.C = C;
  a.ldc = ldc;
  a.status = static_cast<uint32_t*>(ws);
  CUtensorMap tmY, tmXo, tmWo;
  std::memset(&tmY, 0, sizeof(tmY));
  a.y_tma = false;
  prepare_outlier_mma(a, &tmXo, &tmWo, ws, nullptr);  // no outlier product in the raw accumulator dump
  return cuda_status(
      launch_gemm_i8(tmA, tmB, tmY, tmXo, tmWo, a, true, num_sms, static_cast<cudaStream_t>(stream), false));
}

llmint8_status llmint8_unshard_columns(const void* blocks, int64_t world, int64_t M, int64_t ld_block,
                                      const int64_t* bounds, void* Y, int64_t ldy, void* stream) {
  const Range range("llmint8_unshard_columns");
  if (!blocks || !bounds || !Y) return LLMINT8_ERR_INVALID_ARG;
  if (world < 1 || world > kUnshardMaxWorld || M < 1 || ld_block < 1) return LLMINT8_ERR_INVALID_ARG;
  if (!aligned(blocks, 2) || !aligned(Y, 2)) return LLMINT8_ERR_INVALID_ARG;
  UnshardBounds b;
  if (bounds[0] != 0) return LLMINT8_ERR_INVALID_ARG;
  for (int64_t r = 0; r <= world; ++r) {
    b.bounds[r] = bounds[r];
    if (r > 0 && (bounds[r] < bounds[r - 1] || bounds[r] - bounds[r - 1] > ld_block)) return LLMINT8_ERR_INVALID_ARG;
  }
  if (bounds[world] < 1 || ldy < bounds[world]) return LLMINT8_ERR_INVALID_ARG;
  int num_sms = 0;
  llmint8_status st = current_device(&num_sms);
  if (st != LLMINT8_OK) return st;
  return cuda_status(launch_unshard_columns(blocks, static_cast<int>(world), M, ld_block, b, Y, ldy, num_sms,
                                            static_cast<cudaStream_t>(stream)));
}

llmint8_status llmint8_check_status(void* ws, void* stream, uint32_t* flags_out) {
  if (!ws || !aligned(ws, 256)) return LLMINT8_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return LLMINT8_ERR_CUDA;
  uint32_t flags = 0;
  if (cudaMemcpy(&flags, ws, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess) return LLMINT8_ERR_CUDA;
  if (flags != 0 && cudaMemset(ws, 0, sizeof(flags)) != cudaSuccess) return LLMINT8_ERR_CUDA;
  if (flags_out) *flags_out = flags;
  if (flags & LLMINT8_STATUS_TIMEOUT) return LLMINT8_ERR_TIMEOUT;
  if (flags & LLMINT8_STATUS_OUTLIER_OVERFLOW) return LLMINT8_ERR_OUTLIER_OVERFLOW;
  return LLMINT8_OK;
}

}  // extern "C"
