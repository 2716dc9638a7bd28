// noalloc.cu -- llmint8_quantize_act_rowwise_outliers_noalloc: the activation
// step (outlier scan, row quantization, outlier gather) for callers that
// cannot hand the library a device workspace.
//
// Who needs it: code whose device memory is planned once, up front (an
// inference engine's static arena, a C caller without a caching allocator
// where cudaMalloc would synchronise the device, a latency-bounded loop that
// may not allocate).  Such a caller owns its inputs and outputs but has no
// scratch buffer to lend; this entry point keeps its scratch in a file-scope
// device array instead.
//
// The scratch lives in this file's module: every GPU on which the entry point
// is used holds kScratchBytes of device memory for it until the process exits.
// All calls share it and it keeps the last call's contents, so calls that
// overlap on the GPU (two streams, two host threads) race; order them.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "kernels.cuh"
#include "llmint8.h"

namespace {

// 256 KiB: status word, column maxima (4 bytes per column), per-256-column
// counters and the outlier bitmask; enough for K <= LLMINT8_NOALLOC_MAX_K.
constexpr size_t kScratchBytes = 256u * 1024u;
static_assert(kScratchBytes % 256 == 0, "scratch size");

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct ScratchLayout {
  size_t colmax, blk_counter, bitmask, total;
};

ScratchLayout scratch_layout(int64_t K) {
  ScratchLayout L;
  L.colmax = 256;  // [0, 256): status word
  L.blk_counter = align_up(L.colmax + 4 * size_t(K), 256);
  L.bitmask = align_up(L.blk_counter + 4 * size_t((K + 255) / 256), 256);
  L.total = align_up(L.bitmask + 4 * size_t((K + 31) / 32), 256);
  return L;
}

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_zeroed[kMaxDevices] = {};  // per device: the array address last zero-filled

// With the device current: the array's device address (the host-side name
// g_scratch is only a stand-in), looked up on every call, since a device
// reset or a new primary context loads the module again and may place the
// array elsewhere.  The first call that sees an address zero-fills the array,
// since the column maxima and counters must start at zero (the kernels return
// them to zero after every call).
llmint8_status scratch_for_current_device(void** out, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LLMINT8_ERR_CUDA;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return LLMINT8_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_zeroed[dev] != p) {
    if (cudaMemsetAsync(p, 0, kScratchBytes, stream) != cudaSuccess) return LLMINT8_ERR_CUDA;
    g_zeroed[dev] = p;
  }
  *out = p;
  return LLMINT8_OK;
}

bool aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

}  // namespace

extern "C" llmint8_status llmint8_quantize_act_rowwise_outliers_noalloc(
    const void* X, int64_t M, int64_t K, int64_t ldx, float tau, int8_t* Xq, int64_t ldq, float* row_scale,
    int32_t* outlier_idx, int64_t outlier_cap, int32_t* n_outlier, void* Xo, int64_t ldo, void* stream) {
  if (!X || !Xq || !row_scale || !outlier_idx || !n_outlier) return LLMINT8_ERR_INVALID_ARG;
  if (M < 1 || K < 1 || M > (int64_t(1) << 31) - 1 || ldx < K || std::isnan(tau) || tau < 0.0f)
    return LLMINT8_ERR_INVALID_ARG;
  if (outlier_cap < 1 || outlier_cap > K) return LLMINT8_ERR_INVALID_ARG;
  if (ldq < K || ldq % 16 != 0 || !aligned(Xq, 16) || !aligned(X, 2)) return LLMINT8_ERR_INVALID_ARG;
  if (Xo && (ldo < outlier_cap || !aligned(Xo, 2))) return LLMINT8_ERR_INVALID_ARG;
  if (K > LLMINT8_NOALLOC_MAX_K || scratch_layout(K).total > kScratchBytes) return LLMINT8_ERR_WORKSPACE;

  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return LLMINT8_ERR_CUDA;
  if (major != 10 || minor != 0) return LLMINT8_ERR_UNSUPPORTED;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  llmint8_status st = scratch_for_current_device(&scratch, s);
  if (st != LLMINT8_OK) return st;

  const ScratchLayout L = scratch_layout(K);
  unsigned char* b = static_cast<unsigned char*>(scratch);
  llmint8::ActWs ws;
  ws.status = reinterpret_cast<uint32_t*>(b);
  ws.colmax = reinterpret_cast<uint32_t*>(b + L.colmax);
  ws.blk_counter = reinterpret_cast<uint32_t*>(b + L.blk_counter);
  ws.bitmask = reinterpret_cast<uint32_t*>(b + L.bitmask);
  return llmint8::launch_quantize_act(X, M, K, ldx, tau, Xq, ldq, row_scale, outlier_idx, outlier_cap, n_outlier,
                                      Xo, ldo, ws, s, true) == cudaSuccess
             ? LLMINT8_OK
             : LLMINT8_ERR_CUDA;
}
