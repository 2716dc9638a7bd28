// quant_act.cu -- steps a1-a4 on the activation X [M, K] (fp16):
//   a1  outlier feature dimensions: columns with some |x| >= tau;
//   a2  row absmax over the remaining columns;
//   a3  row-wise int8 quantization, outlier columns zero;
//   a4  gather of the outlier columns of X (fp16).
// "Compress your LLMs", bullets Vector-wise quantization (one constant per row
// of the input) and Mixed-precision decomposition (outlier dimensions in
// 16-bit); arXiv abstract of "LLM.int8(): 8-bit Matrix Multiplication for
// Transformers at Scale" (the outlier feature dimensions are isolated).
//
// The outlier set depends on every row, so the work is two kernels:
//  scan:     column maxima of |X| (atomicMax on fp16 bit patterns, which order
//            like the values for non-negative halves); the last CTA to finish
//            turns them into the ascending outlier list and a column bitmask
//            and returns the maxima to zero for the next call;
//  quantize: per row, absmax over non-outlier columns, exact codes, gather.
// Both are HBM-bound streaming kernels: 16-byte loads, warp-shuffle
// reductions, ballot-free prefix sums over 32-column bitmask words.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace llmint8 {

namespace {

constexpr int kScanCols = 256;  // columns per scan CTA (32 lanes x 8)
constexpr int kScanRows = 64;   // rows per scan CTA

__device__ __forceinline__ void load8_bits(const __half* __restrict__ row, int64_t K, int64_t c, bool vec_ok,
                                           __half (&h)[8]) {
  if (vec_ok && c + 8 <= K) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + c));
    const __half* p = reinterpret_cast<const __half*>(&u);
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = p[e];
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = (c + e < K) ? row[c + e] : __ushort_as_half(0);
  }
}

// Block-wide exclusive prefix sum of one int per thread (256 threads).
__device__ __forceinline__ int block_exclusive_scan_256(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int c = s_warp[w];
    base += (w < warp) ? c : 0;
    tot += c;
  }
  __syncthreads();
  total = tot;
  return base + inc - v;
}

__global__ void __launch_bounds__(256) scan_columns_kernel(const __half* __restrict__ X, int64_t M, int64_t K,
                                                           int64_t ldx, bool vec_ok, float tau, ActWs ws,
                                                           int32_t* __restrict__ O, int64_t cap,
                                                           int32_t* __restrict__ n_out) {
  __shared__ uint32_t s_max[8][kScanCols];
  __shared__ int s_warp[8];
  __shared__ int s_last;

  griddep_wait();               // X may come from the previous kernel on the stream
  griddep_launch_dependents();  // let the quantize kernel get resident early

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c = int64_t(blockIdx.x) * kScanCols + 8 * lane;
  const int64_t r0 = int64_t(blockIdx.y) * kScanRows;
  uint32_t m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = 0;
  if (c < K) {
    for (int64_t r = r0 + warp; r < M && r < r0 + kScanRows; r += 8) {
      __half h[8];
      load8_bits(X + r * ldx, K, c, vec_ok, h);
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = max(m[e], abs_bits(h[e]));
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) s_max[warp][8 * lane + e] = m[e];
  __syncthreads();
  {
    uint32_t v = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) v = max(v, s_max[w][threadIdx.x]);
    const int64_t col = int64_t(blockIdx.x) * kScanCols + threadIdx.x;
    if (v != 0 && col < K) atomicMax(ws.colmax + col, v);
  }

  // Last CTA: column flags -> bitmask words and the ascending outlier list.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned total = gridDim.x * gridDim.y;
    s_last = (atomicAdd(ws.counter, 1u) == total - 1u) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int64_t nwords = (K + 31) / 32;
  const int64_t wpt = (nwords + 255) / 256;  // words per thread
  const int64_t w0 = int64_t(threadIdx.x) * wpt;
  int cnt = 0;
  for (int64_t w = w0; w < w0 + wpt && w < nwords; ++w) {
    uint32_t bits = 0;
    for (int b = 0; b < 32; ++b) {
      const int64_t col = w * 32 + b;
      if (col < K) {
        const uint32_t v = __ldcg(ws.colmax + col);
        if (__half2float(__ushort_as_half(static_cast<unsigned short>(v))) >= tau) bits |= 1u << b;
      }
    }
    ws.bitmask[w] = bits;
    cnt += __popc(bits);
  }
  int total = 0;
  int pos = block_exclusive_scan_256(cnt, s_warp, total);
  for (int64_t w = w0; w < w0 + wpt && w < nwords; ++w) {
    uint32_t bits = ws.bitmask[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < cap) O[pos] = static_cast<int32_t>(w * 32 + b);
      ++pos;
    }
    for (int b = 0; b < 32; ++b) {
      const int64_t col = w * 32 + b;
      if (col < K) ws.colmax[col] = 0u;  // ready for the next call
    }
  }
  if (threadIdx.x == 0) {
    *n_out = total;
    *ws.counter = 0u;
    if (total > cap) atomicOr(ws.status, kStatusOverflow);
  }
}

// kWarpsPerRow = 1: one warp per row (large M); 8: one CTA per row (small M).
template <int kWarpsPerRow>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const __half* __restrict__ X, int64_t M, int64_t K,
                                                            int64_t ldx, bool vec_ok, ActWs ws,
                                                            const int32_t* __restrict__ O,
                                                            const int32_t* __restrict__ n_ptr, int64_t cap,
                                                            int8_t* __restrict__ Xq, int64_t ldq,
                                                            float* __restrict__ rs, __half* __restrict__ Xo,
                                                            int64_t ldo) {
  extern __shared__ uint32_t s_mask[];  // K/32 words
  __shared__ float s_part[8];
  constexpr int G = 32 * kWarpsPerRow;
  constexpr int kRowsPerCta = 8 / kWarpsPerRow;

  griddep_wait();  // bitmask, O and n_o come from the scan kernel
  griddep_launch_dependents();

  const int64_t nwords = (K + 31) / 32;
  for (int64_t w = threadIdx.x; w < nwords; w += blockDim.x) s_mask[w] = ws.bitmask[w];
  __syncthreads();
  const int n_o = *n_ptr;
  const int64_t n_gather = n_o < cap ? n_o : cap;

  const int warp = threadIdx.x >> 5;
  const int gt = threadIdx.x % G;  // thread index within the row group
  const int64_t row = int64_t(blockIdx.x) * kRowsPerCta + warp / kWarpsPerRow;
  if (row >= M) return;  // uniform per row group; no CTA-wide barrier follows for kWarpsPerRow == 1
  const __half* xr = X + row * ldx;
  const int64_t nchunks = (K + 7) / 8;

  // a2: absmax over the non-outlier columns
  float m = 0.0f;
  for (int64_t ch = gt; ch < nchunks; ch += G) {
    __half h[8];
    load8_bits(xr, K, 8 * ch, vec_ok, h);
    const uint32_t mw = s_mask[(8 * ch) >> 5] >> ((8 * ch) & 31);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (!((mw >> e) & 1u)) m = fmaxf(m, fabsf(__half2float(h[e])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if constexpr (kWarpsPerRow > 1) {
    if ((threadIdx.x & 31) == 0) s_part[warp] = m;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kWarpsPerRow; ++w) m = fmaxf(m, s_part[w]);
  }
  const float s = m;
  const float inv = s > 0.0f ? __frcp_rn(s) : 0.0f;
  if (gt == 0) rs[row] = s;

  // a3: codes; columns [K, ldq) are written as zero
  int8_t* qr = Xq + row * ldq;
  const int64_t qchunks = ldq / 8;
  for (int64_t ch = gt; ch < qchunks; ch += G) {
    const int64_t c = 8 * ch;
    int q[8];
    if (c < K) {
      __half h[8];
      load8_bits(xr, K, c, vec_ok, h);
      const uint32_t mw = s_mask[c >> 5] >> (c & 31);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const bool keep = (c + e < K) && !((mw >> e) & 1u) && s > 0.0f;
        q[e] = keep ? quantize_exact(__half2float(h[e]), s, inv) : 0;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) q[e] = 0;
    }
    uint2 out;
    out.x = pack4(q[0], q[1], q[2], q[3]);
    out.y = pack4(q[4], q[5], q[6], q[7]);
    *reinterpret_cast<uint2*>(qr + c) = out;
  }

  // a4: gather X[row, O[t]] for the outlier product
  if (Xo != nullptr) {
    for (int64_t t = gt; t < n_gather; t += G) Xo[row * ldo + t] = xr[O[t]];
  }
}

}  // namespace

cudaError_t launch_quantize_act(const void* X, int64_t M, int64_t K, int64_t ldx, float tau, int8_t* Xq,
                                int64_t ldq, float* rs, int32_t* O, int64_t cap, int32_t* n_out, void* Xo,
                                int64_t ldo, ActWs ws, cudaStream_t stream, bool pdl) {
  const __half* x = static_cast<const __half*>(X);
  const bool vec_ok = (ldx % 8 == 0) && (reinterpret_cast<uintptr_t>(X) % 16 == 0);

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;

  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;

  cfg.gridDim = dim3(static_cast<unsigned>((K + kScanCols - 1) / kScanCols),
                     static_cast<unsigned>((M + kScanRows - 1) / kScanRows));
  cfg.dynamicSmemBytes = 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, scan_columns_kernel, x, M, K, ldx, vec_ok, tau, ws, O, cap, n_out);
  if (e != cudaSuccess) return e;

  cfg.dynamicSmemBytes = static_cast<size_t>((K + 31) / 32) * sizeof(uint32_t);
  __half* xo = static_cast<__half*>(Xo);
  if (M <= 512) {
    cfg.gridDim = dim3(static_cast<unsigned>(M));
    e = cudaLaunchKernelEx(&cfg, quantize_rows_kernel<8>, x, M, K, ldx, vec_ok, ws,
                           static_cast<const int32_t*>(O), static_cast<const int32_t*>(n_out), cap, Xq, ldq, rs,
                           xo, ldo);
  } else {
    cfg.gridDim = dim3(static_cast<unsigned>((M + 7) / 8));
    e = cudaLaunchKernelEx(&cfg, quantize_rows_kernel<1>, x, M, K, ldx, vec_ok, ws,
                           static_cast<const int32_t*>(O), static_cast<const int32_t*>(n_out), cap, Xq, ldq, rs,
                           xo, ldo);
  }
  return e;
}

}  // namespace llmint8
