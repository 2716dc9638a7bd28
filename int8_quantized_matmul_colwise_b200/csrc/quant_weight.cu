// quant_weight.cu -- step a0: column-wise absmax int8 quantization of W,
// written transposed (K contiguous) for the tensor-core GEMM.
//
// "Compress your LLMs", Vector-wise quantization: one scaling constant per
// column of the weight matrix.  The arXiv abstract ("LLM.int8(): 8-bit Matrix
// Multiplication for Transformers at Scale") has the 16-bit checkpoint
// converted to int8 once, at load time; this kernel is that conversion.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "quant.cuh"

namespace llmint8 {

namespace {

constexpr int kStripCols = 64;   // columns of W per CTA
constexpr int kMaxRows = 256;    // rows of W per CTA in the column-maximum pass
constexpr int kKBlock = 128;     // rows of W per CTA in the quantize pass (one transposed block)
constexpr int kTStride = 144;    // bytes per transposed row in shared memory

// Load 8 consecutive fp16 of row k starting at column c (zero outside N).
__device__ __forceinline__ uint4 load8w(const __half* __restrict__ W, int64_t ldw, int64_t N, int64_t k, int64_t c,
                                        bool vec_ok) {
  const __half* p = W + k * ldw + c;
  if (vec_ok && c + 8 <= N) return __ldg(reinterpret_cast<const uint4*>(p));
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t lo = (c + 2 * e < N) ? __half_as_ushort(p[2 * e]) : 0u;
    const uint32_t hi = (c + 2 * e + 1 < N) ? __half_as_ushort(p[2 * e + 1]) : 0u;
    w[e] = lo | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Pass 1: column maxima of |W| over a block of kMaxRows rows and a strip of 64
// columns, merged into col_scale (zero-filled first) by an atomic max on the
// bit patterns (non-negative floats order like their bits; NaN never wins).
__global__ void __launch_bounds__(256) weight_colmax_kernel(const __half* __restrict__ W, int64_t K, int64_t N,
                                                            int64_t ldw, bool vec_ok, float* __restrict__ col_scale) {
  __shared__ float s_red[32][kStripCols + 1];
  const int64_t c0 = int64_t(blockIdx.x) * kStripCols;
  const int64_t k0 = int64_t(blockIdx.y) * kMaxRows;
  const int tx = threadIdx.x & 7;   // column group: 8 columns
  const int ty = threadIdx.x >> 3;  // row phase 0..31
  const int64_t cg = c0 + 8 * tx;
  __half2 m[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) m[e] = __half2half2(__ushort_as_half(0));
  uint4 u[kMaxRows / 32];  // all of the thread's loads in flight together
#pragma unroll
  for (int r = 0; r < kMaxRows / 32; ++r) {
    const int64_t k = k0 + ty + 32 * r;
    u[r] = (k < K && cg < N) ? load8w(W, ldw, N, k, cg, vec_ok) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int r = 0; r < kMaxRows / 32; ++r) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&u[r]);
#pragma unroll
    for (int e = 0; e < 4; ++e) m[e] = __hmax2(m[e], __habs2(h2[e]));  // NaN never wins
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(m[e]);
    s_red[ty][8 * tx + 2 * e] = f.x;
    s_red[ty][8 * tx + 2 * e + 1] = f.y;
  }
  __syncthreads();
  if (threadIdx.x < kStripCols && c0 + threadIdx.x < N) {
    float v = 0.0f;
    for (int r = 0; r < 32; ++r) v = fmaxf(v, s_red[r][threadIdx.x]);
    if (v > 0.0f) atomicMax(reinterpret_cast<unsigned int*>(col_scale) + c0 + threadIdx.x, __float_as_uint(v));
  }
}

// Pass 2: codes of a block of 128 rows x 64 columns, transposed through shared
// memory so that each column of W becomes one K-contiguous run of Wq (rows k
// in [K, ldk) are written as zero).  Thread (tx, rg) holds columns 8 tx .. +7
// of rows 4 rg .. 4 rg + 3, so each column's four codes are one 32-bit word;
// the 16-byte pieces of a transposed row are permuted by the writer's column
// group (piece index XOR tx), which puts a warp's 32 stores in 32 different
// banks.  Per value: r = x * fl(127 / s) rounded to the nearest integer, which
// is the exact round-half-away-from-zero result unless r lies within 2^-15 of
// a half-integer; then the exact comparisons decide (quantize_exact).
__global__ void __launch_bounds__(256) weight_quantize_kernel(const __half* __restrict__ W, int64_t K, int64_t N,
                                                              int64_t ldw, bool vec_ok,
                                                              const float* __restrict__ col_scale,
                                                              int8_t* __restrict__ Wq, int64_t ldk) {
  __shared__ float s_scale[kStripCols];
  __shared__ float s_k[kStripCols];
  __shared__ float s_inv[kStripCols];
  __shared__ __align__(16) int8_t s_t[kStripCols][kTStride];
  const int64_t c0 = int64_t(blockIdx.x) * kStripCols;
  const int64_t k0 = int64_t(blockIdx.y) * kKBlock;
  const int tx = threadIdx.x & 7;   // column group: columns 8 tx .. 8 tx + 7
  const int rg = threadIdx.x >> 3;  // row group: rows 4 rg .. 4 rg + 3 of the block
  const int64_t cg = c0 + 8 * tx;
  uint4 u[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t k = k0 + 4 * rg + j;
    u[j] = (k < K && cg < N) ? load8w(W, ldw, N, k, cg, vec_ok) : make_uint4(0u, 0u, 0u, 0u);
  }
  if (threadIdx.x < kStripCols) {
    const float sc = c0 + threadIdx.x < N ? __ldg(col_scale + c0 + threadIdx.x) : 0.0f;
    s_scale[threadIdx.x] = sc;
    s_k[threadIdx.x] = sc > 0.0f ? __fdiv_rn(127.0f, sc) : 0.0f;
    s_inv[threadIdx.x] = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
  }
  __syncthreads();
  constexpr float kSafe = 0.499969482421875f;  // 1/2 - 2^-15
  constexpr float kBias = 12582912.0f;         // 1.5 * 2^23
  // byte offset of rows 4 rg .. 4 rg + 3 inside a transposed row: piece (rg / 4) ^ tx
  const int wofs = 16 * ((rg >> 2) ^ tx) + 4 * (rg & 3);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int c = 8 * tx + e;
    const float kc = s_k[c];
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2* h2 = reinterpret_cast<const __half2*>(&u[j]);
      const float x = (e & 1) ? __high2float(h2[e >> 1]) : __low2float(h2[e >> 1]);
      const float rr = __fmul_rn(x, kc);
      const float t = __fadd_rn(rr, kBias);
      const float qf = __fadd_rn(t, -kBias);
      uint32_t q = __float_as_uint(t) & 0xFFu;  // the low byte of rint(r), two's complement
      if (!(fabsf(__fadd_rn(rr, -qf)) < kSafe))
        q = static_cast<uint32_t>(s_scale[c] > 0.0f ? quantize_exact(x, s_scale[c], s_inv[c]) : 0) & 0xFFu;
      word |= q << (8 * j);
    }
    *reinterpret_cast<uint32_t*>(&s_t[c][wofs]) = word;
  }
  __syncthreads();
  // thread -> (column wc, 32-byte segment): two 16-byte pieces, un-permuted
  const int wc = threadIdx.x >> 2;
  const int wseg = threadIdx.x & 3;
  const int wperm = (wc >> 3) & 7;  // the column group that wrote row wc
  const int64_t col = c0 + wc;
  if (col < N) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int piece = 2 * wseg + h;
      const int64_t kk = k0 + 16 * piece;
      if (kk < ldk)  // ldk % 16 == 0, so a 16-byte piece is either in or out
        *reinterpret_cast<uint4*>(Wq + col * ldk + kk) = *reinterpret_cast<const uint4*>(&s_t[wc][16 * (piece ^ wperm)]);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_weight_colwise(const void* W, int64_t K, int64_t N, int64_t ldw, int8_t* Wq,
                                           int64_t ldk, float* col_scale, cudaStream_t stream) {
  const bool vec_ok = (ldw % 8 == 0) && (reinterpret_cast<uintptr_t>(W) % 16 == 0);
  const __half* w = static_cast<const __half*>(W);
  const unsigned strips = static_cast<unsigned>((N + kStripCols - 1) / kStripCols);
  cudaError_t e = cudaMemsetAsync(col_scale, 0, size_t(N) * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  weight_colmax_kernel<<<dim3(strips, static_cast<unsigned>((K + kMaxRows - 1) / kMaxRows)), 256, 0, stream>>>(
      w, K, N, ldw, vec_ok, col_scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  weight_quantize_kernel<<<dim3(strips, static_cast<unsigned>((ldk + kKBlock - 1) / kKBlock)), 256, 0, stream>>>(
      w, K, N, ldw, vec_ok, col_scale, Wq, ldk);
  return cudaGetLastError();
}

}  // namespace llmint8
