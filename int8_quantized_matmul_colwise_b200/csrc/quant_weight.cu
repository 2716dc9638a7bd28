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
constexpr int kKBlock = 128;     // rows of W per transpose block
constexpr int kTStride = 144;    // bytes per transposed row in shared memory

// Load 8 consecutive fp16 of row k starting at column c (zero outside N).
__device__ __forceinline__ void load8(const __half* __restrict__ W, int64_t ldw, int64_t N, int64_t k, int64_t c,
                                      bool vec_ok, float (&x)[8]) {
  const __half* p = W + k * ldw + c;
  if (vec_ok && c + 8 <= N) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h[e]);
      x[2 * e] = f.x;
      x[2 * e + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = (c + e < N) ? __half2float(p[e]) : 0.0f;
  }
}

// One CTA owns a strip of 64 columns over all K rows: first the exact column
// absmax, then quantization of 128-row blocks transposed through shared memory
// so that each column of W becomes one K-contiguous row of Wq.
__global__ void __launch_bounds__(256) quantize_weight_colwise_kernel(const __half* __restrict__ W, int64_t K,
                                                                      int64_t N, int64_t ldw, bool vec_ok,
                                                                      int8_t* __restrict__ Wq, int64_t ldk,
                                                                      float* __restrict__ col_scale) {
  __shared__ float s_red[32][kStripCols + 1];
  __shared__ float s_scale[kStripCols];
  __shared__ float s_inv[kStripCols];
  __shared__ __align__(16) int8_t s_t[kStripCols][kTStride];

  const int64_t c0 = int64_t(blockIdx.x) * kStripCols;
  const int tx = threadIdx.x & 7;   // column group: 8 columns
  const int ty = threadIdx.x >> 3;  // row phase 0..31
  const int64_t cg = c0 + 8 * tx;

  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = 0.0f;
  for (int64_t k = ty; k < K; k += 32) {
    float x[8];
    load8(W, ldw, N, k, cg, vec_ok, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(x[e]));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) s_red[ty][8 * tx + e] = m[e];
  __syncthreads();
  if (threadIdx.x < kStripCols) {
    float s = 0.0f;
    for (int r = 0; r < 32; ++r) s = fmaxf(s, s_red[r][threadIdx.x]);
    s_scale[threadIdx.x] = s;
    s_inv[threadIdx.x] = s > 0.0f ? __frcp_rn(s) : 0.0f;
    if (c0 + threadIdx.x < N) col_scale[c0 + threadIdx.x] = s;
  }
  __syncthreads();

  // Transposed write-out: thread -> (column wc, 32-byte segment ws).
  const int wc = threadIdx.x >> 2;
  const int wseg = threadIdx.x & 3;
  for (int64_t k0 = 0; k0 < ldk; k0 += kKBlock) {
#pragma unroll
    for (int r = 0; r < kKBlock / 32; ++r) {
      const int kr = ty + 32 * r;
      const int64_t k = k0 + kr;
      float x[8];
      if (k < K) {
        load8(W, ldw, N, k, cg, vec_ok, x);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.0f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int c = 8 * tx + e;
        const float s = s_scale[c];
        s_t[c][kr] = static_cast<int8_t>(s > 0.0f ? quantize_exact(x[e], s, s_inv[c]) : 0);
      }
    }
    __syncthreads();
    const int64_t col = c0 + wc;
    if (col < N) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t kk = k0 + 32 * wseg + 16 * h;
        if (kk < ldk) {  // ldk % 16 == 0, so a 16-byte piece is either in or out
          *reinterpret_cast<uint4*>(Wq + col * ldk + kk) =
              *reinterpret_cast<const uint4*>(&s_t[wc][32 * wseg + 16 * h]);
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_quantize_weight_colwise(const void* W, int64_t K, int64_t N, int64_t ldw, int8_t* Wq,
                                           int64_t ldk, float* col_scale, cudaStream_t stream) {
  const bool vec_ok = (ldw % 8 == 0) && (reinterpret_cast<uintptr_t>(W) % 16 == 0);
  const unsigned grid = static_cast<unsigned>((N + kStripCols - 1) / kStripCols);
  quantize_weight_colwise_kernel<<<grid, 256, 0, stream>>>(static_cast<const __half*>(W), K, N, ldw, vec_ok, Wq,
                                                           ldk, col_scale);
  return cudaGetLastError();
}

}  // namespace llmint8
