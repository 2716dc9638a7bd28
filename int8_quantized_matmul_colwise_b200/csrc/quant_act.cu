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
//            turns them into a column bitmask (one warp ballot per 32 columns)
//            and the ascending outlier list, and returns the maxima to zero
//            for the next call;
//  quantize: per row, absmax over non-outlier columns, exact codes, gather.
//            A row is held in registers by a group of G threads (CPT 16-byte
//            chunks each), so X is read once and all loads are in flight
//            together.
// Both are HBM-bound streaming kernels.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace llmint8 {

namespace {

constexpr int kScanCols = 256;  // columns per scan CTA (32 lanes x 8)
constexpr int kScanRows = 64;   // rows per scan CTA (8 warps x 8 rows)

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

// 8 consecutive fp16 of a row as one 16-byte register quad (zero past K).
__device__ __forceinline__ uint4 load8_packed(const __half* __restrict__ row, int64_t K, int64_t c, bool vec_ok) {
  if (vec_ok && c + 8 <= K) return __ldg(reinterpret_cast<const uint4*>(row + c));
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t lo = (c + 2 * e < K) ? __half_as_ushort(row[c + 2 * e]) : 0u;
    const uint32_t hi = (c + 2 * e + 1 < K) ? __half_as_ushort(row[c + 2 * e + 1]) : 0u;
    w[e] = lo | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ unsigned short half_bits_at(const uint4& u, int e) {
  const uint32_t w = (e < 2) ? u.x : (e < 4) ? u.y : (e < 6) ? u.z : u.w;
  return static_cast<unsigned short>((e & 1) ? (w >> 16) : (w & 0xFFFFu));
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

// Dynamic shared memory of the last CTA: one bitmask word per 32 columns.
__global__ void __launch_bounds__(256, 4) scan_columns_kernel(const __half* __restrict__ X, int64_t M, int64_t K,
                                                           int64_t ldx, bool vec_ok, float tau, ActWs ws,
                                                           int32_t* __restrict__ O, int64_t cap,
                                                           int32_t* __restrict__ n_out) {
  extern __shared__ uint32_t s_bits[];
  __shared__ uint32_t s_max[8][kScanCols];
  __shared__ int s_warp[8];
  __shared__ int s_last;

  griddep_wait();               // X may come from the previous kernel on the stream
  griddep_launch_dependents();  // let the quantize kernel get resident early

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c = int64_t(blockIdx.x) * kScanCols + 8 * lane;
  const int64_t r0 = int64_t(blockIdx.y) * kScanRows + warp;
  // |x| maxima of 8 columns as 4 half2; __hmax2 returns the non-NaN operand,
  // so a NaN never wins (it is mapped to 0 below if nothing else was seen).
  __half2 m2[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) m2[e] = __half2half2(__ushort_as_half(0));
  if (c < K) {
    uint4 u[kScanRows / 8];  // all eight row loads are issued before any is used
#pragma unroll
    for (int j = 0; j < kScanRows / 8; ++j) {
      const int64_t r = r0 + 8 * j;
      u[j] = r < M ? load8_packed(X + r * ldx, K, c, vec_ok) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < kScanRows / 8; ++j) {
      const __half2* h2 = reinterpret_cast<const __half2*>(&u[j]);
#pragma unroll
      for (int e = 0; e < 4; ++e) m2[e] = __hmax2(m2[e], __habs2(h2[e]));
    }
  }
  const uint32_t* mw = reinterpret_cast<const uint32_t*>(m2);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t lo = mw[e] & 0xFFFFu, hi = mw[e] >> 16;
    lo = lo > 0x7C00u ? 0u : lo;  // NaN -> 0
    hi = hi > 0x7C00u ? 0u : hi;
    s_max[warp][8 * lane + 2 * e] = lo;
    s_max[warp][8 * lane + 2 * e + 1] = hi;
  }
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
  // One coalesced read and one ballot per 32 columns (column = 256 i + 32 warp
  // + lane, word = 8 i + warp); the loads of 8 rounds are issued together.
  // The maxima are reset to zero for the next call.
  constexpr int kBatch = 8;
  for (int64_t i0 = 0; i0 * 256 < K; i0 += kBatch) {
    uint32_t v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t col = (i0 + i) * 256 + threadIdx.x;
      v[i] = col < K ? __ldcg(ws.colmax + col) : 0u;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t col = (i0 + i) * 256 + threadIdx.x;
      const bool flag = col < K && __half2float(__ushort_as_half(static_cast<unsigned short>(v[i]))) >= tau;
      const uint32_t bits = __ballot_sync(0xffffffffu, flag);
      const int64_t w = (i0 + i) * 8 + warp;
      if (lane == 0 && w < nwords) {
        s_bits[w] = bits;
        ws.bitmask[w] = bits;
      }
      if (col < K) ws.colmax[col] = 0u;
    }
  }
  __syncthreads();
  const int64_t wpt = (nwords + 255) / 256;  // contiguous words per thread, in column order
  const int64_t w0 = int64_t(threadIdx.x) * wpt;
  int cnt = 0;
  for (int64_t w = w0; w < w0 + wpt && w < nwords; ++w) cnt += __popc(s_bits[w]);
  int total = 0;
  int pos = block_exclusive_scan_256(cnt, s_warp, total);
  for (int64_t w = w0; w < w0 + wpt && w < nwords; ++w) {
    uint32_t bits = s_bits[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < cap) O[pos] = static_cast<int32_t>(w * 32 + b);
      ++pos;
    }
  }
  if (threadIdx.x == 0) {
    *n_out = total;
    *ws.counter = 0u;
    if (total > cap) atomicOr(ws.status, kStatusOverflow);
  }
}

// Row quantizer: a group of G threads owns one row and holds its CPT chunks
// of 8 columns in registers (G * CPT * 8 >= K).  256 threads per CTA, 256 / G
// rows per CTA.
template <int G, int CPT>
__global__ void __launch_bounds__(256, 3) quantize_rows_kernel(const __half* __restrict__ X, int64_t M, int64_t K,
                                                            int64_t ldx, bool vec_ok, ActWs ws,
                                                            const int32_t* __restrict__ O,
                                                            const int32_t* __restrict__ n_ptr, int64_t cap,
                                                            int8_t* __restrict__ Xq, int64_t ldq,
                                                            float* __restrict__ rs, __half* __restrict__ Xo,
                                                            int64_t ldo) {
  extern __shared__ uint32_t s_mask[];  // [nwords] outlier bitmask, then [nwords] exclusive popcount prefix
  constexpr int kWarpsPerRow = G / 32;
  constexpr int kRowsPerCta = 256 / G;
  __shared__ float s_part[8];
  __shared__ int s_warp[8];

  griddep_wait();  // the bitmask comes from the scan kernel
  griddep_launch_dependents();

  const int64_t nwords = (K + 31) / 32;
  uint32_t* s_pre = s_mask + nwords;
  {
    // bitmask into shared memory and, per word, the number of outlier columns
    // before it: the position in O of a column's outlier value
    const int64_t wpt = (nwords + 255) / 256;
    const int64_t w0 = int64_t(threadIdx.x) * wpt;
    int cnt = 0;
    for (int64_t w = w0; w < w0 + wpt && w < nwords; ++w) {
      const uint32_t b = __ldg(ws.bitmask + w);
      s_mask[w] = b;
      cnt += __popc(b);
    }
    int total = 0;
    int pre = block_exclusive_scan_256(cnt, s_warp, total);
    for (int64_t w = w0; w < w0 + wpt && w < nwords; ++w) {
      s_pre[w] = static_cast<uint32_t>(pre);
      pre += __popc(s_mask[w]);
    }
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5;
  const int gt = threadIdx.x % G;
  const int64_t row = int64_t(blockIdx.x) * kRowsPerCta + threadIdx.x / G;
  const bool row_ok = row < M;
  const __half* xr = X + row * ldx;

  uint4 h[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int64_t c = 8 * (int64_t(gt) + int64_t(j) * G);
    h[j] = (row_ok && c < K) ? load8_packed(xr, K, c, vec_ok) : make_uint4(0u, 0u, 0u, 0u);
  }
  // outlier flags of a chunk's 8 columns (chunks past K read as no outliers:
  // their data is zero)
  auto flags = [&](int j) -> uint32_t {
    const int64_t c = 8 * (int64_t(gt) + int64_t(j) * G);
    return c < K ? (s_mask[c >> 5] >> (c & 31)) & 0xFFu : 0u;
  };
  // a2: absmax over the non-outlier columns; packed half2 max on chunks
  // without outliers, element-wise on the rare chunks that have some
  __half2 m2 = __half2half2(__ushort_as_half(0));
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const uint32_t om = flags(j);
    const __half2* h2 = reinterpret_cast<const __half2*>(&h[j]);
    if (om == 0u) {
#pragma unroll
      for (int e = 0; e < 4; ++e) m2 = __hmax2(m2, __habs2(h2[e]));
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (!((om >> e) & 1u)) {
          const __half a = __habs(__ushort_as_half(half_bits_at(h[j], e)));
          m2 = __hmax2(m2, __halves2half2(a, a));
        }
      }
    }
  }
  float m = fmaxf(__low2float(m2), __high2float(m2));
  m = (m == m) ? m : 0.0f;  // all-NaN row segment
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if constexpr (kWarpsPerRow > 1) {
    if ((threadIdx.x & 31) == 0) s_part[warp] = m;
    __syncthreads();
    const int wg0 = (warp / kWarpsPerRow) * kWarpsPerRow;
#pragma unroll
    for (int w = 0; w < kWarpsPerRow; ++w) m = fmaxf(m, s_part[wg0 + w]);
  }
  if (!row_ok) return;
  const float s = m;
  const float inv = s > 0.0f ? __frcp_rn(s) : 0.0f;
  const float k = s > 0.0f ? __fdiv_rn(127.0f, s) : 0.0f;
  if (gt == 0) rs[row] = s;

  // a3: codes; outlier columns are zeroed first (0 quantizes to 0); columns
  // [K, ldq) are written as zero
  int8_t* qr = Xq + row * ldq;
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int64_t c = 8 * (int64_t(gt) + int64_t(j) * G);
    if (c < ldq) {
      const uint32_t om = flags(j);
      uint4 u = h[j];
      if (om != 0u) {
        uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] &= (((om >> (2 * e)) & 1u) ? 0u : 0xFFFFu) | (((om >> (2 * e + 1)) & 1u) ? 0u : 0xFFFF0000u);
      }
      const __half2* h2 = reinterpret_cast<const __half2*>(&u);
      int q[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h2[e]);
        q[2 * e] = quantize_fast(f.x, s, inv, k);
        q[2 * e + 1] = quantize_fast(f.y, s, inv, k);
      }
      uint2 out;
      out.x = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
      out.y = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
      *reinterpret_cast<uint2*>(qr + c) = out;
    }
  }
  // ldq may exceed G * CPT * 8 only by the zero padding beyond K
  for (int64_t c = 8 * (int64_t(gt) + int64_t(CPT) * G); c < ldq; c += 8 * G)
    *reinterpret_cast<uint2*>(qr + c) = make_uint2(0u, 0u);

  // a4: gather X[row, O[t]] for the outlier product, from the registers: the
  // outlier column c sits at position prefix(word) + popcount(lower bits).
  if (Xo != nullptr) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const uint32_t om = flags(j);
      if (om != 0u) {
        const int64_t c = 8 * (int64_t(gt) + int64_t(j) * G);
        const uint32_t word = s_mask[c >> 5];
        const uint32_t base = s_pre[c >> 5];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if ((om >> e) & 1u) {
            const int b = static_cast<int>((c & 31) + e);
            const int64_t pos = base + __popc(word & ((1u << b) - 1u));
            if (pos < cap) Xo[row * ldo + pos] = __ushort_as_half(half_bits_at(h[j], e));
          }
        }
      }
    }
  }
}

// Fallback for very long rows (K > 16384): two passes over the row.
__global__ void __launch_bounds__(256) quantize_rows_long_kernel(const __half* __restrict__ X, int64_t M,
                                                                 int64_t K, int64_t ldx, bool vec_ok, ActWs ws,
                                                                 const int32_t* __restrict__ O,
                                                                 const int32_t* __restrict__ n_ptr, int64_t cap,
                                                                 int8_t* __restrict__ Xq, int64_t ldq,
                                                                 float* __restrict__ rs, __half* __restrict__ Xo,
                                                                 int64_t ldo) {
  extern __shared__ uint32_t s_mask[];
  __shared__ float s_part[8];
  griddep_wait();
  griddep_launch_dependents();
  const int64_t nwords = (K + 31) / 32;
  for (int64_t w = threadIdx.x; w < nwords; w += blockDim.x) s_mask[w] = ws.bitmask[w];
  __syncthreads();
  const int64_t row = blockIdx.x;
  const __half* xr = X + row * ldx;
  const int64_t nchunks = (K + 7) / 8;
  float m = 0.0f;
  for (int64_t ch = threadIdx.x; ch < nchunks; ch += 256) {
    __half h[8];
    load8_bits(xr, K, 8 * ch, vec_ok, h);
    const uint32_t mw = s_mask[(8 * ch) >> 5] >> ((8 * ch) & 31);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (!((mw >> e) & 1u)) m = fmaxf(m, fabsf(__half2float(h[e])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = m;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < 8; ++w) m = fmaxf(m, s_part[w]);
  const float s = m;
  const float inv = s > 0.0f ? __frcp_rn(s) : 0.0f;
  if (threadIdx.x == 0) rs[row] = s;
  int8_t* qr = Xq + row * ldq;
  for (int64_t ch = threadIdx.x; ch < ldq / 8; ch += 256) {
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
  if (Xo != nullptr) {
    const int n_o = *n_ptr;
    const int64_t n_gather = n_o < cap ? n_o : cap;
    for (int64_t t = threadIdx.x; t < n_gather; t += 256) Xo[row * ldo + t] = xr[O[t]];
  }
}

template <int G, int CPT>
cudaError_t launch_rows(cudaLaunchConfig_t& cfg, int64_t M, const __half* x, int64_t K, int64_t ldx, bool vec_ok,
                        ActWs ws, const int32_t* O, const int32_t* n, int64_t cap, int8_t* Xq, int64_t ldq,
                        float* rs, __half* xo, int64_t ldo) {
  constexpr int rows_per_cta = 256 / G;
  cfg.gridDim = dim3(static_cast<unsigned>((M + rows_per_cta - 1) / rows_per_cta));
  return cudaLaunchKernelEx(&cfg, quantize_rows_kernel<G, CPT>, x, M, K, ldx, vec_ok, ws, O, n, cap, Xq, ldq, rs,
                            xo, ldo);
}

}  // namespace

cudaError_t launch_quantize_act(const void* X, int64_t M, int64_t K, int64_t ldx, float tau, int8_t* Xq,
                                int64_t ldq, float* rs, int32_t* O, int64_t cap, int32_t* n_out, void* Xo,
                                int64_t ldo, ActWs ws, cudaStream_t stream, bool pdl) {
  const __half* x = static_cast<const __half*>(X);
  const bool vec_ok = (ldx % 8 == 0) && (reinterpret_cast<uintptr_t>(X) % 16 == 0);
  const size_t mask_bytes = static_cast<size_t>((K + 31) / 32) * sizeof(uint32_t);

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
  cfg.dynamicSmemBytes = mask_bytes;
  cudaError_t e = cudaLaunchKernelEx(&cfg, scan_columns_kernel, x, M, K, ldx, vec_ok, tau, ws, O, cap, n_out);
  if (e != cudaSuccess) return e;

  cfg.dynamicSmemBytes = 2 * mask_bytes;  // bitmask + popcount prefix
  __half* xo = static_cast<__half*>(Xo);
  const int32_t* Oc = O;
  const int32_t* nc = n_out;
  // Row groups: G threads x CPT chunks of 8 columns >= K.  Small M spreads a
  // row over more threads (fewer chunks each) to shorten the critical path.
  const bool small_m = M < 512;
  const int64_t chunks = (K + 7) / 8;
  if (small_m) {
    if (chunks <= 32 * 2) return launch_rows<32, 2>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
    if (chunks <= 64 * 2) return launch_rows<64, 2>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
    if (chunks <= 128 * 2) return launch_rows<128, 2>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
    if (chunks <= 256 * 2) return launch_rows<256, 2>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
    if (chunks <= 256 * 4) return launch_rows<256, 4>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
    if (chunks <= 256 * 8) return launch_rows<256, 8>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
  } else {
    if (chunks <= 32 * 8) return launch_rows<32, 8>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
    if (chunks <= 64 * 8) return launch_rows<64, 8>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
    if (chunks <= 128 * 8) return launch_rows<128, 8>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
    if (chunks <= 256 * 8) return launch_rows<256, 8>(cfg, M, x, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs, xo, ldo);
  }
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  return cudaLaunchKernelEx(&cfg, quantize_rows_long_kernel, x, M, K, ldx, vec_ok, ws, Oc, nc, cap, Xq, ldq, rs,
                            xo, ldo);
}

}  // namespace llmint8
