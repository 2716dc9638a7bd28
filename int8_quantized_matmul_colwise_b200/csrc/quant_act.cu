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
//  scan:     column maxima of |X| over 64 x 256 tiles, merged with atomicMax
//            on fp16 bit patterns (non-negative halves order like their bits)
//            into a workspace array that is zero between calls; the last CTA
//            of each 256-column block writes that block's outlier bitmask
//            words (one ballot per 32 columns) and re-zeroes its maxima;
//  quantize: every CTA issues the loads of its rows, then reads the bitmask
//            and builds its popcount prefix in shared memory while they are in
//            flight; CTA 0 writes the ascending outlier list; each row is then
//            quantized from registers and its outlier values gathered.
// Both are HBM streaming kernels: one 16-byte load per 8 columns, all of a
// thread's loads in flight together, no divergent work on the common path.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace llmint8 {

namespace {

constexpr int kScanCols = 256;  // columns per scan CTA (32 lanes x 8)
constexpr int kScanRows = 64;   // rows per scan CTA (8 warps x 8 rows)

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

// ----------------------------------------------------------------- a1: scan
// Column maxima of |X| over this CTA's 64 rows x 256 columns, merged into the
// workspace with atomicMax.  The last CTA of a column block (per-block
// counter) turns the block's 256 maxima into 8 outlier bitmask words and
// returns the maxima and the counter to zero for the next call.
template <bool kVec>
__global__ void __launch_bounds__(256, 4) scan_columns_kernel(const __half* __restrict__ X, int64_t M, int64_t K,
                                                              int64_t ldx, float tau, ActWs ws) {
  __shared__ uint32_t s_max[8][kScanCols];
  __shared__ int s_last;

  griddep_wait();               // X may come from the previous kernel on the stream
  griddep_launch_dependents();  // let the quantize kernel get resident early

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c = int64_t(blockIdx.x) * kScanCols + 8 * lane;
  const int64_t r0 = int64_t(blockIdx.y) * kScanRows + warp;
  // |x| maxima of 8 columns as 4 half2; __hmax2 returns the non-NaN operand,
  // so a NaN never wins (and is mapped to 0 below if nothing else was seen).
  __half2 m2[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) m2[e] = __half2half2(__ushort_as_half(0));
  if (c < K) {
    uint4 u[kScanRows / 8];  // all eight row loads are issued before any is used
#pragma unroll
    for (int j = 0; j < kScanRows / 8; ++j) {
      const int64_t r = r0 + 8 * j;
      u[j] = r < M ? load8_packed<kVec>(X + r * ldx, K, c) : make_uint4(0u, 0u, 0u, 0u);
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
  uint32_t v = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) v = max(v, s_max[w][threadIdx.x]);
  const int64_t col = int64_t(blockIdx.x) * kScanCols + threadIdx.x;
  if (v != 0 && col < K) atomicMax(ws.colmax + col, v);

  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(ws.blk_counter + blockIdx.x, 1u) == gridDim.y - 1u) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const uint32_t mx = col < K ? __ldcg(ws.colmax + col) : 0u;
  const bool flag = col < K && __half2float(__ushort_as_half(static_cast<unsigned short>(mx))) >= tau;
  const uint32_t bits = __ballot_sync(0xffffffffu, flag);
  const int64_t w = int64_t(blockIdx.x) * (kScanCols / 32) + warp;
  if (lane == 0 && w * 32 < K) ws.bitmask[w] = bits;
  if (col < K) ws.colmax[col] = 0u;
  if (threadIdx.x == 0) ws.blk_counter[blockIdx.x] = 0u;
}

// ----------------------------------------------------------------- a1 -> O
// The outlier bitmask of this call and its popcount prefix into shared memory
// (s_mask[w]: columns 32w..32w+31; s_pre[w]: outliers before word w).  CTA 0
// also writes the ascending outlier list, n_o and the overflow bit.
__device__ __forceinline__ void build_outlier_set(int64_t K, const ActWs& ws, uint32_t* s_mask, uint32_t* s_pre,
                                                  int* s_warp, int32_t* __restrict__ O, int64_t cap,
                                                  int32_t* __restrict__ n_out) {
  const int64_t nwords = (K + 31) / 32;
  const int64_t wpt = (nwords + 255) / 256;  // contiguous words per thread, in column order
  const int64_t w0 = int64_t(threadIdx.x) * wpt;
  int cnt = 0;
  for (int64_t w = w0; w < w0 + wpt && w < nwords; ++w) {
    const uint32_t b = __ldcg(ws.bitmask + w);
    s_mask[w] = b;
    cnt += __popc(b);
  }
  int total = 0;
  int pre = block_exclusive_scan_256(cnt, s_warp, total);
  for (int64_t w = w0; w < w0 + wpt && w < nwords; ++w) {
    s_pre[w] = static_cast<uint32_t>(pre);
    if (blockIdx.x == 0) {
      uint32_t bits = s_mask[w];
      int pos = pre;
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < cap) O[pos] = static_cast<int32_t>(w * 32 + b);
        ++pos;
      }
    }
    pre += __popc(s_mask[w]);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *n_out = total;
    if (total > cap) atomicOr(ws.status, kStatusOverflow);
  }
  __syncthreads();
}

// Every CTA has copied the call's bitmask into shared memory (the caller's
// __syncthreads is behind it): the last one to get here returns the bitmask
// and the counter to zero.
__device__ __forceinline__ void release_bitmask(const ActWs& ws, int64_t nwords, int* s_last) {
  if (threadIdx.x == 0) {
    __threadfence();
    *s_last = atomicAdd(ws.blk_counter, 1u) == gridDim.x - 1u ? 1 : 0;
  }
  __syncthreads();
  if (*s_last) {
    for (int64_t w = threadIdx.x; w < nwords; w += blockDim.x) ws.bitmask[w] = 0u;
    if (threadIdx.x == 0) ws.blk_counter[0] = 0u;
  }
}

// Column of the t-th outlier (t < n_o) from the bitmask and its word prefix.
__device__ __forceinline__ int outlier_col(int t, const uint32_t* mask, const uint32_t* pre, int nwords) {
  int lo = 0, hi = nwords - 1;  // last word whose prefix is <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<int>(pre[mid]) <= t) lo = mid;
    else hi = mid - 1;
  }
  uint32_t bits = mask[lo];
  for (int skip = t - static_cast<int>(pre[lo]); skip > 0; --skip) bits &= bits - 1;
  return lo * 32 + __ffs(bits) - 1;
}

// ----------------------------------------------------------------- a2-a4
// Row quantizer: a group of G threads owns one row and holds its CPT chunks
// of 8 columns in registers (G * CPT * 8 >= K).  256 threads per CTA, 256 / G
// rows per CTA.  Dynamic shared memory: bitmask and prefix, K/32 words each.
template <int G, int CPT, bool kVec>
__global__ void __launch_bounds__(256, 4) quantize_rows_kernel(const __half* __restrict__ X, int64_t M, int64_t K,
                                                               int64_t ldx, float tau, ActWs ws,
                                                               int32_t* __restrict__ O, int32_t* __restrict__ n_out,
                                                               int64_t cap, int8_t* __restrict__ Xq, int64_t ldq,
                                                               float* __restrict__ rs, __half* __restrict__ Xo,
                                                               int64_t ldo) {
  extern __shared__ uint32_t s_mask[];
  constexpr int kWarpsPerRow = G / 32;
  constexpr int kRowsPerCta = 256 / G;
  __shared__ float s_part[8];
  __shared__ int s_warp[8];
  __shared__ int s_last;

  griddep_wait();  // the column maxima come from the scan kernel
  griddep_launch_dependents();

  const int warp = threadIdx.x >> 5;
  const int gt = threadIdx.x % G;
  const int64_t row = int64_t(blockIdx.x) * kRowsPerCta + threadIdx.x / G;
  const bool row_ok = row < M;
  const __half* xr = X + row * ldx;

  // the row loads go out first and overlap the outlier-set construction
  uint4 h[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int64_t c = 8 * (int64_t(gt) + int64_t(j) * G);
    h[j] = (row_ok && c < K) ? load8_packed<kVec>(xr, K, c) : make_uint4(0u, 0u, 0u, 0u);
  }
  const int64_t nwords = (K + 31) / 32;
  uint32_t* s_pre = s_mask + nwords;
  build_outlier_set(K, ws, s_mask, s_pre, s_warp, O, cap, n_out);
  release_bitmask(ws, nwords, &s_last);

  // outlier flags of chunk j's 8 columns (chunks past K: none, data is zero)
  auto flags = [&](int j) -> uint32_t {
    const int64_t c = 8 * (int64_t(gt) + int64_t(j) * G);
    return c < K ? (s_mask[c >> 5] >> (c & 31)) & 0xFFu : 0u;
  };
  uint32_t any_outlier = 0;
#pragma unroll
  for (int j = 0; j < CPT; ++j) any_outlier |= flags(j);

  // a4: gather X[row, O[t]] for the outlier product by outlier number: thread
  // gt of the row's group takes outliers gt, gt + G, .. (the row is in L2:
  // its loads were just issued), so the stores to Xo are contiguous and no
  // thread walks its chunks for outlier bits.
  if (Xo != nullptr && row_ok) {
    const int n_o = static_cast<int>(s_pre[nwords - 1]) + __popc(s_mask[nwords - 1]);
    const int n = static_cast<int>(min(int64_t(n_o), cap));
    for (int t = gt; t < n; t += G) Xo[row * ldo + t] = xr[outlier_col(t, s_mask, s_pre, static_cast<int>(nwords))];
  }
  // outlier columns are zeroed in the registers (0 quantizes to 0)
  if (any_outlier != 0u) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const uint32_t om = flags(j);
      if (om != 0u) {
        uint32_t* w = reinterpret_cast<uint32_t*>(&h[j]);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] &= (((om >> (2 * e)) & 1u) ? 0u : 0xFFFFu) | (((om >> (2 * e + 1)) & 1u) ? 0u : 0xFFFF0000u);
      }
    }
  }

  // a2: absmax over the non-outlier columns (outliers and padding are zero now)
  __half2 m2 = __half2half2(__ushort_as_half(0));
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&h[j]);
#pragma unroll
    for (int e = 0; e < 4; ++e) m2 = __hmax2(m2, __habs2(h2[e]));
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
  const float s = m;
  const float inv = s > 0.0f ? __frcp_rn(s) : 0.0f;
  const float k = s > 0.0f ? __fdiv_rn(127.0f, s) : 0.0f;

  if (row_ok) {
    if (gt == 0) rs[row] = s;
    // a3: codes; columns [K, ldq) are written as zero
    int8_t* qr = Xq + row * ldq;
    uint32_t risk = 0;  // chunks that need the exact rounding
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int64_t c = 8 * (int64_t(gt) + int64_t(j) * G);
      if (c < ldq) {
        bool tie_risk = false;
        *reinterpret_cast<uint2*>(qr + c) = quantize8_fma(h[j], k, tie_risk);
        risk |= static_cast<uint32_t>(tie_risk) << j;
      }
    }
    if (risk != 0u) {  // rare: redo those chunks exactly
#pragma unroll
      for (int j = 0; j < CPT; ++j)
        if ((risk >> j) & 1u)
          *reinterpret_cast<uint2*>(qr + 8 * (int64_t(gt) + int64_t(j) * G)) = quantize8_exact(h[j], s, inv);
    }
    // ldq may exceed G * CPT * 8 only by the zero padding beyond K
    for (int64_t c = 8 * (int64_t(gt) + int64_t(CPT) * G); c < ldq; c += 8 * G)
      *reinterpret_cast<uint2*>(qr + c) = make_uint2(0u, 0u);
  }
}

// ----------------------------------------------------------------- a1-a4 in one kernel
// For shapes whose X fits in shared memory spread over the SMs: one CTA per SM
// (all resident: cooperative launch), each holding a block of rows.  The CTA
// bulk-copies its rows into shared memory; thread t then holds R of those rows
// for one 8-column chunk in registers for the whole kernel (chunks padded to a
// multiple of 32 so that a warp never straddles two row groups).
//
// The outlier set is the union of every CTA's column flags, known only after a
// grid barrier.  The barrier is split: a CTA ORs its own flags into the call's
// global bitmask and arrives, then quantizes its rows against its own flags
// while the other CTAs arrive (row maxima over the columns it has not flagged,
// row scales, codes), and only then waits.  Its own flags are a subset of the
// call's; when the two agree, which is the rule for outlier features that are
// systematic across tokens, the codes already written are the answer.
// Otherwise the CTA zeroes the further columns in its registers and quantizes
// its rows again.  Last, the outlier values are gathered from the rows in
// shared memory into Xo by their position in the call's outlier list.  X is
// read from HBM once.
//
// ws.fused: word 1 is the call generation g, words 0 and 2 are arrival
// counters, words 4.. hold bitmask buffers 0 and 1 of ceil(K/32) words.  A
// call of generation g counts its arrivals in counter g & 1 and ORs into
// buffer g & 1; its CTA 0 zeroes counter and buffer (g + 1) & 1, which the
// previous call used and the next will use, and bumps the generation once
// every CTA has arrived.  A CTA arrives with a release add that returns
// nothing (its flags ORed before the CTA barrier ahead of it), so no CTA waits
// on the arrival itself.
constexpr int kActFusedThreads = 1024;
constexpr int kActFusedMaxRows = 16;  // rows per CTA
constexpr size_t kActFusedSmemMax = 200 * 1024;

// Dynamic shared memory of the kernel: the rows, three bitmask-sized word
// arrays (16-byte multiples) and the column-maximum exchange.
inline size_t act_fused_smem(int64_t rows_per, int64_t K) {
  const size_t words = static_cast<size_t>((K + 31) / 32);
  return size_t(rows_per) * size_t(K) * 2 + 3 * ((words * 4 + 15) / 16 * 16) + size_t(kActFusedThreads) * 16;
}

template <int R>
__global__ void __launch_bounds__(kActFusedThreads, 1)
    act_fused_kernel(const __half* __restrict__ X, int64_t M, int64_t K, int64_t ldx, float tau, ActWs ws,
                     int32_t* __restrict__ O, int32_t* __restrict__ n_out, int64_t cap, int8_t* __restrict__ Xq,
                     int64_t ldq, float* __restrict__ rs, __half* __restrict__ Xo, int64_t ldo, int rows_per,
                     int cpad) {
  extern __shared__ __align__(128) uint8_t smem_a[];
  const int nwords = static_cast<int>((K + 31) / 32);
  const int nw4 = (nwords + 3) & ~3;
  const int nchunks = static_cast<int>(K / 8);  // K % 8 == 0 on this path
  __half* s_x = reinterpret_cast<__half*>(smem_a);  // [rows_per][K]
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem_a + size_t(rows_per) * size_t(K) * 2);  // the call's flags
  uint32_t* s_pre = s_mask + nw4;   // outliers before each word
  uint32_t* s_own = s_pre + nw4;    // this CTA's flags
  uint4* s_cm = reinterpret_cast<uint4*>(s_own + nw4);  // [kActFusedThreads] column maxima
  __shared__ uint64_t bar;
  __shared__ uint32_t s_gen;
  __shared__ int s_more, s_nout;
  __shared__ float s_part[kActFusedThreads / 32][8];  // row maxima per warp
  __shared__ float s_k[kActFusedMaxRows];
  __shared__ float s_sc[kActFusedMaxRows];
  __shared__ float s_inv[kActFusedMaxRows];

  const int tid = static_cast<int>(threadIdx.x);
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t r0 = int64_t(blockIdx.x) * rows_per;
  const int nr = static_cast<int>(min(int64_t(rows_per), M - r0));
  const int groups = kActFusedThreads / cpad;  // row groups; the host's plan gives R * groups >= rows_per
  const int cc = tid % cpad;                    // this thread's chunk
  const int g = tid / cpad;
  const bool col_ok = cc < nchunks && g < groups;
  const int m0 = g * R;                         // its first row (of the CTA's)
  uint32_t* generation = ws.fused + 1;

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  griddep_wait();  // X may be written by the preceding kernel
  griddep_launch_dependents();
  if (tid == 0) {
    // this CTA's rows, one bulk copy each, issued before the generation word
    // is read (an L2 round trip the copies need not wait for)
    mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(nr) * static_cast<uint32_t>(K) * 2u);
    for (int r = 0; r < nr; ++r)
      bulk_load_1d(s_x + size_t(r) * size_t(K), X + (r0 + r) * ldx, static_cast<uint32_t>(K) * 2u, &bar);
    s_gen = ld_acquire_gpu_u32(generation);
  }
  __syncthreads();
  const uint32_t gen = s_gen;
  uint32_t* arrived = ws.fused + 2 * (gen & 1u);
  uint32_t* buf = ws.fused + 4 + (gen & 1u) * uint32_t(nwords);
  uint32_t* other = ws.fused + 4 + ((gen + 1u) & 1u) * uint32_t(nwords);
  if (blockIdx.x == 0) {
    for (int w = tid; w < nwords; w += kActFusedThreads) other[w] = 0u;
    if (tid == 0) ws.fused[2 * ((gen + 1u) & 1u)] = 0u;
  }
  const bool loaded = mbar_wait(&bar, 0, ws.status);

  // this thread's rows of its chunk, kept in registers to the end
  uint4 h[R];
#pragma unroll
  for (int r = 0; r < R; ++r)
    h[r] = (loaded && col_ok && m0 + r < nr) ? *reinterpret_cast<const uint4*>(s_x + size_t(m0 + r) * size_t(K) + 8 * cc)
                                             : make_uint4(0u, 0u, 0u, 0u);

  // a1 (this CTA's rows): column maxima, then over the row groups
  __half2 cm[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) cm[e] = __half2half2(__ushort_as_half(0));
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&h[r]);
#pragma unroll
    for (int e = 0; e < 4; ++e) cm[e] = __hmax2(cm[e], __habs2(h2[e]));  // NaN never wins
  }
  if (groups > 1) {
    s_cm[tid] = *reinterpret_cast<const uint4*>(cm);
    __syncthreads();
    for (int gg = 0; gg < groups; ++gg) {
      const uint4 o = s_cm[gg * cpad + cc];
      const __half2* o2 = reinterpret_cast<const __half2*>(&o);
#pragma unroll
      for (int e = 0; e < 4; ++e) cm[e] = __hmax2(cm[e], o2[e]);
    }
  }
  uint32_t own = 0;  // bit e: column 8 cc + e is an outlier in this CTA's rows
  if (col_ok) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(cm[e]);
      own |= (f.x >= tau ? 1u : 0u) << (2 * e);
      own |= (f.y >= tau ? 1u : 0u) << (2 * e + 1);
    }
  }
  uint32_t word = own << ((8 * cc) & 31);
  word |= __shfl_xor_sync(0xffffffffu, word, 1);
  word |= __shfl_xor_sync(0xffffffffu, word, 2);
  if (g == 0 && col_ok && (cc & 3) == 0) {
    s_own[cc >> 2] = word;
    if (word != 0u) atomicOr(buf + (cc >> 2), word);
  }

  // grid barrier, arrival (every CTA of the grid is resident: cooperative
  // launch); the CTA barrier puts every thread's OR before thread 0's release
  __syncthreads();
  if (tid == 0) red_add_release_gpu_u32(arrived, 1u);

  // a2, a3 for the columns in `flags` (a superset of the ones zeroed so far):
  // zero them, row maxima over the rest, row scales, codes
  auto quantize_rows = [&](uint32_t flags, bool pad) {
    if (flags != 0u) {
      const uint32_t k0 = ((flags & 1u) ? 0u : 0xFFFFu) | ((flags & 2u) ? 0u : 0xFFFF0000u);
      const uint32_t k1 = ((flags & 4u) ? 0u : 0xFFFFu) | ((flags & 8u) ? 0u : 0xFFFF0000u);
      const uint32_t k2 = ((flags & 16u) ? 0u : 0xFFFFu) | ((flags & 32u) ? 0u : 0xFFFF0000u);
      const uint32_t k3 = ((flags & 64u) ? 0u : 0xFFFFu) | ((flags & 128u) ? 0u : 0xFFFF0000u);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        h[r].x &= k0;
        h[r].y &= k1;
        h[r].z &= k2;
        h[r].w &= k3;
      }
    }
    float pm[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const __half2* h2 = reinterpret_cast<const __half2*>(&h[r]);
      const __half2 m2 = __hmax2(__hmax2(__habs2(h2[0]), __habs2(h2[1])), __hmax2(__habs2(h2[2]), __habs2(h2[3])));
      pm[r] = fmaxf(__low2float(m2), __high2float(m2));
    }
    int prow = 0;
    const float pmax = rows_max_transposed<R>(pm, 32, lane, prow);
    if ((lane & (32 / R - 1)) == 0) s_part[warp][prow] = pmax;
    __syncthreads();
    if (tid < nr) {  // row tid: group tid / R, its warps' partial maxima
      const int wpg = cpad / 32;
      const int wa = (tid / R) * wpg;
      float sc = 0.0f;
      for (int w = wa; w < wa + wpg; ++w) sc = fmaxf(sc, s_part[w][tid % R]);
      rs[r0 + tid] = sc;
      s_sc[tid] = sc;
      s_k[tid] = sc > 0.0f ? __fdiv_rn(127.0f, sc) : 0.0f;
      s_inv[tid] = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
    }
    __syncthreads();
    if (col_ok) {
      int8_t* q = Xq + (r0 + m0) * ldq + 8 * cc;
      uint32_t risk_rows = 0;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (m0 + r < nr) {
          bool risk = false;
          const uint2 code = quantize8(h[r], s_k[m0 + r], risk);
          risk_rows |= static_cast<uint32_t>(risk) << r;
          *reinterpret_cast<uint2*>(q) = code;
        }
        q += ldq;
      }
      if (risk_rows != 0u) {  // rare: a value within 2^-15 of a rounding boundary; redo its chunk exactly
#pragma unroll
        for (int r = 0; r < R; ++r)
          if ((risk_rows >> r) & 1u)
            *reinterpret_cast<uint2*>(Xq + (r0 + m0 + r) * ldq + 8 * cc) = quantize8_exact(h[r], s_sc[m0 + r], s_inv[m0 + r]);
      }
    }
    if (pad) {  // Xq columns [K, ldq) are zero
      const int npad = static_cast<int>((ldq - K) / 8);
      for (int i = tid; i < npad * nr; i += kActFusedThreads)
        *reinterpret_cast<uint2*>(Xq + (r0 + i / npad) * ldq + K + 8 * (i % npad)) = make_uint2(0u, 0u);
    }
  };
  quantize_rows(own, true);

  // grid barrier, wait; then warp 0 reads the call's bitmask, compares it with
  // this CTA's flags and builds the popcount prefix (CTA 0 writes O and n_o)
  if (warp == 0) {
    if (lane == 0) {
      // (the stall test hook waits for one arrival more than the grid has:
      // the barrier then never completes and every CTA's wait runs out)
      const uint32_t all = gridDim.x + ((ws.stall & kStallActGridBarrier) ? 1u : 0u);
      const uint64_t t0 = globaltimer_ns();
      uint32_t n = 0;
      bool done = true;
      while (ld_acquire_gpu_u32(arrived) < all) {
        if ((++n & 255u) == 0u && globaltimer_ns() - t0 > wait_limit_ns()) {
          atomicOr(ws.status, kStatusTimeout);
          done = false;
          break;
        }
      }
      if (blockIdx.x == 0 && done) *generation = gen + 1u;  // every CTA has read gen: the next call's
    }
    __syncwarp();
    const int wpl = (nwords + 31) / 32;  // contiguous words per lane
    const int wa = lane * wpl;
    const int wb = min(wa + wpl, nwords);
    int cnt = 0;
    bool more = false;
    for (int w = wa; w < wb; ++w) {
      const uint32_t b = __ldcg(buf + w);
      s_mask[w] = b;
      cnt += __popc(b);
      more |= b != s_own[w];
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int pos = incl - cnt;
    for (int w = wa; w < wb; ++w) {
      s_pre[w] = static_cast<uint32_t>(pos);
      if (blockIdx.x == 0) {
        uint32_t bits = s_mask[w];
        int q = pos;
        while (bits) {
          const int bb = __ffs(bits) - 1;
          bits &= bits - 1;
          if (q < cap) O[q] = w * 32 + bb;
          ++q;
        }
      }
      pos += __popc(s_mask[w]);
    }
    more = __any_sync(0xffffffffu, more);
    if (lane == 0) {
      s_more = more ? 1 : 0;
      s_nout = total;
      if (blockIdx.x == 0) {
        *n_out = total;
        if (total > cap) atomicOr(ws.status, kStatusOverflow);
      }
    }
  }
  __syncthreads();

  // other CTAs flagged columns this one did not: quantize the rows again
  if (s_more) {
    const uint32_t all = col_ok ? (s_mask[cc >> 2] >> ((cc & 3) * 8)) & 0xFFu : 0u;
    quantize_rows(all, false);
  }

  // a4: X[row, O[q]] for this CTA's rows, from the rows in shared memory
  if (Xo != nullptr && loaded) {
    const int nq = static_cast<int>(min(int64_t(s_nout), cap));
    const int items = nq * nr;
    for (int i = tid; i < items; i += kActFusedThreads) {
      const int r = i / nq;
      const int q = i - r * nq;
      const int col = outlier_col(q, s_mask, s_pre, nwords);
      Xo[(r0 + r) * ldo + q] = s_x[size_t(r) * size_t(K) + col];
    }
  }
}

// ----------------------------------------------------------------- outlier statistics
// Values with |x| >= tau, the feature columns they fall in, and the rows that
// hold one -- the quantities the pages report ("8-bit Matrix Multiplication
// for Large Language Models", Summary & Methodology Analysis: 150,000 outliers
// per sequence in 6 feature dimensions at 6.7B).  Rows are split over the
// CTAs; the column bitmask and the counters live in a workspace scratch that
// is zero between calls, and the last CTA counts the bitmask, writes the three
// numbers and returns the scratch to zero.
template <bool kVec>
__global__ void __launch_bounds__(256) outlier_stats_kernel(const __half* __restrict__ X, int64_t M, int64_t K,
                                                            int64_t ldx, float tau, int rows_per,
                                                            uint32_t* __restrict__ scratch,
                                                            int64_t* __restrict__ stats) {
  __shared__ unsigned long long s_val[8];
  __shared__ int s_last;
  const int nwords = static_cast<int>((K + 31) / 32);
  uint32_t* mask = scratch;
  unsigned long long* cnt = reinterpret_cast<unsigned long long*>(scratch + ((nwords + 1) & ~1));
  griddep_wait();
  griddep_launch_dependents();

  unsigned long long my_values = 0;
  unsigned long long my_rows = 0;
  const int64_t r0 = int64_t(blockIdx.x) * rows_per;
  const int64_t r1 = min(M, r0 + rows_per);
  for (int64_t r = r0; r < r1; ++r) {
    const __half* xr = X + r * ldx;
    int any = 0;
    for (int64_t c = 8 * int64_t(threadIdx.x); c < K; c += 8 * 256) {
      const uint4 u = load8_packed<kVec>(xr, K, c);
      uint32_t fl = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float a = fabsf(__half2float(__ushort_as_half(half_bits_at(u, e))));
        if (c + e < K && a >= tau) fl |= 1u << e;  // false for NaN
      }
      if (fl != 0u) {
        my_values += __popc(fl);
        any = 1;
        atomicOr(mask + (c >> 5), fl << (c & 31));
      }
    }
    if (__syncthreads_or(any) && threadIdx.x == 0) ++my_rows;
  }
  // this CTA's value count
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my_values += __shfl_down_sync(0xffffffffu, my_values, o);
  if ((threadIdx.x & 31) == 0) s_val[threadIdx.x >> 5] = my_values;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long v = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += s_val[w];
    if (v) atomicAdd(cnt + 0, v);
    if (my_rows) atomicAdd(cnt + 1, my_rows);
    __threadfence();
    s_last = atomicAdd(cnt + 2, 1ull) == static_cast<unsigned long long>(gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  int cols = 0;
  for (int w = threadIdx.x; w < nwords; w += 256) {
    cols += __popc(__ldcg(mask + w));
    mask[w] = 0u;  // zero for the next call
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cols += __shfl_down_sync(0xffffffffu, cols, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) s_val[threadIdx.x >> 5] = static_cast<unsigned long long>(cols);
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long c = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) c += s_val[w];
    stats[0] = static_cast<int64_t>(__ldcg(cnt + 0));
    stats[1] = static_cast<int64_t>(c);
    stats[2] = static_cast<int64_t>(__ldcg(cnt + 1));
    cnt[0] = 0ull;
    cnt[1] = 0ull;
    cnt[2] = 0ull;
  }
}

// Rows too long for the register-resident kernel (K > 16384): one CTA per row,
// two passes over the row.
__global__ void __launch_bounds__(256) quantize_rows_long_kernel(const __half* __restrict__ X, int64_t M,
                                                                 int64_t K, int64_t ldx, float tau, ActWs ws,
                                                                 int32_t* __restrict__ O,
                                                                 int32_t* __restrict__ n_out, int64_t cap,
                                                                 int8_t* __restrict__ Xq, int64_t ldq,
                                                                 float* __restrict__ rs, __half* __restrict__ Xo,
                                                                 int64_t ldo) {
  extern __shared__ uint32_t s_mask[];
  __shared__ float s_part[8];
  __shared__ int s_warp[8];
  __shared__ int s_last;
  griddep_wait();
  griddep_launch_dependents();
  const int64_t nwords = (K + 31) / 32;
  uint32_t* s_pre = s_mask + nwords;
  build_outlier_set(K, ws, s_mask, s_pre, s_warp, O, cap, n_out);
  release_bitmask(ws, nwords, &s_last);

  const int64_t row = blockIdx.x;
  const __half* xr = X + row * ldx;
  const int64_t nchunks = (K + 7) / 8;
  float m = 0.0f;
  for (int64_t ch = threadIdx.x; ch < nchunks; ch += 256) {
    const uint4 u = load8_scalar(xr, K, 8 * ch);
    const uint32_t mw = s_mask[(8 * ch) >> 5] >> ((8 * ch) & 31);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (!((mw >> e) & 1u)) m = fmaxf(m, fabsf(__half2float(__ushort_as_half(half_bits_at(u, e)))));
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
      const uint4 u = load8_scalar(xr, K, c);
      const uint32_t mw = s_mask[c >> 5] >> (c & 31);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const bool keep = (c + e < K) && !((mw >> e) & 1u) && s > 0.0f;
        q[e] = keep ? quantize_exact(__half2float(__ushort_as_half(half_bits_at(u, e))), s, inv) : 0;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) q[e] = 0;
    }
    *reinterpret_cast<uint2*>(qr + c) = pack8(q);
  }
  if (Xo != nullptr) {
    // positions come from the local bitmask and prefix (O itself is written by CTA 0)
    for (int64_t w = threadIdx.x; w < nwords; w += 256) {
      uint32_t bits = s_mask[w];
      int64_t pos = s_pre[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < cap) Xo[row * ldo + pos] = xr[w * 32 + b];
        ++pos;
      }
    }
  }
}

// ----------------------------------------------------------------- a1-a4 streaming (many rows)
// X with more rows than fit in shared memory over the SMs, rows that allow
// bulk copies (16-byte aligned, K % 8 == 0) and kStreamMinK <= K <=
// kStreamMaxK.  Both kernels are persistent (two CTAs per SM), and each CTA
// streams whole rows of X through a ring of shared-memory stages filled by
// bulk copies, so that several rows per SM are in flight at any time.
//  scan:     column maxima of |X| over the CTA's rows, kept in registers; then
//            one flag per column (maximum >= tau, which a NaN never wins) ORed
//            into the call's bitmask, which is zero between calls;
//  quantize: the CTA copies the bitmask and its popcount prefix into shared
//            memory once (the last CTA to do so returns the bitmask to zero),
//            then quantizes its rows, walking them from the last row up so
//            that the rows the scan read last, still in L2, come first.
constexpr int kStreamThreads = 256;
constexpr int kStreamMaxStages = 8;
constexpr size_t kStreamRing = 96 * 1024;  // bytes of row stages per CTA
constexpr int kStreamListMax = 1024;        // outlier columns listed in shared memory

inline int stream_stages(int64_t K) {
  const int s = static_cast<int>(kStreamRing / (size_t(K) * 2));
  return s > kStreamMaxStages ? kStreamMaxStages : s;
}

// The quantize pass does more work per row: a smaller ring (at least three
// stages, which its one-row lookahead needs) lets three CTAs share an SM for
// rows of up to 8192 columns.
constexpr size_t kStreamRingQ = 64 * 1024;
inline int stream_stages_q(int64_t K) {
  const int s = static_cast<int>(kStreamRingQ / (size_t(K) * 2));
  return s < 3 ? 3 : s > kStreamMaxStages ? kStreamMaxStages : s;
}
// Largest ring of the quantize pass for a CPT instance (its K range).
constexpr size_t stream_ring_q_max(int CPT) {
  return CPT <= 4 ? kStreamRingQ : size_t(3) * 2 * 8 * kStreamThreads * CPT;
}

// Rows of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
__device__ __forceinline__ int64_t stream_rows(int64_t M) {
  return M > int64_t(blockIdx.x) ? (M - 1 - int64_t(blockIdx.x)) / int64_t(gridDim.x) + 1 : 0;
}

// After a wait gave up at row `from` (stage st, phase parity ph): let the
// copies issued for rows [from, to) of this CTA land before the CTA exits.
__device__ __forceinline__ void stream_drain(uint64_t* full, int stages, int64_t from, int64_t to, int st,
                                             uint32_t ph) {
  for (int64_t i = from; i < to; ++i) {
    mbar_wait(&full[st], ph, nullptr);
    if (++st == stages) {
      st = 0;
      ph ^= 1u;
    }
  }
}

template <int CPT>
__global__ void __launch_bounds__(kStreamThreads, 2)
    scan_stream_kernel(const __half* __restrict__ X, int64_t M, int64_t K, int64_t ldx, float tau, ActWs ws,
                       int stages) {
  extern __shared__ __align__(128) uint8_t smem_s[];
  __shared__ uint64_t full[kStreamMaxStages];
  __half* ring = reinterpret_cast<__half*>(smem_s);
  const int tid = static_cast<int>(threadIdx.x);
  const int warp = tid >> 5;
  const int nchunks = static_cast<int>(K / 8);
  const int64_t nrows = stream_rows(M);
  const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // X may be written by the preceding kernel
  griddep_launch_dependents();
  // thread 0 issues row `issued` of this CTA into stage `ist` (rows and stages advance together)
  int64_t issued = 0;
  int ist = 0;
  auto issue = [&]() {
    mbar_arrive_expect_tx(&full[ist], row_bytes);
    bulk_load_1d(ring + size_t(ist) * size_t(K), X + (int64_t(blockIdx.x) + issued * gridDim.x) * ldx, row_bytes,
                 &full[ist]);
    ++issued;
    if (++ist == stages) ist = 0;
  };
  if (tid == 0)
    while (issued < stages && issued < nrows) issue();

  __half2 cm[CPT][4];
#pragma unroll
  for (int j = 0; j < CPT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) cm[j][e] = __half2half2(__ushort_as_half(0));
  // Warp 0 alone waits for each row's copy, the other warps at the row's
  // barrier (which issues nothing), so that no spinning takes issue slots
  // from the other CTA on the SM.
  int st = 0;        // stage of row i
  uint32_t ph = 0;   // its phase parity
  if (!__syncthreads_and(warp != 0 || nrows == 0 || mbar_wait(&full[0], 0, ws.status))) {
    if (tid == 0) stream_drain(full, stages, 0, issued, 0, 0u);  // a copy never landed: timeout bit set
    return;
  }
  for (int64_t i = 0; i < nrows; ++i) {
    const __half* sr = ring + size_t(st) * size_t(K);
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = tid + j * kStreamThreads;
      if (c < nchunks) {
        const uint4 u = *reinterpret_cast<const uint4*>(sr + 8 * c);
        const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) cm[j][e] = __hmax2(cm[j][e], __habs2(h2[e]));  // NaN never wins
      }
    }
    const int nst = st + 1 == stages ? 0 : st + 1;  // row i + 1
    const uint32_t nph = nst == 0 ? ph ^ 1u : ph;
    if (!__syncthreads_and(warp != 0 || i + 1 >= nrows || mbar_wait(&full[nst], nph, ws.status))) {
      if (tid == 0) stream_drain(full, stages, i + 1, issued, nst, nph);
      return;
    }
    if (tid == 0 && issued < nrows) issue();  // every thread is done with row i's stage
    st = nst;
    ph = nph;
  }

  // a1: one flag per column, ORed into the call's bitmask (32 columns per word)
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = tid + j * kStreamThreads;
    uint32_t f = 0;
    if (c < nchunks) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 m = __half22float2(cm[j][e]);
        f |= (m.x >= tau ? 1u : 0u) << (2 * e);
        f |= (m.y >= tau ? 1u : 0u) << (2 * e + 1);
      }
    }
    uint32_t word = f << ((8 * c) & 31);
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    if ((c & 3) == 0 && c < nchunks && word != 0u) atomicOr(ws.bitmask + (c >> 2), word);
  }
}

template <int CPT>
__global__ void __launch_bounds__(kStreamThreads, CPT <= 4 ? 3 : 2)
    quantize_stream_kernel(const __half* __restrict__ X, int64_t M, int64_t K, int64_t ldx, ActWs ws,
                           int32_t* __restrict__ O, int32_t* __restrict__ n_out, int64_t cap, int8_t* __restrict__ Xq,
                           int64_t ldq, float* __restrict__ rs, __half* __restrict__ Xo, int64_t ldo, int stages) {
  extern __shared__ __align__(128) uint8_t smem_s[];
  __shared__ uint64_t full[kStreamMaxStages];
  __shared__ float s_part[2][kStreamThreads / 32];
  __shared__ int s_warp[kStreamThreads / 32];
  __shared__ int s_last;
  const int nwords = static_cast<int>((K + 31) / 32);
  const int nw4 = (nwords + 3) & ~3;
  __half* ring = reinterpret_cast<__half*>(smem_s);
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem_s + size_t(stages) * size_t(K) * 2);
  uint32_t* s_pre = s_mask + nw4;
  int* s_list = reinterpret_cast<int*>(s_pre + nw4);  // [kStreamListMax] the first outlier columns
  const int tid = static_cast<int>(threadIdx.x);
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nchunks = static_cast<int>(K / 8);
  const int64_t nrows = stream_rows(M);
  const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
  auto row_of = [&](int64_t i) { return M - 1 - (int64_t(blockIdx.x) + i * gridDim.x); };  // last row first
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // the bitmask comes from the scan kernel
  griddep_launch_dependents();
  // thread 0 issues row `issued` of this CTA into stage `ist` (rows and stages advance together)
  int64_t issued = 0;
  int ist = 0;
  auto issue = [&]() {
    mbar_arrive_expect_tx(&full[ist], row_bytes);
    bulk_load_1d(ring + size_t(ist) * size_t(K), X + row_of(issued) * ldx, row_bytes, &full[ist]);
    ++issued;
    if (++ist == stages) ist = 0;
  };
  if (tid == 0)
    while (issued < stages && issued < nrows) issue();

  // the call's outlier set, once per CTA (CTA 0 writes O and n_o)
  build_outlier_set(K, ws, s_mask, s_pre, s_warp, O, cap, n_out);
  for (int w = tid; w < nwords; w += kStreamThreads) {
    uint32_t bits = s_mask[w];
    int pos = static_cast<int>(s_pre[w]);
    while (bits && pos < kStreamListMax) {
      s_list[pos++] = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1;
    }
  }
  release_bitmask(ws, nwords, &s_last);  // its barrier also publishes s_list
  const int n_o = static_cast<int>(s_pre[nwords - 1]) + __popc(s_mask[nwords - 1]);
  const int nq = static_cast<int>(min(int64_t(n_o), cap));
  // a thread's chunks are the same columns in every row: their outlier
  // columns as AND masks over the fp16 pairs, once per CTA
  uint4 keep[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = tid + j * kStreamThreads;
    const uint32_t om = c < nchunks ? (s_mask[c >> 2] >> ((c & 3) * 8)) & 0xFFu : 0u;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[e] = (((om >> (2 * e)) & 1u) ? 0u : 0xFFFFu) | (((om >> (2 * e + 1)) & 1u) ? 0u : 0xFFFF0000u);
    keep[j] = make_uint4(w[0], w[1], w[2], w[3]);
  }

  // Warp 0 alone waits for each row's copy (for row i + 1 just before row i's
  // barrier), the other warps at the barrier, which issues nothing.
  int st = 0;        // stage of row i
  uint32_t ph = 0;   // its phase parity
  if (!__syncthreads_and(warp != 0 || nrows == 0 || mbar_wait(&full[0], 0, ws.status))) {
    if (tid == 0) stream_drain(full, stages, 0, issued, 0, 0u);  // a copy never landed: timeout bit set
    return;
  }
  for (int64_t i = 0; i < nrows; ++i) {
    const int64_t row = row_of(i);
    const __half* sr = ring + size_t(st) * size_t(K);
    uint4 h[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = tid + j * kStreamThreads;
      h[j] = c < nchunks ? *reinterpret_cast<const uint4*>(sr + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
    }
    // a3 precondition: outlier columns are zeroed (0 quantizes to 0); a2: row maximum of the rest
    __half2 m2 = __half2half2(__ushort_as_half(0));
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      h[j].x &= keep[j].x;
      h[j].y &= keep[j].y;
      h[j].z &= keep[j].z;
      h[j].w &= keep[j].w;
      const __half2* h2 = reinterpret_cast<const __half2*>(&h[j]);
#pragma unroll
      for (int e = 0; e < 4; ++e) m2 = __hmax2(m2, __habs2(h2[e]));
    }
    float m = fmaxf(__low2float(m2), __high2float(m2));
    m = (m == m) ? m : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_part[i & 1][warp] = m;
    const int nst = st + 1 == stages ? 0 : st + 1;  // row i + 1
    const uint32_t nph = nst == 0 ? ph ^ 1u : ph;
    if (!__syncthreads_and(warp != 0 || i + 1 >= nrows || mbar_wait(&full[nst], nph, ws.status))) {
      if (tid == 0) stream_drain(full, stages, i + 1, issued, nst, nph);  // timeout bit set
      return;
    }
    // every thread is done with row i - 1 (its gather included): refill its stage
    if (tid == 0 && i >= 1 && issued < nrows) issue();
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kStreamThreads / 32; ++w) s = fmaxf(s, s_part[i & 1][w]);
    const float k = s > 0.0f ? __fdiv_rn(127.0f, s) : 0.0f;
    int8_t* qr = Xq + row * ldq;
    uint32_t risk = 0;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = tid + j * kStreamThreads;
      if (c < nchunks) {
        bool r = false;
        *reinterpret_cast<uint2*>(qr + 8 * c) = quantize8_fma(h[j], k, r);
        risk |= static_cast<uint32_t>(r) << j;
      }
    }
    if (risk != 0u) {  // rare: a value within 2^-15 of a rounding boundary; redo its chunk exactly
      const float inv = __frcp_rn(s);
#pragma unroll
      for (int j = 0; j < CPT; ++j)
        if ((risk >> j) & 1u) *reinterpret_cast<uint2*>(qr + 8 * (tid + j * kStreamThreads)) = quantize8_exact(h[j], s, inv);
    }
    for (int64_t c = nchunks + tid; c < ldq / 8; c += kStreamThreads)  // Xq columns [K, ldq) are zero
      *reinterpret_cast<uint2*>(qr + 8 * c) = make_uint2(0u, 0u);
    if (tid == 0) rs[row] = s;
    // a4: X[row, O[t]] from the row in shared memory
    if (Xo != nullptr) {
      for (int t = tid; t < nq; t += kStreamThreads) {
        const int col = t < kStreamListMax ? s_list[t] : outlier_col(t, s_mask, s_pre, nwords);
        Xo[row * ldo + t] = sr[col];
      }
    }
    st = nst;
    ph = nph;
  }
}

template <int CPT>
cudaError_t launch_stream(cudaLaunchConfig_t cfg, int64_t M, const __half* x, int64_t K, int64_t ldx, float tau,
                          ActWs ws, int32_t* O, int32_t* n, int64_t cap, int8_t* Xq, int64_t ldq, float* rs,
                          __half* xo, int64_t ldo, int num_sms) {
  static bool attr_set[64] = {};
  static int per_sm[64][2] = {};  // resident CTAs per SM at the largest ring (scan, quantize), per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int stages = stream_stages(K);
  const int stages_q = stream_stages_q(K);
  const size_t nw4 = static_cast<size_t>(((K + 31) / 32 + 3) & ~int64_t(3));
  const size_t smem_scan = size_t(stages) * size_t(K) * 2;
  const size_t smem_q = size_t(stages_q) * size_t(K) * 2 + 2 * nw4 * 4 + size_t(kStreamListMax) * 4;
  constexpr size_t kSmemQMax = stream_ring_q_max(CPT) + 2 * 4 * 512 + 4 * kStreamListMax;
  if (!attr_set[dev]) {
    // two or three CTAs of 64-100 KB per SM need the largest shared-memory carveout
    e = cudaFuncSetAttribute(scan_stream_kernel<CPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kStreamRing));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(scan_stream_kernel<CPT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(quantize_stream_kernel<CPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSmemQMax));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(quantize_stream_kernel<CPT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    // persistent grids: as many CTAs as are resident at once (one wave)
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[dev][0], scan_stream_kernel<CPT>, kStreamThreads,
                                                        kStreamRing);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[dev][1], quantize_stream_kernel<CPT>, kStreamThreads,
                                                        kSmemQMax);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  auto clamp = [](int v, int hi) { return v < 1 ? 1 : v > hi ? hi : v; };
  const int64_t ctas_scan = int64_t(num_sms) * clamp(per_sm[dev][0], 2);
  const int64_t ctas_q = int64_t(num_sms) * clamp(per_sm[dev][1], 3);
  cfg.blockDim = dim3(kStreamThreads);
  cfg.gridDim = dim3(static_cast<unsigned>(M < ctas_scan ? M : ctas_scan));
  cfg.dynamicSmemBytes = smem_scan;
  e = cudaLaunchKernelEx(&cfg, scan_stream_kernel<CPT>, x, M, K, ldx, tau, ws, stages);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(static_cast<unsigned>(M < ctas_q ? M : ctas_q));
  cfg.dynamicSmemBytes = smem_q;
  return cudaLaunchKernelEx(&cfg, quantize_stream_kernel<CPT>, x, M, K, ldx, ws, O, n, cap, Xq, ldq, rs, xo, ldo,
                            stages_q);
}

template <int G, int CPT>
cudaError_t launch_rows(cudaLaunchConfig_t& cfg, int64_t M, const __half* x, int64_t K, int64_t ldx, bool vec_ok,
                        float tau, ActWs ws, int32_t* O, int32_t* n, int64_t cap, int8_t* Xq, int64_t ldq,
                        float* rs, __half* xo, int64_t ldo) {
  constexpr int rows_per_cta = 256 / G;
  cfg.gridDim = dim3(static_cast<unsigned>((M + rows_per_cta - 1) / rows_per_cta));
  if (vec_ok)
    return cudaLaunchKernelEx(&cfg, quantize_rows_kernel<G, CPT, true>, x, M, K, ldx, tau, ws, O, n, cap, Xq, ldq,
                              rs, xo, ldo);
  return cudaLaunchKernelEx(&cfg, quantize_rows_kernel<G, CPT, false>, x, M, K, ldx, tau, ws, O, n, cap, Xq, ldq,
                            rs, xo, ldo);
}

}  // namespace

bool act_stream_plan(int64_t M, int64_t K, int64_t ldx, const void* X, int num_sms) {
  return num_sms > 0 && ldx % 8 == 0 && K % 8 == 0 && reinterpret_cast<uintptr_t>(X) % 16 == 0 &&
         K >= kStreamMinK && K <= kStreamMaxK && M >= num_sms;
}

bool act_fused_plan(int64_t M, int64_t K, int64_t ldx, const void* X, int num_sms) {
  if (num_sms <= 0 || ldx % 8 != 0 || K % 8 != 0 || reinterpret_cast<uintptr_t>(X) % 16 != 0) return false;
  const int64_t rows_per = (M + num_sms - 1) / num_sms;
  const int64_t cpad = ((K / 8) + 31) / 32 * 32;  // chunks padded to whole warps
  if (cpad > kActFusedThreads) return false;
  const int64_t groups = kActFusedThreads / cpad;
  const int64_t r = (rows_per + groups - 1) / groups;
  const size_t smem = act_fused_smem(rows_per, K);
  return r <= 8 && rows_per <= kActFusedMaxRows && smem <= kActFusedSmemMax;
}

cudaError_t launch_quantize_act(const void* X, int64_t M, int64_t K, int64_t ldx, float tau, int8_t* Xq,
                                int64_t ldq, float* rs, int32_t* O, int64_t cap, int32_t* n_out, void* Xo,
                                int64_t ldo, ActWs ws, cudaStream_t stream, bool pdl, int num_sms) {
  const __half* x = static_cast<const __half*>(X);
  const bool vec_ok = (ldx % 8 == 0) && (K % 8 == 0) && (reinterpret_cast<uintptr_t>(X) % 16 == 0);
  const size_t mask_bytes = static_cast<size_t>((K + 31) / 32) * sizeof(uint32_t);

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;

  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;

  // One kernel when X fits in shared memory over at most num_sms CTAs.
  if (ws.fused != nullptr && act_fused_plan(M, K, ldx, X, num_sms)) {
    const int64_t rows_per = (M + num_sms - 1) / num_sms;
    const int64_t cpad = ((K / 8) + 31) / 32 * 32;  // chunks padded to whole warps
    const int64_t r = (rows_per + kActFusedThreads / cpad - 1) / (kActFusedThreads / cpad);  // rows per thread
    const size_t smem = act_fused_smem(rows_per, K);
    const int ri = r <= 1 ? 0 : r <= 2 ? 1 : r <= 4 ? 2 : 3;
    auto kern = ri == 0 ? act_fused_kernel<1> : ri == 1 ? act_fused_kernel<2> : ri == 2 ? act_fused_kernel<4>
                                                                                        : act_fused_kernel<8>;
    static bool attr_set[4][64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[ri][dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kActFusedSmemMax));
      if (e != cudaSuccess) return e;
      attr_set[ri][dev] = true;
    }
    cfg.blockDim = dim3(kActFusedThreads);
    cfg.gridDim = dim3(static_cast<unsigned>((M + rows_per - 1) / rows_per));
    cfg.dynamicSmemBytes = smem;
    // The grid barrier needs every CTA resident at once: a cooperative launch
    // has the driver guarantee it (the grid is at most one CTA per SM).
    cudaLaunchAttribute fattr[2];
    fattr[0].id = cudaLaunchAttributeCooperative;
    fattr[0].val.cooperative = 1;
    fattr[1] = attr[0];
    cfg.attrs = fattr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, x, M, K, ldx, tau, ws, O, n_out, cap, Xq, ldq, rs, static_cast<__half*>(Xo),
                              ldo, static_cast<int>(rows_per), static_cast<int>(cpad));
  }

  __half* xo = static_cast<__half*>(Xo);
  // Many rows that allow bulk copies: the two streaming kernels.
  if (act_stream_plan(M, K, ldx, X, num_sms)) {
    const int64_t chunks = K / 8;
#define LLMINT8_STREAM(CPT) \
  return launch_stream<CPT>(cfg, M, x, K, ldx, tau, ws, O, n_out, cap, Xq, ldq, rs, xo, ldo, num_sms)
    if (chunks <= kStreamThreads) LLMINT8_STREAM(1);
    if (chunks <= 2 * kStreamThreads) LLMINT8_STREAM(2);
    if (chunks <= 4 * kStreamThreads) LLMINT8_STREAM(4);
    if (chunks <= 6 * kStreamThreads) LLMINT8_STREAM(6);
    LLMINT8_STREAM(8);
#undef LLMINT8_STREAM
  }

  cfg.gridDim = dim3(static_cast<unsigned>((K + kScanCols - 1) / kScanCols),
                     static_cast<unsigned>((M + kScanRows - 1) / kScanRows));
  cfg.dynamicSmemBytes = 0;
  cudaError_t e = vec_ok ? cudaLaunchKernelEx(&cfg, scan_columns_kernel<true>, x, M, K, ldx, tau, ws)
                         : cudaLaunchKernelEx(&cfg, scan_columns_kernel<false>, x, M, K, ldx, tau, ws);
  if (e != cudaSuccess) return e;

  cfg.dynamicSmemBytes = 2 * mask_bytes;  // bitmask + popcount prefix
  // Row groups: G threads x CPT chunks of 8 columns >= K.  Small M spreads a
  // row over more threads (fewer chunks each) to shorten the critical path.
  const int64_t chunks = (K + 7) / 8;
#define LLMINT8_ROWS(G, CPT) \
  return launch_rows<G, CPT>(cfg, M, x, K, ldx, vec_ok, tau, ws, O, n_out, cap, Xq, ldq, rs, xo, ldo)
  if (M < 512) {
    if (chunks <= 32 * 2) LLMINT8_ROWS(32, 2);
    if (chunks <= 64 * 2) LLMINT8_ROWS(64, 2);
    if (chunks <= 128 * 2) LLMINT8_ROWS(128, 2);
    if (chunks <= 256 * 2) LLMINT8_ROWS(256, 2);
    if (chunks <= 256 * 4) LLMINT8_ROWS(256, 4);
    if (chunks <= 256 * 8) LLMINT8_ROWS(256, 8);
  } else {
    if (chunks <= 32 * 8) LLMINT8_ROWS(32, 8);
    if (chunks <= 64 * 8) LLMINT8_ROWS(64, 8);
    if (chunks <= 128 * 8) LLMINT8_ROWS(128, 8);
    if (chunks <= 256 * 8) LLMINT8_ROWS(256, 8);
  }
#undef LLMINT8_ROWS
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  return cudaLaunchKernelEx(&cfg, quantize_rows_long_kernel, x, M, K, ldx, tau, ws, O, n_out, cap, Xq, ldq, rs, xo,
                            ldo);
}

cudaError_t launch_outlier_stats(const void* X, int64_t M, int64_t K, int64_t ldx, float tau, uint32_t* scratch,
                                 int64_t* stats, int num_sms, cudaStream_t stream) {
  const __half* x = static_cast<const __half*>(X);
  const bool vec_ok = (ldx % 8 == 0) && (K % 8 == 0) && (reinterpret_cast<uintptr_t>(X) % 16 == 0);
  const int64_t target = int64_t(num_sms > 0 ? num_sms : 148) * 4;  // CTAs
  const int64_t rows_per = (M + target - 1) / target;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((M + rows_per - 1) / rows_per));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return vec_ok ? cudaLaunchKernelEx(&cfg, outlier_stats_kernel<true>, x, M, K, ldx, tau, static_cast<int>(rows_per),
                                     scratch, stats)
                : cudaLaunchKernelEx(&cfg, outlier_stats_kernel<false>, x, M, K, ldx, tau,
                                     static_cast<int>(rows_per), scratch, stats);
}

// Test hook: this file's wait bound (see ptx.cuh).
cudaError_t set_debug_waits_quant_act(uint64_t limit_ns) { return set_debug_waits_in_this_file(limit_ns); }

}  // namespace llmint8
