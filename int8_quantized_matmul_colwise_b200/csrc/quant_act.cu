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
        *reinterpret_cast<uint2*>(qr + c) = quantize8(h[j], k, tie_risk);
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
// (all resident), each holding a block of rows.  The CTA bulk-copies its rows
// into shared memory; thread t then holds R of those rows for one 8-column
// chunk in registers for the whole kernel (chunks padded to a multiple of 32
// so that a warp never straddles two row groups).  Phase 1 ORs the rows'
// outlier flags (column maxima >= tau) into the call's global bitmask, one
// atomic per non-zero 32-column word; after a grid barrier, phase 2 reads the
// call's bitmask and its prefix, gathers the outlier values, zeroes them, takes
// the row maxima (transposed warp reduction, one shared atomic max per row and
// warp) and writes the codes.  X is read from HBM once.
//
// ws.fused: word 0 counts the CTAs that reached the grid barrier (the last one
// returns it to zero), word 1 is the call generation g (the last CTA bumps
// it, which releases the others), words 4.. hold bitmask buffers 0 and 1 of
// ceil(K/32) words.  A call of generation g ORs into buffer g & 1 and zeroes
// buffer (g + 1) & 1, which the previous call used and the next will use.
constexpr int kActFusedThreads = 1024;
constexpr int kActFusedMaxRows = 16;  // rows per CTA
constexpr size_t kActFusedSmemMax = 200 * 1024;

template <int R>
__global__ void __launch_bounds__(kActFusedThreads, 1)
    act_fused_kernel(const __half* __restrict__ X, int64_t M, int64_t K, int64_t ldx, float tau, ActWs ws,
                     int32_t* __restrict__ O, int32_t* __restrict__ n_out, int64_t cap, int8_t* __restrict__ Xq,
                     int64_t ldq, float* __restrict__ rs, __half* __restrict__ Xo, int64_t ldo, int rows_per,
                     int cpad) {
  extern __shared__ __align__(128) uint8_t smem_a[];
  const int nwords = static_cast<int>((K + 31) / 32);
  const int nchunks = static_cast<int>(K / 8);  // K % 8 == 0 on this path
  __half* s_x = reinterpret_cast<__half*>(smem_a);  // [rows_per][K]
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem_a + size_t(rows_per) * size_t(K) * 2);
  uint32_t* s_pre = s_mask + ((nwords + 3) & ~3);
  uint4* s_cm = reinterpret_cast<uint4*>(s_pre + ((nwords + 3) & ~3));  // [kActFusedThreads] column maxima
  __shared__ uint64_t bar;
  __shared__ int s_warp[kActFusedThreads / 32];
  __shared__ uint32_t s_gen;
  __shared__ int s_ok;
  __shared__ uint32_t s_rmax[kActFusedMaxRows];
  __shared__ float s_k[kActFusedMaxRows];
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
  uint32_t* arrived = ws.fused;
  uint32_t* generation = ws.fused + 1;

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (tid < kActFusedMaxRows) s_rmax[tid] = 0u;
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
  uint32_t* buf = ws.fused + 4 + (gen & 1u) * uint32_t(nwords);
  uint32_t* other = ws.fused + 4 + ((gen + 1u) & 1u) * uint32_t(nwords);
  if (blockIdx.x == 0) {
    for (int w = tid; w < nwords; w += kActFusedThreads) other[w] = 0u;
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
  uint32_t fl = 0;
  if (col_ok) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(cm[e]);
      fl |= (f.x >= tau ? 1u : 0u) << (2 * e);
      fl |= (f.y >= tau ? 1u : 0u) << (2 * e + 1);
    }
  }
  uint32_t word = fl << ((8 * cc) & 31);
  word |= __shfl_xor_sync(0xffffffffu, word, 1);
  word |= __shfl_xor_sync(0xffffffffu, word, 2);
  if (g == 0 && col_ok && (cc & 3) == 0 && word != 0u) atomicOr(buf + (cc >> 2), word);

  // grid barrier (every CTA of the grid is resident: at most one per SM); bounded
  __syncthreads();
  if (tid == 0) {
    int ok = 1;
    // (the stall test hook asks for one arrival more than the grid has: the
    // barrier then never completes and every CTA's wait runs out)
    const uint32_t last = gridDim.x - 1u + ((ws.stall & kStallActGridBarrier) ? 1u : 0u);
    if (atom_add_acq_rel_gpu_u32(arrived, 1u) == last) {
      *arrived = 0u;                             // for the next call
      st_release_gpu_u32(generation, gen + 1u);  // releases the others
    } else {
      const uint64_t t0 = globaltimer_ns();
      uint32_t n = 0;
      while (ld_acquire_gpu_u32(generation) == gen) {
        if ((++n & 255u) == 0u && globaltimer_ns() - t0 > wait_limit_ns()) {
          atomicOr(ws.status, kStatusTimeout);
          ok = 0;
          break;
        }
      }
    }
    s_ok = ok && loaded;
  }
  __syncthreads();

  // phase 2: the call's bitmask and its popcount prefix
  int cnt = 0;
  const int wpt = (nwords + kActFusedThreads - 1) / kActFusedThreads;
  const int w0 = tid * wpt;
  for (int w = w0; w < w0 + wpt && w < nwords; ++w) {
    const uint32_t bw = __ldcg(buf + w);
    s_mask[w] = bw;
    cnt += __popc(bw);
  }
  int x = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kActFusedThreads / 32; ++w) {
    before += w < warp ? s_warp[w] : 0;
    total += s_warp[w];
  }
  int pos = before + x - cnt;
  for (int w = w0; w < w0 + wpt && w < nwords; ++w) {
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
  if (blockIdx.x == 0 && tid == 0) {
    *n_out = total;
    if (total > cap) atomicOr(ws.status, kStatusOverflow);
  }
  __syncthreads();

  // a4: gather this thread's outlier values; then zero them (0 quantizes to 0)
  const uint32_t gfl = col_ok ? (s_mask[cc >> 2] >> ((cc & 3) * 8)) & 0xFFu : 0u;
  if (gfl != 0u) {
    if (Xo != nullptr) {
      const int b0 = (8 * cc) & 31;
      const uint32_t wd = s_mask[cc >> 2];
      const int base = static_cast<int>(s_pre[cc >> 2]);
#pragma unroll 1
      for (int e = 0; e < 8; ++e) {
        if ((gfl >> e) & 1u) {
          const int q = base + __popc(wd & ((1u << (b0 + e)) - 1u));
          if (q < cap) {
#pragma unroll
            for (int r = 0; r < R; ++r)
              if (m0 + r < nr) Xo[(r0 + m0 + r) * ldo + q] = __ushort_as_half(half_bits_at(h[r], e));
          }
        }
      }
    }
    const uint32_t k0 = ((gfl & 1u) ? 0u : 0xFFFFu) | ((gfl & 2u) ? 0u : 0xFFFF0000u);
    const uint32_t k1 = ((gfl & 4u) ? 0u : 0xFFFFu) | ((gfl & 8u) ? 0u : 0xFFFF0000u);
    const uint32_t k2 = ((gfl & 16u) ? 0u : 0xFFFFu) | ((gfl & 32u) ? 0u : 0xFFFF0000u);
    const uint32_t k3 = ((gfl & 64u) ? 0u : 0xFFFFu) | ((gfl & 128u) ? 0u : 0xFFFF0000u);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      h[r].x &= k0;
      h[r].y &= k1;
      h[r].z &= k2;
      h[r].w &= k3;
    }
  }

  // a2: row maxima over the non-outlier columns
  float pm[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&h[r]);
    const __half2 m2 = __hmax2(__hmax2(__habs2(h2[0]), __habs2(h2[1])), __hmax2(__habs2(h2[2]), __habs2(h2[3])));
    pm[r] = fmaxf(__low2float(m2), __high2float(m2));
  }
  int prow = 0;
  const float pmax = rows_max_transposed<R>(pm, 32, lane, prow);
  if ((lane & (32 / R - 1)) == 0 && g < groups && m0 + prow < nr) atomicMax(&s_rmax[m0 + prow], __float_as_uint(pmax));
  __syncthreads();
  if (tid < nr) {
    const float sc = __uint_as_float(s_rmax[tid]);
    rs[r0 + tid] = sc;
    s_k[tid] = sc > 0.0f ? __fdiv_rn(127.0f, sc) : 0.0f;
    s_inv[tid] = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
  }
  __syncthreads();

  // a3: codes
  if (s_ok && col_ok) {
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
          *reinterpret_cast<uint2*>(Xq + (r0 + m0 + r) * ldq + 8 * cc) =
              quantize8_exact(h[r], __uint_as_float(s_rmax[m0 + r]), s_inv[m0 + r]);
    }
  }
  // Xq columns [K, ldq) are zero
  if (s_ok) {
    const int pad = static_cast<int>((ldq - K) / 8);
    for (int i = tid; i < pad * nr; i += kActFusedThreads)
      *reinterpret_cast<uint2*>(Xq + (r0 + i / pad) * ldq + K + 8 * (i % pad)) = make_uint2(0u, 0u);
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
  griddep_wait();
  griddep_launch_dependents();
  const int64_t nwords = (K + 31) / 32;
  uint32_t* s_pre = s_mask + nwords;
  build_outlier_set(K, ws, s_mask, s_pre, s_warp, O, cap, n_out);

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

bool act_fused_plan(int64_t M, int64_t K, int64_t ldx, const void* X, int num_sms) {
  if (num_sms <= 0 || ldx % 8 != 0 || K % 8 != 0 || reinterpret_cast<uintptr_t>(X) % 16 != 0) return false;
  const int64_t rows_per = (M + num_sms - 1) / num_sms;
  const int64_t cpad = ((K / 8) + 31) / 32 * 32;  // chunks padded to whole warps
  if (cpad > kActFusedThreads) return false;
  const int64_t groups = kActFusedThreads / cpad;
  const int64_t r = (rows_per + groups - 1) / groups;
  const size_t mask_bytes = static_cast<size_t>((K + 31) / 32) * sizeof(uint32_t);
  const size_t smem = size_t(rows_per) * size_t(K) * 2 + 2 * ((mask_bytes + 15) / 16 * 16) +
                      size_t(kActFusedThreads) * 16;
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
    const size_t smem = size_t(rows_per) * size_t(K) * 2 + 2 * ((mask_bytes + 15) / 16 * 16) +
                        size_t(kActFusedThreads) * 16;
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

  cfg.gridDim = dim3(static_cast<unsigned>((K + kScanCols - 1) / kScanCols),
                     static_cast<unsigned>((M + kScanRows - 1) / kScanRows));
  cfg.dynamicSmemBytes = 0;
  cudaError_t e = vec_ok ? cudaLaunchKernelEx(&cfg, scan_columns_kernel<true>, x, M, K, ldx, tau, ws)
                         : cudaLaunchKernelEx(&cfg, scan_columns_kernel<false>, x, M, K, ldx, tau, ws);
  if (e != cudaSuccess) return e;

  cfg.dynamicSmemBytes = 2 * mask_bytes;  // bitmask + popcount prefix
  __half* xo = static_cast<__half*>(Xo);
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
