// decode_gemv.cu -- the whole path a1-a7 in one kernel for calls with M <= 8
// rows of X, laid out as a matrix-vector product: no split of K at all.
//
// "8-bit Matrix Multiplication for Large Language Models", Summary &
// Methodology Analysis (outlier feature dimensions in 16-bit, the rest
// vector-wise int8, dequantize by the outer product of row and column
// constants); "Compress your LLMs", bullets Vector-wise quantization and
// Mixed-precision decomposition.
//
// Such a call moves N x K bytes of Wq and does almost no arithmetic, so it is
// bound by HBM.  Each CTA owns a block of consecutive Wq rows (output columns)
// with their whole K range: one contiguous range of bytes, fetched by a single
// bulk copy issued before griddepcontrol.wait, since the weight does not depend
// on the preceding kernel.  The CTA keeps little else in shared memory, so two
// CTAs fit on an SM: while one call computes, the CTAs of the next call (a
// programmatic dependent launch) are already resident and streaming their
// weight rows, and back-to-back calls keep HBM busy.
//
// The activation step runs in registers.  Warp w owns the columns
// [K/8 w, K/8 (w+1)); lane L of it holds 16 consecutive columns for all M rows,
// flags the columns with |x| >= tau in some row, and takes the row maxima over
// the rest; one barrier combines the warps' maxima into the row scales, and
// the lane quantizes its columns.  With at most four rows of X the lane then
// takes the dot products of its own columns with every Wq row on the CUDA
// cores (dp4a) and the warp adds them across its lanes.  With more rows the
// codes go to the lanes that use them as the B operand of the warp-level int8
// MMA (m16n8k32, the X rows as the N side), whose fragments are loaded 16
// bytes at a time: inside each 64-column chunk, lane quarter t supplies
// columns 16t..16t+15, for both operands alike, so the products pair the same
// columns of Wq and Xq.  The int32 sums are exact either way.  The warps'
// partial sums are added in shared memory
// (the weight's space, once it has been used), and one thread per output
// dequantizes, adds the 16-bit outlier product in ascending outlier order and
// the bias, and stores Y.  The first CTA also writes Xq, rs, O, n_o and Xo to
// the workspace.  Every wait is bounded.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace llmint8 {

namespace {

constexpr int kThreadsV = 256;  // 8 warps
constexpr int kWarpsV = kThreadsV / 32;
constexpr int kRowsV = 8;       // rows of X: the MMA's N
constexpr int kChunksV = 8;     // 64-column chunks per warp at most: K <= 4096
constexpr int kTilesV = 4;      // 16-row tiles of Wq per CTA at most
constexpr int kListV = 32;      // outlier columns listed in shared memory
constexpr int kPreV = 8;        // outlier terms whose operands are loaded ahead of the MMA, per output

// Byte offsets in the dynamic shared memory.
struct LayoutV {
  uint32_t w, mask, pmax, cnt, list, rs, bar, total;
  __host__ __device__ LayoutV(int rb, int64_t ldk, int64_t K, int tiles) {
    const uint32_t wbytes = static_cast<uint32_t>(rb) * static_cast<uint32_t>(ldk);
    const uint32_t part = static_cast<uint32_t>(kWarpsV * tiles * 16 * 8 * 4);
    uint32_t o = 0;
    w = o;     // Wq rows [rb][ldk] int8; after the MMA: int32 [warp][tile][16][8] partial sums
    o += wbytes > part ? wbytes : part;
    o = (o + 15u) & ~15u;
    mask = o;  // uint32 [K / 32] the call's outlier bitmask
    o += static_cast<uint32_t>(K / 8);
    pmax = o;  // float [warp][8] row maxima of each warp's columns
    o += kWarpsV * kRowsV * 4;
    cnt = o;   // int [warp] outliers in each warp's columns
    o += kWarpsV * 4;
    list = o;  // int [kListV] the first outlier columns, ascending
    o += kListV * 4;
    rs = o;    // float [8] row scales
    o += kRowsV * 4;
    bar = o;   // mbarriers: Wq landed; a second one nothing arrives on (stall test hook)
    o += 16;
    total = o;
  }
};

// Column index of the t-th outlier (t < n_o), walking the bitmask.  Only used
// past the staged list (more than kListV outliers).
__device__ __noinline__ int outlier_col_at(int t, const uint32_t* s_mask, int nwords) {
  int seen = 0;
  for (int w = 0; w < nwords; ++w) {
    const int c = __popc(s_mask[w]);
    if (seen + c > t) {
      uint32_t bits = s_mask[w];
      for (int skip = t - seen; skip > 0; --skip) bits &= bits - 1;
      return w * 32 + __ffs(bits) - 1;
    }
    seen += c;
  }
  return 0;
}

// Sum of R per-lane values over the 32 lanes, halving the vector at each
// step: afterwards the lane holds the total of value `row`, which is the
// lane's top log2(R) bits (lanes that differ only in the lower 5 - log2(R)
// bits hold the same total).
template <int R>
__device__ __forceinline__ int32_t rows_sum_transposed(int32_t (&v)[R], int lane, int& row) {
  int o = 16;
  row = 0;
#pragma unroll
  for (int half = R >> 1; half > 0; half >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const int32_t mine = up ? v[j + half] : v[j];
      const int32_t other = up ? v[j] : v[j + half];
      v[j] = mine + __shfl_xor_sync(0xffffffffu, other, o);
    }
    row += up ? half : 0;
    o >>= 1;
  }
  int32_t x = v[0];
  for (; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// MR: rows of X (1..8), a template parameter so that every per-row loop is
// straight code of the right length.
template <int MR>
__global__ void __launch_bounds__(kThreadsV, 2) decode_gemv_kernel(const GemvArgs p) {
  constexpr int RP = MR <= 1 ? 1 : MR <= 2 ? 2 : MR <= 4 ? 4 : 8;  // rows rounded up to a power of two
  constexpr bool kDp4a = MR <= 4;  // products by dp4a on the CUDA cores, else warp-level MMAs
  extern __shared__ __align__(128) uint8_t smem_v[];
  const int64_t K = p.K;
  const int64_t ldk = p.ldk;
  const int rb_max = p.rows_per;
  const int T = p.tiles;
  const LayoutV lo(rb_max, ldk, K, T);
  uint8_t* sW = smem_v + lo.w;
  int32_t* s_part = reinterpret_cast<int32_t*>(smem_v + lo.w);
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem_v + lo.mask);
  float* s_pmax = reinterpret_cast<float*>(smem_v + lo.pmax);
  int* s_cnt = reinterpret_cast<int*>(smem_v + lo.cnt);
  int* s_list = reinterpret_cast<int*>(smem_v + lo.list);
  float* s_rs = reinterpret_cast<float*>(smem_v + lo.rs);
  uint64_t* wbar = reinterpret_cast<uint64_t*>(smem_v + lo.bar);
  uint64_t* never = wbar + 1;

  const int tid = static_cast<int>(threadIdx.x);
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int n0 = static_cast<int>(blockIdx.x) * rb_max;
  const int rb = min(rb_max, p.N - n0);  // this CTA's rows of Wq (>= 1)
  const int S = static_cast<int>(K / 512);  // 64-column chunks per warp
  const bool first = blockIdx.x == 0;      // this CTA also writes the workspace outputs

  // The CTA's Wq rows are contiguous in memory: one bulk copy.
  if (tid == 0) {
    mbar_init(wbar, 1);
    mbar_init(never, 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    const uint32_t bytes = static_cast<uint32_t>(rb) * static_cast<uint32_t>(ldk);
    mbar_arrive_expect_tx(wbar, bytes);
    bulk_load_1d(sW, p.Wq + int64_t(n0) * ldk, bytes, wbar);
  }
  griddep_wait();  // X may be written by the preceding kernel; Y and the workspace read by it
  griddep_launch_dependents();

  // a1: lane L < 4S holds columns c0 .. c0 + 15 of every row
  const __half* X = static_cast<const __half*>(p.X);
  const bool act = lane < 4 * S;
  const int c0 = 64 * S * warp + 16 * lane;
  uint4 xv[MR][2];
#pragma unroll
  for (int j = 0; j < MR; ++j) {
    if (act) {
      const uint4* src = reinterpret_cast<const uint4*>(X + int64_t(j) * p.ldx + c0);
      xv[j][0] = src[0];
      xv[j][1] = src[1];
    } else {
      xv[j][0] = make_uint4(0u, 0u, 0u, 0u);
      xv[j][1] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  uint32_t fl = 0;  // bit e: column c0 + e is an outlier
  {
    __half2 cm[8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2* h2 = reinterpret_cast<const __half2*>(&xv[0][h]);
#pragma unroll
      for (int e = 0; e < 4; ++e) cm[4 * h + e] = __habs2(h2[e]);
    }
#pragma unroll
    for (int j = 1; j < MR; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __half2* h2 = reinterpret_cast<const __half2*>(&xv[j][h]);
#pragma unroll
        for (int e = 0; e < 4; ++e) cm[4 * h + e] = __hmax2(cm[4 * h + e], __habs2(h2[e]));  // NaN never wins
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 f = __half22float2(cm[e]);
      fl |= (f.x >= p.tau ? 1u : 0u) << (2 * e);
      fl |= (f.y >= p.tau ? 1u : 0u) << (2 * e + 1);
    }
    if (!act) fl = 0;
  }

  // a2: zero the outlier columns, row maxima over the rest
  float pm[RP];
#pragma unroll
  for (int j = 0; j < RP; ++j) pm[j] = 0.0f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t km[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int b = 8 * h + 2 * e;
      km[e] = (((fl >> b) & 1u) ? 0u : 0xFFFFu) | (((fl >> (b + 1)) & 1u) ? 0u : 0xFFFF0000u);
    }
#pragma unroll
    for (int j = 0; j < MR; ++j) {
      xv[j][h].x &= km[0];
      xv[j][h].y &= km[1];
      xv[j][h].z &= km[2];
      xv[j][h].w &= km[3];
      const __half2* h2 = reinterpret_cast<const __half2*>(&xv[j][h]);
      const __half2 m2 =
          __hmax2(__hmax2(__habs2(h2[0]), __habs2(h2[1])), __hmax2(__habs2(h2[2]), __habs2(h2[3])));
      pm[j] = fmaxf(pm[j], fmaxf(__low2float(m2), __high2float(m2)));
    }
  }
  int prow = 0;
  const float wmax = rows_max_transposed<RP>(pm, 32, lane, prow);
  if ((lane & 3) == 0 && prow < MR) s_pmax[warp * kRowsV + prow] = wmax;

  // outliers of this warp: count, lane prefix, bitmask words
  const int cnt = __popc(fl);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_cnt[warp] = incl;
  const uint32_t pair = fl | (__shfl_xor_sync(0xffffffffu, fl, 1) << 16);
  if (act && (lane & 1) == 0) s_mask[c0 >> 5] = pair;
  __syncthreads();

  // row scales (lane j of every warp computes row j's), outlier positions
  float sc = 0.0f;
  if (lane < MR) {
#pragma unroll
    for (int v = 0; v < kWarpsV; ++v) sc = fmaxf(sc, s_pmax[v * kRowsV + lane]);
  }
  const float kq = sc > 0.0f ? __fdiv_rn(127.0f, sc) : 0.0f;
  const float inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
  if (warp == 0 && lane < MR) {
    s_rs[lane] = sc;
    if (first) p.rs[lane] = sc;
  }
  int base = 0, n_o = 0;
#pragma unroll
  for (int v = 0; v < kWarpsV; ++v) {
    const int c = s_cnt[v];
    base += v < warp ? c : 0;
    n_o += c;
  }
  const bool overflow = n_o > p.cap;

  // a3: codes of this lane's columns, every row
  uint32_t q[MR][4];
#pragma unroll
  for (int j = 0; j < MR; ++j) {
    const float kj = __shfl_sync(0xffffffffu, kq, j);
    const float sj = __shfl_sync(0xffffffffu, sc, j);
    const float ij = __shfl_sync(0xffffffffu, inv, j);
    bool ra = false, rc = false;
    uint2 a = quantize8(xv[j][0], kj, ra);
    uint2 b = quantize8(xv[j][1], kj, rc);
    if (ra) a = quantize8_exact(xv[j][0], sj, ij);  // rare
    if (rc) b = quantize8_exact(xv[j][1], sj, ij);
    q[j][0] = act ? a.x : 0u;
    q[j][1] = act ? a.y : 0u;
    q[j][2] = act ? b.x : 0u;
    q[j][3] = act ? b.y : 0u;
    if (first && act)
      *reinterpret_cast<uint4*>(p.Xq + int64_t(j) * p.ldq + c0) = make_uint4(q[j][0], q[j][1], q[j][2], q[j][3]);
  }

  // a4: the outlier list (ascending), and for the first CTA O, n_o, Xo
  if (fl != 0u) {
    int pos = base + incl - cnt;
    uint32_t bits = fl;
    while (bits) {
      const int col = c0 + __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < kListV) s_list[pos] = col;
      if (first && pos < p.cap) {
        p.O[pos] = col;
        if (p.Xo != nullptr) {
          __half* Xo = static_cast<__half*>(p.Xo);
#pragma unroll 1
          for (int m = 0; m < MR; ++m) Xo[int64_t(m) * p.ldo + pos] = X[int64_t(m) * p.ldx + col];
        }
      }
      ++pos;
    }
  }
  if (first) {
    if (tid == 0) {
      *p.n_out = n_o;
      if (overflow) atomicOr(p.status, kStatusOverflow);
    }
    const int pad = static_cast<int>((p.ldq - K) / 8);  // Xq columns [K, ldq) are zero
#pragma unroll 1
    for (int i = tid; i < pad * MR; i += kThreadsV)
      *reinterpret_cast<uint2*>(p.Xq + int64_t(i / pad) * p.ldq + K + 8 * (i % pad)) = make_uint2(0u, 0u);
  }
  __syncthreads();  // the outlier list

  // output (row r of this CTA, X row m) of this thread: warp w takes X row
  // w % MR and the Wq rows lane + 32 (w / MR) + 32 G i, i = 0, 1
  constexpr int G = kWarpsV / MR;  // warps per X row
  const int em = warp % MR;
  const int eg = warp / MR;
  const bool eact = eg < G;
  const int n_use = overflow ? 0 : n_o;
  const __half* W = static_cast<const __half*>(p.W);
  const __half* bias = static_cast<const __half*>(p.bias);
  // the epilogue's operands from global memory, loaded while the MMAs run:
  // column scales, bias, and the first outlier terms' x and 16-bit w
  const int npre = W != nullptr ? min(n_use, kPreV) : 0;
  // (16-bit values stay one per 32-bit register, unconverted, so that no
  // instruction waits on these loads before the epilogue)
  const unsigned short* Xb = static_cast<const unsigned short*>(p.X);
  const unsigned short* Wb = static_cast<const unsigned short*>(p.W);
  const unsigned short* Bb = static_cast<const unsigned short*>(p.bias);
  float csw[2] = {0.0f, 0.0f};
  uint32_t bv[2] = {0u, 0u};
  uint32_t px[kPreV], pw[2][kPreV];
#pragma unroll
  for (int t = 0; t < kPreV; ++t) px[t] = pw[0][t] = pw[1][t] = 0u;
  if (eact) {
#pragma unroll
    for (int t = 0; t < kPreV; ++t)
      if (t < npre) px[t] = Xb[int64_t(em) * p.ldx + s_list[t]];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = lane + 32 * (eg + G * i);
      if (r < rb) {
        const int n = n0 + r;
        csw[i] = __ldg(p.cs + n);
        if (bias != nullptr) bv[i] = Bb[n];
#pragma unroll
        for (int t = 0; t < kPreV; ++t)
          if (t < npre) pw[i][t] = Wb[int64_t(s_list[t]) * p.ldw + n];
      }
    }
  }

  // a5: int8 products
  // (the stall test hook waits on a barrier that nothing arrives on instead:
  // the wait runs out, the copy itself still lands and is waited for below)
  const bool wok = mbar_wait((p.stall & kStallGemvWeight) ? never : wbar, 0, p.status);
  int32_t d[kTilesV][4];
#pragma unroll
  for (int tl = 0; tl < kTilesV; ++tl) d[tl][0] = d[tl][1] = d[tl][2] = d[tl][3] = 0;
  // few rows of X: each lane takes the dot products of its own 16 columns
  // with every Wq row (dp4a), then the warp sums them over its lanes, in
  // groups of RG Wq rows (lane L ends with row RG gi + (L >> (5 - log2 RG)))
  constexpr int RG = MR <= 2 ? 32 : 16;       // Wq rows per group
  constexpr int NG = 64 / RG;                 // groups at most (rows_per <= 64)
  constexpr int SH = RG == 32 ? 0 : 1;        // lane bits below the row index
  int32_t rsum[NG][MR];
#pragma unroll
  for (int gi = 0; gi < NG; ++gi)
#pragma unroll
    for (int j = 0; j < MR; ++j) rsum[gi][j] = 0;
  if constexpr (kDp4a) {
#pragma unroll 1
    for (int gi = 0; gi < (rb + RG - 1) / RG; ++gi) {
      int32_t acc[MR][RG];
#pragma unroll
      for (int rr = 0; rr < RG; ++rr) {
        const int r = min(RG * gi + rr, rb - 1);  // rows past rb read row rb - 1, unused
        const uint4 wv = *reinterpret_cast<const uint4*>(sW + int64_t(r) * ldk + (act ? c0 : 0));
#pragma unroll
        for (int j = 0; j < MR; ++j) {
          int32_t a = __dp4a(static_cast<int>(wv.x), static_cast<int>(q[j][0]), 0);
          a = __dp4a(static_cast<int>(wv.y), static_cast<int>(q[j][1]), a);
          a = __dp4a(static_cast<int>(wv.z), static_cast<int>(q[j][2]), a);
          acc[j][rr] = __dp4a(static_cast<int>(wv.w), static_cast<int>(q[j][3]), a);
        }
      }
#pragma unroll
      for (int j = 0; j < MR; ++j) {
        int row = 0;
        const int32_t tot = rows_sum_transposed<RG>(acc[j], lane, row);
#pragma unroll
        for (int k = 0; k < NG; ++k) rsum[k][j] = gi == k ? tot : rsum[k][j];
      }
    }
  } else {
    // the B fragment of chunk c (row g, columns 64 ch + 16 t4 .. + 15) comes
    // from lane 4c + t4, which quantized those columns; even and odd chunks
    // accumulate apart (two independent MMA chains per tile)
    int32_t e[kTilesV][4];
#pragma unroll
    for (int tl = 0; tl < kTilesV; ++tl) e[tl][0] = e[tl][1] = e[tl][2] = e[tl][3] = 0;
    int ra[kTilesV], rc[kTilesV];  // rows past this CTA's read row rb - 1 (in bounds; their sums are not used)
#pragma unroll
    for (int tl = 0; tl < kTilesV; ++tl) {
      ra[tl] = min(tl * 16 + g, rb - 1);
      rc[tl] = min(tl * 16 + g + 8, rb - 1);
    }
#pragma unroll 1
    for (int c = 0; c < S; c += 2) {
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const int cc = c + hc;
        if (cc < S) {
          uint32_t bq[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            uint32_t v = 0u;
#pragma unroll
            for (int j = 0; j < MR; ++j) {
              const uint32_t u = __shfl_sync(0xffffffffu, q[j][r], 4 * cc + t4);
              v = g == j ? u : v;
            }
            bq[r] = v;
          }
          const int64_t kof = 64 * int64_t(S * warp + cc) + 16 * t4;
#pragma unroll
          for (int tl = 0; tl < kTilesV; ++tl) {
            if (tl < T) {
              const uint4 ua = *reinterpret_cast<const uint4*>(sW + int64_t(ra[tl]) * ldk + kof);
              const uint4 uc = *reinterpret_cast<const uint4*>(sW + int64_t(rc[tl]) * ldk + kof);
              const uint32_t a0[4] = {ua.x, uc.x, ua.y, uc.y};
              const uint32_t a1[4] = {ua.z, uc.z, ua.w, uc.w};
              if (hc == 0) {
                mma_m16n8k32_s8s32(d[tl], a0, bq[0], bq[1]);
                mma_m16n8k32_s8s32(d[tl], a1, bq[2], bq[3]);
              } else {
                mma_m16n8k32_s8s32(e[tl], a0, bq[0], bq[1]);
                mma_m16n8k32_s8s32(e[tl], a1, bq[2], bq[3]);
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int tl = 0; tl < kTilesV; ++tl) {
      d[tl][0] += e[tl][0];
      d[tl][1] += e[tl][1];
      d[tl][2] += e[tl][2];
      d[tl][3] += e[tl][3];
    }
  }
  if (!__syncthreads_and(wok)) {  // the weight never landed: status has the timeout bit
    if (tid == 0) mbar_wait(wbar, 0, nullptr);  // let the copy finish before the CTA exits
    return;
  }
  // a6: the warps' partial sums, [warp][tile][16][8], in the weight's space
  if constexpr (kDp4a) {
    if ((lane & ((1 << SH) - 1)) == 0) {
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        const int r = RG * gi + (lane >> SH);
        if (r < rb) {
#pragma unroll
          for (int j = 0; j < MR; ++j) s_part[(warp * T + (r >> 4)) * 128 + (r & 15) * 8 + j] = rsum[gi][j];
        }
      }
    }
  } else {
#pragma unroll
    for (int tl = 0; tl < kTilesV; ++tl) {
      if (tl < T) {
        int32_t* pp = s_part + (warp * T + tl) * 128;
        pp[g * 8 + 2 * t4] = d[tl][0];
        pp[g * 8 + 2 * t4 + 1] = d[tl][1];
        pp[(g + 8) * 8 + 2 * t4] = d[tl][2];
        pp[(g + 8) * 8 + 2 * t4 + 1] = d[tl][3];
      }
    }
  }
  __syncthreads();

  // a6-a7: dequantize, add the 16-bit outlier product (ascending) and the bias
  if (!eact) return;
  __half* Y = static_cast<__half*>(p.Y);
  const int nwords = static_cast<int>(K / 32);
  const float rsm = s_rs[em];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = lane + 32 * (eg + G * i);
    if (r < rb) {
      const int n = n0 + r;
      const int tl = r >> 4, rr = r & 15;
      int32_t acc = 0;
#pragma unroll
      for (int v = 0; v < kWarpsV; ++v) acc += s_part[(v * T + tl) * 128 + rr * 8 + em];
      if (p.C != nullptr) {  // test hook: the raw accumulator instead of Y
        p.C[int64_t(em) * p.ldc + n] = acc;
        continue;
      }
      float y = static_cast<float>(acc) * rsm * (csw[i] * (1.0f / 16129.0f));
#pragma unroll
      for (int t = 0; t < kPreV; ++t)
        if (t < npre)
          y = fmaf(__half2float(__ushort_as_half(static_cast<unsigned short>(px[t]))),
                   __half2float(__ushort_as_half(static_cast<unsigned short>(pw[i][t]))), y);
#pragma unroll 1
      for (int t = npre; t < n_use; ++t) {  // many outliers, or no 16-bit weight: fetched one by one
        const int col = t < kListV ? s_list[t] : outlier_col_at(t, s_mask, nwords);
        // without the 16-bit weight, the outlier rows come from the int8 codes
        const float w = W != nullptr ? __half2float(W[int64_t(col) * p.ldw + n])
                                     : __half2float(__ushort_as_half(dequant_weight_bits(
                                           static_cast<int8_t>(p.Wq[int64_t(n) * ldk + col]), csw[i])));
        y = fmaf(__half2float(X[int64_t(em) * p.ldx + col]), w, y);
      }
      y += __half2float(__ushort_as_half(static_cast<unsigned short>(bv[i])));  // the bias, added last (0 without one)
      Y[int64_t(em) * p.ldy + n] = __float2half_rn(overflow ? __int_as_float(0x7fc00000) : y);
    }
  }
}

}  // namespace

bool decode_gemv_plan(int M, int N, int K, int64_t ldk, int num_sms, int* rows_per, int* tiles) {
  if (M < 1 || M > kRowsV || N < 1 || K < 512 || K % 512 != 0 || K > 512 * kChunksV || ldk < K || ldk % 16 != 0 ||
      num_sms < 1)
    return false;
  const int rb = (N + num_sms - 1) / num_sms;
  const int t = (rb + 15) / 16;
  if (t > kTilesV) return false;
  if (LayoutV(rb, ldk, K, t).total > 227u * 1024u) return false;
  *rows_per = rb;
  *tiles = t;
  return true;
}

cudaError_t launch_decode_gemv(const GemvArgs& a, cudaStream_t stream, bool pdl) {
  static int smem_set[64][kRowsV] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (a.M < 1 || a.M > kRowsV) return cudaErrorInvalidValue;
  const LayoutV lo(a.rows_per, a.ldk, a.K, a.tiles);
  if (static_cast<int>(lo.total) > smem_set[dev][a.M - 1]) {
    const void* fn[kRowsV] = {reinterpret_cast<const void*>(decode_gemv_kernel<1>),
                              reinterpret_cast<const void*>(decode_gemv_kernel<2>),
                              reinterpret_cast<const void*>(decode_gemv_kernel<3>),
                              reinterpret_cast<const void*>(decode_gemv_kernel<4>),
                              reinterpret_cast<const void*>(decode_gemv_kernel<5>),
                              reinterpret_cast<const void*>(decode_gemv_kernel<6>),
                              reinterpret_cast<const void*>(decode_gemv_kernel<7>),
                              reinterpret_cast<const void*>(decode_gemv_kernel<8>)};
    e = cudaFuncSetAttribute(fn[a.M - 1], cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(lo.total));
    if (e != cudaSuccess) return e;
    smem_set[dev][a.M - 1] = static_cast<int>(lo.total);
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((a.N + a.rows_per - 1) / a.rows_per));
  cfg.blockDim = dim3(kThreadsV);
  cfg.dynamicSmemBytes = lo.total;
  cfg.stream = stream;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  switch (a.M) {
    case 1: return cudaLaunchKernelEx(&cfg, decode_gemv_kernel<1>, a);
    case 2: return cudaLaunchKernelEx(&cfg, decode_gemv_kernel<2>, a);
    case 3: return cudaLaunchKernelEx(&cfg, decode_gemv_kernel<3>, a);
    case 4: return cudaLaunchKernelEx(&cfg, decode_gemv_kernel<4>, a);
    case 5: return cudaLaunchKernelEx(&cfg, decode_gemv_kernel<5>, a);
    case 6: return cudaLaunchKernelEx(&cfg, decode_gemv_kernel<6>, a);
    case 7: return cudaLaunchKernelEx(&cfg, decode_gemv_kernel<7>, a);
    case 8: return cudaLaunchKernelEx(&cfg, decode_gemv_kernel<8>, a);
    default: return cudaErrorInvalidValue;
  }
}

// Test hook: this file's wait bound (see ptx.cuh).
cudaError_t set_debug_waits_decode_gemv(uint64_t limit_ns) { return set_debug_waits_in_this_file(limit_ns); }

}  // namespace llmint8
