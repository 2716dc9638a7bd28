// decode_fused.cu -- the whole path a1-a7 in one kernel for decode-shaped calls
// (M <= 32 rows of X), where the cost is streaming Wq (N x K bytes) from HBM
// and the launch-to-launch latency of a multi-kernel path would dominate it.
//
// "8-bit Matrix Multiplication for Large Language Models", Summary &
// Methodology Analysis (outlier feature dimensions in 16-bit, the rest
// vector-wise int8, dequantize by the outer product of row and column
// constants); "Compress your LLMs", bullets Vector-wise quantization and
// Mixed-precision decomposition.
//
// Layout of the work.  The N/128 tiles of Wq rows are each given a cluster of
// S CTAs (S = 1, 2, 4 or 8) that split the tile's K range: CTA r owns K
// columns [r*kb*128, (r+1)*kb*128).  The quantized activation a CTA needs is
// exactly that column range of Xq, and the outlier decision for a column needs
// only that column of X, so each CTA
//   1. streams its Wq blocks with TMA (issued before anything else: they do
//      not depend on the preceding kernel),
//   2. loads its column range of X (all M rows) into registers, takes the
//      column maxima (a1) and the row maxima over its non-outlier columns,
//   3. pushes its outlier bitmask words and row maxima into every CTA of its
//      cluster through distributed shared memory (stores and remote atomic
//      max before one cluster barrier, so nothing is read remotely after it),
//      which gives every CTA the call's outlier set O and the row scales rs
//      (a2) -- no grid-wide synchronisation and no workspace round trip,
//   4. quantizes its range (a3) straight into the MMA's shared-memory operand
//      (128-byte swizzle, K-major), and the first cluster also writes Xq, rs,
//      O, n_o and the gathered outlier columns Xo (a4) to the workspace,
//   5. runs tcgen05.mma kind::i8 (M = 128 Wq rows, N = 16 or 32 padded X
//      rows) into TMEM (a5),
//   6. reduces the S partial accumulators exactly in int32 through
//      distributed shared memory: CTA r receives the 128/S rows it owns from
//      every CTA of the cluster (second cluster barrier), then applies the
//      dequantization, the fp16 outlier product over O read from X and W
//      (a6), and stores its rows of Y as fp16 (a7).
// The kernel runs once per call and is latency-bound: K is split finely enough
// that a CTA's whole Wq range fits its ring (no refills after the activation
// step), its shared memory fits two CTAs per SM so that the next call's CTAs
// become resident and start their Wq stream while this call finishes
// (programmatic dependent launch), rows per thread are a template parameter,
// loops that need no register arrays stay rolled, and values fetched for the
// epilogue stay raw until the step that needs them.  Every mbarrier wait is bounded; the cluster barriers are reached by
// every thread on every path.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace llmint8 {

namespace {

constexpr int kTileN = 128;                  // Wq rows per tile (MMA M)
constexpr int kKB = kGemmBK;                 // K bytes per block
constexpr int kThreadsF = 288;               // warp 0 TMA; warps 1-8 activation; warp 1 MMA; warps 5-8 epilogue
constexpr int kActThreads = 256;
constexpr int kOList = 32;                   // outliers whose column index and X values are staged
constexpr int kWS = 16;                      // outliers whose W values are staged
constexpr uint32_t kBytesAF = kTileN * kKB;  // 16 KB
// TMEM columns per CTA (two CTAs may share an SM's 512): the K steps of the
// MMA rotate over kTmemCols / NP independent accumulators (8 or 4), so that
// they do not form one long dependent chain; the epilogue adds them up.
constexpr uint32_t kTmemCols = 128;
// Dynamic shared memory that lets two CTAs share an SM (228 KB per SM, 1 KB
// reserved per CTA).
constexpr uint32_t kTwoPerSmBytes = 113u * 1024u;

// Byte offsets in the (1024-aligned) dynamic shared memory.
struct LayoutF {
  uint32_t a, b, red, xo, w, cm, mask, pre, ol, row, warp, bars, misc, total;
  __host__ __device__ LayoutF(int np, int kb_per, int stages, int nwords) {
    uint32_t o = 0;
    a = o;     // Wq ring: stages x [128 rows][128 B], 128-byte swizzle
    o += stages * kBytesAF;
    b = o;     // Xq of this CTA's K range: kb_per x [np rows][128 B], 128-byte swizzle
    o += kb_per * np * kKB;
    red = o;   // int32 [S][np][128/S]: partial sums of the rows this CTA finishes
    o += kTileN * np * 4;
    xo = o;    // fp16 [np][kOList]: X values of the first outliers
    o += np * kOList * 2;
    w = o;     // fp16 [kWS][128/S]: W values of the first outliers for the finished rows
    o += kWS * kTileN * 2;
    cm = o;    // uint4 [256]: column maxima per row group
    o += kActThreads * 16;
    mask = o;  // uint32 [nwords]: the call's outlier bitmask
    o += ((nwords + 3) & ~3) * 4;
    pre = o;   // uint32 [nwords]: outliers before each word
    o += ((nwords + 3) & ~3) * 4;
    ol = o;    // int32 [kOList]: first outlier columns
    o += kOList * 4;
    row = o;   // 4 x [32]: row maxima (float bits, max over the cluster), rs, 127/rs, 1/rs
    o += 4 * 32 * 4;
    warp = o;  // int [8]: scan partials
    o += 8 * 4;
    bars = (o + 7u) & ~7u;  // full[stages], empty[stages], tmem full, drain
    o = bars + (2 * stages + 2) * 8;
    misc = o;  // TMEM address, abort flag
    o += 16;
    total = o + 1024;  // alignment slack
  }
};

__device__ __forceinline__ void red_max_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.max.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Exclusive prefix sum over the 256 activation threads (warps 1-8).
__device__ __forceinline__ int act_exclusive_scan(int v, int* s_warp, int& total) {
  const int lane = static_cast<int>(threadIdx.x & 31u);
  const int aw = static_cast<int>(threadIdx.x >> 5) - 1;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[aw] = x;
  named_bar_sync(1, kActThreads);
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int t = s_warp[w];
    before += w < aw ? t : 0;
    total += t;
  }
  return before + x - v;
}

// Column index of the t-th outlier (t < n_o) from the bitmask and its prefix.
__device__ __noinline__ int outlier_at(int t, const uint32_t* s_mask, const uint32_t* s_pre, int nwords) {
  int lo = 0, hi = nwords - 1;  // last word whose prefix is <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<int>(s_pre[mid]) <= t) lo = mid;
    else hi = mid - 1;
  }
  uint32_t bits = s_mask[lo];
  for (int skip = t - static_cast<int>(s_pre[lo]); skip > 0; --skip) bits &= bits - 1;
  return lo * 32 + __ffs(bits) - 1;
}

template <int NP, int R, int MINB>
__global__ void __launch_bounds__(kThreadsF, MINB)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tmA, const FusedArgs p) {
  extern __shared__ uint8_t smem_raw[];
  const int nwords = (p.K + 31) / 32;
  const int P = p.stages;
  const LayoutF lo(NP, p.kb_per, P, nwords);
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base + lo.a;
  uint8_t* sB = base + lo.b;
  int32_t* s_red = reinterpret_cast<int32_t*>(base + lo.red);
  __half* s_xo = reinterpret_cast<__half*>(base + lo.xo);
  __half* s_w = reinterpret_cast<__half*>(base + lo.w);
  uint4* s_cm = reinterpret_cast<uint4*>(base + lo.cm);
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(base + lo.mask);
  uint32_t* s_pre = reinterpret_cast<uint32_t*>(base + lo.pre);
  int32_t* s_ol = reinterpret_cast<int32_t*>(base + lo.ol);
  uint32_t* s_rmax = reinterpret_cast<uint32_t*>(base + lo.row);
  float* s_rs = reinterpret_cast<float*>(base + lo.row) + 32;
  float* s_k = s_rs + 32;
  float* s_inv = s_k + 32;
  int* s_warp = reinterpret_cast<int*>(base + lo.warp);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + lo.bars);
  uint64_t* empty = full + P;
  uint64_t* tfull = empty + P;
  uint64_t* drain = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + lo.misc);
  volatile int* abort = reinterpret_cast<volatile int*>(base + lo.misc + 4);

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const int S = p.splits;
  const int log2s = __ffs(S) - 1;
  const int RO = kTileN >> log2s;  // Wq rows of the tile each CTA of the cluster finishes
  const int tile = static_cast<int>(blockIdx.x) / S;
  const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
  const bool first_tile = tile == 0;  // this cluster also writes the workspace outputs
  const int nkb_total = (p.K + kKB - 1) / kKB;
  const int kb0 = static_cast<int>(rank) * p.kb_per;
  const int nkb = max(0, min(p.kb_per, nkb_total - kb0));
  const int n0 = tile * kTileN;
  const int c0 = kb0 * kKB;                 // first column of this CTA's K range
  const int c1 = min(p.K, c0 + nkb * kKB);  // end of the range
  const int pre = min(nkb, P);
  bool mma_issued = false;     // warp 1, lane 0: MMAs were issued
  uint32_t issued_phase = 0u;  // warp 0, lane 0: bit st = phase of the last Wq load into stage st

  if (threadIdx.x == 0) {
    for (int i = 0; i < P; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
  }
  if (threadIdx.x < 32) s_rmax[threadIdx.x] = 0u;
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Weight stream first: it does not depend on the preceding kernel.
  if (warp == 0 && lane == 0) {
    const uint64_t hint_w = policy_evict_first();  // Wq is streamed once
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&full[i], kBytesAF);
      tma_load_2d(sA + i * kBytesAF, &tmA, &full[i], (kb0 + i) * kKB, n0, hint_w);
    }
    // the rest of the range (when it is longer than the ring) into L2
    for (int i = pre; i < nkb; ++i) tma_prefetch_l2_2d(&tmA, (kb0 + i) * kKB, n0);
  }
  // barrier 0 (arrive now, wait before the first remote access): every CTA of
  // the cluster has started and initialised its shared memory
  if (S > 1) {
    __syncwarp();
    cluster_arrive();
  }

  griddep_wait();  // X may be written by the preceding kernel; Y and the workspace read by it
  // The next launch on the stream may get resident now: every kernel of this
  // library waits (griddepcontrol.wait) for this grid to complete before it
  // touches memory this grid reads or writes.
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------ Wq producer (ring refills)
    if (S > 1) {
      cluster_wait();    // barrier 0
      cluster_arrive();  // barrier 1: nothing to publish
    }
    if (lane == 0) {
      const uint64_t hint_w = policy_evict_first();
      for (int i = P; i < nkb; ++i) {
        const int st = i % P;
        const uint32_t ph = static_cast<uint32_t>(i / P - 1) & 1u;
        if (!mbar_wait_abortable(&empty[st], ph, p.status, abort)) break;
        mbar_arrive_expect_tx(&full[st], kBytesAF);
        tma_load_2d(sA + st * kBytesAF, &tmA, &full[st], (kb0 + i) * kKB, n0, hint_w);
        issued_phase = (issued_phase & ~(1u << st)) | ((static_cast<uint32_t>(i / P) & 1u) << st);
      }
    }
    __syncwarp();
    if (S > 1) {
      cluster_wait();
      cluster_arrive();  // barrier 2: nothing to send
      cluster_wait();
    }
  } else {
    // ------------------------------------------------ activation: warps 1-8
    const int at = static_cast<int>(threadIdx.x) - 32;
    const int C = p.kb_per * (kKB / 8);  // 8-column chunks in a full range: 16 .. 256, a power of two
    const int log2c = __ffs(C) - 1;
    const int Gq = kActThreads >> log2c;  // row groups; the host's plan gives R * Gq >= M
    const int cc = at & (C - 1);
    const int g = at >> log2c;
    const int c = c0 + 8 * cc;           // first of this thread's 8 columns
    const bool col_ok = c < c1;
    const int m0 = g * R;
    const __half* X = static_cast<const __half*>(p.X);
    const __half* W = static_cast<const __half*>(p.W);

    uint4 h[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int m = m0 + r;
      h[r] = (col_ok && m < p.M) ? __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * p.ldx + c))
                                 : make_uint4(0u, 0u, 0u, 0u);
    }

    // a1: column maxima of |x| over this thread's rows, then over the row groups
    __half2 cm[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) cm[e] = __half2half2(__ushort_as_half(0));
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const __half2* h2 = reinterpret_cast<const __half2*>(&h[r]);
#pragma unroll
      for (int e = 0; e < 4; ++e) cm[e] = __hmax2(cm[e], __habs2(h2[e]));
    }
    if (Gq > 1) {
      s_cm[at] = *reinterpret_cast<const uint4*>(cm);
      named_bar_sync(1, kActThreads);
      for (int gg = 0; gg < Gq; ++gg) {
        const uint4 o = s_cm[gg * C + cc];
        const __half2* o2 = reinterpret_cast<const __half2*>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) cm[e] = __hmax2(cm[e], o2[e]);
      }
    }
    uint32_t fl = 0;  // outlier flags of the 8 columns (|x| >= tau in some row)
    if (col_ok) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float v = (e & 1) ? __high2float(cm[e >> 1]) : __low2float(cm[e >> 1]);
        if (c + e < c1 && v >= p.tau) fl |= 1u << e;
      }
    }
    // the 32-bit outlier word of columns [c & ~31, +32): four neighbouring lanes
    uint32_t word = fl << (c & 31);
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    uint32_t keep[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      keep[e] = (((fl >> (2 * e)) & 1u) ? 0u : 0xFFFFu) | (((fl >> (2 * e + 1)) & 1u) ? 0u : 0xFFFF0000u);

    // outlier columns are zeroed in the registers (0 quantizes to 0); a2 on
    // this range: row maxima of |x| over the non-outlier columns
    float pm[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      h[r].x &= keep[0];
      h[r].y &= keep[1];
      h[r].z &= keep[2];
      h[r].w &= keep[3];
      const __half2* h2 = reinterpret_cast<const __half2*>(&h[r]);
      __half2 m2 = __habs2(h2[0]);
#pragma unroll
      for (int e = 1; e < 4; ++e) m2 = __hmax2(m2, __habs2(h2[e]));
      pm[r] = fmaxf(__low2float(m2), __high2float(m2));  // NaN never wins
    }
    const int width = C < 32 ? C : 32;  // lanes of a warp that share a row group
    int prow = 0;
    const float pmax = rows_max_transposed<R>(pm, width, static_cast<int>(lane), prow);
    const bool row_writer = (static_cast<int>(lane) & (width / R - 1)) == 0 && m0 + prow < p.M;
    const bool word_writer = g == 0 && (cc & 3) == 0 && col_ok;

    // push this CTA's outlier words and row maxima into every CTA of the
    // cluster (itself included); barrier 1 then makes them visible
    if (S > 1) {
      __syncwarp();
      cluster_wait();  // barrier 0
      for (int r = 0; r < S; ++r) {
        if (word_writer) st_cluster_u32(mapa_shared(smem_u32(&s_mask[c >> 5]), static_cast<uint32_t>(r)), word);
        if (row_writer)
          red_max_cluster_u32(mapa_shared(smem_u32(&s_rmax[m0 + prow]), static_cast<uint32_t>(r)), __float_as_uint(pmax));
      }
      __syncwarp();
      cluster_arrive();
      cluster_wait();
    } else {
      if (word_writer) s_mask[c >> 5] = word;
      if (row_writer) atomicMax(&s_rmax[m0 + prow], __float_as_uint(pmax));
      named_bar_sync(1, kActThreads);
    }

    // positions of the outliers: popcount prefix over the words
    uint32_t mw[2];
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int w = 2 * at + j;
      mw[j] = w < nwords ? s_mask[w] : 0u;
      cnt += __popc(mw[j]);
    }
    int n_o = 0;
    const int before = act_exclusive_scan(cnt, s_warp, n_o);
    const bool write_ws = first_tile && rank == 0u;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int w = 2 * at + j;
      if (w < nwords) {
        int pos = before + (j ? __popc(mw[0]) : 0);
        s_pre[w] = static_cast<uint32_t>(pos);
        uint32_t bits = mw[j];
        while (bits) {
          const int col = w * 32 + __ffs(bits) - 1;
          bits &= bits - 1;
          if (pos < kOList) s_ol[pos] = col;
          if (write_ws && pos < p.cap) p.O[pos] = col;
          ++pos;
        }
      }
    }
    if (at < 32) {  // a2: the row scales of the call
      const float s = at < p.M ? __uint_as_float(s_rmax[at]) : 0.0f;
      if (write_ws && at < p.M) p.rs[at] = s;
      s_rs[at] = s;
      s_k[at] = s > 0.0f ? __fdiv_rn(127.0f, s) : 0.0f;
      s_inv[at] = s > 0.0f ? __frcp_rn(s) : 0.0f;
    }
    if (write_ws && at == 0) {
      *p.n_out = n_o;
      if (n_o > p.cap) atomicOr(p.status, kStatusOverflow);
    }
    named_bar_sync(1, kActThreads);
    const bool overflow = n_o > p.cap;
    const int n_use = overflow ? 0 : n_o;

    // What the finishing step reads for the first outliers, loaded now (kept
    // as raw fp16 bits, so nothing waits for them) to overlap the
    // quantization: W[O[t], n] for the rows this CTA finishes (s_w [t][RO])
    // and X[m, O[t]] (s_xo [m][kOList]).
    constexpr int kPW = kWS * kTileN / kActThreads;  // 8
    constexpr int kPX = NP * kOList / kActThreads;   // 2 or 4
    const int tw = min(n_use, kWS);
    const int tx = min(n_use, kOList);
    const unsigned short* Wb = reinterpret_cast<const unsigned short*>(W);
    const unsigned short* Xb = reinterpret_cast<const unsigned short*>(X);
    // (no fp16 weight kept: the code Wq[n, O[t]] and cs[n] instead, turned
    // into the recovered fp16 value when stored)
    unsigned short pf_w[kPW], pf_x[kPX];
    float pf_c[kPW];
#pragma unroll
    for (int u = 0; u < kPW; ++u) {
      const int k = at + u * kActThreads;
      const int t = k >> (7 - log2s), i = k & (RO - 1);
      const int n = n0 + static_cast<int>(rank) * RO + i;
      const bool use = t < tw && n < p.N;
      if (W != nullptr) {
        pf_w[u] = use ? Wb[static_cast<int64_t>(s_ol[t]) * p.ldw + n] : static_cast<unsigned short>(0);
        pf_c[u] = 0.0f;
      } else {
        pf_w[u] = use ? static_cast<unsigned short>(static_cast<uint8_t>(p.Wq[int64_t(n) * p.ldk + s_ol[t]]))
                      : static_cast<unsigned short>(0);
        pf_c[u] = use ? __ldg(p.cs + n) : 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kPX; ++u) {
      const int k = at + u * kActThreads;
      const int m = k / kOList, t = k % kOList;
      pf_x[u] = (m < p.M && t < tx) ? Xb[static_cast<int64_t>(m) * p.ldx + s_ol[t]] : static_cast<unsigned short>(0);
    }

    // a4: the first cluster gathers the outlier columns of X into Xo
    if (first_tile && fl != 0u && p.Xo != nullptr) {
      __half* Xo = static_cast<__half*>(p.Xo);
      const uint32_t wd = s_mask[c >> 5];
      const int wbase = static_cast<int>(s_pre[c >> 5]);
#pragma unroll 1
      for (int e = 0; e < 8; ++e) {
        if ((fl >> e) & 1u) {
          const int pos = wbase + __popc(wd & ((1u << ((c & 31) + e)) - 1u));
          if (pos < p.cap) {
#pragma unroll 1
            for (int m = m0; m < min(m0 + R, p.M); ++m)
              Xo[static_cast<int64_t>(m) * p.ldo + pos] = X[static_cast<int64_t>(m) * p.ldx + c + e];
          }
        }
      }
    }

    // a3: codes into the MMA operand (row m, K-major, 128-byte swizzle) and,
    // for the first cluster, into the workspace's Xq
    if (col_ok) {
      const int kb = cc >> 4;          // K block within the range
      const int u16 = (cc & 15) >> 1;  // 16-byte unit within the 128-byte row
      const uint32_t half8 = (cc & 1) * 8u;
      uint8_t* blk = sB + kb * (NP * kKB);
      uint32_t risk_rows = 0;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int m = m0 + r;
        if (m < p.M) {
          bool risk = false;
          const uint2 code = quantize8(h[r], s_k[m], risk);
          risk_rows |= static_cast<uint32_t>(risk) << r;
          *reinterpret_cast<uint2*>(blk + m * kKB + ((u16 ^ (m & 7)) << 4) + half8) = code;
          if (first_tile) *reinterpret_cast<uint2*>(p.Xq + static_cast<int64_t>(m) * p.ldq + c) = code;
        }
      }
      if (risk_rows != 0u) {  // rare: a value within 2^-15 of a rounding boundary; redo its chunk exactly
#pragma unroll 1
        for (int r = 0; r < R; ++r) {
          if ((risk_rows >> r) & 1u) {
            const int m = m0 + r;
            uint4 u = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * p.ldx + c));
            u.x &= keep[0];
            u.y &= keep[1];
            u.z &= keep[2];
            u.w &= keep[3];
            const uint2 code = quantize8_exact(u, s_rs[m], s_inv[m]);
            *reinterpret_cast<uint2*>(blk + m * kKB + ((u16 ^ (m & 7)) << 4) + half8) = code;
            if (first_tile) *reinterpret_cast<uint2*>(p.Xq + static_cast<int64_t>(m) * p.ldq + c) = code;
          }
        }
      }
    } else if (first_tile && c == p.K && c < p.ldq) {  // Xq columns [K, ldq) are zero
#pragma unroll 1
      for (int m = m0; m < min(m0 + R, p.M); ++m)
        *reinterpret_cast<uint2*>(p.Xq + static_cast<int64_t>(m) * p.ldq + c) = make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kPW; ++u)
      s_w[at + u * kActThreads] = __ushort_as_half(
          W != nullptr ? pf_w[u] : dequant_weight_bits(static_cast<int8_t>(pf_w[u] & 0xFFu), pf_c[u]));
#pragma unroll
    for (int u = 0; u < kPX; ++u) s_xo[at + u * kActThreads] = __ushort_as_half(pf_x[u]);
    fence_proxy_async_smem();  // the operand was written by the generic proxy
    named_bar_sync(1, kActThreads);

    if (warp == 1) {
      // ---------------------------------------------- MMA issue
      if (lane == 0 && nkb > 0) {
        constexpr uint32_t idesc = idesc_i8(kTileN, NP);
        constexpr int kAcc = kTmemCols / NP;  // independent accumulators
        bool ok = true;
        mma_issued = true;
        for (int i = 0; i < nkb; ++i) {
          const int st = i % P;
          const uint32_t ph = static_cast<uint32_t>(i / P) & 1u;
          if (!mbar_wait_abortable(&full[st], ph, p.status, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = smem_desc_k_sw128(smem_u32(sA + st * kBytesAF));
          const uint64_t db = smem_desc_k_sw128(smem_u32(sB + i * (NP * kKB)));
#pragma unroll
          for (int kk = 0; kk < kKB / 32; ++kk) {
            const int step = i * (kKB / 32) + kk;
            mma_i8(tmem_base + static_cast<uint32_t>((step % kAcc) * NP), da + 2u * kk, db + 2u * kk, idesc,
                   step >= kAcc);
          }
          mma_commit(&empty[st]);
        }
        mma_commit(ok ? tfull : drain);
        if (!ok) mbar_wait(drain, 0, nullptr);
      }
      __syncwarp();
      if (S > 1) {
        cluster_arrive();  // barrier 2: nothing to send
        cluster_wait();
      }
    } else if (warp >= 5) {
      // ---------------------------------------------- epilogue: warps 5-8
      const uint32_t q = warp & 3u;                       // TMEM lanes 32q .. 32q+31
      const int et = static_cast<int>((q << 5) | lane);  // accumulator row of this thread
      const int i = et & (RO - 1);                        // row of this CTA's share it finishes
      const int cg = et >> (7 - log2s);                   // and its columns m = cg, cg + S, ...
      const int n = n0 + static_cast<int>(rank) * RO + i;
      const float csw = n < p.N ? __ldg(p.cs + n) : 0.0f;
      const float csn = csw * (1.0f / 16129.0f);
      const float bn = (p.bias != nullptr && n < p.N) ? __half2float(static_cast<const __half*>(p.bias)[n]) : 0.0f;
      uint32_t v[32];
#pragma unroll
      for (int m = 0; m < 32; ++m) v[m] = 0u;
      if (nkb > 0) {
        bool got = mbar_wait_abortable(tfull, 0, p.status, abort);
        got = named_bar_and(2, 128, got);  // the warp-wide TMEM loads need one answer
        if (got) {
          // add up the accumulators that received K steps (32 columns per load)
          const int used = min(4 * nkb, static_cast<int>(kTmemCols) / NP) * NP;
          tc_fence_after();
          for (int col = 0; col < used; col += 32) {
            uint32_t u[32];
            tmem_ld_32x32b_x32(tmem_base + ((q * 32u) << 16) + static_cast<uint32_t>(col), u);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const bool in = col + j < used;
              v[j % NP] += in ? u[j] : 0u;  // int32 sums: exact
            }
          }
        }
      }
      tc_fence_before();

      // exact split-K reduction: accumulator row et goes to the CTA that
      // finishes it, as the slice of this CTA's rank
      const int li = i;
      if (S > 1) {
        const uint32_t dst = mapa_shared(smem_u32(s_red), static_cast<uint32_t>(cg)) +
                             static_cast<uint32_t>((static_cast<int>(rank) * NP * RO + li) * 4);
#pragma unroll
        for (int m = 0; m < NP; ++m) st_cluster_u32(dst + static_cast<uint32_t>(m * RO * 4), v[m]);
        __syncwarp();
        cluster_arrive();  // barrier 2: the partial sums have landed
        cluster_wait();
      } else {
#pragma unroll
        for (int m = 0; m < NP; ++m) s_red[m * kTileN + et] = static_cast<int32_t>(v[m]);
        named_bar_sync(2, 128);
      }

      // a6-a7 for row n and columns m = cg, cg + S, ...: dequantize, add the
      // outlier product in ascending outlier order, store
      __half* Y = static_cast<__half*>(p.Y);
#pragma unroll 1
      for (int m = cg; m < p.M; m += S) {
        int32_t part[8];
#pragma unroll
        for (int src = 0; src < 8; ++src) part[src] = src < S ? s_red[(src * NP + m) * RO + i] : 0;
        const int32_t acc = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
        if (p.C != nullptr) {  // test hook: the raw accumulator instead of Y
          if (n < p.N) p.C[static_cast<int64_t>(m) * p.ldc + n] = acc;
          continue;
        }
        float y = static_cast<float>(acc) * s_rs[m] * csn;
#pragma unroll 4
        for (int t = 0; t < tw; ++t) y = fmaf(__half2float(s_xo[m * kOList + t]), __half2float(s_w[t * RO + i]), y);
#pragma unroll 1
        for (int t = kWS; t < n_use; ++t) {  // outliers past the staged ones
          const int col = t < kOList ? s_ol[t] : outlier_at(t, s_mask, s_pre, nwords);
          const float w = n >= p.N ? 0.0f
                          : W != nullptr
                              ? __half2float(W[static_cast<int64_t>(col) * p.ldw + n])
                              : __half2float(__ushort_as_half(dequant_weight_bits(p.Wq[int64_t(n) * p.ldk + col], csw)));
          const float xv =
              t < kOList ? __half2float(s_xo[m * kOList + t]) : __half2float(X[static_cast<int64_t>(m) * p.ldx + col]);
          y = fmaf(xv, w, y);
        }
        if (p.bias != nullptr) y += bn;  // the linear layer's bias, added last
        if (n < p.N) Y[static_cast<int64_t>(m) * p.ldy + n] = __float2half_rn(overflow ? __int_as_float(0x7fc00000) : y);
      }
    } else {
      // warps 2-4: done
      if (S > 1) {
        __syncwarp();
        cluster_arrive();  // barrier 2
        cluster_wait();
      }
    }
  }

  __syncthreads();
  if (warp == 0 && lane == 0 && *abort) {
    // after a timeout anywhere in the CTA, let the copies in flight land
    // before the CTA exits
    for (int st = 0; st < pre; ++st) mbar_wait(&full[st], (issued_phase >> st) & 1u, nullptr);
  }
  if (warp == 1) {
    // after a timeout the epilogue may not have waited for the MMAs: wait for
    // them (bounded) before the accumulator is freed
    if (lane == 0 && mma_issued && *abort) {
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Rows of X per activation thread for a plan: 256 threads cover the CTA's
// 16 * kb_per chunks of 8 columns in 16 / kb_per row groups.
int rows_per_thread(int M, int kb_per) {
  const int groups = (kActThreads / (kKB / 8)) / kb_per;
  int r = (M + groups - 1) / groups, t = 1;
  while (t < r) t <<= 1;
  return t;
}

template <int NP, int R, int MINB>
cudaError_t launch_fused_variant(const CUtensorMap& tmA, const FusedArgs& a, cudaStream_t stream, bool pdl) {
  static int smem_set[64] = {};
  auto kern = decode_fused_kernel<NP, R, MINB>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const LayoutF lo(NP, a.kb_per, a.stages, (a.K + 31) / 32);
  if (static_cast<int>(lo.total) > smem_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(lo.total));
    if (e != cudaSuccess) return e;
    // all of the SM's unified memory as shared memory, so that two CTAs fit
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    smem_set[dev] = static_cast<int>(lo.total);
  }
  const int tiles = (a.N + kTileN - 1) / kTileN;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (a.splits > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(a.splits);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * a.splits));
  cfg.blockDim = dim3(kThreadsF);
  cfg.dynamicSmemBytes = lo.total;
  cfg.stream = stream;
  cfg.attrs = na ? attr : nullptr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, tmA, a);
}

}  // namespace

bool decode_fused_plan(int M, int N, int K, int num_sms, int* splits, int* kb_per, int* stages) {
  if (M < 1 || M > kDecodeMaxM || N < 1 || K < 1 || K > kFusedMaxK) return false;
  const int np = decode_rows_padded(M);
  const int tiles = (N + kTileN - 1) / kTileN;
  const int nkb = (K + kKB - 1) / kKB;
  const int nwords = (K + 31) / 32;
  auto split = [&](int ctas_per_sm, int* s_out, int* per_out) {
    int s = 8;
    while (s > 1 && (tiles * s > ctas_per_sm * num_sms || s > nkb)) s >>= 1;
    int per = 1;
    while (per * s < nkb) per <<= 1;
    *s_out = s;
    *per_out = per;
  };
  // Two CTAs per SM, each CTA's whole K range in a 4-deep ring (no refills):
  // the next call's CTAs get resident while this call runs.
  int s = 1, per = 1;
  split(2, &s, &per);
  if (per <= 4 && rows_per_thread(M, per) <= 8 && LayoutF(np, per, 4, nwords).total <= kTwoPerSmBytes) {
    *splits = s;
    *kb_per = per;
    *stages = 4;
    return true;
  }
  // Otherwise one CTA per SM with an 8-deep ring (refills come from L2).
  split(1, &s, &per);
  if (per * np * kKB > kFusedXqBytes || per * (kKB / 8) > kActThreads || rows_per_thread(M, per) > 16) return false;
  *splits = s;
  *kb_per = per;
  *stages = 8;
  return LayoutF(np, per, 8, nwords).total <= 227u * 1024u;
}

cudaError_t launch_decode_fused(const CUtensorMap& tmA, const FusedArgs& a, cudaStream_t stream, bool pdl) {
  const int r = rows_per_thread(a.M, a.kb_per);
  const bool np16 = decode_rows_padded(a.M) == 16;
  if (a.stages == 4) {  // two CTAs per SM
    switch (r) {
      case 1: return np16 ? launch_fused_variant<16, 1, 2>(tmA, a, stream, pdl) : cudaErrorInvalidValue;
      case 2: return np16 ? launch_fused_variant<16, 2, 2>(tmA, a, stream, pdl)
                          : launch_fused_variant<32, 2, 2>(tmA, a, stream, pdl);
      case 4: return np16 ? launch_fused_variant<16, 4, 2>(tmA, a, stream, pdl)
                          : launch_fused_variant<32, 4, 2>(tmA, a, stream, pdl);
      case 8: return np16 ? launch_fused_variant<16, 8, 2>(tmA, a, stream, pdl)
                          : launch_fused_variant<32, 8, 2>(tmA, a, stream, pdl);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (r) {
    case 1: return np16 ? launch_fused_variant<16, 1, 1>(tmA, a, stream, pdl) : cudaErrorInvalidValue;
    case 2: return np16 ? launch_fused_variant<16, 2, 1>(tmA, a, stream, pdl)
                        : launch_fused_variant<32, 2, 1>(tmA, a, stream, pdl);
    case 4: return np16 ? launch_fused_variant<16, 4, 1>(tmA, a, stream, pdl)
                        : launch_fused_variant<32, 4, 1>(tmA, a, stream, pdl);
    case 8: return np16 ? launch_fused_variant<16, 8, 1>(tmA, a, stream, pdl)
                        : launch_fused_variant<32, 8, 1>(tmA, a, stream, pdl);
    case 16: return np16 ? launch_fused_variant<16, 16, 1>(tmA, a, stream, pdl)
                         : launch_fused_variant<32, 16, 1>(tmA, a, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

// Test hook: this file's wait bound (see ptx.cuh).
cudaError_t set_debug_waits_decode_fused(uint64_t limit_ns) { return set_debug_waits_in_this_file(limit_ns); }

}  // namespace llmint8
