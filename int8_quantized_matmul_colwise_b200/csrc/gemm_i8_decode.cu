// gemm_i8_decode.cu -- steps a5-a7 for decode-shaped calls (M <= 32 rows of X):
// the int8 GEMM is HBM-bound on streaming Wq (N x K bytes), so the kernel is
// laid out to put every SM on that stream.
//
// "8-bit Matrix Multiplication for Large Language Models", Summary &
// Methodology Analysis (dequantize by the outer product of row and column
// constants, add the 16-bit outlier product, 16-bit output); "Compress your
// LLMs", Mixed-precision decomposition.
//
// Swap-AB: the MMA computes D^T = Wq * Xq^T with Wq's rows on the MMA's M side
// (128 per tile) and the M <= 32 activation rows, padded to NP = 16 or 32, on
// its N side (tcgen05.mma kind::i8, M=128 N=NP K=32, int32 accumulator in 32
// TMEM columns).  The N/128 tiles are split along K into S slices so that
// tiles x S CTAs cover the SMs; each CTA adds its int32 partial sums into a
// zero-initialised workspace buffer laid out [m][n] (red.global.add: exact,
// order-free, coalesced) and the last CTA of a tile (per-tile counter) applies
// the dequantize + outlier epilogue, writes Y and returns the buffer and the
// counter to zero.  While the MMAs stream Wq, the epilogue warps fetch what
// the epilogue needs (row scales, Xo, and each thread's W values of the
// outlier rows into registers), so the tile's last CTA finishes quickly.
// The Wq loads of the first ring stages are issued before
// griddepcontrol.wait: they do not depend on the activation kernels, so the
// weight stream overlaps them.  Every mbarrier wait is bounded.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace llmint8 {

namespace {

constexpr int kRowsA = 128;            // Wq rows per tile (MMA M)
constexpr int kBK = kGemmBK;           // K bytes per stage
constexpr int kStagesD = 10;           // ring depth
constexpr int kThreadsD = 192;         // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr uint32_t kBytesAD = kRowsA * kBK;  // 16 KB
constexpr int kXoCols = 64;            // outlier values staged per pass (epilogue)

template <int NP>
struct GeoD {
  static constexpr uint32_t kBytesB = NP * kBK;  // 2 or 4 KB
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kOffA + kStagesD * kBytesAD;
  static constexpr uint32_t kOffXo = kOffB + kStagesD * kBytesB;            // fp32 [32][kXoCols]
  static constexpr uint32_t kOffRs = kOffXo + 32 * kXoCols * 4;             // fp32 [32]
  static constexpr uint32_t kOffBars = kOffRs + 32 * 4;
  static constexpr uint32_t kNumBars = 2 * kStagesD + 2;                    // full, empty, tmem full, drain
  static constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
  static constexpr size_t kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kBytesB % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void red_add_s32(int32_t* p, int32_t v) {
  asm volatile("red.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

constexpr int kWReg = 32;  // outlier W values a thread keeps in registers

// Final epilogue of one Wq row n (this thread) for all M activation rows:
// Y[m, n] = acc[m] * rs[m] * cs[n] / 127^2 + sum_t Xo[m, t] * W[O[t], n].
// s_xo holds Xo[m, t] for t < min(n_use, kXoCols) and wreg the W values for
// t < min(n_use, kWReg); outliers beyond those are read here.
template <bool kRaw, int NP>
__device__ void finish_row(const DecodeArgs& p, const float* s_rs, float* s_xo, int n, const int32_t (&acc)[NP],
                           const float (&wreg)[kWReg], int n_use, bool overflow, int et) {
  if constexpr (kRaw) {
    if (n < p.N) {
#pragma unroll
      for (int m = 0; m < NP; ++m)
        if (m < p.M) p.C[static_cast<int64_t>(m) * p.ldc + n] = acc[m];
    }
    return;
  } else {
    float y[NP];
    const float csn = n < p.N ? __ldg(p.cs + n) * (1.0f / 16129.0f) : 0.0f;
#pragma unroll
    for (int m = 0; m < NP; ++m) y[m] = static_cast<float>(acc[m]) * s_rs[m] * csn;
    // outliers already staged: Xo in s_xo, W in registers
#pragma unroll
    for (int t = 0; t < kWReg; ++t) {
      if (t < n_use && t < kXoCols) {
#pragma unroll
        for (int m = 0; m < NP; ++m) y[m] = fmaf(s_xo[m * kXoCols + t], wreg[t], y[m]);
      }
    }
    // any further outliers (more than kWReg): loads here
    const __half* W = static_cast<const __half*>(p.W);
    const __half* Xo = static_cast<const __half*>(p.Xo);
    for (int t0 = kWReg; t0 < n_use; t0 += kXoCols) {
      const int tn = min(kXoCols, n_use - t0);
      named_bar_sync(1, 128);  // previous readers of s_xo are done
      for (int i = et; i < NP * kXoCols; i += 128) {
        const int m = i / kXoCols, t = i % kXoCols;
        s_xo[m * kXoCols + t] = (t < tn && m < p.M) ? __half2float(Xo[static_cast<int64_t>(m) * p.ldo + t0 + t]) : 0.0f;
      }
      named_bar_sync(1, 128);
      for (int t = 0; t < tn; ++t) {
        const int64_t k = __ldg(p.O + t0 + t);
        const float w = n >= p.N ? 0.0f
                        : W != nullptr ? __half2float(W[k * p.ldw + n])
                                       : __half2float(__ushort_as_half(dequant_weight_bits(p.Wq[int64_t(n) * p.ldk + k],
                                                                                           __ldg(p.cs + n))));
#pragma unroll
        for (int m = 0; m < NP; ++m) y[m] = fmaf(s_xo[m * kXoCols + t], w, y[m]);
      }
    }
    if (n < p.N) {
      if (p.bias != nullptr) {  // the linear layer's bias, added last
        const float bn = __half2float(static_cast<const __half*>(p.bias)[n]);
#pragma unroll
        for (int m = 0; m < NP; ++m) y[m] += bn;
      }
      __half* Y = static_cast<__half*>(p.Y);
#pragma unroll
      for (int m = 0; m < NP; ++m)
        if (m < p.M) Y[static_cast<int64_t>(m) * p.ldy + n] = __float2half_rn(overflow ? __int_as_float(0x7fc00000) : y[m]);
    }
  }
}

template <bool kRaw, int NP>
__global__ void __launch_bounds__(kThreadsD, 1)
    gemm_i8_decode_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const DecodeArgs p) {
  using G = GeoD<NP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base + G::kOffA;
  uint8_t* sB = base + G::kOffB;
  float* s_xo = reinterpret_cast<float*>(base + G::kOffXo);
  float* s_rs = reinterpret_cast<float*>(base + G::kOffRs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + G::kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStagesD;
  uint64_t* tfull = bars + 2 * kStagesD;
  uint64_t* drain = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + G::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(base + G::kOffMisc + 4);
  int* s_last = reinterpret_cast<int*>(base + G::kOffMisc + 8);

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const int tile = static_cast<int>(blockIdx.x) / p.splits;
  const int split = static_cast<int>(blockIdx.x) % p.splits;
  const int nkb_total = (p.K + kBK - 1) / kBK;
  const int kb0 = split * p.kb_per_split;
  const int nkb = max(0, min(p.kb_per_split, nkb_total - kb0));
  const int n0 = tile * kRowsA;
  constexpr uint32_t kTx = kBytesAD + G::kBytesB;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesD; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const uint64_t hint_w = policy_evict_first();  // Wq is streamed once
  const uint64_t hint_x = policy_evict_last();   // Xq is read by every tile
  // Weight stream first: it does not depend on the activation kernels.
  const int pre = min(nkb, kStagesD);
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&full[i], kTx);
      tma_load_2d(sA + i * kBytesAD, &tmA, &full[i], (kb0 + i) * kBK, n0, hint_w);
    }
  }

  griddep_wait();  // Xq, rs, O, n_o and Xo are written by the quantize kernel
  // The next launch on the stream may get resident now: every kernel of this
  // library waits (griddepcontrol.wait) for this grid to complete before it
  // touches memory this grid reads or writes.
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < pre; ++i) tma_load_2d(sB + i * G::kBytesB, &tmB, &full[i], (kb0 + i) * kBK, 0, hint_x);
      uint32_t issued = (1u << pre) - 1u;  // bit st: stage st has had a load issued
      uint32_t issued_phase = 0;           // bit st: the phase of its last load
      bool ok = true;
      for (int i = kStagesD; i < nkb && ok; ++i) {
        const int st = i % kStagesD;
        const uint32_t ph = static_cast<uint32_t>(i / kStagesD - 1) & 1u;
        if (!mbar_wait_abortable(&empty[st], ph, p.status, abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[st], kTx);
        tma_load_2d(sA + st * kBytesAD, &tmA, &full[st], (kb0 + i) * kBK, n0, hint_w);
        tma_load_2d(sB + st * G::kBytesB, &tmB, &full[st], (kb0 + i) * kBK, 0, hint_x);
        const uint32_t phase = static_cast<uint32_t>(i / kStagesD) & 1u;
        issued_phase = (issued_phase & ~(1u << st)) | (phase << st);
      }
      if (!ok) {  // let the copies in flight land before the CTA exits
        for (int st = 0; st < kStagesD; ++st)
          if (issued & (1u << st)) mbar_wait(&full[st], (issued_phase >> st) & 1u, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kRowsA, NP);
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int st = i % kStagesD;
        const uint32_t ph = static_cast<uint32_t>(i / kStagesD) & 1u;
        if (!mbar_wait_abortable(&full[st], ph, p.status, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = smem_desc_k_sw128(smem_u32(sA + st * kBytesAD));
        const uint64_t db = smem_desc_k_sw128(smem_u32(sB + st * G::kBytesB));
#pragma unroll
        for (int kk = 0; kk < kBK / 32; ++kk) mma_i8(tmem_base, da + 2u * kk, db + 2u * kk, idesc, (i | kk) != 0);
        mma_commit(&empty[st]);
      }
      if (ok) {
        mma_commit(tfull);
      } else if (nkb > 0) {
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr);
      }
    }
  } else {
    // ---------------- epilogue warps: thread <-> Wq row n (TMEM lane)
    const uint32_t q = warp & 3u;
    const int et = static_cast<int>(threadIdx.x) - 64;
    const int n = n0 + static_cast<int>(q * 32 + lane);
    // Fetch what the epilogue reads while the MMAs run.
    const int n_o = kRaw ? 0 : *p.n_o;
    const bool overflow = n_o > p.cap;
    const int n_use = overflow ? 0 : n_o;
    float wreg[kWReg];
    if constexpr (!kRaw) {
      if (et < 32) s_rs[et] = et < p.M ? __ldg(p.rs + et) : 0.0f;
      const __half* Xo = static_cast<const __half*>(p.Xo);
      const int tx = min(n_use, kXoCols);
      for (int i = et; i < NP * kXoCols; i += 128) {
        const int m = i / kXoCols, t = i % kXoCols;
        s_xo[m * kXoCols + t] = (t < tx && m < p.M) ? __half2float(Xo[static_cast<int64_t>(m) * p.ldo + t]) : 0.0f;
      }
      const __half* W = static_cast<const __half*>(p.W);
      int orow[kWReg];
#pragma unroll
      for (int t = 0; t < kWReg; ++t) orow[t] = t < n_use ? __ldg(p.O + t) : 0;
      if (W != nullptr) {
#pragma unroll
        for (int t = 0; t < kWReg; ++t)
          wreg[t] = (t < n_use && n < p.N) ? __half2float(W[static_cast<int64_t>(orow[t]) * p.ldw + n]) : 0.0f;
      } else {  // no fp16 weight kept: the outlier rows recovered from Wq
        const float csw = n < p.N ? __ldg(p.cs + n) : 0.0f;
#pragma unroll
        for (int t = 0; t < kWReg; ++t)
          wreg[t] = (t < n_use && n < p.N)
                        ? __half2float(__ushort_as_half(dequant_weight_bits(p.Wq[int64_t(n) * p.ldk + orow[t]], csw)))
                        : 0.0f;
      }
    } else {
#pragma unroll
      for (int t = 0; t < kWReg; ++t) wreg[t] = 0.0f;
    }
    int32_t acc[NP];
    bool got = true;
    if (nkb > 0) {
      got = mbar_wait_abortable(tfull, 0, p.status, abort);
      got = named_bar_and(2, 128, got);  // also makes s_rs / s_xo visible
      if (got) {
        tc_fence_after();
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + ((q * 32u) << 16), v);  // NP <= 32 columns are valid
        tmem_ld_wait();
#pragma unroll
        for (int m = 0; m < NP; ++m) acc[m] = static_cast<int32_t>(v[m]);
      }
    } else {
      named_bar_sync(1, 128);
#pragma unroll
      for (int m = 0; m < NP; ++m) acc[m] = 0;
    }
    tc_fence_before();
    if (got) {
      bool finish = true;
      if (p.splits > 1) {
        // exact split-K reduction: add the partial sums ([m][n], coalesced), count the tile
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < NP; ++m)
            if (m < p.M) red_add_s32(p.partial + static_cast<int64_t>(m) * p.N + n, acc[m]);
        }
        __threadfence();
        named_bar_sync(1, 128);
        if (et == 0) *s_last = (atomicAdd(p.tile_counter + tile, 1u) == static_cast<uint32_t>(p.splits - 1)) ? 1 : 0;
        named_bar_sync(1, 128);
        finish = *s_last != 0;
        if (finish) {
          __threadfence();
          if (n < p.N) {
#pragma unroll
            for (int m = 0; m < NP; ++m) {
              int32_t* pm = p.partial + static_cast<int64_t>(m) * p.N + n;
              acc[m] = m < p.M ? __ldcg(pm) : 0;
              if (m < p.M) *pm = 0;  // zero for the next call
            }
          }
          if (et == 0) p.tile_counter[tile] = 0u;
        }
      }
      if (finish) finish_row<kRaw, NP>(p, s_rs, s_xo, n, acc, wreg, n_use, overflow, et);
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 32);
  }
}

template <bool kRaw, int NP>
cudaError_t launch_decode_variant(const CUtensorMap& tmA, const CUtensorMap& tmB, const DecodeArgs& a,
                                  cudaStream_t stream, bool pdl) {
  using G = GeoD<NP>;
  static bool attr_set[64] = {};
  auto kern = gemm_i8_decode_kernel<kRaw, NP>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int tiles = (a.N + kRowsA - 1) / kRowsA;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * a.splits));
  cfg.blockDim = dim3(kThreadsD);
  cfg.dynamicSmemBytes = G::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, a);
}

}  // namespace

int decode_rows_padded(int M) { return M <= 16 ? 16 : 32; }

void decode_split(int M, int N, int K, int num_sms, bool can_split, int* splits, int* kb_per_split) {
  const int tiles = (N + kRowsA - 1) / kRowsA;
  const int nkb = (K + kBK - 1) / kBK;
  int s = can_split ? num_sms / tiles : 1;
  s = s < 1 ? 1 : (s > nkb ? nkb : s);
  const int per = (nkb + s - 1) / s;
  *kb_per_split = per;
  *splits = (nkb + per - 1) / per;  // no empty slices
  (void)M;
}

cudaError_t launch_gemm_i8_decode(const CUtensorMap& tmA, const CUtensorMap& tmB, const DecodeArgs& a, bool raw_i32,
                                  cudaStream_t stream, bool pdl) {
  if (decode_rows_padded(a.M) == 16)
    return raw_i32 ? launch_decode_variant<true, 16>(tmA, tmB, a, stream, pdl)
                   : launch_decode_variant<false, 16>(tmA, tmB, a, stream, pdl);
  return raw_i32 ? launch_decode_variant<true, 32>(tmA, tmB, a, stream, pdl)
                 : launch_decode_variant<false, 32>(tmA, tmB, a, stream, pdl);
}

// Test hook: this file's wait bound (see ptx.cuh).
cudaError_t set_debug_waits_gemm_i8_decode(uint64_t limit_ns) { return set_debug_waits_in_this_file(limit_ns); }

}  // namespace llmint8
