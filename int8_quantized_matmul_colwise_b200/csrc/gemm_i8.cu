// gemm_i8.cu -- steps a5-a7: int8 x int8 -> int32 GEMM on the 5th-generation
// tensor cores (tcgen05.mma kind::i8, accumulators in TMEM), with an epilogue
// that dequantizes by the outer product of row and column scales and adds the
// 16-bit product of the outlier feature dimensions before the fp16 store.
//
// "8-bit Matrix Multiplication for Large Language Models", Summary &
// Methodology Analysis: int8 outputs are dequantized by the outer product of
// the row and column normalization constants and accumulated with the outlier
// (16-bit) matmul into 16-bit outputs.  "Compress your LLMs",
// Mixed-precision decomposition: 16-bit matmul for the ~0.1 % outlier
// dimensions, 8-bit for the other 99.9 %.
//
// Structure (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: Xq tile [128 x 128 B] + Wq tile [256 x 128 B]
//               per stage into a 4-stage shared-memory ring (128-byte swizzle);
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma kind::i8
//               (M=128, N=256, K=32) from one thread; accumulators are double
//               buffered (2 x 256 int32 columns) so the epilogue of tile i
//               overlaps the main loop of tile i+1;
//   warps 2-5   epilogue: tcgen05.ld of 32 columns at a time, dequantize with
//               rs[i] * cs[j] / 127^2, add sum_t Xo[i,t] * W[O[t], j] (fp16
//               operands, fp32 accumulation; W rows staged through shared
//               memory), round once to fp16 and store.
// Every mbarrier wait is bounded; a wait that gives up sets the status
// word's timeout bit, raises a CTA abort flag and the CTA drains and exits.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace llmint8 {

namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kBytesA = BM * BK;
constexpr uint32_t kBytesB = BN * BK;
constexpr uint32_t kAccCols = BN;
constexpr uint32_t kTmemCols = 2 * kAccCols;
constexpr int kOutT = 32;      // outlier rows of W staged per step
constexpr int kChunk = 32;     // accumulator columns per tcgen05.ld

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kBytesA;
constexpr uint32_t kOffWo = kOffB + kStages * kBytesB;
constexpr uint32_t kOffBars = kOffWo + kOutT * kChunk * 2;
constexpr uint32_t kNumBars = 2 * kStages + 2 + 2 + 1;  // full, empty, tmem full, tmem empty, drain
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr size_t kSmemBytes = kSmemUsed + 1024;  // slack for 1024-byte alignment

static_assert(kBytesA % 1024 == 0 && kBytesB % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

struct Shared {
  uint8_t* a;
  uint8_t* b;
  __half* wo;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint32_t* tmem_slot;
  volatile int* abort;
};

__device__ __forceinline__ Shared carve(uint8_t* raw) {
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  Shared s;
  s.a = base + kOffA;
  s.b = base + kOffB;
  s.wo = reinterpret_cast<__half*>(base + kOffWo);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = bars + 2 * kStages + 2;
  s.drain = bars + 2 * kStages + 4;
  s.tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  s.abort = reinterpret_cast<volatile int*>(base + kOffMisc + 4);
  return s;
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, uint32_t* status,
                                              volatile int* abort) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if ((++n & 63u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicOr(status, kStatusTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tile_coords(int tile, int num_m, int& mb, int& nb) {
  mb = tile % num_m;
  nb = tile / num_m;
}

__device__ void run_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const Shared& s, int num_m,
                             int num_tiles, int num_k, uint32_t* status) {
  const uint64_t hint = policy_evict_last();
  uint32_t stage = 0, phase = 0;
  uint32_t issued = 0;            // bit s: stage s has had a load issued
  uint32_t issued_phase = 0;      // bit s: the phase of that load
  bool ok = true;
  for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
    int mb, nb;
    tile_coords(tile, num_m, mb, nb);
    for (int kb = 0; kb < num_k; ++kb) {
      if (!wait_or_abort(&s.empty[stage], phase ^ 1u, status, s.abort)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&s.full[stage], kBytesA + kBytesB);
      tma_load_2d(s.a + stage * kBytesA, tmA, &s.full[stage], kb * BK, mb * BM, hint);
      tma_load_2d(s.b + stage * kBytesB, tmB, &s.full[stage], kb * BK, nb * BN, hint);
      issued |= 1u << stage;
      issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  if (!ok) {
    // Let the copies already in flight land before the CTA exits.
    for (int st = 0; st < kStages; ++st)
      if (issued & (1u << st)) mbar_wait(&s.full[st], (issued_phase >> st) & 1u, nullptr);
  }
}

__device__ void run_mma(const Shared& s, uint32_t tmem_base, int num_tiles, int num_k, uint32_t* status) {
  constexpr uint32_t idesc = idesc_i8(BM, BN);
  uint32_t stage = 0, phase = 0, it = 0;
  bool ok = true;
  bool any = false;
  for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
    const uint32_t b = it & 1u;
    const uint32_t use = (it >> 1) & 1u;
    if (!wait_or_abort(&s.tempty[b], use ^ 1u, status, s.abort)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t d = tmem_base + b * kAccCols;
    for (int kb = 0; kb < num_k; ++kb) {
      if (!wait_or_abort(&s.full[stage], phase, status, s.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t da = smem_desc_k_sw128(smem_u32(s.a + stage * kBytesA));
      const uint64_t db = smem_desc_k_sw128(smem_u32(s.b + stage * kBytesB));
#pragma unroll
      for (int kk = 0; kk < BK / 32; ++kk) {
        // +32 bytes along K inside the 128-byte swizzle atom = +2 in the
        // descriptor's 16-byte address units.
        mma_i8(d, da + 2u * kk, db + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
      }
      any = true;
      mma_commit(&s.empty[stage]);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (ok) mma_commit(&s.tfull[b]);
  }
  if (!ok && any) {
    // Make sure no MMA is still writing TMEM before it is freed.
    mma_commit(s.drain);
    mbar_wait(s.drain, 0, nullptr);
  }
}

template <bool kRaw>
__device__ void run_epilogue(const GemmArgs& p, const Shared& s, uint32_t tmem_base, int num_m, int num_tiles,
                             uint32_t warp, uint32_t lane) {
  const uint32_t q = warp & 3u;  // TMEM lane quarter this warp may access
  const int et = static_cast<int>(threadIdx.x) - 64;  // 0..127
  const int n_o = kRaw ? 0 : *p.n_o;
  const bool overflow = n_o > p.cap;
  const int n_use = overflow ? 0 : n_o;
  const __half* W = static_cast<const __half*>(p.W);
  const __half* Xo = static_cast<const __half*>(p.Xo);
  __half* Y = static_cast<__half*>(p.Y);
  const bool y_vec = (p.ldy % 8 == 0) && (reinterpret_cast<uintptr_t>(p.Y) % 16 == 0);
  const bool w_vec = (p.ldw % 8 == 0) && (reinterpret_cast<uintptr_t>(p.W) % 16 == 0);
  const bool c_vec = (p.ldc % 4 == 0) && (reinterpret_cast<uintptr_t>(p.C) % 16 == 0);

  uint32_t it = 0;
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
    const uint32_t b = it & 1u;
    const uint32_t use = (it >> 1) & 1u;
    const bool got = wait_or_abort(&s.tfull[b], use, p.status, s.abort);
    if (!named_bar_and(2, kEpiThreads, got)) break;  // all epilogue threads stop together
    tc_fence_after();
    int mb, nb;
    tile_coords(tile, num_m, mb, nb);
    const int row = mb * BM + static_cast<int>(q * 32 + lane);
    const bool row_ok = row < p.M;
    float rsc = 0.0f;
    if (!kRaw && row_ok) rsc = p.rs[row] * (1.0f / 16129.0f);

#pragma unroll 1
    for (int c = 0; c < BN / kChunk; ++c) {
      const int col0 = nb * BN + c * kChunk;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_base + ((q * 32u) << 16) + b * kAccCols + c * kChunk, v);
      tmem_ld_wait();

      if constexpr (kRaw) {
        if (row_ok) {
          int32_t* dst = p.C + static_cast<int64_t>(row) * p.ldc + col0;
          if (c_vec && col0 + kChunk <= p.N) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<uint4*>(dst + j) = make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          } else {
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.N) dst[j] = static_cast<int32_t>(v[j]);
          }
        }
        continue;
      } else {
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float csj = (col0 + j < p.N) ? __ldg(p.cs + col0 + j) : 0.0f;
          y[j] = static_cast<float>(static_cast<int32_t>(v[j])) * rsc * csj;
        }
        // 16-bit outlier product: y += sum_t Xo[row, t] * W[O[t], cols]
        for (int t0 = 0; t0 < n_use; t0 += kOutT) {
          named_bar_sync(1, kEpiThreads);  // previous step's readers are done
          {
            const int tt = et >> 2;
            const int seg = (et & 3) * 8;
            const int t = t0 + tt;
            __half h[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) h[e] = __ushort_as_half(0);
            if (t < n_use) {
              const __half* wr = W + static_cast<int64_t>(p.O[t]) * p.ldw + col0 + seg;
              if (w_vec && col0 + seg + 8 <= p.N) {
                const uint4 u = __ldg(reinterpret_cast<const uint4*>(wr));
                const __half* hp = reinterpret_cast<const __half*>(&u);
#pragma unroll
                for (int e = 0; e < 8; ++e) h[e] = hp[e];
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  if (col0 + seg + e < p.N) h[e] = wr[e];
              }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) s.wo[tt * kChunk + seg + e] = h[e];
          }
          named_bar_sync(1, kEpiThreads);
          const int tn = min(kOutT, n_use - t0);
          for (int tt = 0; tt < tn; ++tt) {
            const float xo = row_ok ? __half2float(Xo[static_cast<int64_t>(row) * p.ldo + t0 + tt]) : 0.0f;
            const __half2* wv = reinterpret_cast<const __half2*>(s.wo + tt * kChunk);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float2 w2 = __half22float2(wv[j]);
              y[2 * j] = fmaf(xo, w2.x, y[2 * j]);
              y[2 * j + 1] = fmaf(xo, w2.y, y[2 * j + 1]);
            }
          }
        }
        if (overflow) {
#pragma unroll
          for (int j = 0; j < 32; ++j) y[j] = __int_as_float(0x7fc00000);
        }
        if (row_ok) {
          __half* dst = Y + static_cast<int64_t>(row) * p.ldy + col0;
          if (y_vec && col0 + kChunk <= p.N) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 u;
              __half2* h2 = reinterpret_cast<__half2*>(&u);
              h2[0] = __floats2half2_rn(y[j], y[j + 1]);
              h2[1] = __floats2half2_rn(y[j + 2], y[j + 3]);
              h2[2] = __floats2half2_rn(y[j + 4], y[j + 5]);
              h2[3] = __floats2half2_rn(y[j + 6], y[j + 7]);
              *reinterpret_cast<uint4*>(dst + j) = u;
            }
          } else {
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.N) dst[j] = __float2half_rn(y[j]);
          }
        }
      }
    }
    tc_fence_before();
    mbar_arrive(&s.tempty[b]);
  }
}

template <bool kRaw>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  const Shared s = carve(smem_raw);
  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const int num_m = (p.M + BM - 1) / BM;
  const int num_n = (p.N + BN - 1) / BN;
  const int num_k = (p.K + BK - 1) / BK;
  const int num_tiles = num_m * num_n;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], kEpiThreads);
    }
    mbar_init(s.drain, 1);
    *s.abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(s.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;

  griddep_wait();  // Xq, rs, O, n_o and Xo are written by the quantize kernel

  if (warp == 0) {
    if (lane == 0) run_producer(&tmA, &tmB, s, num_m, num_tiles, num_k, p.status);
  } else if (warp == 1) {
    if (lane == 0) run_mma(s, tmem_base, num_tiles, num_k, p.status);
  } else {
    run_epilogue<kRaw>(p, s, tmem_base, num_m, num_tiles, warp, lane);
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_i8(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, bool raw_i32,
                           int num_sms, cudaStream_t stream, bool pdl) {
  static bool attr_set[2][64] = {};  // per kernel variant and device
  auto kern = raw_i32 ? gemm_i8_kernel<true> : gemm_i8_kernel<false>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[raw_i32][dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[raw_i32][dev] = true;
  }
  const int num_tiles = ((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  const int grid = num_tiles < num_sms ? num_tiles : num_sms;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, a);
}

}  // namespace llmint8
