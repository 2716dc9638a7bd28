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
// Two tile shapes share one code path (kPair):
//   single CTA   128 x 256 tile per CTA, MMA M=128 N=256 K=32, 4-stage ring of
//                48 KB (Xq 128 x 128 B, Wq 256 x 128 B);
//   CTA pair     256 x 256 tile per 2-CTA cluster (tcgen05 cta_group::2): each
//                CTA loads 128 rows of Xq and 128 rows of Wq per stage (6-stage
//                ring of 32 KB), the leader issues M=256 N=256 K=32 MMAs that
//                read both CTAs' shared memory, and each CTA holds its 128 x 256
//                half of the accumulator in its own TMEM.  Per-SM operand
//                traffic per MAC is two thirds of the single-CTA tile's.
// Roles (320 threads per CTA, one persistent CTA per SM):
//   warp 0      TMA producer (128-byte swizzle, zero fill past the edges);
//   warp 1      TMEM allocation (512 columns = 2 accumulators of 256 int32
//               columns, so the epilogue of tile i overlaps the main loop of
//               tile i+1) and, in the single CTA or the pair leader, the MMA
//               issuer (one thread);
//   warps 2-9   epilogue, two warps per TMEM lane quarter, 16 rows each:
//               tcgen05.ld in the mma.m16n8 fragment layout, dequantize with
//               rs[i] * cs[j] / 127^2, add the 16-bit outlier product
//               sum_t Xo[i,t] * W[O[t], j] (fp16 operands, fp32 accumulation;
//               see below for where it runs), round once to fp16 and store
//               through a shared-memory staging tile.  The tile's W rows,
//               column scales, row scales and Xo fragments are fetched before
//               the accumulator wait.
// The outlier product: n_o <= K/256 on the CUDA cores in the epilogue;
// K/256 < n_o <= 256 on the tensor cores (the epilogue writes the dequantized
// tile back to TMEM as fp32, the MMA thread accumulates kind::f16 MMAs onto it
// from operands the epilogue warps gather into the workspace before their
// first tile, and the epilogue rounds the sum); past that, or without room in
// the workspace, warp-level mma.sync in the epilogue.
// Every mbarrier wait is bounded; a wait that gives up sets the status word's
// timeout bit, raises a CTA abort flag and the CTA drains and exits.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace llmint8 {

namespace {

constexpr int BM = kGemmBM;   // accumulator rows per CTA (TMEM lanes)
constexpr int BN = kGemmBN;   // accumulator columns per CTA
constexpr int BK = kGemmBK;   // K bytes per stage
constexpr int kEpiWarps = 8;     // two per TMEM lane quarter, 16 rows each
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint32_t kAccCols = BN;
constexpr uint32_t kTmemCols = 2 * kAccCols;
constexpr int kChunk = 32;     // accumulator columns per tcgen05.ld (raw int32 epilogue)
constexpr int kSG = 16;        // outlier rows of W staged per pass over a tile (one k16 MMA step)
constexpr int kWoStride = BN + 8;  // halves per staged row: 528 bytes, conflict-free ldmatrix
// More than kSG outliers: the epilogue walks the tile's 64-column chunks
// outermost and stages up to kRound outlier rows of W for one chunk at a time,
// so that each accumulator chunk is read from TMEM once and every pass's MMAs
// run on it in registers.
constexpr int kRound = 96;
constexpr int kWo2Stride = 72;  // halves per staged row of a chunk: 144 bytes, conflict-free ldmatrix
// Many outliers (K/256 < n_o <= kOutlierMmaMax): the outlier product runs on
// the tensor cores.  The epilogue dequantizes the tile in TMEM (int32 -> fp32
// in place) and the MMA thread accumulates Xo * W[O, :] onto it with kind::f16
// MMAs (fp16 operands, fp32 accumulation).  Each block of 64 outlier columns
// is one ring stage with the int8 stage's geometry (the tile's rows of Xo and
// of the gathered W^T, 128 bytes each), and a tile's blocks enter the ring
// om_insert() blocks into the next tile's main loop (kOmLag, or half of a
// shorter one), by which time the epilogue has the tile dequantized and still
// has half a main loop to finish it before its accumulator is needed again.
constexpr int kOmLag = 8;
__host__ __device__ constexpr int om_insert(int num_k) {
  return (num_k + 1) / 2 < kOmLag ? (num_k + 1) / 2 : kOmLag;
}
constexpr int kOmCols = kOutlierMmaMax;   // fp16 columns (row stride) of the gathered operands
constexpr int kOmUnit = 16;               // rows of W^T or Xo per gather unit
constexpr int kOmStride = kOmCols + 8;    // halves per row of the transposing tile: 528 bytes

template <bool kPair>
struct Geo {
  static constexpr int kTileM = kPair ? 2 * BM : BM;      // rows of Y per tile
  static constexpr int kRowsB = kPair ? BN / 2 : BN;      // rows of Wq loaded per CTA per stage
  static constexpr int kStages = kPair ? 6 : 4;
  static constexpr uint32_t kBytesA = BM * BK;
  static constexpr uint32_t kBytesB = kRowsB * BK;
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kOffA + kStages * kBytesA;
  static constexpr uint32_t kOffWo = kOffB + kStages * kBytesB;     // fp16 [kSG][kWoStride] or [kRound][kWo2Stride]
  static constexpr uint32_t kWoBytes =
      kSG * kWoStride * 2 > kRound * kWo2Stride * 2 ? kSG * kWoStride * 2 : kRound * kWo2Stride * 2;
  static constexpr uint32_t kOffCs = kOffWo + kWoBytes;  // fp32 [BN]
  static constexpr uint32_t kOffBias = kOffCs + BN * 4;              // fp32 [BN]
  // per epilogue warp, 16 rows x 64 fp16 columns of Y in the 128-byte swizzle
  static constexpr uint32_t kOffY = (kOffBias + BN * 4 + 1023) & ~1023u;
  static constexpr uint32_t kYBytes = 16 * 128;
  static constexpr uint32_t kOffBars = kOffY + kEpiWarps * kYBytes;
  // full, empty, tmem full/empty, drain, dequantized (pair leader), outlier product done
  static constexpr uint32_t kNumBars = 2 * kStages + 2 + 2 + 1 + 2 + 2;
  static constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
  static constexpr size_t kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
  // Arrivals that free a TMEM accumulator: one per epilogue warp of each CTA.
  static constexpr uint32_t kTmemEmptyArrivals = kPair ? 2 * kEpiWarps : kEpiWarps;
  static_assert(kBytesA % 1024 == 0 && kBytesB % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kOmUnit * kOmStride * 2 <= kWoBytes, "the gather's transposing tile fits the staging area");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct Shared {
  uint8_t* a;
  uint8_t* b;
  __half* wo;  // outlier rows of W over the tile's columns
  float* cs;  // column scales of the tile
  float* bias;  // bias of the tile's columns (zero without a bias)
  uint8_t* ystage;  // Y staging tiles for the TMA store, one per epilogue warp
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint64_t* deq;    // [2] the epilogue has written the dequantized tile to TMEM (pair leader)
  uint64_t* ofull;  // [2] the outlier MMAs on that tile are done
  uint32_t* tmem_slot;
  volatile int* abort;
};

template <bool kPair>
__device__ __forceinline__ Shared carve(uint8_t* raw) {
  using G = Geo<kPair>;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  Shared s;
  s.a = base + G::kOffA;
  s.b = base + G::kOffB;
  s.wo = reinterpret_cast<__half*>(base + G::kOffWo);
  s.cs = reinterpret_cast<float*>(base + G::kOffCs);
  s.bias = reinterpret_cast<float*>(base + G::kOffBias);
  s.ystage = base + G::kOffY;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + G::kOffBars);
  s.full = bars;
  s.empty = bars + G::kStages;
  s.tfull = bars + 2 * G::kStages;
  s.tempty = bars + 2 * G::kStages + 2;
  s.drain = bars + 2 * G::kStages + 4;
  s.deq = bars + 2 * G::kStages + 5;
  s.ofull = bars + 2 * G::kStages + 7;
  s.tmem_slot = reinterpret_cast<uint32_t*>(base + G::kOffMisc);
  s.abort = reinterpret_cast<volatile int*>(base + G::kOffMisc + 4);
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
      if (globaltimer_ns() - t0 > wait_limit_ns()) {
        atomicOr(status, kStatusTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

// Tile order: the M tiles are split into groups of group_m consecutive tiles
// (Xq strips of at most kGroupBytes together); a group's tiles run before the
// next group's, M index fastest within it.  The tiles in flight at one time
// then share a few Wq strips, and the group's Xq strips stay in L2 for all of
// its N tiles, so that Xq is read from HBM once and Wq once per group.  With
// M fastest over all of M every wave reads all of Xq, and once that is more
// than L2 keeps, each wave re-reads it from HBM.
constexpr int64_t kGroupBytes = int64_t(20) << 20;

struct Sched {
  int first, stride, num_tiles, num_m, num_k, group_m;
};

// M tiles per group for tiles of tile_m rows and K bytes per row: groups of
// equal size (the last one may be smaller) under the byte budget.
__device__ __forceinline__ int tile_group_m(int num_m, int tile_m, int K) {
  const int64_t by_bytes = kGroupBytes / (int64_t(tile_m) * int64_t(K > 0 ? K : 1));
  const int cap = by_bytes < 1 ? 1 : (by_bytes > num_m ? num_m : static_cast<int>(by_bytes));
  const int groups = (num_m + cap - 1) / cap;
  return (num_m + groups - 1) / groups;
}

__device__ __forceinline__ void tile_coords(int tile, const Sched& sc, int& mb, int& nb) {
  const int num_n = sc.num_tiles / sc.num_m;
  const int per_group = sc.group_m * num_n;
  const int g = tile / per_group;
  const int r = tile - g * per_group;
  const int m0 = g * sc.group_m;
  const int rows = sc.num_m - m0 < sc.group_m ? sc.num_m - m0 : sc.group_m;
  mb = m0 + r % rows;
  nb = r / rows;
}

// Blocks of 64 outlier columns the tensor-core outlier product takes for this
// call (0: the epilogue computes the product itself).  Every role of every CTA
// derives the same value from n_o.
__device__ __forceinline__ int outlier_mma_blocks(const GemmArgs& p) {
  if (!p.om_ok) return 0;
  const int n_o = *p.n_o;
  if (n_o > p.cap || n_o > kOmCols || int64_t(n_o) * 256 <= int64_t(p.K)) return 0;
  return (n_o + 63) / 64;
}

// Bounded wait until a global counter reaches `target` (acquire).
__device__ __forceinline__ bool wait_counter(const uint32_t* ctr, uint32_t target, uint32_t* status,
                                             volatile int* abort) {
  const uint64_t t0 = globaltimer_ns();
  uint32_t n = 0;
  while (ld_acquire_gpu_u32(ctr) < target) {
    if ((++n & 63u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > wait_limit_ns()) {
        atomicOr(status, kStatusTimeout);
        *abort = 1;
        return false;
      }
    }
  }
  return true;
}

template <bool kPair>
__device__ void run_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const CUtensorMap* tmXo,
                             const CUtensorMap* tmWo, const Shared& s, const Sched& sc, uint32_t rank,
                             const GemmArgs& p, bool om_possible) {
  using G = Geo<kPair>;
  const uint64_t hint = policy_evict_last();
  uint32_t stage = 0, phase = 0;
  uint32_t issued = 0;        // bit s: stage s has had a load issued
  uint32_t issued_phase = 0;  // bit s: the phase of that load
  uint32_t* const status = p.status;
  // Blocks of the tensor-core outlier product, read where they are first
  // needed (one tile into the main loop), so n_o's load never delays the
  // first copies.
  int om = om_possible ? -1 : 0;
  auto om_blocks = [&]() {
    if (om < 0) om = outlier_mma_blocks(p);
    return om;
  };
  bool gathered = false;      // the gathered outlier operands are complete in global memory
  // one ring stage: the box at column x of both maps
  auto load = [&](const CUtensorMap* ta, const CUtensorMap* tb, int x, int ya, int yb) -> bool {
    if (!wait_or_abort(&s.empty[stage], phase ^ 1u, status, s.abort)) return false;
    if constexpr (kPair) {
      // both CTAs' bytes are counted on the leader's full barrier
      if (rank == 0) mbar_arrive_expect_tx(&s.full[stage], 2 * (G::kBytesA + G::kBytesB));
      const uint32_t bar = mapa_shared(smem_u32(&s.full[stage]), 0);
      tma_load_2d_pair(s.a + stage * G::kBytesA, ta, bar, x, ya, hint);
      tma_load_2d_pair(s.b + stage * G::kBytesB, tb, bar, x, yb, hint);
    } else {
      mbar_arrive_expect_tx(&s.full[stage], G::kBytesA + G::kBytesB);
      tma_load_2d(s.a + stage * G::kBytesA, ta, &s.full[stage], x, ya, hint);
      tma_load_2d(s.b + stage * G::kBytesB, tb, &s.full[stage], x, yb, hint);
    }
    issued |= 1u << stage;
    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
    if (++stage == G::kStages) {
      stage = 0;
      phase ^= 1u;
    }
    return true;
  };
  // a tile's outlier blocks: 64 columns of Xo (A) and of W^T (B) each
  auto load_outliers = [&](int ya, int yb) -> bool {
    if (!gathered) {  // every CTA's share of the gather, then TMA reads of it
      if (!wait_counter(p.om_sync, gridDim.x, status, s.abort)) return false;
      fence_proxy_async_global();
      gathered = true;
    }
    for (int ob = 0; ob < om; ++ob)
      if (!load(tmXo, tmWo, ob * 64, ya, yb)) return false;
    return true;
  };
  bool ok = true;
  bool prev = false;
  int pya = 0, pyb = 0;  // the previous tile's rows
  const int ins = om_insert(sc.num_k);
  for (int tile = sc.first; tile < sc.num_tiles && ok; tile += sc.stride) {
    int mb, nb;
    tile_coords(tile, sc, mb, nb);
    const int ya = mb * G::kTileM + (kPair ? static_cast<int>(rank) * BM : 0);
    const int yb = nb * BN + (kPair ? static_cast<int>(rank) * G::kRowsB : 0);
    // the main loop's blocks in two runs, the previous tile's outlier blocks between them
    for (int run = 0; run < 2 && ok; ++run) {
      if (run == 1 && prev && om != 0 && om_blocks() > 0) ok = load_outliers(pya, pyb);
      const int k_end = run == 0 ? ins : sc.num_k;
      for (int kb = run == 0 ? 0 : ins; kb < k_end && ok; ++kb) ok = load(tmA, tmB, kb * BK, ya, yb);
    }
    prev = true;
    pya = ya;
    pyb = yb;
  }
  if (ok && prev && om != 0 && om_blocks() > 0) ok = load_outliers(pya, pyb);
  if (!ok && (!kPair || rank == 0)) {
    // Let the copies already in flight land before the CTA exits.
    for (int st = 0; st < G::kStages; ++st)
      if (issued & (1u << st)) mbar_wait(&s.full[st], (issued_phase >> st) & 1u, nullptr);
  }
}

template <bool kPair>
__device__ void run_mma(const Shared& s, uint32_t tmem_base, const Sched& sc, const GemmArgs& p, bool om_possible) {
  using G = Geo<kPair>;
  uint32_t* const status = p.status;
  const uint32_t stall = p.stall;
  int om = om_possible ? -1 : 0;  // read where first needed, as in the producer
  auto om_blocks = [&]() {
    if (om < 0) om = outlier_mma_blocks(p);
    return om;
  };
  constexpr uint32_t idesc = idesc_i8(G::kTileM, BN);
  uint32_t stage = 0, phase = 0, it = 0;
  bool ok = true;
  bool any = false;
  // The outlier product of the tile in accumulator pb (its use-th use): once
  // both CTAs' epilogues have dequantized it in TMEM, fp16 MMAs accumulate
  // onto it, and the commit tells both epilogues that it is done.
  auto outliers = [&](uint32_t pb, uint32_t puse) -> bool {
    constexpr uint32_t idesc_o = idesc_f16(G::kTileM, BN);
    if (!wait_or_abort(&s.deq[pb], puse, status, s.abort)) return false;
    tc_fence_after();
    const uint32_t d = tmem_base + pb * kAccCols;
    for (int ob = 0; ob < om; ++ob) {
      if (!wait_or_abort(&s.full[stage], phase, status, s.abort)) return false;
      tc_fence_after();
      const uint64_t da = smem_desc_k_sw128(smem_u32(s.a + stage * G::kBytesA));
      const uint64_t db = smem_desc_k_sw128(smem_u32(s.b + stage * G::kBytesB));
#pragma unroll
      for (int kk = 0; kk < BK / 32; ++kk) {  // K = 16 fp16 = 32 bytes per MMA, as for int8
        if constexpr (kPair)
          mma_f16_pair(d, da + 2u * kk, db + 2u * kk, idesc_o, 1u);
        else
          mma_f16(d, da + 2u * kk, db + 2u * kk, idesc_o, 1u);
      }
      any = true;
      if constexpr (kPair)
        mma_commit_pair(&s.empty[stage], 0x3);
      else
        mma_commit(&s.empty[stage]);
      if (++stage == G::kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if constexpr (kPair)
      mma_commit_pair(&s.ofull[pb], 0x3);
    else
      mma_commit(&s.ofull[pb]);
    return true;
  };
  // (the stall test hook first waits on the drain barrier, which nothing has
  // arrived on yet: the wait runs out before any MMA is issued and the CTA
  // takes the abort path)
  if ((stall & kStallGemmOperands) && !wait_or_abort(s.drain, 0, status, s.abort)) ok = false;
  const int ins = om_insert(sc.num_k);
  for (int tile = sc.first; tile < sc.num_tiles && ok; tile += sc.stride, ++it) {
    const uint32_t b = it & 1u;
    const uint32_t use = (it >> 1) & 1u;
    if (!wait_or_abort(&s.tempty[b], use ^ 1u, status, s.abort)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t d = tmem_base + b * kAccCols;
    // the main loop's blocks in two runs, the previous tile's outlier blocks between them
    for (int run = 0; run < 2 && ok; ++run) {
      if (run == 1 && it > 0 && om != 0 && om_blocks() > 0 && !outliers(b ^ 1u, ((it - 1) >> 1) & 1u)) {
        ok = false;
        break;
      }
      const int k_end = run == 0 ? ins : sc.num_k;
      for (int kb = run == 0 ? 0 : ins; kb < k_end; ++kb) {
        if (!wait_or_abort(&s.full[stage], phase, status, s.abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = smem_desc_k_sw128(smem_u32(s.a + stage * G::kBytesA));
        const uint64_t db = smem_desc_k_sw128(smem_u32(s.b + stage * G::kBytesB));
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk) {
          // +32 bytes along K inside the 128-byte swizzle atom = +2 in the
          // descriptor's 16-byte address units.
          if constexpr (kPair)
            mma_i8_pair(d, da + 2u * kk, db + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          else
            mma_i8(d, da + 2u * kk, db + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        any = true;
        if constexpr (kPair)
          mma_commit_pair(&s.empty[stage], 0x3);
        else
          mma_commit(&s.empty[stage]);
        if (++stage == G::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (ok) {
      if constexpr (kPair)
        mma_commit_pair(&s.tfull[b], 0x3);
      else
        mma_commit(&s.tfull[b]);
    }
  }
  // the last tile's outlier product
  if (ok && it > 0 && om != 0 && om_blocks() > 0 && !outliers((it - 1) & 1u, ((it - 1) >> 1) & 1u)) ok = false;
  if (!ok && any) {
    // Make sure no MMA is still writing TMEM before it is freed.
    if constexpr (kPair)
      mma_commit_pair(s.drain, 0x1);
    else
      mma_commit(s.drain);
    mbar_wait(s.drain, 0, nullptr);
  }
}

// Column scales of the tile into shared memory.
__device__ __forceinline__ void stage_scales(const GemmArgs& p, const Shared& s, int nb, int et, bool cs_vec) {
  const int n0 = nb * BN;
  if (et < BN / 4) {
    const int c = n0 + 4 * et;
    float4 v;
    if (cs_vec && c + 4 <= p.N) {
      v = __ldg(reinterpret_cast<const float4*>(p.cs + c));
    } else {
      v.x = c < p.N ? __ldg(p.cs + c) : 0.0f;
      v.y = c + 1 < p.N ? __ldg(p.cs + c + 1) : 0.0f;
      v.z = c + 2 < p.N ? __ldg(p.cs + c + 2) : 0.0f;
      v.w = c + 3 < p.N ? __ldg(p.cs + c + 3) : 0.0f;
    }
    *reinterpret_cast<float4*>(s.cs + 4 * et) = v;
    // the linear layer's bias (fp16), zero without one
    const __half* bias = static_cast<const __half*>(p.bias);
    float4 bv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (bias != nullptr) {
      bv.x = c < p.N ? __half2float(bias[c]) : 0.0f;
      bv.y = c + 1 < p.N ? __half2float(bias[c + 1]) : 0.0f;
      bv.z = c + 2 < p.N ? __half2float(bias[c + 2]) : 0.0f;
      bv.w = c + 3 < p.N ? __half2float(bias[c + 3]) : 0.0f;
    }
    *reinterpret_cast<float4*>(s.bias + 4 * et) = bv;
  }
}

// Outlier rows O[t0 .. t0+tn) of W over the tile's BN columns, as the pieces
// (8 columns each) this epilogue thread stages: rows up to the next multiple
// of 16 are zero so that a partly used k16 step adds exact zeros.  Loaded into
// registers first (load_outlier_rows), so that the loads of the next pass are
// in flight while the current pass computes, then stored to shared memory
// (store_outlier_rows, rows kWoStride apart).
constexpr int kWoPieces = (kSG * (BN / 8) + kEpiThreads - 1) / kEpiThreads;  // pieces per thread (2)

__device__ __forceinline__ void load_outlier_rows(const GemmArgs& p, int nb, int t0, int tn, int et, bool w_vec,
                                                  uint4 (&u)[kWoPieces]) {
  const __half* W = static_cast<const __half*>(p.W);
  const int n0 = nb * BN;
#pragma unroll
  for (int k = 0; k < kWoPieces; ++k) {
    const int pc = et + k * kEpiThreads;
    const int t = pc / (BN / 8);
    const int cc = 8 * (pc % (BN / 8));
    const int c = n0 + cc;
    u[k] = make_uint4(0u, 0u, 0u, 0u);
    if (t < tn && W == nullptr) {  // no fp16 weight kept: the rows recovered from Wq
      const int64_t kk = __ldg(p.O + t0 + t);
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = c + 2 * e;
        const uint32_t lo = n < p.N ? dequant_weight_bits(p.Wq[int64_t(n) * p.ldk + kk], __ldg(p.cs + n)) : 0u;
        const uint32_t hi =
            n + 1 < p.N ? dequant_weight_bits(p.Wq[int64_t(n + 1) * p.ldk + kk], __ldg(p.cs + n + 1)) : 0u;
        w[e] = lo | (hi << 16);
      }
      u[k] = make_uint4(w[0], w[1], w[2], w[3]);
    } else if (t < tn) {
      const __half* wr = W + static_cast<int64_t>(__ldg(p.O + t0 + t)) * p.ldw + c;
      if (w_vec && c + 8 <= p.N) {
        u[k] = __ldg(reinterpret_cast<const uint4*>(wr));
      } else {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t lo = (c + 2 * e < p.N) ? __half_as_ushort(wr[2 * e]) : 0u;
          const uint32_t hi = (c + 2 * e + 1 < p.N) ? __half_as_ushort(wr[2 * e + 1]) : 0u;
          w[e] = lo | (hi << 16);
        }
        u[k] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

__device__ __forceinline__ void store_outlier_rows(const Shared& s, int et, const uint4 (&u)[kWoPieces]) {
#pragma unroll
  for (int k = 0; k < kWoPieces; ++k) {
    const int pc = et + k * kEpiThreads;
    if (pc < kSG * (BN / 8)) {
      const int t = pc / (BN / 8);
      const int cc = 8 * (pc % (BN / 8));
      *reinterpret_cast<uint4*>(s.wo + t * kWoStride + cc) = u[k];
    }
  }
}

// The same for one 64-column chunk c of the tile and up to kRound outlier rows
// O[t0 .. t0+tn) (rows kWo2Stride apart, zero up to the next multiple of 16).
constexpr int kWo2Pieces = (kRound * 8 + kEpiThreads - 1) / kEpiThreads;  // pieces per thread (3)

__device__ __forceinline__ void load_outlier_chunk(const GemmArgs& p, int nb, int c, int t0, int tn, int et,
                                                   bool w_vec, uint4 (&u)[kWo2Pieces]) {
  const __half* W = static_cast<const __half*>(p.W);
  const int n0 = nb * BN + 64 * c;
#pragma unroll
  for (int k = 0; k < kWo2Pieces; ++k) {
    const int pc = et + k * kEpiThreads;
    const int t = pc >> 3;
    const int col = n0 + 8 * (pc & 7);
    u[k] = make_uint4(0u, 0u, 0u, 0u);
    if (t < tn && W == nullptr) {  // no fp16 weight kept: the rows recovered from Wq
      const int64_t kk = __ldg(p.O + t0 + t);
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = col + 2 * e;
        const uint32_t lo = n < p.N ? dequant_weight_bits(p.Wq[int64_t(n) * p.ldk + kk], __ldg(p.cs + n)) : 0u;
        const uint32_t hi =
            n + 1 < p.N ? dequant_weight_bits(p.Wq[int64_t(n + 1) * p.ldk + kk], __ldg(p.cs + n + 1)) : 0u;
        w[e] = lo | (hi << 16);
      }
      u[k] = make_uint4(w[0], w[1], w[2], w[3]);
    } else if (t < tn) {
      const __half* wr = W + static_cast<int64_t>(__ldg(p.O + t0 + t)) * p.ldw + col;
      if (w_vec && col + 8 <= p.N) {
        u[k] = __ldg(reinterpret_cast<const uint4*>(wr));
      } else {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t lo = (col + 2 * e < p.N) ? __half_as_ushort(wr[2 * e]) : 0u;
          const uint32_t hi = (col + 2 * e + 1 < p.N) ? __half_as_ushort(wr[2 * e + 1]) : 0u;
          w[e] = lo | (hi << 16);
        }
        u[k] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

__device__ __forceinline__ void store_outlier_chunk(const Shared& s, int et, int tn, const uint4 (&u)[kWo2Pieces]) {
  const int rows = (tn + 15) & ~15;
#pragma unroll
  for (int k = 0; k < kWo2Pieces; ++k) {
    const int pc = et + k * kEpiThreads;
    if ((pc >> 3) < rows) *reinterpret_cast<uint4*>(s.wo + (pc >> 3) * kWo2Stride + 8 * (pc & 7)) = u[k];
  }
}

// Exact int32 -> fp32 for |a| < 2^22 by the exponent-bias trick (two full-rate
// operations instead of one conversion-pipe instruction); falls back to the
// conversion instruction otherwise.  Both give the exact value whenever it is
// representable; the int32 accumulator needs |a| <= 127^2 K.
__device__ __forceinline__ float i2f_exact(int32_t a) {
  if (static_cast<uint32_t>(a) + (1u << 22) < (1u << 23))
    return __fsub_rn(__int_as_float(0x4B400000 + a), 12582912.0f);
  return static_cast<float>(a);
}

// A fragment (16 rows x 16 outliers, fp16) of mma.m16n8k16 for rows r0..r0+15
// and outliers k0..k0+15 of the gathered Xo; outliers at or past `kend` and
// rows past M read as zero.
__device__ __forceinline__ void load_xo_fragment(const GemmArgs& p, int r0, int k0, int kend, uint32_t lane,
                                                 uint32_t (&a)[4]) {
  const __half* Xo = static_cast<const __half*>(p.Xo);
  const int g = static_cast<int>(lane >> 2), t4 = static_cast<int>(lane & 3);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + g + ((i & 1) ? 8 : 0);
    const int k = k0 + 2 * t4 + ((i & 2) ? 8 : 0);
    uint32_t lo = 0u, hi = 0u;
    if (r < p.M) {
      const __half* x = Xo + static_cast<int64_t>(r) * p.ldo;
      if (k < kend) lo = __half_as_ushort(x[k]);
      if (k + 1 < kend) hi = __half_as_ushort(x[k + 1]);
    }
    a[i] = lo | (hi << 16);
  }
}

// This CTA's share of the operands of the tensor-core outlier product, by all
// epilogue threads before the first tile: W^T [N, 256] (row j of column n is
// W[O[j], n], or the row recovered from Wq without an fp16 weight) and Xo
// [M, 256], zero from n_o up to the 64-column blocks the MMAs read (columns
// past them are never read), in units of kOmUnit rows.  W rows are read along
// N and transposed through shared memory so that both sides are coalesced.
__device__ void gather_outlier_operands(const GemmArgs& p, const Shared& s, int et, int om) {
  const int n_o = *p.n_o;
  const int ncol = 64 * om;  // columns written per row
  const int units_n = (p.N + kOmUnit - 1) / kOmUnit;
  const int units = units_n + (p.M + kOmUnit - 1) / kOmUnit;
  const __half* W = static_cast<const __half*>(p.W);
  const __half* Xo = static_cast<const __half*>(p.Xo);
  uint16_t* wt = static_cast<uint16_t*>(p.wo_t);
  uint16_t* xp = static_cast<uint16_t*>(p.xo_p);
  const bool w_vec = (p.ldw % 8 == 0) && (reinterpret_cast<uintptr_t>(p.W) % 16 == 0);
  uint16_t* tile = reinterpret_cast<uint16_t*>(s.wo);  // [kOmUnit][kOmStride]
  for (int u = static_cast<int>(blockIdx.x); u < units; u += static_cast<int>(gridDim.x)) {
    if (u >= units_n) {  // Xo rows
      const int m0 = (u - units_n) * kOmUnit;
      for (int i = et; i < kOmUnit * kOmCols; i += kEpiThreads) {
        const int m = m0 + i / kOmCols, j = i % kOmCols;
        if (m < p.M && j < ncol) xp[int64_t(m) * kOmCols + j] = j < n_o ? __half_as_ushort(Xo[int64_t(m) * p.ldo + j]) : 0;
      }
      continue;
    }
    const int n0 = u * kOmUnit;
    if (W == nullptr) {  // no fp16 weight kept: the rows recovered from Wq
      for (int i = et; i < kOmUnit * kOmCols; i += kEpiThreads) {
        const int n = n0 + i / kOmCols, j = i % kOmCols;
        if (n < p.N && j < ncol)
          wt[int64_t(n) * kOmCols + j] =
              j < n_o ? dequant_weight_bits(p.Wq[int64_t(n) * p.ldk + __ldg(p.O + j)], __ldg(p.cs + n)) : 0;
      }
      continue;
    }
    // pieces of 8 columns of a W row into the transposing tile
    for (int pc = et; pc < kOmCols * (kOmUnit / 8); pc += kEpiThreads) {
      const int j = pc / (kOmUnit / 8), c = 8 * (pc % (kOmUnit / 8));
      if (j >= ncol) continue;
      uint16_t v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (j < n_o) {
        const __half* wr = W + int64_t(__ldg(p.O + j)) * p.ldw + n0 + c;
        if (w_vec && n0 + c + 8 <= p.N) {
          const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(wr));
          const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[2 * e] = static_cast<uint16_t>(w[e] & 0xFFFFu);
            v[2 * e + 1] = static_cast<uint16_t>(w[e] >> 16);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (n0 + c + e < p.N) v[e] = __half_as_ushort(wr[e]);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) tile[(c + e) * kOmStride + j] = v[e];
    }
    named_bar_sync(1, kEpiThreads);
    for (int pc = et; pc < kOmUnit * (kOmCols / 8); pc += kEpiThreads) {
      const int r = pc / (kOmCols / 8), c = 8 * (pc % (kOmCols / 8));
      if (n0 + r < p.N && c < ncol)
        *reinterpret_cast<uint4*>(wt + int64_t(n0 + r) * kOmCols + c) =
            *reinterpret_cast<const uint4*>(tile + r * kOmStride + c);
    }
    named_bar_sync(1, kEpiThreads);  // the tile is free for the next unit
  }
}

template <bool kRaw, bool kPair>
__device__ void run_epilogue(const GemmArgs& p, const CUtensorMap& tmY, const Shared& s, uint32_t tmem_base,
                             const Sched& sc, uint32_t rank, uint32_t warp, uint32_t lane, int om) {
  using G = Geo<kPair>;
  const uint32_t q = warp & 3u;             // TMEM lane quarter this warp may access
  const int ab = static_cast<int>(warp - 2) >> 2;  // which 16 rows of the quarter
  const int et = static_cast<int>(threadIdx.x) - 64;  // 0..kEpiThreads-1
  const int n_o = kRaw ? 0 : *p.n_o;
  const bool overflow = n_o > p.cap;
  const int n_use = overflow ? 0 : n_o;
  const int passes = n_use > 0 ? (n_use + kSG - 1) / kSG : 1;  // outlier row groups staged per tile
  // Where the 16-bit outlier product runs.  As mma.sync it shares the tensor
  // cores with the next tile's tcgen05 MMAs and waits behind them (with six
  // outliers on the 6.7B FFN shape that stretched the first tile's epilogue
  // past the next main loop and held every later tile back); on the CUDA
  // cores it costs about 0.56 us per outlier and tile, against a main loop of
  // about 2.7 ns per unit of K.  So: the CUDA cores while n_o <= K / 256 (the
  // epilogue stays inside the next main loop), mma.sync past that.
  const bool core_product = int64_t(n_use) * 256 <= int64_t(p.K);
  __half* Y = static_cast<__half*>(p.Y);
  const bool y_pair = (p.ldy % 2 == 0) && (reinterpret_cast<uintptr_t>(p.Y) % 4 == 0);
  const bool w_vec = (p.ldw % 8 == 0) && (reinterpret_cast<uintptr_t>(p.W) % 16 == 0);
  const bool c_vec = (p.ldc % 4 == 0) && (reinterpret_cast<uintptr_t>(p.C) % 16 == 0);
  const bool cs_vec = (reinterpret_cast<uintptr_t>(p.cs) % 16 == 0);
  const int g = static_cast<int>(lane >> 2), t4 = static_cast<int>(lane & 3);
  // the pair leader's TMEM-empty barriers collect the arrivals of both CTAs
  const uint32_t tempty_leader = kPair ? mapa_shared(smem_u32(s.tempty), 0) : smem_u32(s.tempty);
  // ldmatrix row address of this lane inside a 16 x 16 block of staged W rows
  const uint32_t wo_lane = smem_u32(s.wo) + 2u * static_cast<uint32_t>(((lane & 7) + 8 * ((lane >> 3) & 1)) *
                                                                          kWoStride + 8 * (lane >> 4));
  // this warp's Y staging tile (1024-byte aligned: the 128-byte swizzle repeats every 8 rows)
  const uint32_t ystage_off = static_cast<uint32_t>(warp - 2) * G::kYBytes;
  const uint32_t ystage = smem_u32(s.ystage) + ystage_off;
  // the dequantized-tile barriers (tensor-core outlier product; the pair leader's for CTA pairs)
  const uint32_t deq_leader = kPair ? mapa_shared(smem_u32(s.deq), 0) : smem_u32(s.deq);
  if (om > 0) {
    // this CTA's share of the gathered operands, then one release per CTA
    // (the producers wait for all of them before their first outlier block)
    gather_outlier_operands(p, s, et, om);
    fence_proxy_async_global();
    named_bar_sync(1, kEpiThreads);
    if (et == 0) red_add_release_gpu_u32(p.om_sync, 1u);
  }

  uint32_t it = 0;
  for (int tile = sc.first; tile < sc.num_tiles; tile += sc.stride, ++it) {
    const uint32_t b = it & 1u;
    const uint32_t use = (it >> 1) & 1u;
    int mb, nb;
    tile_coords(tile, sc, mb, nb);
    const int wrow0 = mb * G::kTileM + (kPair ? static_cast<int>(rank) * BM : 0) + static_cast<int>(q * 32);
    const int r0 = wrow0 + 16 * ab;  // this warp's 16 rows
    const uint32_t tacc = tmem_base + ((q * 32u + 16u * ab) << 16) + b * kAccCols;

    // Everything but the accumulator is fetched before waiting for it.
    float rsc[2] = {0.0f, 0.0f};  // rows g, g + 8
    uint32_t afr[4];              // Xo fragment of the first pass
    if constexpr (!kRaw) {
      named_bar_sync(1, kEpiThreads);  // the previous tile's readers of the staged data are done
      stage_scales(p, s, nb, et, cs_vec);
      if (om > 0) {
        // the outlier product runs on the tensor cores: nothing to stage
      } else if (passes > 1) {  // many outliers: the first chunk's rows of the first round
        uint4 u[kWo2Pieces];
        load_outlier_chunk(p, nb, 0, 0, min(n_use, kRound), et, w_vec, u);
        store_outlier_chunk(s, et, min(n_use, kRound), u);
      } else {
        uint4 u[kWoPieces];
        load_outlier_rows(p, nb, 0, min(n_use, kSG), et, w_vec, u);
        store_outlier_rows(s, et, u);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = r0 + g + 8 * h;
        if (r < p.M) rsc[h] = __ldg(p.rs + r) * (1.0f / 16129.0f);
      }
      if (n_use > 0 && om == 0) load_xo_fragment(p, r0, 0, min(n_use, kSG), lane, afr);
    }

    const bool got = wait_or_abort(&s.tfull[b], use, p.status, s.abort);
    if (!named_bar_and(2, kEpiThreads, got)) break;  // all epilogue threads stop together; staged data visible
    tc_fence_after();

    if constexpr (kRaw) {
      // the lane quarter's 32 rows, columns split between its two warps
      const int row = wrow0 + static_cast<int>(lane);
      const uint32_t traw = tmem_base + ((q * 32u) << 16) + b * kAccCols;
#pragma unroll 1
      for (int c = ab * (BN / kChunk / 2); c < (ab + 1) * (BN / kChunk / 2); ++c) {
        const int col0 = nb * BN + c * kChunk;
        uint32_t v[32];
        tmem_ld_32x32b_x32(traw + c * kChunk, v);
        tmem_ld_wait();
        if (row < p.M) {
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
      }
    } else {
      // a finished 64-column chunk: the bias, then fp16 Y (TMA store through
      // the swizzled staging tile, or direct stores); an unfinished one (more
      // rounds of outliers to come) is parked in its own TMEM columns
      auto finish = [&](int c, float (&d)[8][4], bool last, uint32_t taddr, uint32_t (&v)[32]) {
        if (last && p.bias != nullptr) {  // the linear layer's bias, added last
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            const float2 b2 = *reinterpret_cast<const float2*>(s.bias + c * 64 + 8 * n + 2 * t4);
            d[n][0] += b2.x;
            d[n][1] += b2.y;
            d[n][2] += b2.x;
            d[n][3] += b2.y;
          }
        }
        if (last) {
          // fp16 Y through the warp's 16 x 64 staging tile (128-byte swizzle):
          // a TMA store when Y's rows are 16-byte aligned; otherwise one row
          // at a time, each store instruction covering 64 consecutive columns
          // of a row (stores from the fragment layout would scatter over
          // eight rows each)
          uint32_t lo[8], hi[8];
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            float y0 = d[n][0], y1 = d[n][1], y2 = d[n][2], y3 = d[n][3];
            if (overflow) y0 = y1 = y2 = y3 = __int_as_float(0x7fc00000);
            const __half2 a = __floats2half2_rn(y0, y1), bb = __floats2half2_rn(y2, y3);
            lo[n] = *reinterpret_cast<const uint32_t*>(&a);
            hi[n] = *reinterpret_cast<const uint32_t*>(&bb);
          }
          // the previous store (TMA) or row reads (direct) have left the staging tile
          if (p.y_tma && lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t rr = (lane & 7) + 8 * ((lane >> 3) & 1);
            const uint32_t nn = 2 * i + (lane >> 4);
            stmatrix_x4(ystage + rr * 128u + ((nn ^ (rr & 7)) << 4), lo[2 * i], hi[2 * i], lo[2 * i + 1],
                        hi[2 * i + 1]);
          }
          if (p.y_tma) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, s.ystage + ystage_off, nb * BN + c * 64, r0);
              bulk_commit();
            }
          } else {
            __syncwarp();
            const int col = nb * BN + c * 64 + 2 * static_cast<int>(lane);  // this lane's two columns
#pragma unroll 1
            for (int rr = 0; rr < 16; ++rr) {
              const int r = r0 + rr;
              if (r >= p.M) break;
              const uint32_t w = ld_shared_u32(ystage + static_cast<uint32_t>(rr) * 128u +
                                               (((lane >> 2) ^ static_cast<uint32_t>(rr & 7)) << 4) + (lane & 3) * 4u);
              __half* yr = Y + static_cast<int64_t>(r) * p.ldy;
              if (y_pair && col + 1 < p.N) {
                *reinterpret_cast<uint32_t*>(yr + col) = w;
              } else {
                if (col < p.N) yr[col] = __ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu));
                if (col + 1 < p.N) yr[col + 1] = __ushort_as_half(static_cast<unsigned short>(w >> 16));
              }
            }
          }
        } else {
#pragma unroll
          for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) v[4 * n + e] = __float_as_uint(d[n][e]);
          tmem_st_16x256b_x8(taddr, v);
        }
      };
      // dequantize: acc * rs[row] * cs[col] / 127^2
      auto dequant = [&](int c, const uint32_t (&v)[32], float (&d)[8][4]) {
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          const float2 c2 = *reinterpret_cast<const float2*>(s.cs + c * 64 + 8 * n + 2 * t4);
          d[n][0] = i2f_exact(static_cast<int32_t>(v[4 * n + 0])) * rsc[0] * c2.x;
          d[n][1] = i2f_exact(static_cast<int32_t>(v[4 * n + 1])) * rsc[0] * c2.y;
          d[n][2] = i2f_exact(static_cast<int32_t>(v[4 * n + 2])) * rsc[1] * c2.x;
          d[n][3] = i2f_exact(static_cast<int32_t>(v[4 * n + 3])) * rsc[1] * c2.y;
        }
      };
      if (om > 0) {
        // Tensor-core outlier product: dequantize the tile in place (fp32 over
        // the int32 accumulator), hand it to the MMA thread, and finish each
        // chunk once the outlier MMAs have accumulated onto it.
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {
          const uint32_t taddr = tacc + c * 64;
          uint32_t v[32];
          tmem_ld_16x256b_x8(taddr, v);
          tmem_ld_wait();
#pragma unroll
          for (int n = 0; n < 8; ++n) {  // acc * rs[row] * cs[col] / 127^2, in place
            const float2 c2 = *reinterpret_cast<const float2*>(s.cs + c * 64 + 8 * n + 2 * t4);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              v[4 * n + e] = __float_as_uint(i2f_exact(static_cast<int32_t>(v[4 * n + e])) * rsc[e >> 1] *
                                             ((e & 1) ? c2.y : c2.x));
          }
          tmem_st_16x256b_x8(taddr, v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kPair)
            mbar_arrive_cluster(deq_leader + b * 8u);
          else
            mbar_arrive(&s.deq[b]);
        }
        const bool done = wait_or_abort(&s.ofull[b], use, p.status, s.abort);
        if (!named_bar_and(2, kEpiThreads, done)) break;
        tc_fence_after();
      }
      if (om > 0 || passes <= 1) {
        // At most 16 outliers: their W rows over the whole tile were staged
        // before the accumulator wait; one k16 step of the 16-bit product.
        // On the CUDA cores: fp32 fused multiply-adds of the exact fp16
        // products; the four lanes of a row pair hold all 16 outlier values of
        // rows g and g + 8 in their A fragments, a pair of them is one shuffle
        // per row.
        const __half* wo = s.wo + 2 * t4;
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {  // 64 accumulator columns at a time
          const uint32_t taddr = tacc + c * 64;
          uint32_t v[32];
          tmem_ld_16x256b_x8(taddr, v);
          tmem_ld_wait();
          float d[8][4];
          if (om > 0) {  // dequantized, with the outlier product added by the tensor cores
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
              for (int e = 0; e < 4; ++e) d[n][e] = __uint_as_float(v[4 * n + e]);
          } else {
            dequant(c, v, d);
          }
          // d += Xo[rows, k] * W[O[k], cols], k < n_use
          if (!core_product && om == 0) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4_trans(wo_lane + 2u * static_cast<uint32_t>(c * 64 + 16 * np), b0, b1, b2, b3);
              mma_m16n8k16_f16f32(d[2 * np], afr, b0, b1);
              mma_m16n8k16_f16f32(d[2 * np + 1], afr, b2, b3);
            }
          }
#pragma unroll 1
          for (int kp = 0; core_product && 2 * kp < n_use; ++kp) {  // k = 2 kp, 2 kp + 1 (a W row past n_use is zero)
            const int src = 4 * g + (kp & 3);
            const uint32_t xa = __shfl_sync(0xffffffffu, kp < 4 ? afr[0] : afr[2], src);  // row g
            const uint32_t xb = __shfl_sync(0xffffffffu, kp < 4 ? afr[1] : afr[3], src);  // row g + 8
            const float2 xg = __half22float2(*reinterpret_cast<const __half2*>(&xa));
            const float2 xh = __half22float2(*reinterpret_cast<const __half2*>(&xb));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float2 x0 = h ? make_float2(xg.y, xg.y) : make_float2(xg.x, xg.x);
              const float2 x8 = h ? make_float2(xh.y, xh.y) : make_float2(xh.x, xh.x);
              const __half* wr = wo + (2 * kp + h) * kWoStride + c * 64;
#pragma unroll
              for (int n = 0; n < 8; ++n) {
                const float2 w2 = __half22float2(*reinterpret_cast<const __half2*>(wr + 8 * n));
                const float2 lo = __ffma2_rn(x0, w2, make_float2(d[n][0], d[n][1]));
                const float2 hi = __ffma2_rn(x8, w2, make_float2(d[n][2], d[n][3]));
                d[n][0] = lo.x;
                d[n][1] = lo.y;
                d[n][2] = hi.x;
                d[n][3] = hi.y;
              }
            }
          }
          finish(c, d, true, taddr, v);
        }
      } else {
        // more than 16 outliers: rounds of up to kRound, and inside a round
        // the 64-column chunks outermost, each staging the round's W rows for
        // its 64 columns (the next chunk's rows loaded into registers while this
        // one computes); the accumulator chunk is read once per round and all
        // the round's k16 steps run on it in registers
        const int rounds = (n_use + kRound - 1) / kRound;
        const uint32_t wo2_lane =
            smem_u32(s.wo) + 2u * static_cast<uint32_t>(((lane & 7) + 8 * ((lane >> 3) & 1)) * kWo2Stride + 8 * (lane >> 4));
        uint4 wn[kWo2Pieces];
        uint32_t ax[kRound / kSG][4];  // Xo fragments of the round's k16 steps
#pragma unroll 1
        for (int rnd = 0; rnd < rounds; ++rnd) {
          const int tr0 = rnd * kRound;
          const int trn = min(kRound, n_use - tr0);
          const int pr = (trn + kSG - 1) / kSG;
          const bool last = rnd == rounds - 1;
#pragma unroll
          for (int q = 0; q < kRound / kSG; ++q)
            if (q < pr) load_xo_fragment(p, r0, tr0 + kSG * q, tr0 + min(kSG * (q + 1), trn), lane, ax[q]);
#pragma unroll 1
          for (int c = 0; c < BN / 64; ++c) {
            if (rnd > 0 || c > 0) {
              named_bar_sync(1, kEpiThreads);  // the previous chunk's rows are no longer read
              store_outlier_chunk(s, et, trn, wn);
              named_bar_sync(1, kEpiThreads);
            }
            {
              int nrd = rnd, nc = c + 1;
              if (nc == BN / 64) {
                nc = 0;
                ++nrd;
              }
              if (nrd < rounds)
                load_outlier_chunk(p, nb, nc, nrd * kRound, min(kRound, n_use - nrd * kRound), et, w_vec, wn);
            }
            const uint32_t taddr = tacc + c * 64;
            uint32_t v[32];
            tmem_ld_16x256b_x8(taddr, v);
            tmem_ld_wait();
            float d[8][4];
            if (rnd == 0) {
              dequant(c, v, d);
            } else {
#pragma unroll
              for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) d[n][e] = __uint_as_float(v[4 * n + e]);
            }
            if (core_product) {
              // on the CUDA cores (k = 16 q + 2 kp + h)
#pragma unroll
              for (int q = 0; q < kRound / kSG; ++q) {
                if (q < pr) {
#pragma unroll 1
                  for (int kp = 0; kSG * q + 2 * kp < trn && kp < kSG / 2; ++kp) {
                    const int src = 4 * g + (kp & 3);
                    const uint32_t xa = __shfl_sync(0xffffffffu, kp < 4 ? ax[q][0] : ax[q][2], src);
                    const uint32_t xb = __shfl_sync(0xffffffffu, kp < 4 ? ax[q][1] : ax[q][3], src);
                    const float2 xg = __half22float2(*reinterpret_cast<const __half2*>(&xa));
                    const float2 xh = __half22float2(*reinterpret_cast<const __half2*>(&xb));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                      const float2 x0 = h ? make_float2(xg.y, xg.y) : make_float2(xg.x, xg.x);
                      const float2 x8 = h ? make_float2(xh.y, xh.y) : make_float2(xh.x, xh.x);
                      const __half* wr = s.wo + (kSG * q + 2 * kp + h) * kWo2Stride + 2 * t4;
#pragma unroll
                      for (int n = 0; n < 8; ++n) {
                        const float2 w2 = __half22float2(*reinterpret_cast<const __half2*>(wr + 8 * n));
                        const float2 lo = __ffma2_rn(x0, w2, make_float2(d[n][0], d[n][1]));
                        const float2 hi = __ffma2_rn(x8, w2, make_float2(d[n][2], d[n][3]));
                        d[n][0] = lo.x;
                        d[n][1] = lo.y;
                        d[n][2] = hi.x;
                        d[n][3] = hi.y;
                      }
                    }
                  }
                }
              }
            } else {
#pragma unroll
              for (int q = 0; q < kRound / kSG; ++q) {
                if (q < pr) {
#pragma unroll
                  for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(wo2_lane + 2u * static_cast<uint32_t>(q * kSG * kWo2Stride + 16 * np), b0,
                                      b1, b2, b3);
                    mma_m16n8k16_f16f32(d[2 * np], ax[q], b0, b1);
                    mma_m16n8k16_f16f32(d[2 * np + 1], ax[q], b2, b3);
                  }
                }
              }
            }
            finish(c, d, last, taddr, v);
          }
          if (!last) tmem_st_wait();
        }
      }
    }
    // this warp's TMEM reads of buffer b are complete: free it for the MMA
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if constexpr (kPair)
        mbar_arrive_cluster(tempty_leader + b * 8u);
      else
        mbar_arrive(&s.tempty[b]);
    }
  }
  if (lane == 0) bulk_wait_all();  // Y stores complete before the CTA exits
  __syncwarp();
}

template <bool kRaw, bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmXo,
                   const __grid_constant__ CUtensorMap tmWo, const GemmArgs p) {
  using G = Geo<kPair>;
  extern __shared__ uint8_t smem_raw[];
  const Shared s = carve<kPair>(smem_raw);
  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  Sched sc;
  sc.num_m = (p.M + G::kTileM - 1) / G::kTileM;
  sc.num_k = (p.K + BK - 1) / BK;
  sc.num_tiles = sc.num_m * ((p.N + BN - 1) / BN);
  sc.group_m = tile_group_m(sc.num_m, G::kTileM, p.K);
  sc.first = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  sc.stride = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < G::kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], G::kTmemEmptyArrivals);
    }
    mbar_init(s.drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.deq[i], G::kTmemEmptyArrivals);
      mbar_init(&s.ofull[i], 1);
    }
    *s.abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (p.y_tma) tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(s.tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(s.tmem_slot, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // the peer's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;

  griddep_wait();  // Xq, rs, O, n_o and Xo are written by the quantize kernel
  // The next launch on the stream may get resident now: every kernel of this
  // library waits (griddepcontrol.wait) for this grid to complete before it
  // touches memory this grid reads or writes.
  griddep_launch_dependents();
  const bool om_possible = !kRaw && p.om_ok;

  if (warp == 0) {
    if (lane == 0) {
      if (om_possible) {
        prefetch_l1(p.n_o);
        tma_prefetch_desc(&tmXo);
        tma_prefetch_desc(&tmWo);
      }
      run_producer<kPair>(&tmA, &tmB, &tmXo, &tmWo, s, sc, rank, p, om_possible);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      if (om_possible) prefetch_l1(p.n_o);
      run_mma<kPair>(s, tmem_base, sc, p, om_possible);
    }
  } else {
    run_epilogue<kRaw, kPair>(p, tmY, s, tmem_base, sc, rank, warp, lane, om_possible ? outlier_mma_blocks(p) : 0);
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // no CTA leaves while its pair may still signal it
  if (om_possible && threadIdx.x == 0 && outlier_mma_blocks(p) > 0) {
    // the last CTA out returns the gather counters to zero for the next call
    // (every CTA has released its gather share and no producer waits any more)
    if (atomicAdd(p.om_sync + 1, 1u) == gridDim.x - 1) {
      p.om_sync[0] = 0u;
      p.om_sync[1] = 0u;
    }
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (kPair)
      tmem_dealloc_pair(tmem_base, kTmemCols);
    else
      tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <bool kRaw, bool kPair>
cudaError_t launch_variant(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmY,
                           const CUtensorMap& tmXo, const CUtensorMap& tmWo, const GemmArgs& a, int num_sms,
                           cudaStream_t stream, bool pdl) {
  using G = Geo<kPair>;
  static bool attr_set[64] = {};  // per device
  static int max_units[64] = {};  // CTAs (or CTA pairs) that fit at once, per device
  auto kern = gemm_i8_kernel<kRaw, kPair>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::kSmemBytes));
    if (e != cudaSuccess) return e;
    if (kPair) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
      if (e != cudaSuccess) return e;
    }
    max_units[dev] = kPair ? num_sms / 2 : num_sms;
    if (kPair) {
      // a persistent grid must be co-resident: ask how many pairs fit
      cudaLaunchAttribute ca;
      ca.id = cudaLaunchAttributeClusterDimension;
      ca.val.clusterDim.x = 2;
      ca.val.clusterDim.y = 1;
      ca.val.clusterDim.z = 1;
      cudaLaunchConfig_t oc = {};
      oc.gridDim = dim3(static_cast<unsigned>(num_sms));
      oc.blockDim = dim3(kThreads);
      oc.dynamicSmemBytes = G::kSmemBytes;
      oc.attrs = &ca;
      oc.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &oc) == cudaSuccess && n > 0 && n < max_units[dev])
        max_units[dev] = n;
      (void)cudaGetLastError();
    }
    attr_set[dev] = true;
  }
  const int num_tiles = ((a.M + G::kTileM - 1) / G::kTileM) * ((a.N + BN - 1) / BN);
  const int units = max_units[dev];  // CTAs or CTA pairs that run at once
  const int grid = (num_tiles < units ? num_tiles : units) * (kPair ? 2 : 1);

  cudaLaunchAttribute attr[2];
  int n_attr = 0;
  if (pdl) {
    attr[n_attr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n_attr].val.programmaticStreamSerializationAllowed = 1;
    ++n_attr;
  }
  if (kPair) {
    attr[n_attr].id = cudaLaunchAttributeClusterDimension;
    attr[n_attr].val.clusterDim.x = 2;
    attr[n_attr].val.clusterDim.y = 1;
    attr[n_attr].val.clusterDim.z = 1;
    ++n_attr;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = G::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = n_attr ? attr : nullptr;
  cfg.numAttrs = n_attr;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmY, tmXo, tmWo, a);
}

}  // namespace

bool gemm_uses_pair(int M) { return M > BM; }

cudaError_t launch_gemm_i8(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmY,
                           const CUtensorMap& tmXo, const CUtensorMap& tmWo, const GemmArgs& a, bool raw_i32,
                           int num_sms, cudaStream_t stream, bool pdl) {
  const bool pair = gemm_uses_pair(a.M);
  GemmArgs b = a;
  b.om_ok = a.om_ok && !raw_i32 && a.xo_p != nullptr && a.wo_t != nullptr && a.om_sync != nullptr;
  if (raw_i32) {
    return pair ? launch_variant<true, true>(tmA, tmB, tmY, tmXo, tmWo, b, num_sms, stream, pdl)
                : launch_variant<true, false>(tmA, tmB, tmY, tmXo, tmWo, b, num_sms, stream, pdl);
  }
  return pair ? launch_variant<false, true>(tmA, tmB, tmY, tmXo, tmWo, b, num_sms, stream, pdl)
              : launch_variant<false, false>(tmA, tmB, tmY, tmXo, tmWo, b, num_sms, stream, pdl);
}

// Test hook: this file's wait bound (see ptx.cuh).
cudaError_t set_debug_waits_gemm_i8(uint64_t limit_ns) { return set_debug_waits_in_this_file(limit_ns); }

}  // namespace llmint8
