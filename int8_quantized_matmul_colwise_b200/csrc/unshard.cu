// unshard.cu -- reassembly of a column-sharded output after an all-gather.
//
// When the output columns (the rows of Wq) are split across GPUs, each GPU
// computes Y[:, n_r .. n_{r+1}) for the same replicated X ("Compress your
// LLMs": the deployments the pages describe serve one model from 8 GPUs).  An
// all-gather then leaves every GPU holding the blocks side by side, block r as
// fp16 [M, ld_block] with its first n_{r+1} - n_r columns valid.  This kernel
// copies them into Y [M, N] (row-major, ldy): a pure data move, bound by HBM.
// 16-byte loads and stores when every block start and both row strides are
// multiples of 8 halves; 2-byte moves otherwise.
#include <cuda_fp16.h>

#include "kernels.cuh"

namespace llmint8 {

namespace {

template <bool kVec>
__global__ void __launch_bounds__(256) unshard_columns_kernel(const __half* __restrict__ blocks, int64_t M,
                                                              int64_t ld_block, UnshardBounds b,
                                                              __half* __restrict__ Y, int64_t ldy) {
  const int r = static_cast<int>(blockIdx.y);
  const int64_t n0 = b.bounds[r];
  const int64_t w = b.bounds[r + 1] - n0;
  const __half* src = blocks + int64_t(r) * M * ld_block;
  constexpr int E = kVec ? 8 : 1;                // halves per move
  const int64_t per_row = (w + E - 1) / E;
  const int64_t total = M * per_row;
  for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = t / per_row;
    const int64_t j = (t - i * per_row) * E;
    if constexpr (kVec) {
      // w is a multiple of 8 except in the last block; its tail is moved singly
      if (j + 8 <= w) {
        *reinterpret_cast<uint4*>(Y + i * ldy + n0 + j) = __ldg(reinterpret_cast<const uint4*>(src + i * ld_block + j));
      } else {
        for (int64_t e = j; e < w; ++e) Y[i * ldy + n0 + e] = src[i * ld_block + e];
      }
    } else {
      Y[i * ldy + n0 + j] = src[i * ld_block + j];
    }
  }
}

}  // namespace

cudaError_t launch_unshard_columns(const void* blocks, int world, int64_t M, int64_t ld_block, const UnshardBounds& b,
                                   void* Y, int64_t ldy, int num_sms, cudaStream_t stream) {
  bool vec = ld_block % 8 == 0 && ldy % 8 == 0 && reinterpret_cast<uintptr_t>(blocks) % 16 == 0 &&
             reinterpret_cast<uintptr_t>(Y) % 16 == 0;
  for (int r = 0; r < world; ++r) vec = vec && b.bounds[r] % 8 == 0;
  int64_t widest = 0;
  for (int r = 0; r < world; ++r) widest = b.bounds[r + 1] - b.bounds[r] > widest ? b.bounds[r + 1] - b.bounds[r] : widest;
  const int64_t moves = M * ((widest + (vec ? 7 : 0)) / (vec ? 8 : 1));
  // enough CTAs per block to fill the SMs a few times over, no more than the work
  const int64_t want = (int64_t(num_sms) * 4 + world - 1) / world;
  const int64_t need = (moves + 255) / 256;
  const unsigned gx = static_cast<unsigned>(need < want ? (need > 0 ? need : 1) : want);
  const dim3 grid(gx, static_cast<unsigned>(world));
  const __half* src = static_cast<const __half*>(blocks);
  __half* dst = static_cast<__half*>(Y);
  if (vec)
    unshard_columns_kernel<true><<<grid, 256, 0, stream>>>(src, M, ld_block, b, dst, ldy);
  else
    unshard_columns_kernel<false><<<grid, 256, 0, stream>>>(src, M, ld_block, b, dst, ldy);
  return cudaGetLastError();
}

}  // namespace llmint8
