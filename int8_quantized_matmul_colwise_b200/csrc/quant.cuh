// quant.cuh -- exact absmax int8 quantizer shared by the weight and the
// activation kernels.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

namespace llmint8 {

// q = round-half-away-from-zero(127 * x / s) for fp16 values |x| <= s, s > 0,
// computed without a division and exactly:
//  * t = 127 |x| is exact in binary32 (11-bit times 7-bit significands);
//  * r = t * (1/s) is within 2^-22 relative of t/s, so rint(r) is within one
//    of the answer;
//  * the answer is the integer q with (q - 1/2) s <= t < (q + 1/2) s (halves
//    go up, i.e. away from zero); (q +- 1/2) s has at most 9 + 11 significant
//    bits and is exact in binary32, so the two comparisons below decide it
//    exactly.  __fmul_rn/__fadd_rn keep the compiler from fusing them.
__device__ __forceinline__ int quantize_exact(float x, float s, float inv_s) {
  const float t = __fmul_rn(127.0f, fabsf(x));
  if (!(t == t)) return 0;  // NaN input: code 0
  float q = rintf(__fmul_rn(t, inv_s));
  if (__fmul_rn(__fadd_rn(q, 0.5f), s) <= t) {
    q = __fadd_rn(q, 1.0f);
  } else if (__fmul_rn(__fadd_rn(q, -0.5f), s) > t) {
    q = __fadd_rn(q, -1.0f);
  }
  q = fminf(q, 127.0f);
  const int qi = __float2int_rz(q);
  return x < 0.0f ? -qi : qi;
}

// Pack four codes (low byte first) into a 32-bit word.
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (uint32_t(a) & 0xFFu) | ((uint32_t(b) & 0xFFu) << 8) | ((uint32_t(c) & 0xFFu) << 16) |
         ((uint32_t(d) & 0xFFu) << 24);
}

// |h| as the bit pattern of a non-negative fp16; NaN maps to 0 so that it never
// wins a max (NaN compares false against the threshold).
__device__ __forceinline__ uint32_t abs_bits(__half h) {
  const uint32_t b = __half_as_ushort(h) & 0x7FFFu;
  return b > 0x7C00u ? 0u : b;
}

}  // namespace llmint8
