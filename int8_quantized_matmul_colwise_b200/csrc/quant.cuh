// quant.cuh -- exact absmax int8 quantizer shared by the weight and the
// activation kernels.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

namespace llmint8 {

// q = round-half-away-from-zero(127 * x / s) for fp16 values |x| <= s, s > 0
// (s = 0, a vector whose values are all zero or NaN, and NaN x give 0),
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
  if (!(t == t) || !(s > 0.0f)) return 0;  // NaN input, or a vector without a finite nonzero value: code 0
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

// A weight value recovered from its int8 code, for callers that keep no fp16
// weight: fp16_RNE(q * cs / 127), as the bits of the fp16.  q * cs is exact in
// binary32 (7- and 11-bit significands, a = |q| * significand(cs) < 2^18) and
// the quotient is correctly rounded.  Unless the exact quotient is itself an
// fp16 rounding boundary, it lies at least 2^-19 (relative) from one, since
// a * 2^j / 127 is at least 1/127 from every odd integer; the binary32
// rounding moves it by at most 2^-24, so rounding the binary32 quotient to
// fp16 gives the fp16 rounding of the exact value.
__device__ __forceinline__ unsigned short dequant_weight_bits(int q, float cs) {
  return __half_as_ushort(__float2half_rn(__fdiv_rn(__fmul_rn(static_cast<float>(q), cs), 127.0f)));
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

// 8 consecutive fp16 of a row by scalar loads (unaligned rows or a ragged end).
__device__ __forceinline__ uint4 load8_scalar(const __half* __restrict__ row, int64_t K, int64_t c) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t lo = (c + 2 * e < K) ? __half_as_ushort(row[c + 2 * e]) : 0u;
    const uint32_t hi = (c + 2 * e + 1 < K) ? __half_as_ushort(row[c + 2 * e + 1]) : 0u;
    w[e] = lo | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 8 consecutive fp16 of a row as one 16-byte register quad (zero past K).
// kVec: rows are 16-byte aligned and K % 8 == 0, so every chunk that starts
// before K is one aligned 16-byte load (decided on the host).
template <bool kVec>
__device__ __forceinline__ uint4 load8_packed(const __half* __restrict__ row, int64_t K, int64_t c) {
  if constexpr (kVec) return __ldg(reinterpret_cast<const uint4*>(row + c));
  else return load8_scalar(row, K, c);
}

__device__ __forceinline__ unsigned short half_bits_at(const uint4& u, int e) {
  const uint32_t w = (e < 2) ? u.x : (e < 4) ? u.y : (e < 6) ? u.z : u.w;
  return static_cast<unsigned short>((e & 1) ? (w >> 16) : (w & 0xFFFFu));
}

__device__ __forceinline__ uint2 pack8(const int (&q)[8]) {
  uint2 out;
  out.x = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
  return out;
}

// Codes of 8 values (fp16 pairs in u) by the exact comparisons.
__device__ __forceinline__ uint2 quantize8_exact(uint4 u, float s, float inv) {
  const __half2* h2 = reinterpret_cast<const __half2*>(&u);
  int q[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(h2[e]);
    q[2 * e] = quantize_exact(f.x, s, inv);
    q[2 * e + 1] = quantize_exact(f.y, s, inv);
  }
  return pack8(q);
}

// Codes of 8 values by rounding x * (127 / s).  With k = fl(127/s) and
// r = fl(x k), |r - 127x/s| <= 127 (2^-24 + 2^-24)(1 + 2^-24) < 2^-16, so when
// |r - rint(r)| < 1/2 - 2^-15 the exact value is strictly nearer to rint(r)
// than to any other integer and rint(r) is its rounding (no tie possible).
// Otherwise (about one value in 16000, or NaN) tie_risk is set and the caller
// redoes the chunk with quantize8_exact.
// rint is taken as t = r + 1.5 * 2^23: for |r| < 2^22 the sum lies in
// [2^23, 2^24) where the spacing is 1, so it is rounded to the nearest integer
// (ties to even), t - 1.5 * 2^23 is exact, and the low byte of t's bit pattern
// is the integer's low byte (two's complement) -- all on the FMA pipe.
__device__ __forceinline__ uint2 quantize8(uint4 u, float k, bool& tie_risk) {
  constexpr float kSafe = 0.499969482421875f;  // 1/2 - 2^-15
  constexpr float kBias = 12582912.0f;         // 1.5 * 2^23
  const __half2* h2 = reinterpret_cast<const __half2*>(&u);
  uint32_t t[8];
  const float2 k2 = make_float2(k, k);
  const float2 b2 = make_float2(kBias, kBias);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 r = __fmul2_rn(__half22float2(h2[e]), k2);
    const float2 tb = __fadd2_rn(r, b2);
    const float2 q = __fadd2_rn(tb, make_float2(-kBias, -kBias));
    const float2 d = __fadd2_rn(r, make_float2(-q.x, -q.y));
    tie_risk |= !(fabsf(d.x) < kSafe) | !(fabsf(d.y) < kSafe);  // true for NaN as well
    t[2 * e] = __float_as_uint(tb.x);
    t[2 * e + 1] = __float_as_uint(tb.y);
  }
  uint2 out;
  out.x = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
  return out;
}

// max(a, b) that returns NaN when either is NaN (fmaxf drops a NaN operand).
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// quantize8 with fused multiply-adds (fewer instructions, more registers:
// for kernels with registers to spare).  With k = fl(127/s), the exact
// product x k is within 127 * 2^-24 < 2^-17 of v = 127 x / s (|x| <= s).  One
// fused multiply-add gives t = fl(x k + 1.5 * 2^23): for |x k| < 2^22 the sum
// lies in [2^23, 2^24) where the spacing is 1, so t - 1.5 * 2^23 = q is x k
// rounded to an integer (ties to even), exactly, and the low byte of t's bit
// pattern is q's low byte (two's complement).  A second one, with -k, gives
// d = fl(q - x k), within 2^-25 of q - x k.  When |d| < 1/2 - 2^-15,
// |v - q| < 1/2 - 2^-15 + 2^-25 + 2^-17 < 1/2: q is the integer nearest to v
// and v is no tie, so q is its round-half-away-from-zero value.  Otherwise
// (about one value in 16000, or NaN: the maximum of |d| over the chunk
// propagates NaN) tie_risk is set and the caller redoes the chunk with quantize8_exact.  The
// arithmetic runs two values per instruction on the FMA pipe.
__device__ __forceinline__ uint2 quantize8_fma(uint4 u, float k, bool& tie_risk) {
  constexpr float kSafe = 0.499969482421875f;  // 1/2 - 2^-15
  constexpr float kBias = 12582912.0f;         // 1.5 * 2^23
  const __half2* h2 = reinterpret_cast<const __half2*>(&u);
  uint32_t t[8];
  const float2 k2 = make_float2(k, k);
  const float2 nk2 = make_float2(-k, -k);
  const float2 b2 = make_float2(kBias, kBias);
  const float2 nb2 = make_float2(-kBias, -kBias);
  float dmax = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __half22float2(h2[e]);
    const float2 tb = __ffma2_rn(x, k2, b2);
    const float2 q = __fadd2_rn(tb, nb2);
    const float2 d = __ffma2_rn(x, nk2, q);
    dmax = fmax_nan(dmax, fmax_nan(fabsf(d.x), fabsf(d.y)));
    t[2 * e] = __float_as_uint(tb.x);
    t[2 * e + 1] = __float_as_uint(tb.y);
  }
  tie_risk |= !(dmax < kSafe);  // true for NaN as well
  uint2 out;
  out.x = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
  out.y = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
  return out;
}

// Maximum of R per-lane values over `width` lanes (a power of two >= R),
// halving the vector at each step: after the call the lane holds the maximum
// of row `row` over its width lanes (lanes that agree on the low bits below
// width / R hold the same row).
template <int R>
__device__ __forceinline__ float rows_max_transposed(float (&v)[R], int width, int lane, int& row) {
  int o = width >> 1;
  row = 0;
#pragma unroll
  for (int half = R >> 1; half > 0; half >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float mine = up ? v[j + half] : v[j];
      const float other = up ? v[j] : v[j + half];
      v[j] = fmaxf(mine, __shfl_xor_sync(0xffffffffu, other, o));
    }
    row += up ? half : 0;
    o >>= 1;
  }
  float x = v[0];
  for (; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

}  // namespace llmint8
