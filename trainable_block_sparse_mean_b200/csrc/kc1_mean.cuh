// Mean of 32 bf16 key rows (one stage-1 kernel, one 8-element slice of the
// head dim), summed in fp64 in token order and rounded once to bf16.  Shared
// by the prefill compression kernel and the decode step's incremental update,
// so both produce bit-identical K^C1.
#pragma once
#include <stdint.h>

namespace infv2 {

// Nearest bf16 to a double, ties to the even significand, from the double's
// bit fields: keep the top 8 significant bits (fewer in the bf16 subnormal
// range) and round on the dropped bits.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(x);
  const uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
  const unsigned long long a = u & 0x7FFFFFFFFFFFFFFFull;
  if (a > 0x7FF0000000000000ull) return 0x7FC0;                 // NaN
  if (a == 0x7FF0000000000000ull) return (uint16_t)(sign | 0x7F80u);  // inf
  const int e = (int)(a >> 52);
  if (e == 0) return sign;  // fp64 subnormal: far below half the least bf16
  const unsigned long long M = (a & 0xFFFFFFFFFFFFFull) | (1ull << 52);  // value = M * 2^(E-52)
  const int E = e - 1023;
  int q = E - 7;             // exponent of the bf16 quantum at this magnitude
  if (q < -133) q = -133;    // bf16 subnormal quantum
  const int shift = q - (E - 52);  // low bits of M below the quantum (>= 45)
  unsigned long long r;
  if (shift >= 64) {
    r = 0;  // below a quarter quantum: rounds to zero
  } else {
    r = M >> shift;
    const unsigned long long rem = M & ((1ull << shift) - 1ull);
    const unsigned long long half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (r & 1ull))) ++r;
  }
  if (r == 0) return sign;
  // r * 2^q with r <= 256 is exact in fp32 (or overflows to inf)
  const float f = ldexpf((float)r, q);
  return (uint16_t)(sign | (uint16_t)((__float_as_uint(f) >> 16) & 0x7FFFu));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// src points at token 16j's slice; rows are `row_stride` elements apart.  If
// subst_row >= 0, that row (0..31) is read from `subst` instead (the decode
// step's new token, written in the same kernel).
__device__ __forceinline__ uint4 kc1_mean_slice(const uint16_t* src, size_t row_stride,
                                                const uint16_t* subst, int subst_row) {
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 4
  for (int t = 0; t < 32; ++t) {
    const uint16_t* p = (t == subst_row) ? subst : src + (size_t)t * row_stride;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
    acc[0] += (double)bf16_lo(w.x);
    acc[1] += (double)bf16_hi(w.x);
    acc[2] += (double)bf16_lo(w.y);
    acc[3] += (double)bf16_hi(w.y);
    acc[4] += (double)bf16_lo(w.z);
    acc[5] += (double)bf16_hi(w.z);
    acc[6] += (double)bf16_lo(w.w);
    acc[7] += (double)bf16_hi(w.w);
  }
  uint16_t o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) o[e] = f64_to_bf16_rne(acc[e] * (1.0 / 32.0));
  uint4 r;
  r.x = (uint32_t)o[0] | ((uint32_t)o[1] << 16);
  r.y = (uint32_t)o[2] | ((uint32_t)o[3] << 16);
  r.z = (uint32_t)o[4] | ((uint32_t)o[5] << 16);
  r.w = (uint32_t)o[6] | ((uint32_t)o[7] << 16);
  return r;
}

}  // namespace infv2
