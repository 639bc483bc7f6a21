// 2^x on the FMA pipe, for two lanes at once (Blackwell packed f32x2).
//
// The Softmax needs one exponential per score; at head dim 128 the MUFU
// (ex2.approx) rate equals the tensor-core rate per score, so part of the
// exponentials are computed here instead, with FMA-pipe instructions only:
//   1. clamp x >= -125 (keeps the result a normal float; 2^-125 is far below
//      anything a bf16 probability or the fp32 row sum can see),
//   2. split x = n + f with n = rint(x), f in [-1/2, 1/2]: adding 1.5 * 2^23
//      rounds x to an integer held in the low mantissa bits of t,
//   3. 2^f by a cubic whose coefficients were fitted for this file by
//      iteratively reweighted least squares on 4000 Chebyshev nodes of
//      [-1/2, 1/2] (max relative error 7.5e-5),
//   4. multiply by 2^n by adding n << 23 to the bits of the cubic's value;
//      (bits(t) << 23) equals n << 23 because the shift constant's own bits
//      vanish under the shift.
#pragma once

#include <stdint.h>

namespace vdn {

__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}

__device__ __forceinline__ float f32x2_lo(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v));
}

__device__ __forceinline__ float f32x2_hi(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v >> 32));
}

__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// max(a, b, c) as one instruction (the three-input form of sm_100); like
// fmaxf, a NaN operand is ignored when another operand is a number.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// MUFU exponential (hardware ex2.approx).
__device__ __forceinline__ float exp2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for both lanes of x2 on the FMA pipe (see the file comment).
__device__ __forceinline__ uint64_t exp2_fma_x2(uint64_t x2) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  const float x0 = fmaxf(f32x2_lo(x2), -125.f);
  const float x1 = fmaxf(f32x2_hi(x2), -125.f);
  const uint64_t xc = f32x2_pack(x0, x1);
  const uint64_t t = f32x2_add(xc, f32x2_pack(kShift, kShift));
  const uint64_t n = f32x2_add(t, f32x2_pack(-kShift, -kShift));   // rint(x), exact
  const uint64_t f = f32x2_fma(n, f32x2_pack(-1.f, -1.f), xc);      // x - rint(x)
  uint64_t p = f32x2_fma(f32x2_pack(0.055171653628349304f, 0.055171653628349304f), f,
                         f32x2_pack(0.2426111251115799f, 0.2426111251115799f));
  p = f32x2_fma(p, f, f32x2_pack(0.6932609677314758f, 0.6932609677314758f));
  p = f32x2_fma(p, f, f32x2_pack(0.9999280571937561f, 0.9999280571937561f));
  const uint32_t lo = static_cast<uint32_t>(p) + (static_cast<uint32_t>(t) << 23);
  const uint32_t hi = static_cast<uint32_t>(p >> 32) + (static_cast<uint32_t>(t >> 32) << 23);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

}  // namespace vdn
