// 2^x on the FMA pipe, two values per instruction (packed f32x2 arithmetic, sm_100).
//
// The softmax passes of the compress kernels take one exponential per attention logit; on the
// MUFU unit alone (16 per clock per SM) that is their binding rate. A fixed share of the
// exponentials is computed here instead, on the FMA pipe, which runs beside the MUFU unit.
//
// Method: the exact base-2 argument reduction of Cody and Waite ("Software Manual for the
// Elementary Functions", 1980), 2^x = 2^n * 2^f with n = rint(x) and f = x - n in [-1/2, 1/2],
// then 2^f by a degree-5 polynomial whose coefficients minimise the maximum relative error on
// [-1/2, 1/2] (Remez exchange; fit_exp2_poly.py beside this file prints them: 7.5e-8 in exact
// arithmetic, about 2.1e-7 with fp32 coefficients and fp32 Horner steps). rint(x) is read from the
// low mantissa bits of x + 1.5 * 2^23 (round to nearest), and n is added to the exponent field of
// the polynomial's value. x is clamped at -126 first, so the exponent field cannot wrap: inputs
// below -126 give 2^-126 instead of 0, which only matters when the caller does not sum the value
// with a term of order 1.
#pragma once

#include <cstdint>

namespace iamap {

// fit_exp2_poly.py 5
constexpr float kExp2C0 = 1.000000119e+00f;
constexpr float kExp2C1 = 6.931469440e-01f;
constexpr float kExp2C2 = 2.402212024e-01f;
constexpr float kExp2C3 = 5.550713092e-02f;
constexpr float kExp2C4 = 9.675540961e-03f;
constexpr float kExp2C5 = 1.327647245e-03f;
constexpr float kExp2Round = 12582912.0f;   // 1.5 * 2^23
constexpr float kExp2Floor = -126.0f;

__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_splat(float a) { return f2_pack(a, a); }

// (2^x0, 2^x1) for a packed pair x.
__device__ __forceinline__ uint64_t exp2_fma_x2(uint64_t x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  x = f2_pack(fmaxf(x0, kExp2Floor), fmaxf(x1, kExp2Floor));
  const uint64_t rnd = f2_splat(kExp2Round);
  const uint64_t t = f2_add(x, rnd);          // low mantissa bits: rint(x)
  const uint64_t f = f2_sub(x, f2_sub(t, rnd));   // x - rint(x), exact
  uint64_t p = f2_fma(f2_splat(kExp2C5), f, f2_splat(kExp2C4));
  p = f2_fma(p, f, f2_splat(kExp2C3));
  p = f2_fma(p, f, f2_splat(kExp2C2));
  p = f2_fma(p, f, f2_splat(kExp2C1));
  p = f2_fma(p, f, f2_splat(kExp2C0));
  float t0, t1, p0, p1;
  f2_unpack(t, t0, t1);
  f2_unpack(p, p0, p1);
  // n * 2^23 added to the exponent field: (bits(t) << 23) is n << 23 modulo 2^32
  return f2_pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

__device__ __forceinline__ float exp2_fma(float x) {
  float y0, y1;
  f2_unpack(exp2_fma_x2(f2_pack(x, x)), y0, y1);
  return y0;
}

}  // namespace iamap
