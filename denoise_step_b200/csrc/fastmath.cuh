// Softmax arithmetic helpers for the attention kernels: packed f32x2 ops,
// MUFU exp2, fp16x2 packing, 3-input max and an FMA-pipe exp2 polynomial.
#pragma once
#include <cstdint>

namespace pl {

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float ex2_f32(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// fp16x2 of (lo, hi), lo in the low half
__device__ __forceinline__ uint32_t h2_from(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// 2^x for a pair on the FMA pipe: n = nearest integer (1.5 * 2^23 shifter),
// f = x - n in [-0.5, 0.5], 2^f by a degree-3 polynomial, 2^n added into the
// exponent field. x is clamped to >= -126 so 2^n stays a normal number.
// The cubic is a weighted least-squares fit of 2^f on 4096 Chebyshev nodes of
// [-0.5, 0.5] (relative error minimised; max 7.7e-5, below the 4.9e-4 of the
// fp16 rounding that P gets next); exp2_poly.py beside this file prints it.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  const uint64_t shift = f2_pack(12582912.f, 12582912.f);
  const uint64_t xc = f2_pack(x0, x1);
  const uint64_t y = f2_add(xc, shift);
  const uint64_t n = f2_add(y, f2_pack(-12582912.f, -12582912.f));
  float n0, n1;
  f2_unpack(n, n0, n1);
  const uint64_t f = f2_add(xc, f2_pack(-n0, -n1));
  uint64_t pz = f2_fma(f, f2_pack(0.055088684f, 0.055088684f), f2_pack(0.242604047f, 0.242604047f));
  pz = f2_fma(pz, f, f2_pack(0.693276227f, 0.693276227f));
  pz = f2_fma(pz, f, f2_pack(0.999928951f, 0.999928951f));
  float y0, y1, p0, p1;
  f2_unpack(y, y0, y1);
  f2_unpack(pz, p0, p1);
  const uint32_t r0 = __float_as_uint(p0) + (__float_as_uint(y0) << 23);
  const uint32_t r1 = __float_as_uint(p1) + (__float_as_uint(y1) << 23);
  return f2_pack(__uint_as_float(r0), __uint_as_float(r1));
}


}  // namespace pl
