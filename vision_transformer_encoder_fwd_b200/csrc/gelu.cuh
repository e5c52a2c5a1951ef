// Exact-form GELU for the FC1 epilogue and the dense head: GELU(x) = x * Phi(x) =
// x (1 + erf(x / sqrt 2)) / 2 ([diagram] "Encoder block": GELU; erf form, not the tanh one).
//
// erf is evaluated with formula 7.1.28 of Abramowitz & Stegun, Handbook of Mathematical
// Functions (1964):  for z >= 0,
//   erf(z) = 1 - (1 + a1 z + a2 z^2 + a3 z^3 + a4 z^4 + a5 z^5 + a6 z^6)^(-16) + e(z),
//   |e(z)| <= 3e-7,
// with the handbook's coefficients below, and erf(-z) = -erf(z).  Writing r for the (-16)th
// power at z = |x| / sqrt 2:
//   GELU(x) = x - x r / 2   (x >= 0),      GELU(x) = x r / 2   (x < 0),
// so the absolute error is at most |x| * 1.5e-7 plus the rounding of the single-precision
// evaluation (one reciprocal and four squarings).  Two values are processed together with the
// packed f32x2 FMA/multiply of sm_100a; the reciprocal runs on the MUFU.
#pragma once

#include "common.cuh"

namespace vit {

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float2 gelu2(float2 x) {
  // Abramowitz & Stegun 7.1.28 coefficients
  constexpr float a1 = 0.0705230784f, a2 = 0.0422820123f, a3 = 0.0092705272f;
  constexpr float a4 = 0.0001520143f, a5 = 0.0002765672f, a6 = 0.0000430638f;
  constexpr float kInvSqrt2 = 0.70710678118654752f;
  const float2 z = make_float2(fabsf(x.x) * kInvSqrt2, fabsf(x.y) * kInvSqrt2);
  float2 p = ffma2(z, make_float2(a6, a6), make_float2(a5, a5));
  p = ffma2(z, p, make_float2(a4, a4));
  p = ffma2(z, p, make_float2(a3, a3));
  p = ffma2(z, p, make_float2(a2, a2));
  p = ffma2(z, p, make_float2(a1, a1));
  p = ffma2(z, p, make_float2(1.f, 1.f));
  float2 r = make_float2(rcp_approx(p.x), rcp_approx(p.y));
  r = fmul2(r, r);  // ^2
  r = fmul2(r, r);  // ^4
  r = fmul2(r, r);  // ^8
  r = fmul2(r, r);  // ^16
  const float2 h = fmul2(fmul2(x, make_float2(0.5f, 0.5f)), r);  // x r / 2
  const float2 pos = fadd2(x, make_float2(-h.x, -h.y));
  return make_float2(x.x >= 0.f ? pos.x : h.x, x.y >= 0.f ? pos.y : h.y);
}

}  // namespace vit
