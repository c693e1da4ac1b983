// Packed fp32 arithmetic and the base-2 exponentials of the attention softmax.
//
// poly_exp2x2 is this library's own 2^x for the FMA pipe (it relieves the MUFU unit,
// which the softmax would otherwise saturate):
//   - range reduction: adding 1.5 * 2^23 rounds x to the nearest integer n and leaves n
//     in the low mantissa bits; f = x - n is exact and lies in [-1/2, 1/2];
//   - 2^f from a cubic c0 + c1 f + c2 f^2 + c3 f^3 whose coefficients minimise the largest
//     RELATIVE error over [-1/2, 1/2] (a minimax fit: minimise t subject to
//     |p(f) / 2^f - 1| <= t on a dense grid, a linear program in (c0..c3, t)); the
//     optimum is 7.475e-5 and the rounded fp32 coefficients below reach 7.48e-5, below
//     the bf16 rounding (2^-9 = 1.95e-3) that P goes through before the PV product;
//   - the exponent: n << 23 is added to the bit pattern of 2^f.
// x is clamped to -126.  Below -125.5 the result leaves the normal range and is only
// good to an absolute 2^-125 (it stays in [0, 2^-125]); the softmax's largest term is 1,
// so such terms add nothing, and callers zero masked columns themselves.
// tests/test_fastmath.py checks the coefficients and the error bound on the host and,
// through msa_exp2_poly_eval, this very device code against exp2 on a GPU.
#pragma once

#include <stdint.h>

namespace msa {
namespace fastmath {

// Packed two-lane fp32 arithmetic (sm_100: one instruction for both lanes).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                      float c0, float c1) {
  asm("{\n.reg .b64 a, b, c, d;\nmov.b64 a, {%2, %3};\nmov.b64 b, {%4, %5};\n"
      "mov.b64 c, {%6, %7};\nfma.rn.f32x2 d, a, b, c;\nmov.b64 {%0, %1}, d;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0,
                                      float b1) {
  asm("{\n.reg .b64 a, b, d;\nmov.b64 a, {%2, %3};\nmov.b64 b, {%4, %5};\n"
      "add.rn.f32x2 d, a, b;\nmov.b64 {%0, %1}, d;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fmul2(float& d0, float& d1, float a0, float a1, float b0,
                                      float b1) {
  asm("{\n.reg .b64 a, b, d;\nmov.b64 a, {%2, %3};\nmov.b64 b, {%4, %5};\n"
      "mul.rn.f32x2 d, a, b;\nmov.b64 {%0, %1}, d;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Hardware base-2 exponential (MUFU).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Minimax cubic for 2^f on [-1/2, 1/2] (relative error), highest degree first.
constexpr float kExp2C3 = 0.0551716573536396f;
constexpr float kExp2C2 = 0.2426111400127411f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C0 = 0.9999280571937561f;

// 2^x for two lanes on the FMA pipe (see the file comment).
__device__ __forceinline__ void poly_exp2x2(float x0, float x1, float& p0, float& p1) {
  constexpr float kShift = 12582912.f;            // 1.5 * 2^23
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  float t0, t1, n0, n1, f0, f1;
  fadd2(t0, t1, x0, x1, kShift, kShift);
  fadd2(n0, n1, t0, t1, -kShift, -kShift);        // exact: n as a float
  ffma2(f0, f1, n0, n1, -1.f, -1.f, x0, x1);      // exact: x - n
  float q0, q1;
  ffma2(q0, q1, kExp2C3, kExp2C3, f0, f1, kExp2C2, kExp2C2);
  ffma2(q0, q1, q0, q1, f0, f1, kExp2C1, kExp2C1);
  ffma2(q0, q1, q0, q1, f0, f1, kExp2C0, kExp2C0);
  // the low 9 bits of t's pattern are n's; shifted by 23 only n << 23 remains
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

}  // namespace fastmath
}  // namespace msa
