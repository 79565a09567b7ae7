// softmax_math.cuh -- packed fp32 arithmetic and the FMA-pipe exponential used by
// the softmax of the tensor-core kernels (and by its self-test kernel).
#pragma once

#include <stdint.h>

namespace swa {

// ------------------------------------------------------------------ packed fp32 helpers
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                      float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^a for a pair of arguments <= 2^7 on the FMA pipe: round to the nearest
// integer i (adding 1.5*2^23 leaves i in the low mantissa bits), f = a - i in
// [-1/2, 1/2], 2^f by a degree-3 polynomial (coefficients fitted for this
// kernel by iterated weighted least squares on Chebyshev nodes, c0 = 1 exactly;
// relative error at most 1.02e-4, largest near f = -0.342), then i is added to
// the exponent field.  The bound holds while the result is a normal number
// (a >= -125.5); below that the result is a value in [0, 2^-125].  Arguments
// below -127 (masked scores are -inf) are clamped to -127, which yields +0.
__device__ __forceinline__ void exp2_poly2(float& y0, float& y1, float a0, float a1) {
  constexpr float kRound = 12582912.0f;         // 1.5 * 2^23
  constexpr float c1 = 0.6932829022407532f, c2 = 0.2422109693288803f, c3 = 0.05500892549753189f;
  a0 = fmaxf(a0, -127.f);
  a1 = fmaxf(a1, -127.f);
  float r0, r1, i0, i1, f0, f1, q0, q1;
  fadd2(r0, r1, a0, a1, kRound, kRound);
  fadd2(i0, i1, r0, r1, -kRound, -kRound);
  fadd2(f0, f1, a0, a1, -i0, -i1);
  ffma2(q0, q1, f0, f1, c3, c3, c2, c2);
  ffma2(q0, q1, q0, q1, f0, f1, c1, c1);
  ffma2(q0, q1, q0, q1, f0, f1, 1.f, 1.f);
  y0 = __int_as_float(__float_as_int(q0) + (__float_as_int(r0) << 23));
  y1 = __int_as_float(__float_as_int(q1) + (__float_as_int(r1) << 23));
}

}  // namespace swa
