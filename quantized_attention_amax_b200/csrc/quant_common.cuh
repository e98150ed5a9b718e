// quant_common.cuh -- arithmetic shared by the FP8 quantizers (per token, per block, rotate + block).
#pragma once

#include <cuda_runtime.h>

namespace faq {

// x / s rounded to fp32 as IEEE division does, for an FP8 scale s = fl(amax / 448) with
// s >= kFastDivMin and a bf16 |x| <= amax: q0 = x * r with r the correctly rounded 1 / s, then one
// FMA for the negated residual q0 * s - x (exact) and one FMA correction q0 - that * r.  This is
// the FMA-based quotient correction published by P. Markstein ("Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; and "IA-64 and
// Elementary Functions", 2000): given the correctly rounded reciprocal, one residual and one
// correction step round the quotient as the division would.  Taking the
// residual negated keeps the sign of a zero x (-0 gives -0 where x - q0 * s would give +0); for a
// nonzero result the two forms round identically, the sign flips being exact.
// Its E4M3 codes equal those of IEEE division for every bf16 amax whose scale reaches kFastDivMin
// and every bf16 |x| <= amax (an exhaustive check on the GPU); scales below it use IEEE division.
constexpr float kFastDivMin = 0x1p-90f;

__device__ __forceinline__ float fp8_div(float x, float s, float r) {
  const float q0 = x * r;
  return fmaf(-fmaf(q0, s, -x), r, q0);
}

// The same for a static scale that x can exceed (FP8 per head): quotients of 2^20 or more keep the
// plain product (they saturate to +-448 either way; the correction would overflow).  Same E4M3
// codes as IEEE division for every bf16 amax with s >= kFastDivMin and every finite bf16 x.
__device__ __forceinline__ float fp8_div_sat(float x, float s, float r) {
  const float q0 = x * r;
  return fabsf(q0) < 0x1p20f ? fmaf(-fmaf(q0, s, -x), r, q0) : q0;
}

// INT8 (s = fl(amax / 127)): x / s before round-to-integer and saturation, as IEEE division
// rounds it where that decides the code, for every bf16 amax with s >= kFastDivMin and every
// finite bf16 x (the exhaustive check covers this too).
__device__ __forceinline__ float int8_div(float x, float s, float r) {
  const float q0 = x * r;
  return fabsf(q0) < 0x1p20f ? fmaf(fmaf(-q0, s, x), r, q0) : q0;
}

// INT8 where |x| <= amax is known (per-token scales, or a per-head row inside its calibrated
// range): |x / s| <= 127 (1 + 2^-23), so the overflow guard of int8_div is never taken and the
// correction applies unconditionally.  Same codes as IEEE division on that domain (exhaustive).
__device__ __forceinline__ float int8_div_bounded(float x, float s, float r) {
  const float q0 = x * r;
  return fmaf(fmaf(-q0, s, x), r, q0);
}

// int8_div_bounded on a pair in packed f32x2 arithmetic: two lanes per instruction, each with the
// scalar form's three roundings (-q0 * s written as q0 * (-s), an exact sign change).
__device__ __forceinline__ void int8_div_bounded_x2(float& a, float& b, float s, float r) {
  asm("{\n\t.reg .b64 x, q, e, ns, rv;\n\t"
      "mov.b64 x, {%0, %1};\n\tmov.b64 ns, {%2, %2};\n\tmov.b64 rv, {%3, %3};\n\t"
      "mul.rn.f32x2 q, x, rv;\n\t"
      "fma.rn.f32x2 e, q, ns, x;\n\t"
      "fma.rn.f32x2 q, e, rv, q;\n\t"
      "mov.b64 {%0, %1}, q;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(-s), "f"(r));
}

}  // namespace faq
