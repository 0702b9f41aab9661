// exp2_poly.cuh -- 2^x on the FMA pipe, for the share of the scan's decays
// that the special-function unit (16 lanes/SM/clk against 128 FP32 lanes)
// cannot absorb.
//
// Range reduction j = rint(x), f = x - j in [-1/2, 1/2]; 2^x = 2^j p(f) with
// p(f) = 1 + f q(f) of degree 5, fitted for minimum maximum relative error on
// [-1/2, 1/2] with p(0) = 1 exactly (gen_exp2_poly.py: 9.2e-8 in exact
// arithmetic, 1.9e-7 with float32 Horner steps).  rint uses the 1.5 * 2^23
// shifter; 2^j is added to the exponent field.  Valid for x in [-126, 126]:
// callers clamp the argument first.
#pragma once
#include <cuda_runtime.h>

namespace ssm {

constexpr float kExp2C1 = 6.931470037e-01f;
constexpr float kExp2C2 = 2.402224243e-01f;
constexpr float kExp2C3 = 5.550733581e-02f;
constexpr float kExp2C4 = 9.671516716e-03f;
constexpr float kExp2C5 = 1.326473663e-03f;
constexpr float kShifter = 12582912.0f;  // 1.5 * 2^23

// 2^(a * b) for a pair; a * b must lie in [-126, 126].
__device__ __forceinline__ float2 exp2_poly2(float2 a, float2 b) {
  const float2 sh = make_float2(kShifter, kShifter);
  const float2 t = __ffma2_rn(a, b, sh);                         // shifter + rint(ab)
  const float2 jn = __fadd2_rn(sh, make_float2(-t.x, -t.y));     // -rint(ab)
  const float2 f = __ffma2_rn(a, b, jn);                         // ab - rint(ab)
  float2 p = __ffma2_rn(make_float2(kExp2C5, kExp2C5), f, make_float2(kExp2C4, kExp2C4));
  p = __ffma2_rn(p, f, make_float2(kExp2C3, kExp2C3));
  p = __ffma2_rn(p, f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(1.0f, 1.0f));
  float2 r;
  r.x = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
  r.y = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
  return r;
}

}  // namespace ssm
