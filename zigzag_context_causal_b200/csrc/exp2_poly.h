// 2^x on the FMA and integer pipes, for the share of softmax exponentials the
// kernel keeps off the MUFU unit.  2^x = 2^n * p(f), n = round(x), f = x - n in
// [-1/2, 1/2], p = degree-3 Chebyshev interpolant of 2^f on that interval
// (coefficients printed by gen_exp2_poly.py; max relative error 1.0e-4, far
// below the 2^-9 of the bf16 rounding that P goes through next).
#pragma once

namespace zz {
namespace dev {

constexpr float kExp2C0 = 0.99992454f;
constexpr float kExp2C1 = 0.69313675f;
constexpr float kExp2C2 = 0.24263948f;
constexpr float kExp2C3 = 0.055838283f;

// Two values at once.  Inputs are clamped at -126 so that n << 23 never leaves
// the exponent field (results there are ~1e-38, i.e. zero for the softmax).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 magic = make_float2(12582912.f, 12582912.f);   // 1.5 * 2^23: x + magic rounds x
  const float2 t = fadd2(x, magic);
  const float2 r = fadd2(t, make_float2(-12582912.f, -12582912.f));  // round(x)
  const float2 f = ffma2(r, make_float2(-1.f, -1.f), x);             // x - round(x)
  float2 p = ffma2(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = ffma2(p, f, make_float2(kExp2C1, kExp2C1));
  p = ffma2(p, f, make_float2(kExp2C0, kExp2C0));
  // The low mantissa bits of t hold round(x); shifted by 23 they land in the exponent.
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

}  // namespace dev
}  // namespace zz
