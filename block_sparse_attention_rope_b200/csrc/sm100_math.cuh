// sm100_math.cuh -- arithmetic helpers shared by the tensor-core kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lcsm100 {

// 2^x on the FMA pipe, two lanes at once: x = n + f with n = rint(x) (by the
// 1.5*2^23 rounding constant) and f in [-1/2, 1/2]; 2^f by a degree-3
// polynomial fitted here by the Remez exchange for least maximum relative
// error (7.5e-5, far below bf16's 2^-9); 2^n by adding n to the exponent
// field.  Inputs below -126 are clamped (the result is then < 2^-125).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 rnd = make_float2(12582912.f, 12582912.f);
  const float2 t = __fadd2_rn(x, rnd);
  const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(make_float2(0.0551716685f, 0.0551716685f), f,
                        make_float2(0.242611125f, 0.242611125f));
  p = __ffma2_rn(p, f, make_float2(0.693260968f, 0.693260968f));
  p = __ffma2_rn(p, f, make_float2(0.999928057f, 0.999928057f));
  float2 r;
  r.x = __uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23));
  r.y = __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23));
  return r;
}

}  // namespace lcsm100
