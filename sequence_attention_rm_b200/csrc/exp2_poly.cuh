// 2^x on the FMA pipe: the polynomial exponential that the tensor-core
// forward uses for part of its softmax (shared with the test hook that checks
// it against the exact value over its whole input range).
#pragma once

#include <cuda_runtime.h>

namespace rm {

// 2^x for two values at once on the FMA pipe, to take part of the softmax's
// exponentials off the SFU (which runs ex2 at 16 results per clock per SM,
// the forward's limit next to the tensor pipe).  x = j + f with j the nearest
// integer (adding 1.5 * 2^23 leaves j in the low mantissa bits of the sum)
// and f in [-1/2, 1/2]; 2^f from a cubic fitted to 2^f on [-1/2, 1/2] by the
// Remez exchange (relative error 7.5e-5; P is rounded to bf16, relative
// 3.9e-3, before the PV product); 2^j added to the exponent field.  x is
// clamped below at -125 so that the exponent stays normal: an input of
// -inf gives 2^-125 instead of 0 (a row that never sees a key is detected
// from its running max instead).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 shift = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
  const float2 t = __fadd2_rn(x, shift);
  const float2 j = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __fadd2_rn(x, make_float2(-j.x, -j.y));
  float2 q = __ffma2_rn(make_float2(0.0551716685f, 0.0551716685f), f,
                        make_float2(0.242611125f, 0.242611125f));
  q = __ffma2_rn(q, f, make_float2(0.693260968f, 0.693260968f));
  q = __ffma2_rn(q, f, make_float2(0.999928057f, 0.999928057f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}
}  // namespace rm
