// fa_exp2.cuh -- 2^x on the FMA pipe, shared by the forward and backward
// softmax so part of the exponentials can bypass the special-function unit.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

// ---------------------------------------------------------------- exp2 on the FMA pipe
// 2^x for a pair: x = n + f with n = round(x) (the 1.5 * 2^23 addition rounds
// to an integer in the low mantissa bits), f in [-1/2, 1/2]; 2^f by a minimax
// polynomial of degree 3 (relative error 7.5e-5, see fit_exp2_poly.py); 2^n
// built directly in the exponent field.  x is clamped
// at -127 first, where the exponent field becomes 0 and the result is +0, so
// masked (-inf) scores give exactly 0.
template <bool BF16>
__device__ __forceinline__ float2 exp2_fma_pair(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -127.0f);
  x.y = fmaxf(x.y, -127.0f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
  const float2 n = __fadd2_rn(t, make_float2(-kRound, -kRound));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);
  // degree 3 (relative error 7.5e-5): below the rounding of P to bf16 (2^-9)
  // and to fp16 (2^-12, 6.5x larger)
  float2 p = __ffma2_rn(make_float2(5.517166853e-02f, 5.517166853e-02f), f,
                        make_float2(2.426111251e-01f, 2.426111251e-01f));
  p = __ffma2_rn(p, f, make_float2(6.932609677e-01f, 6.932609677e-01f));
  p = __ffma2_rn(p, f, make_float2(9.999280572e-01f, 9.999280572e-01f));
  // (n + 127) << 23: the low bits of t hold n + 2^22 + 2^23, whose shifted-out
  // high part vanishes modulo 2^32
  const float sx = __uint_as_float((__float_as_uint(t.x) << 23) + (127u << 23));
  const float sy = __uint_as_float((__float_as_uint(t.y) << 23) + (127u << 23));
  return __fmul2_rn(p, make_float2(sx, sy));
}

}  // namespace fa
