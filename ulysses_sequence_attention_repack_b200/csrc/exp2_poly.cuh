// exp2 on the FMA pipe, for part of the softmax exponentials (the rest go to
// the MUFU ex2 unit, whose throughput otherwise matches the tensor core's and
// limits the attention loop).
//
// 2^x = 2^j * p(f), x = j + f, j = round(x), f in [-1/2, 1/2]:
//   * j by the round-to-nearest shifter: t = x + 1.5*2^23 holds j in its low
//     mantissa bits, and (bits(t) << 23) is j shifted into the exponent field;
//   * p: degree-3 polynomial minimising the maximum relative error against
//     2^f on [-1/2, 1/2] (Remez exchange; exp2_poly_fit.py reproduces the
//     coefficients); max relative error 7.5e-5;
//   * 2^j applied by adding j to p's exponent field (integer add).
// x is clamped to >= -125 so the result stays a normal number; inputs below
// that give 2^-125 (callers use MUFU ex2 where exact zeros matter, i.e.
// for masked -inf logits).
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace ulysses {

constexpr float kExp2C0 = 9.999280572e-01f;
constexpr float kExp2C1 = 6.932609677e-01f;
constexpr float kExp2C2 = 2.426111251e-01f;
constexpr float kExp2C3 = 5.517166853e-02f;
constexpr float kRoundShifter = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ f2 exp2_poly2(f2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const f2 t = fadd2(x, f2{kRoundShifter, kRoundShifter});
  const f2 j = fadd2(t, f2{-kRoundShifter, -kRoundShifter});
  const f2 fr = ffma2(j, f2{-1.0f, -1.0f}, x);   // x - j, exact
  f2 p = ffma2(fr, f2{kExp2C3, kExp2C3}, f2{kExp2C2, kExp2C2});
  p = ffma2(p, fr, f2{kExp2C1, kExp2C1});
  p = ffma2(p, fr, f2{kExp2C0, kExp2C0});
  f2 r;
  r.x = __uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23));
  r.y = __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23));
  return r;
}

}  // namespace ulysses
