// 2^x on the FMA pipe, for kernels bound by the MUFU exp2 rate: a share of their
// exponentials is computed here instead of by ex2.approx, so both pipes work.
//
// Method (range reduction plus a minimax polynomial):
//   x = r + f with r = rint(x) and f in [-1/2, 1/2]; 2^x = 2^r * p(f).
//   rint comes from the 1.5 * 2^23 shifter: in t = x + 1.5 * 2^23 the low mantissa bits
//   of t hold r as a two's-complement integer, so shifting the bits of t left by 23 puts
//   r into the exponent field, and an integer add of that to the bits of p(f) (a normal
//   number in [2^-1/2, 2^1/2]) scales it by 2^r.
//   p is the degree-5 polynomial that minimises the relative error of p(f) / 2^f on
//   [-1/2, 1/2] (Remez exchange on the equioscillating reference; minimax relative
//   error 7.5e-8).  Evaluated in fp32 by Horner's rule its relative error is within
//   2.2e-7 (< 2 ulp of 1), the accuracy class of ex2.approx.
//   x is clamped to [-125, 0]: every argument here is a logit minus an upper bound
//   (<= 0), and below 2^-125 the result stays about 2.4e-38 instead of 0, which no sum
//   it enters can see.
#pragma once

namespace kvc {

__device__ __forceinline__ float exp2_poly(float x) {
  x = fminf(fmaxf(x, -125.f), 0.f);
  const float shifter = 12582912.f;                 // 1.5 * 2^23
  const float t = x + shifter;                      // rounds x to the nearest integer r
  const float f = x - (t - shifter);                // f = x - r in [-1/2, 1/2]
  float p = 1.3276472454890609e-3f;
  p = fmaf(p, f, 9.675540961325169e-3f);
  p = fmaf(p, f, 5.550713092088699e-2f);
  p = fmaf(p, f, 2.4022120237350464e-1f);
  p = fmaf(p, f, 6.931469440460205e-1f);
  p = fmaf(p, f, 1.0000001192092896f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

}  // namespace kvc
