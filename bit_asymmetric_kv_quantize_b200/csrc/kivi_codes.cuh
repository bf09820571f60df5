// kivi_codes.cuh -- the code of one quantized element, shared by the
// quantize kernels and a host build that tests the rule.
#pragma once

#include <math.h>
#include <stdint.h>

#ifdef __CUDACC__
#include <cuda_runtime.h>
#define KIVI_HD __host__ __device__
#else
#define KIVI_HD
#endif

namespace kivi {

// round_half_even(fl(d / s)) clamped to [0, L], without a division for most
// elements: q = fl(d * rs) with rs = fl(1/s) differs from fl(d / s) by at
// most |d/s|(2^-23 + 2^-24 + 2^-48) (two roundings against one), below 3e-6
// for |d/s| <= 16; so when q is more than 4e-6 from the nearest half-integer
// both round to the same integer and neither is a tie.  Otherwise (and for
// inf or NaN q) the quotient is taken by the IEEE division.  Quotients far
// outside [-0.5, L + 0.5] (|d/s| > 16, which binary16 scales and zeros can
// produce, or d < 0 when the rounded zero lies above an element) are safe
// although the bound no longer holds there: with L <= 15 both q and fl(d/s)
// then lie beyond the same end of the range, so both clamp to the same code
// (0 or L).
KIVI_HD inline int code_of(float d, float s, float rs, int L) {
#ifdef __CUDA_ARCH__
  const float q = __fmul_rn(d, rs);
  const float f = q - floorf(q);
  const int c = fabsf(f - 0.5f) > 4e-6f ? __float2int_rn(q) : __float2int_rn(__fdiv_rn(d, s));
#else
  // host build (tests): binary32 operations rounded to nearest-even
  volatile float qv = d * rs;
  const float q = qv;
  const float f = q - floorf(q);
  volatile float dq = d / s;
  const int c = fabsf(f - 0.5f) > 4e-6f ? (int)nearbyintf(q) : (int)nearbyintf(dq);
#endif
  return c < 0 ? 0 : (c > L ? L : c);
}

// code_of's rounding without the conversion to an integer, for loops that
// check a whole group at once: q = fl(d * rs) clamped to [0, L], plus
// 1.5 * 2^23 (whose ulp is 1) rounds it to an integer half to even, and the
// low bits of the sum's encoding are that integer (returned: 0x4B400000 +
// code).  fmax(*ae, |q - rint(q)|) goes to *ae.  For q in [0, L] that
// difference is exact and 0.5 - *ae is q's distance to the nearest
// half-integer, so when 0.5 - *ae > 4e-6 over a group whose rs is finite,
// every code equals code_of's (the same rounding of the same q, which
// code_of's bound makes the exact code); outside [0, L] both clamp to the
// same end.  Otherwise code_of decides.  (A NaN q -- 0 * inf, inf * 0 --
// clamps to 0, as code_of's conversion of a NaN quotient gives 0.)
KIVI_HD inline uint32_t code_bits(float d, float rs, float Lf, float* ae) {
  const float kRound = 12582912.0f;  // 1.5 * 2^23
#ifdef __CUDA_ARCH__
  const float q = fminf(fmaxf(__fmul_rn(d, rs), 0.0f), Lf);
  const float m = __fadd_rn(q, kRound);
  *ae = fmaxf(*ae, fabsf(__fsub_rn(q, __fsub_rn(m, kRound))));
  return __float_as_uint(m);
#else
  volatile float qv = d * rs;
  float q = qv;
  q = q > 0.0f ? q : 0.0f;  // also maps a NaN to 0, as fmaxf does
  q = q < Lf ? q : Lf;
  volatile float mv = q + kRound;
  const float m = mv;
  volatile float rv = m - kRound;
  volatile float ev = q - rv;
  const float e = fabsf(ev);
  if (e > *ae) *ae = e;
  uint32_t u;
  __builtin_memcpy(&u, &m, 4);
  return u;
#endif
}

// Whether a group coded by code_bits needs code_of: some element within
// 4e-6 of a half-integer, or a reciprocal that is not finite.
KIVI_HD inline bool codes_need_exact(float ae, float rs) {
  return !(0.5f - ae > 4e-6f) || !(rs <= 3.0e38f);
}

// fl(1/s), the reciprocal code_of takes.
KIVI_HD inline float recip_rn(float s) {
#ifdef __CUDA_ARCH__
  return __frcp_rn(s);
#else
  volatile float r = 1.0f / s;
  return r;
#endif
}

}  // namespace kivi
