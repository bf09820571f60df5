// kivi_codes.cuh -- the code of one quantized element, shared by the
// quantize kernels and a host build that tests the rule.
#pragma once

#include <math.h>

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
