// kivi_sparse.cuh -- dense-and-sparse quantization of one group held by one
// thread (the format variant that keeps each group's largest magnitudes
// exactly; KVQuant's per-vector dense-and-sparse quantization, as read in
// the design notes).  Host and device build; the host build is checked bit
// for bit against the CPU oracle.
#pragma once

#include <math.h>

#include "kivi_codes.cuh"

namespace kivi {

KIVI_HD inline float sub_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fsub_rn(a, b);
#else
  volatile float r = a - b;
  return r;
#endif
}
KIVI_HD inline float div_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fdiv_rn(a, b);
#else
  volatile float r = a / b;
  return r;
#endif
}

// One group of N entries x[0..N-1], K outliers at most (k <= K, k < N):
//   the k largest magnitudes (the lower index first among equal ones) go to
//   out_idx / out_val in ascending index order, their codes are 0;
//   the others are quantized with s = fl(fl(mx - mn) / L), z = mn (strict
//   compares in index order, so the first of equal extremes is kept) and the
//   code rule of kivi_codes.cuh.
template <int N, int K>
KIVI_HD inline void quantize_group_sparse(const float (&x)[N], int k, int bits, float* scale,
                                          float* zero, int (&codes)[N], int (&out_idx)[K],
                                          float (&out_val)[K]) {
  bool out[N];
  for (int i = 0; i < N; ++i) out[i] = false;
  for (int m = 0; m < k; ++m) {  // k arg-max passes over the magnitudes
    int best = -1;
    for (int i = 0; i < N; ++i)
      if (!out[i] && (best < 0 || fabsf(x[i]) > fabsf(x[best]))) best = i;
    out[best] = true;
  }
  float mn = 0.f, mx = 0.f;
  bool first = true;
  for (int i = 0; i < N; ++i) {
    if (out[i]) continue;
    if (first) {
      mn = mx = x[i];
      first = false;
    } else {
      if (x[i] < mn) mn = x[i];
      if (x[i] > mx) mx = x[i];
    }
  }
  const int L = (1 << bits) - 1;
  const float s = div_rn(sub_rn(mx, mn), (float)L);
  const float rs = recip_rn(s);
  *scale = s;
  *zero = mn;
  int j = 0;
  for (int i = 0; i < N; ++i) {
    if (out[i]) {
      codes[i] = 0;
      out_idx[j] = i;
      out_val[j] = x[i];
      ++j;
    } else {
      codes[i] = s != 0.0f ? code_of(sub_rn(x[i], mn), s, rs, L) : 0;
    }
  }
}

}  // namespace kivi
