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

#if defined(__CUDA_ARCH__)
#define KIVI_UNROLL _Pragma("unroll")
#else
#define KIVI_UNROLL
#endif

// quantize_group_sparse with every array indexed at positions known when the
// loops are unrolled: the kept set is a bit mask, each pass remembers its pick
// by value, and the picks are sorted by index at the end (a kernel then keeps
// the group in registers instead of local memory).  The same selection (k
// passes, larger magnitude first, lower index on ties), bounds, codes and
// lists bit for bit; out_idx / out_val entries past k are N / 0.  N <= 32.
template <int N, int K>
KIVI_HD inline void quantize_group_sparse_reg(const float (&x)[N], int k, int bits, float* scale,
                                              float* zero, int (&codes)[N], int (&out_idx)[K],
                                              float (&out_val)[K]) {
  static_assert(N <= 32, "one mask bit per element");
  uint32_t outm = 0u;
  int pi[K];
  float pv[K];
  KIVI_UNROLL
  for (int m = 0; m < K; ++m) {  // k arg-max passes over the magnitudes
    pi[m] = N;
    pv[m] = 0.f;
    if (m < k) {
      int best = -1;
      float ba = 0.f, bx = 0.f;
      KIVI_UNROLL
      for (int i = 0; i < N; ++i) {
        const float a = fabsf(x[i]);
        const bool pick = !((outm >> i) & 1u) && (best < 0 || a > ba);
        best = pick ? i : best;
        ba = pick ? a : ba;
        bx = pick ? x[i] : bx;
      }
      outm |= 1u << best;
      pi[m] = best;
      pv[m] = bx;
    }
  }
  KIVI_UNROLL
  for (int a = 0; a < K; ++a) {  // the lists in index order
    KIVI_UNROLL
    for (int b = 0; b + 1 < K - a; ++b) {
      if (pi[b] > pi[b + 1]) {
        const int ti = pi[b];
        pi[b] = pi[b + 1];
        pi[b + 1] = ti;
        const float tv = pv[b];
        pv[b] = pv[b + 1];
        pv[b + 1] = tv;
      }
    }
  }
  float mn = 0.f, mx = 0.f;
  bool first = true;
  KIVI_UNROLL
  for (int i = 0; i < N; ++i) {
    if ((outm >> i) & 1u) continue;
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
  KIVI_UNROLL
  for (int i = 0; i < N; ++i)
    codes[i] = ((outm >> i) & 1u) || s == 0.0f ? 0 : code_of(sub_rn(x[i], mn), s, rs, L);
  KIVI_UNROLL
  for (int m = 0; m < K; ++m) {
    out_idx[m] = pi[m];
    out_val[m] = pv[m];
  }
}

}  // namespace kivi
