/*
 * kivi_oracle.c -- plain, slow, single-threaded CPU oracle for the KIVI
 * asymmetric 2/4-bit KV cache and its decode attention.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load this file.  It shares nothing with the
 * CUDA library and the CUDA library never calls it.
 *
 * Build: gcc -std=c99 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (every float operation below is one IEEE binary32 operation rounded to
 * nearest-even; no contraction into fused multiply-adds).
 *
 * The four steps, in the order the method applies them:
 *   Q  quantize a group with an asymmetric min/max scale and zero
 *      (KIVI, study.space summary: the method is asymmetric; mlsanity.com
 *      index page, "Abstract (arXiv)": 2-bit codes, keys per channel,
 *      values per token);
 *   P  pack the codes 32/bits to a 32-bit word;
 *   S  split the cache into a quantized part and a full-precision residual
 *      window of R recent tokens, flushing the window into the quantized
 *      part every R tokens (study.space summary: grouped and residual
 *      parts, value codes appended along tokens, key quantization grouped
 *      across tokens; scholarfeed.org "KIVI" page, third quote:
 *      fixed-length residual buffer);
 *   A  decode attention over the dequantized quantized part and the
 *      residual part together (study.space summary: the residual part is
 *      combined with the grouped part when attention is computed).
 *
 * Parity pins for every function are in tests/test_oracle_*.py.
 */
#include "kivi_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

static int valid_bits(int bits) {
  return bits == 1 || bits == 2 || bits == 3 || bits == 4 || bits == 8 || bits == 16;
}

/* Code blocks of the packed layout: CB codes in WB words.  Widths that
 * divide 32 pack CB = 32/bits codes into one word; 3 bits packs CB = 32
 * codes into three bit-plane words. */
static int block_codes(int bits) { return bits == 3 ? 32 : 32 / bits; }
static int block_words(int bits) { return bits == 3 ? 3 : 1; }

/*
 * Q.  The pages name the quantizer only as asymmetric (a scale and an
 * offset per group).  Reading: the plain min/max form, in binary32:
 *   mn = min x_i, mx = max x_i   (strict compares, first occurrence kept)
 *   L  = 2^bits - 1
 *   s  = (mx - mn) / L           (one rounded subtraction, one rounded
 *                                 division)
 *   z  = mn                      (a float offset, not an integer zero-point)
 *   c_i = clamp(round_half_even((x_i - mn) / s), 0, L), or 0 when s == 0.
 * The quotient is a true division, not a multiply by 1/s.
 */
/*
 * Binary16 rounding, from the format's definition: 11 significant bits for
 * normal values (|x| >= 2^-14), a fixed quantum of 2^-24 below that, round
 * to nearest with ties to even, and magnitudes that round above 65504 (the
 * largest finite binary16 value) become infinite.  The division by the
 * quantum q (a power of two) and the product by q are exact in binary64.
 */
float kivi_oracle_round_half(float x) {
  double a, q, r;
  int e;
  if (x == 0.0f || !isfinite(x)) return x;
  a = fabs((double)x);
  (void)frexp(a, &e); /* a = m 2^e, 0.5 <= m < 1 */
  e -= 11;            /* quantum of an 11-bit significand */
  if (e < -24) e = -24;
  q = ldexp(1.0, e);
  r = nearbyint(a / q) * q; /* default rounding mode: half to even */
  if (r > 65504.0) r = INFINITY;
  return (float)(x < 0.0f ? -r : r);
}

int kivi_oracle_quantize_group(const float *x, long long n, long long stride,
                               int bits, float *scale, float *zero,
                               uint16_t *codes) {
  return kivi_oracle_quantize_group_meta(x, n, stride, bits, 0, scale, zero, codes);
}

/*
 * Format variant (metadata in binary16).  Reading: the binary32 scale and
 * zero above are rounded to binary16 (round to nearest even), and the codes
 * are chosen against the rounded values, so that the stored (scale, zero)
 * reconstruct the codes as closely as the grid allows:
 *   s16 = half(s), z16 = half(mn), c_i = clamp(rhe((x_i - z16) / s16), 0, L),
 *   or 0 when s16 == 0.
 */
int kivi_oracle_quantize_group_meta(const float *x, long long n, long long stride,
                                    int bits, int meta_f16, float *scale,
                                    float *zero, uint16_t *codes) {
  long long i;
  float mn, mx, L, range, s, z;
  if (!x || !scale || !zero || !codes || n <= 0 || !valid_bits(bits) ||
      (meta_f16 != 0 && meta_f16 != 1))
    return KIVI_ORACLE_ERR_ARG;
  mn = x[0];
  mx = x[0];
  for (i = 1; i < n; ++i) {
    float v = x[i * stride];
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  L = (float)((1u << bits) - 1u);
  range = mx - mn;
  s = range / L;
  z = mn;
  if (meta_f16) {
    s = kivi_oracle_round_half(s);
    z = kivi_oracle_round_half(mn);
  }
  *scale = s;
  *zero = z;
  for (i = 0; i < n; ++i) {
    if (s == 0.0f) {
      codes[i] = 0;
    } else {
      float t = (x[i * stride] - z) / s;
      float c = nearbyintf(t); /* default rounding mode: half to even */
      if (c < 0.0f) c = 0.0f;
      if (c > L) c = L;
      codes[i] = (uint16_t)c;
    }
  }
  return KIVI_ORACLE_OK;
}

/*
 * Q, dense-and-sparse variant (KVQuant on the codewithpapers.app page,
 * abstract item (iv): outliers are isolated separately for each vector so
 * that they do not skew its quantization range).  Reading: the vector is
 * the quantization group; its k entries of largest magnitude (equal
 * magnitudes: the lower index first) are kept exactly in a sparse list, in
 * ascending index order, and Q runs over the other n - k entries in their
 * order; an outlier's dense code is 0.  Requires 0 <= k < n.
 */
int kivi_oracle_quantize_group_sparse(const float *x, long long n, long long stride, int bits,
                                      int k, float *scale, float *zero, uint16_t *codes,
                                      long long *out_idx, float *out_val) {
  long long i, j, m, picked;
  unsigned char *is_out;
  float *rest;
  uint16_t *rest_codes;
  int rc;
  if (!x || !scale || !zero || !codes || n <= 0 || !valid_bits(bits) || k < 0 || k >= n ||
      (k > 0 && (!out_idx || !out_val)))
    return KIVI_ORACLE_ERR_ARG;
  is_out = (unsigned char *)calloc((size_t)n, 1);
  rest = (float *)malloc((size_t)n * sizeof(float));
  rest_codes = (uint16_t *)malloc((size_t)n * sizeof(uint16_t));
  if (!is_out || !rest || !rest_codes) {
    free(is_out);
    free(rest);
    free(rest_codes);
    return KIVI_ORACLE_ERR_ARG;
  }
  /* k passes, each taking the largest magnitude not yet taken */
  for (picked = 0; picked < k; ++picked) {
    long long best = -1;
    for (i = 0; i < n; ++i) {
      if (is_out[i]) continue;
      if (best < 0 || fabsf(x[i * stride]) > fabsf(x[best * stride])) best = i;
    }
    is_out[best] = 1;
  }
  /* the remaining entries, in order, through Q */
  for (i = 0, m = 0; i < n; ++i)
    if (!is_out[i]) rest[m++] = x[i * stride];
  rc = kivi_oracle_quantize_group(rest, m, 1, bits, scale, zero, rest_codes);
  if (rc == KIVI_ORACLE_OK) {
    for (i = 0, j = 0, m = 0; i < n; ++i) {
      if (is_out[i]) {
        codes[i] = 0;
        out_idx[j] = i;
        out_val[j] = x[i * stride];
        ++j;
      } else {
        codes[i] = rest_codes[m++];
      }
    }
  }
  free(is_out);
  free(rest);
  free(rest_codes);
  return rc;
}

/*
 * P.  Reading (the pages give no bit layout): E = 32/bits codes per word,
 * the first code in the least significant bits.
 */
uint32_t kivi_oracle_pack_word(const uint16_t *codes, int bits) {
  int i, E = 32 / bits;
  uint32_t mask = (uint32_t)((1u << bits) - 1u);
  uint32_t w = 0;
  for (i = 0; i < E; ++i) w |= ((uint32_t)codes[i] & mask) << (bits * i);
  return w;
}

/*
 * P for 3 bits (a format variant; the pages name 3-bit quantization only in
 * KVQuant's abstract).  Reading: 3 does not divide 32, so a block of 32
 * codes is stored as three bit planes, word b holding bit b of code i in
 * its bit i.
 */
void kivi_oracle_pack_planes(const uint16_t *codes, uint32_t *words) {
  int i, b;
  for (b = 0; b < 3; ++b) {
    uint32_t w = 0;
    for (i = 0; i < 32; ++i) w |= (uint32_t)((codes[i] >> b) & 1u) << i;
    words[b] = w;
  }
}

static void pack_block(const uint16_t *codes, int bits, uint32_t *words) {
  if (bits == 3)
    kivi_oracle_pack_planes(codes, words);
  else
    words[0] = kivi_oracle_pack_word(codes, bits);
}

/* code at position pos of a block whose first word is w[0] */
static uint32_t unpack_block(const uint32_t *w, int pos, int bits) {
  if (bits == 3)
    return ((w[0] >> pos) & 1u) | (((w[1] >> pos) & 1u) << 1) | (((w[2] >> pos) & 1u) << 2);
  return (w[0] >> (bits * pos)) & (uint32_t)((1u << bits) - 1u);
}

/* D.  x_hat = c * s + z, evaluated in real arithmetic (binary64 holds
 * c * s exactly; the one remaining rounding is far below binary32). */
double kivi_oracle_dequant(uint32_t c, float scale, float zero) {
  return (double)c * (double)scale + (double)zero;
}

int kivi_oracle_check_unit(const kivi_oracle_unit *u) {
  int E;
  if (!u || !valid_bits(u->bits)) return KIVI_ORACLE_ERR_ARG;
  E = block_codes(u->bits);
  if (u->D <= 0 || u->G <= 0 || u->Gv <= 0 || u->R <= 0 || u->Tq < 0)
    return KIVI_ORACLE_ERR_ARG;
  if (u->D % E || u->D % u->Gv || u->R % u->G || u->R % E || u->Tq % u->R)
    return KIVI_ORACLE_ERR_ARG;
  if (u->Tq > 0 && (!u->k_codes || !u->k_scale || !u->k_zero ||
                    !u->v_codes || !u->v_scale || !u->v_zero))
    return KIVI_ORACLE_ERR_ARG;
  if (!u->k_res || !u->v_res) return KIVI_ORACLE_ERR_ARG;
  /* dense-and-sparse: fewer outliers than group entries (and at most 64),
   * binary32 metadata, the lists present */
  if (u->k_out < 0 || u->k_out >= u->G || u->k_out > 64 || u->v_out < 0 || u->v_out >= u->Gv ||
      u->v_out > 64)
    return KIVI_ORACLE_ERR_ARG;
  if ((u->k_out > 0 || u->v_out > 0) && u->meta_f16) return KIVI_ORACLE_ERR_ARG;
  if (u->Tq > 0 && ((u->k_out > 0 && (!u->k_out_idx || !u->k_out_val)) ||
                    (u->v_out > 0 && (!u->v_out_idx || !u->v_out_val))))
    return KIVI_ORACLE_ERR_ARG;
  return KIVI_ORACLE_OK;
}

/*
 * Q + P over a block of n tokens (n a multiple of G and of E), written to
 * token positions t0 .. t0+n-1 of the quantized store.  K and V are [n][D].
 *   keys:   per channel d, groups of G consecutive tokens (per-channel key
 *           quantization, grouped across tokens);
 *   values: per token t, groups of Gv consecutive channels (per-token value
 *           quantization).
 * Codes are first produced for every (token, channel), then packed: keys
 * along channels within a token, values along tokens within a channel.
 */
static int quantize_block(kivi_oracle_unit *u, const float *K, const float *V,
                          long long t0, long long n) {
  const int D = u->D, bits = u->bits, G = u->G, Gv = u->Gv;
  /* E codes per block of WB words; a token's keys take WK words */
  const int E = block_codes(bits), WB = block_words(bits), WK = (D / E) * WB, NJ = D / Gv;
  uint16_t *ck = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(n * D));
  uint16_t *cv = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(n * D));
  uint16_t *tmp = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(G > E ? G : E));
  long long t, g, i;
  int d, j, w;
  if (!ck || !cv || !tmp) {
    free(ck);
    free(cv);
    free(tmp);
    return KIVI_ORACLE_ERR_NOMEM;
  }

  long long oi[64];
  float ov[64];
  int m;
  /* keys: one group per (key group g, channel d) over G tokens */
  for (g = 0; g < n / G; ++g) {
    for (d = 0; d < D; ++d) {
      long long gq = (t0 / G) + g;
      if (u->k_out > 0) {
        kivi_oracle_quantize_group_sparse(&K[(g * G) * D + d], G, D, bits, u->k_out,
                                          &u->k_scale[gq * D + d], &u->k_zero[gq * D + d], tmp,
                                          oi, ov);
        for (m = 0; m < u->k_out; ++m) {
          u->k_out_idx[(gq * D + d) * u->k_out + m] = (int32_t)oi[m];
          u->k_out_val[(gq * D + d) * u->k_out + m] = ov[m];
        }
      } else {
        kivi_oracle_quantize_group_meta(&K[(g * G) * D + d], G, D, bits, u->meta_f16,
                                        &u->k_scale[gq * D + d],
                                        &u->k_zero[gq * D + d], tmp);
      }
      for (i = 0; i < G; ++i) ck[(g * G + i) * D + d] = tmp[i];
    }
  }
  /* values: one group per (token t, value group j) over Gv channels */
  for (t = 0; t < n; ++t) {
    for (j = 0; j < NJ; ++j) {
      const long long mo = (t0 + t) * NJ + j;
      if (u->v_out > 0) {
        kivi_oracle_quantize_group_sparse(&V[t * D + j * Gv], Gv, 1, bits, u->v_out,
                                          &u->v_scale[mo], &u->v_zero[mo], tmp, oi, ov);
        for (m = 0; m < u->v_out; ++m) {
          u->v_out_idx[mo * u->v_out + m] = (int32_t)oi[m];
          u->v_out_val[mo * u->v_out + m] = ov[m];
        }
      } else {
        kivi_oracle_quantize_group_meta(&V[t * D + j * Gv], Gv, 1, bits, u->meta_f16,
                                        &u->v_scale[mo], &u->v_zero[mo], tmp);
      }
      for (i = 0; i < Gv; ++i) cv[t * D + j * Gv + i] = tmp[i];
    }
  }
  /* pack keys along channels: block w of token t holds channels wE..wE+E-1
   * in words [w WB, w WB + WB) of the token's WK words */
  for (t = 0; t < n; ++t)
    for (w = 0; w < D / E; ++w)
      pack_block(&ck[t * D + w * E], bits, &u->k_codes[(t0 + t) * WK + w * WB]);
  /* pack values along tokens: block (tb, d) holds tokens tb*E..tb*E+E-1 of
   * channel d in word rows tb WB .. tb WB + WB - 1 */
  for (t = 0; t < n / E; ++t) {
    for (d = 0; d < D; ++d) {
      uint32_t words[3];
      int b;
      for (i = 0; i < E; ++i) tmp[i] = cv[(t * E + i) * D + d];
      pack_block(tmp, bits, words);
      for (b = 0; b < WB; ++b) u->v_codes[(((t0 / E) + t) * WB + b) * D + d] = words[b];
    }
  }
  free(ck);
  free(cv);
  free(tmp);
  return KIVI_ORACLE_OK;
}

/*
 * S, prefill.  Reading of "residual window of R recent tokens, flushed every
 * R": the window is flushed just before a token would not fit, so a
 * non-empty cache always holds 1..R residual tokens.  A prompt of T tokens
 * therefore leaves r = ((T-1) mod R) + 1 tokens in the window and quantizes
 * the first n_q = T - r, exactly the state T single appends would reach.
 */
int kivi_oracle_prefill(kivi_oracle_unit *u, const float *K, const float *V,
                        long long T) {
  int rc = kivi_oracle_check_unit(u);
  long long r, nq;
  if (rc) return rc;
  if (T < 0 || (T > 0 && (!K || !V))) return KIVI_ORACLE_ERR_ARG;
  if (u->n_q != 0 || u->r != 0) return KIVI_ORACLE_ERR_STATE;
  r = (T == 0) ? 0 : ((T - 1) % u->R) + 1;
  nq = T - r;
  if (nq > u->Tq) return KIVI_ORACLE_ERR_CAPACITY;
  if (nq > 0) {
    rc = quantize_block(u, K, V, 0, nq);
    if (rc) return rc;
  }
  memcpy(u->k_res, &K[nq * u->D], sizeof(float) * (size_t)(r * u->D));
  memcpy(u->v_res, &V[nq * u->D], sizeof(float) * (size_t)(r * u->D));
  u->n_q = nq;
  u->r = (int)r;
  return KIVI_ORACLE_OK;
}

/*
 * S, append one token.  If the window is full, its R tokens are quantized
 * (Q + P, R/G key groups and R value tokens) into token positions
 * n_q .. n_q+R-1 and the window is emptied; then the token is written to the
 * next window slot.
 */
int kivi_oracle_append(kivi_oracle_unit *u, const float *k, const float *v) {
  int rc = kivi_oracle_check_unit(u);
  if (rc) return rc;
  if (!k || !v) return KIVI_ORACLE_ERR_ARG;
  if (u->r == u->R) {
    if (u->n_q + u->R > u->Tq) return KIVI_ORACLE_ERR_CAPACITY;
    rc = quantize_block(u, u->k_res, u->v_res, u->n_q, u->R);
    if (rc) return rc;
    u->n_q += u->R;
    u->r = 0;
  }
  memcpy(&u->k_res[(long long)u->r * u->D], k, sizeof(float) * (size_t)u->D);
  memcpy(&u->v_res[(long long)u->r * u->D], v, sizeof(float) * (size_t)u->D);
  u->r += 1;
  return KIVI_ORACLE_OK;
}

/* D over the whole unit: token t < n_q from codes, t >= n_q from the window. */
int kivi_oracle_dequant_keys(const kivi_oracle_unit *u, double *out) {
  int rc = kivi_oracle_check_unit(u);
  const int D = u ? u->D : 0;
  long long t;
  int d;
  if (rc) return rc;
  if (!out) return KIVI_ORACLE_ERR_ARG;
  for (t = 0; t < u->n_q; ++t) {
    const int E = block_codes(u->bits), WB = block_words(u->bits);
    for (d = 0; d < D; ++d) {
      const uint32_t *blk = &u->k_codes[t * (D / E) * WB + (d / E) * WB];
      uint32_t c = unpack_block(blk, d % E, u->bits);
      long long g = t / u->G;
      out[t * D + d] = kivi_oracle_dequant(c, u->k_scale[g * D + d], u->k_zero[g * D + d]);
    }
  }
  /* dense-and-sparse: the kept outliers replace their dense values */
  for (t = 0; u->k_out > 0 && t < u->n_q / u->G; ++t) {
    int m;
    for (d = 0; d < D; ++d)
      for (m = 0; m < u->k_out; ++m) {
        const long long e = (t * D + d) * u->k_out + m;
        out[(t * u->G + u->k_out_idx[e]) * D + d] = (double)u->k_out_val[e];
      }
  }
  for (t = 0; t < u->r; ++t)
    for (d = 0; d < D; ++d) out[(u->n_q + t) * D + d] = (double)u->k_res[t * D + d];
  return KIVI_ORACLE_OK;
}

int kivi_oracle_dequant_values(const kivi_oracle_unit *u, double *out) {
  int rc = kivi_oracle_check_unit(u);
  const int D = u ? u->D : 0;
  long long t;
  int d;
  if (rc) return rc;
  if (!out) return KIVI_ORACLE_ERR_ARG;
  for (t = 0; t < u->n_q; ++t) {
    const int E = block_codes(u->bits), WB = block_words(u->bits), NJ = D / u->Gv;
    for (d = 0; d < D; ++d) {
      uint32_t blk[3];
      int b;
      for (b = 0; b < WB; ++b) blk[b] = u->v_codes[((t / E) * WB + b) * D + d];
      uint32_t c = unpack_block(blk, (int)(t % E), u->bits);
      int j = d / u->Gv;
      out[t * D + d] = kivi_oracle_dequant(c, u->v_scale[t * NJ + j], u->v_zero[t * NJ + j]);
    }
  }
  /* dense-and-sparse: the kept outliers replace their dense values */
  for (t = 0; u->v_out > 0 && t < u->n_q; ++t) {
    const int NJ = D / u->Gv;
    int j, m;
    for (j = 0; j < NJ; ++j)
      for (m = 0; m < u->v_out; ++m) {
        const long long e = (t * NJ + j) * u->v_out + m;
        out[t * D + j * u->Gv + u->v_out_idx[e]] = (double)u->v_out_val[e];
      }
  }
  for (t = 0; t < u->r; ++t)
    for (d = 0; d < D; ++d) out[(u->n_q + t) * D + d] = (double)u->v_res[t * D + d];
  return KIVI_ORACLE_OK;
}

/*
 * A.  Plain two-pass softmax attention over all n_q + r tokens, with the
 * quantized and the residual tokens in one softmax (not two normalised
 * parts):
 *   l_t   = sigma * sum_d q_d * Khat_{t,d}
 *   p_t   = exp(l_t - max_t l_t)
 *   out_d = sum_t p_t * Vhat_{t,d} / sum_t p_t
 * in binary64, sums in index order.
 */
int kivi_oracle_decode(const kivi_oracle_unit *u, const float *q, int n_heads,
                       double sigma, double *out) {
  int rc = kivi_oracle_check_unit(u);
  long long T, t;
  int h, d;
  double *Kh, *Vh, *p;
  if (rc) return rc;
  if (!q || !out || n_heads <= 0) return KIVI_ORACLE_ERR_ARG;
  T = u->n_q + u->r;
  if (T == 0) return KIVI_ORACLE_ERR_STATE;
  Kh = (double *)malloc(sizeof(double) * (size_t)(T * u->D));
  Vh = (double *)malloc(sizeof(double) * (size_t)(T * u->D));
  p = (double *)malloc(sizeof(double) * (size_t)T);
  if (!Kh || !Vh || !p) {
    free(Kh);
    free(Vh);
    free(p);
    return KIVI_ORACLE_ERR_NOMEM;
  }
  kivi_oracle_dequant_keys(u, Kh);
  kivi_oracle_dequant_values(u, Vh);
  for (h = 0; h < n_heads; ++h) {
    const float *qh = &q[(long long)h * u->D];
    double m = -INFINITY, l = 0.0;
    for (t = 0; t < T; ++t) {
      double acc = 0.0;
      for (d = 0; d < u->D; ++d) acc += (double)qh[d] * Kh[t * u->D + d];
      p[t] = sigma * acc;
      if (p[t] > m) m = p[t];
    }
    for (t = 0; t < T; ++t) {
      p[t] = exp(p[t] - m);
      l += p[t];
    }
    for (d = 0; d < u->D; ++d) {
      double o = 0.0;
      for (t = 0; t < T; ++t) o += p[t] * Vh[t * u->D + d];
      out[(long long)h * u->D + d] = o / l;
    }
  }
  free(Kh);
  free(Vh);
  free(p);
  return KIVI_ORACLE_OK;
}
