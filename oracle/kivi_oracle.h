/*
 * kivi_oracle.h -- declarations of the plain CPU oracle for the KIVI
 * asymmetric 2/4-bit KV cache.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load this code.  It shares no source, header
 * or table with the CUDA library (include/kivi.h, the package's csrc/), and
 * the CUDA library never calls it.
 *
 * Method sources (pages about "KIVI: A Tuning-Free Asymmetric 2bit
 * Quantization for KV Cache"):
 *   - mlsanity.com index page, section "Abstract (arXiv)": keys quantized
 *     per channel, values per token, 2-bit codes.
 *   - study.space summary page (single summary paragraph): asymmetric
 *     quantization, key quantization grouped over tokens, value codes
 *     appended along the token axis, caches split into a quantized
 *     ("grouped") part and a full-precision residual part that is merged
 *     with the quantized part in decode attention.
 *   - scholarfeed.org "KIVI" page, third quote: the residual is a
 *     fixed-length buffer of recent tokens kept unquantized.
 * Where the pages say nothing (the scale/zero formula, rounding, packing
 * order, flush timing) the oracle takes the plainest reading, stated in
 * kivi_oracle.c beside the function that applies it.
 */
#ifndef KIVI_ORACLE_H
#define KIVI_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  KIVI_ORACLE_OK = 0,
  KIVI_ORACLE_ERR_ARG = 1,
  KIVI_ORACLE_ERR_STATE = 2,
  KIVI_ORACLE_ERR_CAPACITY = 3,
  KIVI_ORACLE_ERR_NOMEM = 4
};

/*
 * One (batch element, KV head) unit of the cache, in host memory.
 * Let E = 32 / bits codes per 32-bit word and Tq = the quantized-store
 * capacity in tokens.  The arrays are this unit's slices of the cache
 * buffers, laid out as:
 *   k_codes [Tq][D/E]   word w of token t holds channels wE..wE+E-1,
 *                       channel wE+i in bits [bits*i, bits*i+bits)
 *   k_scale [Tq/G][D]   one (scale, zero) per key group (G tokens) and channel
 *   k_zero  [Tq/G][D]
 *   v_codes [Tq/E][D]   word (tb, d) holds tokens tb*E..tb*E+E-1 of channel
 *                       d, token tb*E+i in bits [bits*i, bits*i+bits)
 *   v_scale [Tq][D/Gv]  one (scale, zero) per token and value group (Gv
 *   v_zero  [Tq][D/Gv]  channels)
 *   k_res   [R][D]      residual keys, full precision (fp32 values)
 *   v_res   [R][D]      residual values
 * 3 bits (E = 32 codes per block of three bit-plane words,
 * kivi_oracle_pack_planes): k_codes [Tq][D/32*3], block w of a token in
 * words 3w..3w+2; v_codes [Tq/32*3][D], block tb of channel d in rows
 * 3tb..3tb+2.
 * Dense-and-sparse variant (k_out / v_out > 0, binary32 metadata only): every
 * key group keeps its k_out largest magnitudes exactly and every value group
 * its v_out largest (kivi_oracle_quantize_group_sparse), listed in
 *   k_out_idx, k_out_val [Tq/G][D][k_out]   token within the group, value
 *   v_out_idx, v_out_val [Tq][D/Gv][v_out]  channel within the group, value
 * in ascending index order; their dense codes are 0.
 */
typedef struct {
  int D;
  int bits;
  int G;
  int Gv;
  int R;
  long long Tq;
  uint32_t *k_codes;
  float *k_scale;
  float *k_zero;
  uint32_t *v_codes;
  float *v_scale;
  float *v_zero;
  float *k_res;
  float *v_res;
  long long n_q; /* tokens held in the quantized store */
  int r;         /* tokens held in the residual window */
  int meta_f16;  /* 1: scales and zeros stored in binary16 (format variant) */
  int k_out;     /* outliers kept per key group (dense-and-sparse variant), 0: none */
  int v_out;     /* outliers kept per value group */
  int32_t *k_out_idx;
  float *k_out_val;
  int32_t *v_out_idx;
  float *v_out_val;
} kivi_oracle_unit;

/* Q: quantize one group of n values x[0], x[stride], ..., x[(n-1)*stride]. */
int kivi_oracle_quantize_group(const float *x, long long n, long long stride,
                               int bits, float *scale, float *zero,
                               uint16_t *codes);

/* Q with the metadata stored in binary16 when meta_f16 is 1: the scale and
 * zero are rounded to binary16 and the codes are chosen against the rounded
 * values (a format variant; meta_f16 = 0 is kivi_oracle_quantize_group). */
int kivi_oracle_quantize_group_meta(const float *x, long long n, long long stride,
                                    int bits, int meta_f16, float *scale,
                                    float *zero, uint16_t *codes);

/* Q, dense-and-sparse variant: the k entries of largest magnitude (ties:
 * lower index first) go to out_idx / out_val in ascending index order with
 * dense code 0; the other n - k entries are quantized by Q in their order.
 * Requires 0 <= k < n. */
int kivi_oracle_quantize_group_sparse(const float *x, long long n, long long stride, int bits,
                                      int k, float *scale, float *zero, uint16_t *codes,
                                      long long *out_idx, float *out_val);

/* x rounded to the nearest IEEE binary16 value (ties to even), as a float. */
float kivi_oracle_round_half(float x);

/* P: pack 32/bits codes into one word, codes[0] in the least significant bits. */
uint32_t kivi_oracle_pack_word(const uint16_t *codes, int bits);

/* P for 3 bits: 32 codes as three bit planes, words[b] bit i = bit b of codes[i]. */
void kivi_oracle_pack_planes(const uint16_t *codes, uint32_t *words);

/* D: the dequantized value of code c with (scale, zero), in real arithmetic. */
double kivi_oracle_dequant(uint32_t c, float scale, float zero);

/* S: state machine of one unit. */
int kivi_oracle_check_unit(const kivi_oracle_unit *u);
int kivi_oracle_prefill(kivi_oracle_unit *u, const float *K, const float *V,
                        long long T);
int kivi_oracle_append(kivi_oracle_unit *u, const float *k, const float *v);

/* Full-precision view of the unit's keys / values: out[(n_q + r) * D]. */
int kivi_oracle_dequant_keys(const kivi_oracle_unit *u, double *out);
int kivi_oracle_dequant_values(const kivi_oracle_unit *u, double *out);

/* A: decode attention of n_heads query heads q[n_heads][D] against the
 * unit, out[n_heads][D]. */
int kivi_oracle_decode(const kivi_oracle_unit *u, const float *q, int n_heads,
                       double sigma, double *out);

#ifdef __cplusplus
}
#endif

#endif
