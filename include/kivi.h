/*
 * kivi.h -- C ABI of libkivi.so: a KIVI-style asymmetric 1/2/4-bit KV cache
 * with a full-precision residual window and fused decode attention, for
 * NVIDIA B200 (sm_100a).
 *
 * Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache".
 *   - mlsanity.com index page, section "Abstract (arXiv)": keys are
 *     quantized per channel, values per token, to 2 bits; loading the KV
 *     cache, not arithmetic, limits decode speed.
 *   - study.space summary page (one summary paragraph): the quantizer is
 *     asymmetric; key groups span tokens; value codes are appended along the
 *     token axis; each cache is split into a quantized ("grouped") part and
 *     a full-precision residual part, and decode attention over the
 *     quantized part is combined with the residual part.
 *   - scholarfeed.org "KIVI" page, third quote: the residual is a
 *     fixed-length buffer of the most recent tokens, kept unquantized
 *     (a mixed-precision cache).
 *   - same page, first quote: a 4-bit variant of KIVI exists.
 *
 * Conventions shared by every entry point
 *   - Every pointer named "device" is CUDA device memory on the current
 *     device; the library never allocates, frees or copies host memory on
 *     the caller's behalf, never allocates device memory and never
 *     synchronizes.  All work is enqueued on `stream` (a cudaStream_t passed
 *     as void*; NULL is the legacy default stream) and is asynchronous.
 *   - Every call returns a kivi_status.  Argument, shape, state and capacity
 *     errors are detected on the host before anything is enqueued and leave
 *     the cache state unchanged.  KIVI_ERR_CUDA reports a launch error
 *     (cudaGetLastError after the launch); the host counters are then not
 *     advanced.  Nothing throws across this boundary.
 *   - A kivi_cache is not thread safe: calls on one cache must be
 *     serialized by the caller (they update its host-side counters).
 *
 * Cache layout (part of the ABI; all arrays dense, row-major).  With
 * E = 32/bits codes per 32-bit word, Tq = capacity - R quantized tokens per
 * sequence, NG = Tq/G key groups and NJ = D/Gv value groups per token:
 *   k_codes  uint32 [B][Hkv][Tq][D/E]   word w of token t packs channels
 *                                        wE..wE+E-1; channel wE+i in bits
 *                                        [bits*i, bits*i+bits)
 *   k_scale  meta   [B][Hkv][NG][D]     one scale and zero per key group
 *   k_zero   meta   [B][Hkv][NG][D]     (G consecutive tokens) and channel
 *   v_codes  uint32 [B][Hkv][Tq/E][D]   word (tb, d) packs tokens
 *                                        tb*E..tb*E+E-1 of channel d;
 *                                        token tb*E+i in bits
 *                                        [bits*i, bits*i+bits)
 *   v_scale  meta   [B][Hkv][Tq][NJ]    one scale and zero per token and
 *   v_zero   meta   [B][Hkv][Tq][NJ]    value group (Gv consecutive channels)
 *   k_res    dtype  [B][Hkv][R][D]      residual window, input precision;
 *   v_res    dtype  [B][Hkv][R][D]      slots 0..r-1 hold the newest tokens
 * Each code packs along the axis its attention product contracts over
 * (channels for keys, tokens for values).  "meta" is binary32 (float), or
 * binary16 when dims.meta = KIVI_META_F16 (see kivi_meta).
 * 3 bits (a format variant; 3 does not divide 32): codes come in blocks of
 * E = 32 held as three bit-plane words, plane p holding bit p of code i in
 * its bit i.  k_codes [B][Hkv][Tq][D/32*3]: block w of token t (channels
 * 32w..32w+31) in words 3w..3w+2; v_codes [B][Hkv][Tq/32*3][D]: block tb of
 * channel d (tokens 32tb..32tb+31) in rows 3tb..3tb+2.  (KVQuant page,
 * abstract: 3-bit KV cache quantization.)
 *
 * Quantizer (fixed binary32 formula; codes, scales and zeros are bit-exact
 * functions of the inputs): for a group x_0..x_{n-1},
 *   mn = min x_i, mx = max x_i (first occurrence kept among equal values),
 *   s = (mx - mn) / (2^bits - 1), z = mn  (each op rounded to nearest),
 *   c_i = clamp(round_half_even((x_i - mn) / s), 0, 2^bits - 1), or 0 if s == 0.
 * Dequantized value: c * s + z.  (With binary16 metadata s and z are first
 * rounded to binary16; see kivi_meta.)
 *
 * Residual window ("flush before write"): a non-empty cache holds
 * r in [1, R] residual tokens.  Prefill of T tokens leaves
 * r = ((T-1) mod R) + 1 and quantizes the first n_q = T - r; appending to a
 * full window first quantizes its R tokens into positions n_q..n_q+R-1.
 * prefill(T) and T single appends therefore produce identical bytes.
 */
#ifndef KIVI_H
#define KIVI_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KIVI_API __attribute__((visibility("default")))
#else
#define KIVI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KIVI_OK = 0,
  KIVI_ERR_ARG = 1,         /* null pointer, negative size, Hq not a multiple of Hkv */
  KIVI_ERR_UNSUPPORTED = 2, /* bits, G, Gv, D, R or dtype outside the built kernels */
  KIVI_ERR_STATE = 3,       /* prefill on a non-empty cache; decode on an empty one */
  KIVI_ERR_CAPACITY = 4,    /* the tokens would not fit in `capacity` */
  KIVI_ERR_WORKSPACE = 5,   /* workspace missing, too small or misaligned */
  KIVI_ERR_CUDA = 6,        /* a CUDA launch or device query failed */
  KIVI_ERR_SCRATCH_LIMIT = 7 /* request exceeds the fixed scratch of the _noalloc call */
} kivi_status;

typedef enum { KIVI_F16 = 0, KIVI_F32 = 1 } kivi_dtype;

/* Element type of the scales and zeros.  KIVI_META_F16 is the format
 * variant with binary16 metadata (fp16 caches only): the binary32 scale s
 * and minimum mn of a group are rounded to nearest-even binary16, s16 and
 * z16, and the codes are chosen against them:
 *   c_i = clamp(round_half_even((x_i - z16) / s16), 0, 2^bits - 1), or 0 if
 *   s16 == 0; dequantized value c * s16 + z16.
 * It halves the metadata bytes; at 2 bits the binary32 scales and zeros are
 * half of what the decode streams per quantized token, so binary16 cuts
 * those bytes by a quarter.  (KIVI, study.space summary:
 * each group keeps an asymmetric scale and offset; the pages fix no
 * storage precision for them.) */
typedef enum { KIVI_META_F32 = 0, KIVI_META_F16 = 1 } kivi_meta;

/* Shape of one cache (one attention layer).  k_out = v_out = 0 (a
 * zero-filled struct) is the plain format; see the dense-and-sparse
 * variant below for other values.  Supported: bits in {1, 2, 3, 4}
 * (3 bits: the tensor-core decode only; kivi_decode_attention_simt refuses
 * it with KIVI_ERR_UNSUPPORTED),
 * G = 32, Gv = 32, D in {32, 64, 128}, R a positive multiple of 32,
 * capacity a positive multiple of R, dtype KIVI_F16 or KIVI_F32, meta
 * KIVI_META_F32 or (with dtype KIVI_F16) KIVI_META_F16.  A zero-filled
 * meta field selects binary32 metadata. */
typedef struct {
  int B;              /* sequences (batch) */
  int Hkv;            /* key/value heads */
  int D;              /* head dimension (channels) */
  int bits;           /* code width */
  int G;              /* key group: tokens sharing one scale/zero per channel */
  int Gv;             /* value group: channels sharing one scale/zero per token */
  int R;              /* residual window length in tokens */
  long long capacity; /* max tokens per sequence, quantized + residual */
  int dtype;          /* kivi_dtype of K, V, q, out and the residual window */
  int meta;           /* kivi_meta of k_scale, k_zero, v_scale, v_zero */
  int k_out;          /* dense-and-sparse variant: entries kept exactly per key
                         group (0: plain codes; see kivi_outlier_buffer_sizes) */
  int v_out;          /* ... per value group */
} kivi_dims;

enum {
  KIVI_BUF_K_CODES = 0,
  KIVI_BUF_K_SCALE = 1,
  KIVI_BUF_K_ZERO = 2,
  KIVI_BUF_V_CODES = 3,
  KIVI_BUF_V_SCALE = 4,
  KIVI_BUF_V_ZERO = 5,
  KIVI_BUF_K_RES = 6,
  KIVI_BUF_V_RES = 7,
  KIVI_NUM_BUFFERS = 8
};

/* A cache: the caller's device buffers (layout above) plus host counters
 * that the library owns and advances.  n_q and r are the same for every
 * sequence of the batch. */
typedef struct {
  kivi_dims dims;
  uint32_t *k_codes;
  void *k_scale; /* float, or uint16_t binary16 bits when dims.meta = KIVI_META_F16 */
  void *k_zero;
  uint32_t *v_codes;
  void *v_scale;
  void *v_zero;
  void *k_res;
  void *v_res;
  long long n_q; /* tokens per sequence in the quantized store */
  int r;         /* tokens per sequence in the residual window */
  /* paged store (kivi_paged_cache_init); NULL / 0 for a contiguous cache */
  const int32_t *block_table; /* device, [B][pages_per_seq] pool page ids */
  int pages_per_seq;
  long long num_pages;        /* pages in the pool */
  /* dense-and-sparse variant (kivi_cache_set_outliers); NULL otherwise */
  int32_t *k_out_idx;
  float *k_out_val;
  int32_t *v_out_idx;
  float *v_out_val;
} kivi_cache;

/* Byte size of each of the KIVI_NUM_BUFFERS buffers for `dims`, written to
 * out_bytes[KIVI_BUF_*].  Pure host arithmetic.
 * Errors: KIVI_ERR_ARG (null), KIVI_ERR_UNSUPPORTED (dims not supported). */
KIVI_API int kivi_buffer_sizes(const kivi_dims *dims, size_t out_bytes[KIVI_NUM_BUFFERS]);

/* Bind `buffers[KIVI_BUF_*]` (device pointers, each 16-byte aligned and at
 * least kivi_buffer_sizes() bytes; the caller keeps ownership) to `cache`
 * and set n_q = r = 0.  No device work; buffer contents are not read until
 * written by prefill/append.
 * Errors: KIVI_ERR_ARG (null or misaligned pointer), KIVI_ERR_UNSUPPORTED. */
KIVI_API int kivi_cache_init(kivi_cache *cache, const kivi_dims *dims,
                    void *const buffers[KIVI_NUM_BUFFERS]);

/* Prefill: quantize a prompt of T tokens into an empty cache.
 * K, V: device, dims.dtype, [B][Hkv][T][D] contiguous.  Tokens 0..n_q-1
 * (n_q = T - r, r = ((T-1) mod R) + 1) are quantized: keys per (key group,
 * channel) over G tokens, values per (token, value group) over Gv channels;
 * tokens n_q..T-1 are copied unmodified into the residual window.
 * (KIVI, study.space summary: grouped parts quantized, residual parts kept
 * in full precision; mlsanity.com abstract: per-channel keys, per-token
 * values.)
 * Any element alignment is accepted.  K and V 16-byte aligned (and no outlier
 * lists) take the fast path, which stages each 32-token tile in shared memory
 * by 16-byte asynchronous copies; the result is the same bit for bit.
 * Inputs are expected finite: with a NaN in a group the scale, zero and codes
 * of that group are unspecified.
 * Errors: KIVI_ERR_ARG, KIVI_ERR_STATE (cache not empty),
 * KIVI_ERR_CAPACITY (T > capacity), KIVI_ERR_CUDA. */
KIVI_API int kivi_quantize_prefill(kivi_cache *cache, const void *K, const void *V,
                          long long T, void *stream);

/* Append one token per sequence.  k, v: device, dims.dtype, [B][Hkv][D].
 * If the window is full (r == R) its R tokens are first quantized into the
 * store (R/G key groups, R value tokens) and the window emptied (one kernel
 * launch either way).  (KIVI, study.space summary: new codes appended along
 * the token axis, key groups formed across tokens; scholarfeed.org "KIVI"
 * page: fixed-length residual buffer.)
 * Errors: KIVI_ERR_ARG, KIVI_ERR_CAPACITY (n_q + r + 1 > capacity),
 * KIVI_ERR_CUDA. */
KIVI_API int kivi_append_token(kivi_cache *cache, const void *k, const void *v,
                      void *stream);

/* Bytes of device workspace kivi_decode_attention needs for Hq query heads
 * at any fill level of this cache (0 on error).  Host arithmetic only. */
KIVI_API size_t kivi_decode_workspace_bytes(const kivi_cache *cache, int Hq);

/* Decode attention for one new query per sequence and head, computed
 * directly over the packed codes plus the residual window, with one softmax
 * over all n_q + r tokens:
 *   out[b][h] = sum_t p_t * Vhat_t / sum_t p_t,
 *   p_t = exp(softmax_scale * <q[b][h], Khat_t> - max),
 * where Khat/Vhat are the dequantized codes for t < n_q and the stored
 * window tokens after that.  Query head h reads KV head h / (Hq/Hkv).
 * q, out: device, dims.dtype, [B][Hq][D] contiguous.  workspace: device,
 * 16-byte aligned, at least kivi_decode_workspace_bytes(cache, Hq) bytes,
 * scratch that is fully written before it is read.
 * (KIVI, study.space summary: attention over the quantized part, then
 * combined with the residual part; mlsanity.com abstract: cache loading
 * bounds decode.)
 * Errors: KIVI_ERR_ARG (null, Hq % Hkv != 0, Hq/Hkv > 8), KIVI_ERR_STATE
 * (empty cache), KIVI_ERR_WORKSPACE, KIVI_ERR_CUDA. */
KIVI_API int kivi_decode_attention(const kivi_cache *cache, const void *q, int Hq,
                          float softmax_scale, void *out, void *workspace,
                          size_t workspace_bytes, void *stream);

/* Same result as kivi_decode_attention (same arguments, same workspace
 * rule) computed by the plain CUDA-core (SIMT) kernel instead of the
 * tensor-core kernel; kept as the measured alternative. */
KIVI_API int kivi_decode_attention_simt(const kivi_cache *cache, const void *q,
                               int Hq, float softmax_scale, void *out,
                               void *workspace, size_t workspace_bytes,
                               void *stream);

/* One decode step of a streaming loop: kivi_append_token(cache, k, v)
 * followed by kivi_decode_attention over the cache that now holds the new
 * token -- same arguments as the two calls, same result, same counter
 * update -- in one kernel launch: when the window is full (r == R) the
 * decode kernel first quantizes it into the store (every CTA takes a share
 * of the window tiles, then a grid-wide barrier), and the warp that reads
 * the window tile holding the new token's slot (r, or 0 after a flush)
 * writes the token there, into shared memory and the cache.  Only a k or v
 * that is not 16-byte aligned takes two launches (the append on its own
 * first).  All argument checks of both calls happen before any launch, so
 * an error leaves the cache unchanged.  The counters stay on the host, so a loop of
 * these calls is not graph-capturable.  (KIVI, study.space summary: new
 * tokens enter the full-precision residual part; decode attends over both
 * parts.)
 * Errors: those of kivi_append_token and kivi_decode_attention. */
KIVI_API int kivi_append_decode(kivi_cache *cache, const void *k, const void *v,
                       const void *q, int Hq, float softmax_scale, void *out,
                       void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of device staging kivi_append_decode_host needs for Hq query heads
 * (0 on error).  Host arithmetic only. */
KIVI_API size_t kivi_host_step_bytes(const kivi_cache *cache, int Hq);

/* kivi_append_decode from host memory: one step of a decode loop whose
 * token and query arrive from, and whose output goes back to, the host.
 * host_kvq: host, dims.dtype, k [B][Hkv][D], v [B][Hkv][D] and q [B][Hq][D]
 * back to back.  host_out: host, dims.dtype, [B][Hq][D].  Both should be
 * page-locked (cudaHostAlloc or registered) for the copies to be
 * asynchronous.  staging: device, 16-byte aligned, at least
 * kivi_host_step_bytes(cache, Hq) bytes, owned by the caller; its contents
 * are scratch.  On `stream`: one host-to-device copy of the inputs into
 * staging, the fused step of kivi_append_decode on them (one launch), one
 * device-to-host copy of out into host_out.  All are asynchronous: host_out
 * holds the result once the stream has reached the end of the call.  The
 * host counters advance as for kivi_append_decode.
 * Errors: KIVI_ERR_ARG (null pointer, misaligned staging, Hq not a multiple
 * of Hkv), KIVI_ERR_WORKSPACE (staging too small), those of
 * kivi_append_decode (nothing is copied back and the counters stay as they
 * were), KIVI_ERR_CUDA (a copy failed to enqueue). */
KIVI_API int kivi_append_decode_host(kivi_cache *cache, const void *host_kvq, int Hq,
                                     float softmax_scale, void *host_out, void *staging,
                                     size_t staging_bytes, void *workspace,
                                     size_t workspace_bytes, void *stream);

/* Device-resident counters of a cache: 16 bytes of device memory, 16-byte
 * aligned, laid out as { long long n_q; int r; int status; }.  With them a
 * decode loop runs without host round trips and can be captured in a CUDA
 * graph: kivi_append_decode_dev reads and advances them on the device and
 * never touches the host counters of `cache`.  status becomes 1 (and the
 * call does nothing) once an append finds the cache full.
 * kivi_dev_state_init: write the host counters of `cache` into `state`
 * (asynchronously, on `stream`) and clear status.
 * To continue with the host-counter calls afterwards, copy n_q and r back
 * from `state` into the cache struct.  No counterpart on the pages.
 * Errors: KIVI_ERR_ARG (null or misaligned state), KIVI_ERR_CUDA. */
KIVI_API int kivi_dev_state_init(const kivi_cache *cache, void *state, void *stream);

/* kivi_append_decode with the counters in `state` (device memory, see
 * kivi_dev_state_init) instead of cache->n_q / cache->r, in one kernel
 * launch per step: the decode kernel reads the counters, quantizes a full
 * window (r == R) into the store before it reads the store (all CTAs, then a
 * grid-wide barrier), writes the token into its window slot, plans its split
 * on the device, and its last CTA advances the counters.  Launch arguments
 * do not depend on the counters, so the launch can be captured once and
 * replayed.  (A k or v that is not 16-byte aligned takes two launches: the
 * append on its own, then the decode.)  The workspace
 * (kivi_decode_workspace_bytes) must be zero-filled before first use and
 * used only by these calls: they count arrivals in counters that every call
 * leaves at zero.  (KIVI, study.space summary: append to the residual part,
 * flush every R tokens, attend over both parts.)
 * Errors: KIVI_ERR_ARG, KIVI_ERR_UNSUPPORTED, KIVI_ERR_WORKSPACE,
 * KIVI_ERR_CUDA (the capacity check happens on the device: status). */
KIVI_API int kivi_append_decode_dev(const kivi_cache *cache, void *state, const void *k,
                           const void *v, const void *q, int Hq, float softmax_scale,
                           void *out, void *workspace, size_t workspace_bytes,
                           void *stream);

/* Ragged batches: every sequence b has its own length, held on the device
 * in state[b] (B entries of the kivi_dev_state_init layout:
 * { long long n_q; int r; int status; }, 16 bytes each, 16-byte aligned).
 * A cache filled by kivi_ragged_prefill is used only with the kivi_ragged_*
 * calls (the host-counter calls refuse it with KIVI_ERR_STATE); the buffer
 * layout is unchanged, each sequence filling its own units from position 0.
 * A sequence whose counters are not a valid fill, or that ran out of room
 * (status 1), is left untouched by later appends and decodes to NaN.
 * All decode work is planned on the device from the sequences' lengths
 * (tensor-core kernel; the same stream-K split over every unit's own tiles
 * and window), so launch arguments never depend on the lengths.
 * The workspace (kivi_decode_workspace_bytes) must be zero-filled before
 * first use and shared only with other kivi_ragged_* / *_dev calls.
 * (KIVI, study.space summary: a grouped part plus a residual part per
 * sequence; scholarfeed.org "KIVI" page: mixed-precision caches do not fit
 * uniform paged blocks, hence per-sequence counters here.) */

/* Paged store (ragged batches only).  The quantized store of every
 * sequence is a list of pages of R tokens (one flushed window each) taken
 * from a shared pool: page l of sequence b is pool page
 * block_table[b * pages_per_seq + l] (device int32, owned and filled by the
 * caller; distinct sequences must not share a page).  Pool layout, per
 * page and KV head, the contiguous layout above with Tq = R:
 *   k_codes uint32 [num_pages][Hkv][R][D/E]   k_scale, k_zero [num_pages][Hkv][R/G][D]
 *   v_codes uint32 [num_pages][Hkv][R/E][D]   v_scale, v_zero [num_pages][Hkv][R][NJ]
 * The residual windows stay per sequence, [B][Hkv][R][D] (a mixed-precision
 * cache keeps its full-precision part apart from the uniform pages:
 * scholarfeed.org "KIVI" page, second quote).  dims.capacity must be
 * (pages_per_seq + 1) * R.  A page id outside [0, num_pages) where a
 * sequence needs a page refuses that sequence (status 1) at prefill or
 * flush time.
 * kivi_paged_buffer_sizes: byte sizes of the 8 buffers for a pool of
 * num_pages pages.  Errors: KIVI_ERR_ARG, KIVI_ERR_UNSUPPORTED. */
KIVI_API int kivi_paged_buffer_sizes(const kivi_dims *dims, long long num_pages,
                            size_t out_bytes[KIVI_NUM_BUFFERS]);

/* Bind a pool (buffers as sized by kivi_paged_buffer_sizes, 16-byte
 * aligned) and a block table to `cache`; the cache is then filled with
 * kivi_ragged_prefill and used with the kivi_ragged_* calls only.
 * Errors: KIVI_ERR_ARG (null or misaligned pointer, capacity not
 * (pages_per_seq + 1) * R, num_pages < 1), KIVI_ERR_UNSUPPORTED. */
KIVI_API int kivi_paged_cache_init(kivi_cache *cache, const kivi_dims *dims,
                          void *const buffers[KIVI_NUM_BUFFERS], const int32_t *block_table,
                          int pages_per_seq, long long num_pages);

/* Prefill of a ragged batch into an empty cache.  K, V: device, dims.dtype,
 * [B][Hkv][T_max][D] (padded; sequence b uses its first lens[b] tokens).
 * lens: device, int64 [B].  Writes state[b] = { n_q_b, r_b, 0 } with
 * r_b = ((lens[b]-1) mod R) + 1 and n_q_b = lens[b] - r_b, or { 0, 0, 1 }
 * when lens[b] is outside [1, min(T_max, capacity)] (nothing else written).
 * Errors: KIVI_ERR_ARG, KIVI_ERR_STATE (cache not empty), KIVI_ERR_CUDA. */
KIVI_API int kivi_ragged_prefill(kivi_cache *cache, void *state, const void *K, const void *V,
                        long long T_max, const long long *lens, void *stream);

/* One token per sequence (k, v: device, dims.dtype, [B][Hkv][D]); a sequence
 * whose window is full flushes it first, on its own.  Two launches (the
 * append, then a B-thread counter update).  A sequence without room gets
 * status 1 and takes nothing.
 * Errors: KIVI_ERR_ARG, KIVI_ERR_STATE, KIVI_ERR_CUDA. */
KIVI_API int kivi_ragged_append(const kivi_cache *cache, void *state, const void *k,
                       const void *v, void *stream);

/* Decode attention of a ragged batch over each sequence's own n_q + r
 * tokens (arguments as kivi_decode_attention; state is only read).
 * Errors: KIVI_ERR_ARG, KIVI_ERR_UNSUPPORTED, KIVI_ERR_STATE,
 * KIVI_ERR_WORKSPACE, KIVI_ERR_CUDA. */
KIVI_API int kivi_ragged_decode(const kivi_cache *cache, const void *state, const void *q,
                       int Hq, float softmax_scale, void *out, void *workspace,
                       size_t workspace_bytes, void *stream);

/* kivi_ragged_append then kivi_ragged_decode as two launches: the decode
 * reads the counters as the append found them, decodes the cache with the
 * new tokens in it, and its last CTA advances every sequence's counters.
 * Capturable in a CUDA graph.  Same errors as kivi_ragged_decode. */
KIVI_API int kivi_ragged_append_decode(const kivi_cache *cache, void *state, const void *k,
                              const void *v, const void *q, int Hq, float softmax_scale,
                              void *out, void *workspace, size_t workspace_bytes,
                              void *stream);

/* Optional timing hook: if start/stop are non-NULL cudaEvent_t handles,
 * later decode calls on this thread record `start` just before and `stop`
 * just after the launch of the dominant (split) decode kernel, on the
 * call's stream.  Pass NULL, NULL to turn it off. */
KIVI_API void kivi_set_timing_events(void *start_event, void *stop_event);

/* Number of context splits the decode kernel would use for this cache's
 * current fill level and Hq (>= 1), or 0 on error. */
KIVI_API int kivi_decode_num_splits(const kivi_cache *cache, int Hq);

/* Dense-and-sparse variant (dims.k_out > 0 or dims.v_out > 0; KVQuant page,
 * abstract item (iv): outliers isolated per vector so that they do not skew
 * its quantization range).  Every key group (channel d over G tokens) keeps
 * its k_out largest magnitudes exactly, and every value group (token t over
 * Gv channels) its v_out largest; among equal magnitudes the lower index
 * goes first.  Those entries get dense code 0 and are listed, in ascending
 * index order, in four more device buffers:
 *   k_out_idx int32 [B][Hkv][Tq/G][D][k_out]   token within the key group
 *   k_out_val float [B][Hkv][Tq/G][D][k_out]   its exact value
 *   v_out_idx int32 [B][Hkv][Tq][D/Gv][v_out]  channel within the value group
 *   v_out_val float [B][Hkv][Tq][D/Gv][v_out]  its exact value
 * The other entries are quantized as usual over the remaining ones (min and
 * max taken without the kept entries).  Decode reconstructs a kept entry as
 * its value and every other one as c * s + z.  Supported: k_out and v_out
 * in [0, 4], binary32 metadata, bits 1, 2 or 4, contiguous caches (uniform
 * or ragged batches; not the paged store), the tensor-core decode (the
 * CUDA-core kernel and kivi_paged_cache_init refuse it with
 * KIVI_ERR_UNSUPPORTED).
 * kivi_outlier_buffer_sizes: byte sizes of the four buffers (0 for a list
 * that is not kept).  kivi_cache_set_outliers: bind them to a cache made by
 * kivi_cache_init (before its prefill); buffers[i] may be NULL only where
 * its size is 0.  Errors: KIVI_ERR_ARG, KIVI_ERR_UNSUPPORTED. */
KIVI_API int kivi_outlier_buffer_sizes(const kivi_dims *dims, size_t out_bytes[4]);
KIVI_API int kivi_cache_set_outliers(kivi_cache *cache, void *const buffers[4]);

/* Size of the fixed device scratch used by kivi_decode_attention_noalloc. */
#define KIVI_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

/* Decode attention for callers that cannot allocate device memory.
 * No counterpart on the pages: this is a library convenience, not part of
 * the method.  Same arguments and result as kivi_decode_attention, minus the
 * workspace: the cross-split partials go to a static device array of
 * KIVI_NOALLOC_SCRATCH_BYTES (4 MiB) that the library reserves on every GPU
 * it is loaded on, for the life of the process.  It is meant for callers
 * that run where device allocation is unavailable or not allowed once they
 * are running -- for example a plugin inside an inference engine that has
 * already reserved all device memory for its own pool, or a latency-bound
 * loop that must not call cudaMalloc because it can synchronize the device.
 *   - Nothing is allocated or freed: no cudaMalloc, cudaFree or allocating
 *     library call.  The scratch array's device address is looked up
 *     (cudaGetSymbolAddress) once per device, with that device current, by
 *     the first call on that device that launches work: a prefill, an append
 *     or a decode of any kind, this one included.  Under CUDA's lazy module
 *     loading (the default) that first lookup is also when the array's 4 MiB
 *     is reserved on the device.  So make one such call on each device
 *     (filling a cache is enough) before reserving the rest of the device
 *     for a pool of your own, and before any stream capture.
 *   - The split count is capped so that B * Hq * splits * (D + 2) * 4 bytes
 *     fit; if even one split does not fit, the call returns
 *     KIVI_ERR_SCRATCH_LIMIT and launches nothing.
 *   - All calls on a device share the one array, and it keeps whatever the
 *     last call wrote (every byte a call reads it first writes itself).
 *     Calls whose kernels overlap on the GPU (for example on two streams
 *     without ordering between them) race on it: serialize them.
 * Errors: as kivi_decode_attention (without KIVI_ERR_WORKSPACE), plus
 * KIVI_ERR_SCRATCH_LIMIT. */
KIVI_API int kivi_decode_attention_noalloc(const kivi_cache *cache, const void *q, int Hq,
                                           float softmax_scale, void *out, void *stream);

/* Human-readable name of a kivi_status. */
KIVI_API const char *kivi_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KIVI_H */
