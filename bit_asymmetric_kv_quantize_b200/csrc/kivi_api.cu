// kivi_api.cu -- the extern "C" boundary of libkivi.so (declared in
// include/kivi.h): argument and state validation, the residual-window state
// machine, the decode split heuristic, and kernel launches.  No device
// memory is allocated and no call synchronizes.
#include <limits.h>
#include <stdint.h>

#include <atomic>

#include "kivi.h"
#include "kivi_internal.cuh"

namespace {

using kivi::CacheView;
using kivi::DecodeArgs;

thread_local cudaEvent_t g_ev0 = nullptr;
thread_local cudaEvent_t g_ev1 = nullptr;

constexpr int kMaxSplits = 64;

int check_dims(const kivi_dims* d) {
  if (!d) return KIVI_ERR_ARG;
  if (d->B <= 0 || d->Hkv <= 0 || d->D <= 0 || d->R <= 0 || d->capacity <= 0)
    return KIVI_ERR_ARG;
  if (d->bits != 1 && d->bits != 2 && d->bits != 3 && d->bits != 4) return KIVI_ERR_UNSUPPORTED;
  if (d->G != kivi::kG || d->Gv != kivi::kGv) return KIVI_ERR_UNSUPPORTED;
  if (d->D != 32 && d->D != 64 && d->D != 128) return KIVI_ERR_UNSUPPORTED;
  if (d->R % kivi::kTile != 0) return KIVI_ERR_UNSUPPORTED;
  if (d->capacity % d->R != 0) return KIVI_ERR_UNSUPPORTED;
  if (d->dtype != KIVI_F16 && d->dtype != KIVI_F32) return KIVI_ERR_UNSUPPORTED;
  if (d->meta != KIVI_META_F32 && d->meta != KIVI_META_F16) return KIVI_ERR_UNSUPPORTED;
  if (d->meta == KIVI_META_F16 && d->dtype != KIVI_F16) return KIVI_ERR_UNSUPPORTED;
  if ((long long)d->B * d->Hkv > 65535) return KIVI_ERR_UNSUPPORTED;  // grid y limit
  // dense-and-sparse variant: a few kept entries per group, binary32 metadata
  if (d->k_out < 0 || d->v_out < 0) return KIVI_ERR_ARG;
  if (d->k_out > kivi::kMaxOut || d->v_out > kivi::kMaxOut) return KIVI_ERR_UNSUPPORTED;
  if ((d->k_out > 0 || d->v_out > 0) && (d->meta != KIVI_META_F32 || d->bits == 3))
    return KIVI_ERR_UNSUPPORTED;
  return KIVI_OK;
}

bool sparse(const kivi_dims& d) { return d.k_out > 0 || d.v_out > 0; }

// n_q of a cache filled by kivi_ragged_prefill: its counters live in the
// caller's device state, and the host-counter calls refuse it.
constexpr long long kRaggedMark = -1;
bool is_ragged(const kivi_cache* c) { return c->n_q == kRaggedMark; }
// Caches whose counters live on the device: ragged-filled or paged ones.
bool device_counted(const kivi_cache* c) { return is_ragged(c) || c->block_table != nullptr; }

int check_cache(const kivi_cache* c) {
  if (!c) return KIVI_ERR_ARG;
  int rc = check_dims(&c->dims);
  if (rc) return rc;
  const long long Tq = c->dims.capacity - c->dims.R;
  if (Tq > 0 && (!c->k_codes || !c->k_scale || !c->k_zero || !c->v_codes || !c->v_scale ||
                 !c->v_zero))
    return KIVI_ERR_ARG;
  if (!c->k_res || !c->v_res) return KIVI_ERR_ARG;
  if (Tq > 0 && ((c->dims.k_out > 0 && (!c->k_out_idx || !c->k_out_val)) ||
                 (c->dims.v_out > 0 && (!c->v_out_idx || !c->v_out_val))))
    return KIVI_ERR_ARG;  // the outlier lists are not bound
  return KIVI_OK;
}

size_t elem_bytes(int dtype) { return dtype == KIVI_F32 ? 4 : 2; }
size_t meta_bytes(int meta) { return meta == KIVI_META_F16 ? 2 : 4; }

CacheView view(const kivi_cache* c) {
  CacheView v;
  v.k_codes = c->k_codes;
  v.k_scale = c->k_scale;
  v.k_zero = c->k_zero;
  v.v_codes = c->v_codes;
  v.v_scale = c->v_scale;
  v.v_zero = c->v_zero;
  v.k_res = c->k_res;
  v.v_res = c->v_res;
  v.Tq = c->dims.capacity - c->dims.R;
  v.R = c->dims.R;
  v.meta = c->dims.meta;
  v.bt = c->block_table;
  v.pps = c->pages_per_seq;
  v.n_pages = c->num_pages;
  v.Hkv = c->dims.Hkv;
  v.k_out = c->dims.k_out;
  v.v_out = c->dims.v_out;
  v.k_oi = c->k_out_idx;
  v.k_ov = c->k_out_val;
  v.v_oi = c->v_out_idx;
  v.v_ov = c->v_out_val;
  return v;
}

// SM count of the current device, queried once per device.
int device_sms() {
  static int cached[128] = {0};
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 128 && cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 128) cached[dev] = sms;
  return sms;
}

// Upper bound on splits for this cache shape: enough CTAs for ~4 per SM,
// never more than kMaxSplits or than the tiles a full cache holds.
int max_splits(const kivi_dims& d, int sms) {
  const long long units = (long long)d.B * d.Hkv;
  long long want = (4LL * sms + units - 1) / units;
  long long tiles = d.capacity / kivi::kTile;
  long long s = want < tiles ? want : tiles;
  if (s > kMaxSplits) s = kMaxSplits;
  return s < 1 ? 1 : (int)s;
}

// Splits for the current fill: at most max_splits, each split a contiguous
// range of whole 32-token tiles (quantized tiles first, then the window).
void plan_splits(const kivi_cache* c, int sms, int* n_split, int* tiles_per_split) {
  const long long tiles = c->n_q / kivi::kTile + (c->r + kivi::kTile - 1) / kivi::kTile;
  int s = max_splits(c->dims, sms);
  if (s > tiles) s = (int)tiles;
  if (s < 1) s = 1;
  long long tps = (tiles + s - 1) / s;
  *tiles_per_split = (int)tps;
  *n_split = (int)((tiles + tps - 1) / tps);
}

// Tensor-core kernel: persistent stream-K plan (kivi::plan_stream_core, the
// same function the kernel runs in device-counter mode).  A unit is covered
// by the CTAs whose ranges meet its tiles or its window start index -- at
// most ceil((n_q/32 + 1) / W) + 1 CTA segments, each writing one partial --
// and the last of them also takes the window.
constexpr int kTcCtasPerSm = 3;  // upper bound; the kernel instance decides
using kivi::StreamPlan;

long long ceil_div(long long x, long long y) { return (x + y - 1) / y; }

// Partial slots per unit that any fill level of this cache can need.
int tc_seg_cap(const kivi_dims& d, int sms) {
  const long long units = (long long)d.B * d.Hkv;
  long long s = ceil_div((long long)kTcCtasPerSm * sms, units);
  const long long t = ceil_div((d.capacity - d.R) / kivi::kTile + 1, 4);
  if (t < s) s = t;
  return (int)s + 1;
}

// CTAs of the tensor-core kernel instance that run at once.
long long tc_ctas(int sms, int ctas_per_sm) {
  return (long long)(ctas_per_sm < kTcCtasPerSm ? ctas_per_sm : kTcCtasPerSm) * sms;
}

// ctas_per_sm: resident CTAs per SM of the kernel instance (<= kTcCtasPerSm);
// seg_cap: largest number of partial slots per unit the workspace holds.
void plan_stream(const kivi_cache* c, int sms, int ctas_per_sm, int seg_cap, StreamPlan* p) {
  *p = kivi::plan_stream_core((long long)c->dims.B * c->dims.Hkv, c->n_q, c->r,
                              c->dims.dtype == KIVI_F16, tc_ctas(sms, ctas_per_sm), seg_cap);
}

// Workspace: per-unit arrival counters, a grid arrival counter and a grid
// barrier counter (8 bytes each, 16-byte aligned block) followed by the split
// partials [B*Hq][n_split][D + 2] floats.
size_t counter_bytes(const kivi_dims& d) {
  return ((size_t)(d.B * d.Hkv + 2) * 8 + 15) / 16 * 16;
}

int ws_splits(const kivi_dims& d, int sms) {
  int s = max_splits(d, sms);
  const int t = tc_seg_cap(d, sms);
  return t > s ? t : s;
}

size_t workspace_bytes(const kivi_dims& d, int Hq, int sms) {
  return counter_bytes(d) + (size_t)d.B * Hq * ws_splits(d, sms) * (d.D + 2) * sizeof(float);
}

std::atomic<unsigned int> g_epoch{0};

unsigned int next_epoch() {
  unsigned int e = ++g_epoch;
  if (e == 0) e = ++g_epoch;  // 0 never tags a call
  return e;
}

void touch_noalloc_scratch();

// Validate, plan and launch one decode.  `ws` holds the arrival counters and
// the partials; the split count is capped at `split_cap`.
int decode_launch(const kivi_cache* c, const void* q, int Hq, float softmax_scale, void* out,
                  void* ws, int split_cap, int sms, void* stream, bool simt,
                  const void* new_k = nullptr, const void* new_v = nullptr, int new_slot = 0,
                  void* dev_state = nullptr, bool ragged = false, bool pending = false,
                  bool flush = false) {
  touch_noalloc_scratch();
  const int gq = Hq / c->dims.Hkv;
  DecodeArgs a;
  a.ragged = ragged ? 1 : 0;
  a.pending = pending ? 1 : 0;
  a.flush = flush ? 1 : 0;
  a.new_k = new_k;
  a.new_v = new_v;
  a.new_slot = new_slot;
  a.dev_state = (kivi::DevState*)dev_state;
  a.seg_cap = split_cap;
  a.c = view(c);
  a.q = q;
  a.out = out;
  a.ctr = (unsigned long long*)ws;
  a.ws = (float*)((char*)ws + counter_bytes(c->dims));
  a.units = c->dims.B * c->dims.Hkv;
  a.Hkv = c->dims.Hkv;
  a.gq = gq;
  a.D = c->dims.D;
  a.bits = c->dims.bits;
  a.dtype = c->dims.dtype;
  a.meta = c->dims.meta;
  a.n_q = c->n_q;
  a.r = c->r;
  a.qscale = softmax_scale * kivi::kLog2e;
  a.epoch = next_epoch();
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t err;
  if (simt) {
    plan_splits(c, sms, &a.n_split, &a.tiles_per_split);
    if (a.n_split > split_cap) {  // re-plan with fewer, longer splits
      const long long tiles = c->n_q / kivi::kTile + (c->r + kivi::kTile - 1) / kivi::kTile;
      const long long tps = (tiles + split_cap - 1) / split_cap;
      a.tiles_per_split = (int)tps;
      a.n_split = (int)((tiles + tps - 1) / tps);
    }
    err = kivi::launch_decode_simt(a, s, g_ev0, g_ev1);
  } else {
    int occ = 0;
    if (kivi::decode_tc_ctas_per_sm(a, &occ) != cudaSuccess) return KIVI_ERR_CUDA;
    StreamPlan sp;
    plan_stream(c, sms, occ, split_cap, &sp);
    // device counters: the kernel plans on the device over a full grid
    a.n_cta = dev_state ? (int)tc_ctas(sms, occ) : sp.n_cta;
    if (dev_state) a.r = 1;  // any post-append cache has a window (tensor maps)
    a.tiles_per_cta = sp.W;
    a.max_seg = sp.max_seg;
    a.win_weight = sp.win_weight;
    a.n_split = sp.max_seg;
    a.tiles_per_split = 0;
    err = kivi::launch_decode_tc(a, s, g_ev0, g_ev1);
  }
  return err == cudaSuccess ? KIVI_OK : KIVI_ERR_CUDA;
}

int decode_checks(const kivi_cache* c, const void* q, int Hq, const void* out) {
  int rc = check_cache(c);
  if (rc) return rc;
  if (!q || !out || Hq <= 0 || Hq % c->dims.Hkv != 0) return KIVI_ERR_ARG;
  const int gq = Hq / c->dims.Hkv;
  if (gq != 1 && gq != 2 && gq != 4 && gq != 8) return KIVI_ERR_UNSUPPORTED;
  if (device_counted(c) || c->n_q + c->r == 0) return KIVI_ERR_STATE;
  return KIVI_OK;
}

// Checks of the ragged calls: a cache filled by kivi_ragged_prefill, a
// 16-byte aligned state, and (decode) a query shape and workspace.
int ragged_checks(const kivi_cache* c, const void* state, const void* q, int Hq, const void* out,
                  const void* workspace, size_t ws_bytes, int* sms) {
  int rc = check_cache(c);
  if (rc) return rc;
  if (!state || ((uintptr_t)state & 15)) return KIVI_ERR_ARG;
  if (!is_ragged(c)) return KIVI_ERR_STATE;
  if (!q) return KIVI_OK;  // append only
  if (!out || Hq <= 0 || Hq % c->dims.Hkv != 0) return KIVI_ERR_ARG;
  const int gq = Hq / c->dims.Hkv;
  if (gq != 1 && gq != 2 && gq != 4 && gq != 8) return KIVI_ERR_UNSUPPORTED;
  *sms = device_sms();
  if (*sms <= 0) return KIVI_ERR_CUDA;
  if (!workspace || ((uintptr_t)workspace & 15) || ws_bytes < workspace_bytes(c->dims, Hq, *sms))
    return KIVI_ERR_WORKSPACE;
  return KIVI_OK;
}

int decode_common(const kivi_cache* c, const void* q, int Hq, float softmax_scale, void* out,
                  void* workspace, size_t ws_bytes, void* stream, bool simt) {
  int rc = decode_checks(c, q, Hq, out);
  if (rc) return rc;
  // the CUDA-core kernel: 1, 2, 4 bits, plain codes
  if (simt && (c->dims.bits == 3 || sparse(c->dims))) return KIVI_ERR_UNSUPPORTED;
  const int sms = device_sms();
  if (sms <= 0) return KIVI_ERR_CUDA;
  if (!workspace || ((uintptr_t)workspace & 15) || ws_bytes < workspace_bytes(c->dims, Hq, sms))
    return KIVI_ERR_WORKSPACE;
  return decode_launch(c, q, Hq, softmax_scale, out, workspace, ws_splits(c->dims, sms), sms,
                       stream, simt);
}

// ---- static scratch for kivi_decode_attention_noalloc ----------------------
// One fixed array per device.  It exists on a device once this file's device
// module is loaded there; under CUDA's lazy module loading (the default) that
// happens at the first use of the symbol, i.e. the first
// cudaGetSymbolAddress below, which also reserves the array's 4 MiB.  So that
// this happens early, at a point the caller controls, every call that
// launches work (prefill, append, decode of any kind) resolves the address on
// its device first (touch_noalloc_scratch); a caller that later reserves the
// whole device for its own pool has the array already.  Host code must not
// use the symbol itself as a device address: its device address is looked up
// once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[KIVI_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::atomic<void*> g_noalloc_ptr[kMaxDevices];

int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KIVI_ERR_CUDA;
  void* p = g_noalloc_ptr[dev].load();
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return KIVI_ERR_CUDA;
    }
    g_noalloc_ptr[dev].store(p);
  }
  *out = p;
  return KIVI_OK;
}

// Resolve the scratch on the current device if not done yet (best effort:
// a failure here is reported by the no-allocation call itself).
void touch_noalloc_scratch() {
  void* p = nullptr;
  (void)noalloc_scratch(&p);
}

}  // namespace

extern "C" {

int kivi_buffer_sizes(const kivi_dims* dims, size_t out_bytes[KIVI_NUM_BUFFERS]) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!out_bytes) return KIVI_ERR_ARG;
  const long long units = (long long)dims->B * dims->Hkv;
  const long long Tq = dims->capacity - dims->R;
  // E codes per block of WB words: 32/b in one word, or 32 as three bit planes at 3 bits
  const int E = dims->bits == 3 ? 32 : 32 / dims->bits;
  const int WB = dims->bits == 3 ? 3 : 1;
  const size_t f = meta_bytes(dims->meta);
  out_bytes[KIVI_BUF_K_CODES] = (size_t)(units * Tq * (dims->D / E) * WB) * sizeof(uint32_t);
  out_bytes[KIVI_BUF_K_SCALE] = (size_t)(units * (Tq / dims->G) * dims->D) * f;
  out_bytes[KIVI_BUF_K_ZERO] = out_bytes[KIVI_BUF_K_SCALE];
  out_bytes[KIVI_BUF_V_CODES] = (size_t)(units * (Tq / E) * WB * dims->D) * sizeof(uint32_t);
  out_bytes[KIVI_BUF_V_SCALE] = (size_t)(units * Tq * (dims->D / dims->Gv)) * f;
  out_bytes[KIVI_BUF_V_ZERO] = out_bytes[KIVI_BUF_V_SCALE];
  out_bytes[KIVI_BUF_K_RES] = (size_t)(units * dims->R * dims->D) * elem_bytes(dims->dtype);
  out_bytes[KIVI_BUF_V_RES] = out_bytes[KIVI_BUF_K_RES];
  return KIVI_OK;
}

int kivi_cache_init(kivi_cache* cache, const kivi_dims* dims,
                    void* const buffers[KIVI_NUM_BUFFERS]) {
  if (!cache || !buffers) return KIVI_ERR_ARG;
  int rc = check_dims(dims);
  if (rc) return rc;
  const bool has_store = dims->capacity > dims->R;
  for (int i = 0; i < KIVI_NUM_BUFFERS; ++i) {
    const bool needed = has_store || i == KIVI_BUF_K_RES || i == KIVI_BUF_V_RES;
    if (needed && !buffers[i]) return KIVI_ERR_ARG;
    if (((uintptr_t)buffers[i] & 15) != 0) return KIVI_ERR_ARG;
  }
  cache->dims = *dims;
  cache->k_codes = (uint32_t*)buffers[KIVI_BUF_K_CODES];
  cache->k_scale = buffers[KIVI_BUF_K_SCALE];
  cache->k_zero = buffers[KIVI_BUF_K_ZERO];
  cache->v_codes = (uint32_t*)buffers[KIVI_BUF_V_CODES];
  cache->v_scale = buffers[KIVI_BUF_V_SCALE];
  cache->v_zero = buffers[KIVI_BUF_V_ZERO];
  cache->k_res = buffers[KIVI_BUF_K_RES];
  cache->v_res = buffers[KIVI_BUF_V_RES];
  cache->n_q = 0;
  cache->r = 0;
  cache->block_table = nullptr;
  cache->pages_per_seq = 0;
  cache->num_pages = 0;
  cache->k_out_idx = nullptr;
  cache->k_out_val = nullptr;
  cache->v_out_idx = nullptr;
  cache->v_out_val = nullptr;
  return KIVI_OK;
}

int kivi_outlier_buffer_sizes(const kivi_dims* dims, size_t out_bytes[4]) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!out_bytes) return KIVI_ERR_ARG;
  const long long units = (long long)dims->B * dims->Hkv;
  const long long Tq = dims->capacity - dims->R;
  out_bytes[0] = (size_t)(units * (Tq / dims->G) * dims->D * dims->k_out) * 4;
  out_bytes[1] = out_bytes[0];
  out_bytes[2] = (size_t)(units * Tq * (dims->D / dims->Gv) * dims->v_out) * 4;
  out_bytes[3] = out_bytes[2];
  return KIVI_OK;
}

int kivi_cache_set_outliers(kivi_cache* cache, void* const buffers[4]) {
  if (!cache || !buffers) return KIVI_ERR_ARG;
  int rc = check_dims(&cache->dims);
  if (rc) return rc;
  if (!sparse(cache->dims) || cache->block_table) return KIVI_ERR_UNSUPPORTED;
  if (cache->n_q != 0 || cache->r != 0) return KIVI_ERR_STATE;
  const bool has_store = cache->dims.capacity > cache->dims.R;
  for (int i = 0; i < 4; ++i) {
    const bool needed = has_store && (i < 2 ? cache->dims.k_out > 0 : cache->dims.v_out > 0);
    if (needed && !buffers[i]) return KIVI_ERR_ARG;
    if (((uintptr_t)buffers[i] & 15) != 0) return KIVI_ERR_ARG;
  }
  cache->k_out_idx = (int32_t*)buffers[0];
  cache->k_out_val = (float*)buffers[1];
  cache->v_out_idx = (int32_t*)buffers[2];
  cache->v_out_val = (float*)buffers[3];
  return KIVI_OK;
}

int kivi_paged_buffer_sizes(const kivi_dims* dims, long long num_pages,
                            size_t out_bytes[KIVI_NUM_BUFFERS]) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!out_bytes || num_pages < 1) return KIVI_ERR_ARG;
  // a pool of num_pages pages of R tokens is the contiguous layout of
  // num_pages * Hkv units of R tokens each; the windows are per sequence
  kivi_dims pool = *dims;
  pool.B = 1;
  pool.capacity = 2 * (long long)dims->R;  // Tq = R
  size_t one[KIVI_NUM_BUFFERS];
  rc = kivi_buffer_sizes(&pool, one);
  if (rc) return rc;
  for (int i = 0; i < KIVI_BUF_K_RES; ++i) out_bytes[i] = one[i] * (size_t)num_pages;
  const long long units = (long long)dims->B * dims->Hkv;
  out_bytes[KIVI_BUF_K_RES] = (size_t)(units * dims->R * dims->D) * elem_bytes(dims->dtype);
  out_bytes[KIVI_BUF_V_RES] = out_bytes[KIVI_BUF_K_RES];
  return KIVI_OK;
}

int kivi_paged_cache_init(kivi_cache* cache, const kivi_dims* dims,
                          void* const buffers[KIVI_NUM_BUFFERS], const int32_t* block_table,
                          int pages_per_seq, long long num_pages) {
  if (!cache || !buffers || !block_table || ((uintptr_t)block_table & 3)) return KIVI_ERR_ARG;
  int rc = check_dims(dims);
  if (rc) return rc;
  if (sparse(*dims)) return KIVI_ERR_UNSUPPORTED;  // outlier lists are per unit, not paged
  if (pages_per_seq < 1 || num_pages < 1 || num_pages > (long long)INT_MAX ||
      dims->capacity != ((long long)pages_per_seq + 1) * dims->R)
    return KIVI_ERR_ARG;
  for (int i = 0; i < KIVI_NUM_BUFFERS; ++i)
    if (!buffers[i] || ((uintptr_t)buffers[i] & 15) != 0) return KIVI_ERR_ARG;
  rc = kivi_cache_init(cache, dims, buffers);
  if (rc) return rc;
  cache->block_table = block_table;
  cache->pages_per_seq = pages_per_seq;
  cache->num_pages = num_pages;
  return KIVI_OK;
}

int kivi_quantize_prefill(kivi_cache* cache, const void* K, const void* V, long long T,
                          void* stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (T < 0 || (T > 0 && (!K || !V))) return KIVI_ERR_ARG;
  if (cache->n_q != 0 || cache->r != 0 || cache->block_table) return KIVI_ERR_STATE;
  if (T > cache->dims.capacity) return KIVI_ERR_CAPACITY;
  if (T == 0) return KIVI_OK;
  const int R = cache->dims.R;
  const int r = (int)((T - 1) % R) + 1;
  const long long n_q = T - r;
  if (n_q / kivi::kTile + 1 > (long long)INT_MAX) return KIVI_ERR_UNSUPPORTED;
  touch_noalloc_scratch();
  cudaError_t err = kivi::launch_prefill(view(cache), cache->dims.B * cache->dims.Hkv,
                                         cache->dims.D, cache->dims.bits, cache->dims.dtype, K,
                                         V, T, n_q, r, (cudaStream_t)stream);
  if (err != cudaSuccess) return KIVI_ERR_CUDA;
  cache->n_q = n_q;
  cache->r = r;
  return KIVI_OK;
}

int kivi_append_token(kivi_cache* cache, const void* k, const void* v, void* stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!k || !v) return KIVI_ERR_ARG;
  if (device_counted(cache)) return KIVI_ERR_STATE;
  if (cache->n_q + cache->r + 1 > cache->dims.capacity) return KIVI_ERR_CAPACITY;
  const bool flush = cache->r == cache->dims.R;
  const int slot = flush ? 0 : cache->r;
  touch_noalloc_scratch();
  cudaError_t err = kivi::launch_append(view(cache), cache->dims.B * cache->dims.Hkv,
                                        cache->dims.D, cache->dims.bits, cache->dims.dtype, k, v,
                                        cache->n_q, slot, flush, (cudaStream_t)stream);
  if (err != cudaSuccess) return KIVI_ERR_CUDA;
  if (flush) cache->n_q += cache->dims.R;
  cache->r = slot + 1;
  return KIVI_OK;
}

size_t kivi_decode_workspace_bytes(const kivi_cache* cache, int Hq) {
  if (check_cache(cache) != KIVI_OK || Hq <= 0 || Hq % cache->dims.Hkv != 0) return 0;
  const int sms = device_sms();
  if (sms <= 0) return 0;
  return workspace_bytes(cache->dims, Hq, sms);
}

int kivi_decode_attention(const kivi_cache* cache, const void* q, int Hq, float softmax_scale,
                          void* out, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_common(cache, q, Hq, softmax_scale, out, workspace, workspace_bytes, stream,
                       false);
}

// Staging layout of kivi_append_decode_host: k | v | q back to back (each a
// whole number of 16-byte chunks, since D * element size is), then out at the
// next 16-byte boundary.
size_t kivi_host_step_bytes(const kivi_cache* cache, int Hq) {
  if (check_cache(cache) != KIVI_OK || Hq <= 0 || Hq % cache->dims.Hkv != 0) return 0;
  const kivi_dims& d = cache->dims;
  const size_t es = d.dtype == KIVI_F16 ? 2 : 4;
  const size_t kv = (size_t)d.B * d.Hkv * d.D * es, qo = (size_t)d.B * Hq * d.D * es;
  const size_t in = (2 * kv + qo + 15) / 16 * 16;
  return in + (qo + 15) / 16 * 16;
}

int kivi_append_decode_host(kivi_cache* cache, const void* host_kvq, int Hq, float softmax_scale,
                            void* host_out, void* staging, size_t staging_bytes, void* workspace,
                            size_t ws_bytes, void* stream) {
  const size_t need = kivi_host_step_bytes(cache, Hq);
  if (need == 0 || !host_kvq || !host_out || !staging || ((uintptr_t)staging & 15))
    return KIVI_ERR_ARG;
  if (staging_bytes < need) return KIVI_ERR_WORKSPACE;
  // the refusals that need no device, before the copy (kivi_append_decode
  // checks everything again)
  if (device_counted(cache)) return KIVI_ERR_STATE;
  if (cache->n_q + cache->r + 1 > cache->dims.capacity) return KIVI_ERR_CAPACITY;
  const kivi_dims& d = cache->dims;
  const size_t es = d.dtype == KIVI_F16 ? 2 : 4;
  const size_t kv = (size_t)d.B * d.Hkv * d.D * es, qo = (size_t)d.B * Hq * d.D * es;
  unsigned char* st = static_cast<unsigned char*>(staging);
  unsigned char* out = st + (2 * kv + qo + 15) / 16 * 16;
  cudaStream_t s = (cudaStream_t)stream;
  // inputs in one copy, the fused step on them, out back in one copy
  if (cudaMemcpyAsync(st, host_kvq, 2 * kv + qo, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return KIVI_ERR_CUDA;
  const int rc = kivi_append_decode(cache, st, st + kv, st + 2 * kv, Hq, softmax_scale, out,
                                    workspace, ws_bytes, stream);
  if (rc != KIVI_OK) return rc;
  if (cudaMemcpyAsync(host_out, out, qo, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return KIVI_ERR_CUDA;
  return KIVI_OK;
}

int kivi_append_decode(kivi_cache* cache, const void* k, const void* v, const void* q, int Hq,
                       float softmax_scale, void* out, void* workspace, size_t ws_bytes,
                       void* stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!k || !v) return KIVI_ERR_ARG;
  if (device_counted(cache)) return KIVI_ERR_STATE;
  if (cache->n_q + cache->r + 1 > cache->dims.capacity) return KIVI_ERR_CAPACITY;
  // the decode half sees the cache with the new token in it
  kivi_cache after = *cache;
  if (after.r == after.dims.R) {
    after.n_q += after.dims.R;
    after.r = 1;
  } else {
    after.r += 1;
  }
  rc = decode_checks(&after, q, Hq, out);
  if (rc) return rc;
  const int sms = device_sms();
  if (sms <= 0) return KIVI_ERR_CUDA;
  if (!workspace || ((uintptr_t)workspace & 15) || ws_bytes < workspace_bytes(cache->dims, Hq, sms))
    return KIVI_ERR_WORKSPACE;
  // a token not 16-byte aligned (the kernel copies it in 16-byte pieces):
  // the append as its own launch, then decode
  if (((uintptr_t)k & 15) || ((uintptr_t)v & 15)) {
    rc = kivi_append_token(cache, k, v, stream);
    if (rc) return rc;
    return decode_launch(cache, q, Hq, softmax_scale, out, workspace, ws_splits(cache->dims, sms),
                         sms, stream, false);
  }
  // one launch: a due flush (full window) is quantized into the store by the
  // decode kernel itself before it reads the store; the token goes to window
  // slot r (slot 0 after a flush)
  const bool flush = cache->r == cache->dims.R;
  rc = decode_launch(&after, q, Hq, softmax_scale, out, workspace, ws_splits(cache->dims, sms), sms,
                     stream, false, k, v, flush ? 0 : cache->r, nullptr, false, false, flush);
  if (rc == KIVI_OK) {
    cache->n_q = after.n_q;
    cache->r = after.r;
  }
  return rc;
}

int kivi_dev_state_init(const kivi_cache* cache, void* state, void* stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!state || ((uintptr_t)state & 15)) return KIVI_ERR_ARG;
  if (device_counted(cache)) return KIVI_ERR_STATE;
  return kivi::launch_set_state((kivi::DevState*)state, cache->n_q, cache->r,
                                (cudaStream_t)stream) == cudaSuccess
             ? KIVI_OK
             : KIVI_ERR_CUDA;
}

int kivi_append_decode_dev(const kivi_cache* cache, void* state, const void* k, const void* v,
                           const void* q, int Hq, float softmax_scale, void* out,
                           void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!state || ((uintptr_t)state & 15) || !k || !v) return KIVI_ERR_ARG;
  if (device_counted(cache)) return KIVI_ERR_STATE;
  kivi_cache after = *cache;  // any post-append state passes the decode checks
  after.r = 1;
  rc = decode_checks(&after, q, Hq, out);
  if (rc) return rc;
  const int sms = device_sms();
  if (sms <= 0) return KIVI_ERR_CUDA;
  if (!workspace || ((uintptr_t)workspace & 15) || ws_bytes < workspace_bytes(cache->dims, Hq, sms))
    return KIVI_ERR_WORKSPACE;
  if (((uintptr_t)k & 15) || ((uintptr_t)v & 15)) {
    // a token not 16-byte aligned: the append as its own launch, then decode
    if (kivi::launch_append_dev(view(cache), cache->dims.B * cache->dims.Hkv, cache->dims.D,
                                cache->dims.bits, cache->dims.dtype, k, v,
                                (const kivi::DevState*)state, (cudaStream_t)stream) != cudaSuccess)
      return KIVI_ERR_CUDA;
    return decode_launch(&after, q, Hq, softmax_scale, out, workspace, ws_splits(cache->dims, sms),
                         sms, stream, false, nullptr, nullptr, 0, state);
  }
  // one launch: the decode kernel reads the counters, flushes a full window
  // into the store, writes the token into its window slot, decodes, and its
  // last CTA advances the counters
  return decode_launch(&after, q, Hq, softmax_scale, out, workspace, ws_splits(cache->dims, sms),
                       sms, stream, false, k, v, 0, state);
}

int kivi_ragged_prefill(kivi_cache* cache, void* state, const void* K, const void* V,
                        long long T_max, const long long* lens, void* stream) {
  int rc = check_cache(cache);
  if (rc) return rc;
  if (!state || ((uintptr_t)state & 15) || !K || !V || !lens || T_max < 1) return KIVI_ERR_ARG;
  if (cache->n_q != 0 || cache->r != 0) return KIVI_ERR_STATE;
  if (T_max / kivi::kTile + 1 > (long long)INT_MAX) return KIVI_ERR_UNSUPPORTED;
  touch_noalloc_scratch();
  cudaError_t err = kivi::launch_prefill_ragged(
      view(cache), cache->dims.B * cache->dims.Hkv, cache->dims.Hkv, cache->dims.D,
      cache->dims.bits, cache->dims.dtype, K, V, T_max, lens, (kivi::DevState*)state,
      (cudaStream_t)stream);
  if (err != cudaSuccess) return KIVI_ERR_CUDA;
  cache->n_q = kRaggedMark;
  cache->r = 0;
  return KIVI_OK;
}

int kivi_ragged_append(const kivi_cache* cache, void* state, const void* k, const void* v,
                       void* stream) {
  int sms = 0;
  int rc = ragged_checks(cache, state, nullptr, 0, nullptr, nullptr, 0, &sms);
  if (rc) return rc;
  if (!k || !v) return KIVI_ERR_ARG;
  const int units = cache->dims.B * cache->dims.Hkv;
  if (kivi::launch_append_ragged(view(cache), units, cache->dims.Hkv, cache->dims.D,
                                 cache->dims.bits, cache->dims.dtype, k, v,
                                 (const kivi::DevState*)state, (cudaStream_t)stream) != cudaSuccess)
    return KIVI_ERR_CUDA;
  return kivi::launch_advance_ragged((kivi::DevState*)state, cache->dims.B,
                                     cache->dims.capacity - cache->dims.R, cache->dims.R,
                                     (cudaStream_t)stream) == cudaSuccess
             ? KIVI_OK
             : KIVI_ERR_CUDA;
}

int kivi_ragged_decode(const kivi_cache* cache, const void* state, const void* q, int Hq,
                       float softmax_scale, void* out, void* workspace, size_t ws_bytes,
                       void* stream) {
  int sms = 0;
  int rc = ragged_checks(cache, state, q, Hq, out, workspace, ws_bytes, &sms);
  if (rc) return rc;
  kivi_cache any = *cache;  // host counters unused: every length is read on the device
  any.n_q = 0;
  any.r = 1;
  return decode_launch(&any, q, Hq, softmax_scale, out, workspace, ws_splits(cache->dims, sms),
                       sms, stream, false, nullptr, nullptr, 0, const_cast<void*>(state), true,
                       false);
}

int kivi_ragged_append_decode(const kivi_cache* cache, void* state, const void* k,
                              const void* v, const void* q, int Hq, float softmax_scale,
                              void* out, void* workspace, size_t ws_bytes, void* stream) {
  if (!k || !v) return KIVI_ERR_ARG;
  int sms = 0;
  int rc = ragged_checks(cache, state, q, Hq, out, workspace, ws_bytes, &sms);
  if (rc) return rc;
  const int units = cache->dims.B * cache->dims.Hkv;
  if (kivi::launch_append_ragged(view(cache), units, cache->dims.Hkv, cache->dims.D,
                                 cache->dims.bits, cache->dims.dtype, k, v,
                                 (const kivi::DevState*)state, (cudaStream_t)stream) != cudaSuccess)
    return KIVI_ERR_CUDA;
  kivi_cache any = *cache;
  any.n_q = 0;
  any.r = 1;
  return decode_launch(&any, q, Hq, softmax_scale, out, workspace, ws_splits(cache->dims, sms),
                       sms, stream, false, nullptr, nullptr, 0, state, true, true);
}

int kivi_decode_attention_simt(const kivi_cache* cache, const void* q, int Hq,
                               float softmax_scale, void* out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return decode_common(cache, q, Hq, softmax_scale, out, workspace, workspace_bytes, stream,
                       true);
}

int kivi_decode_attention_noalloc(const kivi_cache* cache, const void* q, int Hq,
                                  float softmax_scale, void* out, void* stream) {
  int rc = decode_checks(cache, q, Hq, out);
  if (rc) return rc;
  // the scratch holds the per-unit counters, then the partials of at most
  // `fit` splits
  const size_t per_split = (size_t)cache->dims.B * Hq * (cache->dims.D + 2) * sizeof(float);
  const size_t cbytes = counter_bytes(cache->dims);
  if (cbytes + per_split > KIVI_NOALLOC_SCRATCH_BYTES) return KIVI_ERR_SCRATCH_LIMIT;
  const int sms = device_sms();
  if (sms <= 0) return KIVI_ERR_CUDA;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  const long long fit = (long long)((KIVI_NOALLOC_SCRATCH_BYTES - cbytes) / per_split);
  const int cap = (int)(fit < ws_splits(cache->dims, sms) ? fit : ws_splits(cache->dims, sms));
  return decode_launch(cache, q, Hq, softmax_scale, out, scratch, cap, sms, stream, false);
}

void kivi_set_timing_events(void* start_event, void* stop_event) {
  g_ev0 = (cudaEvent_t)start_event;
  g_ev1 = (cudaEvent_t)stop_event;
}

int kivi_decode_num_splits(const kivi_cache* cache, int Hq) {
  if (check_cache(cache) != KIVI_OK || Hq <= 0 || Hq % cache->dims.Hkv != 0) return 0;
  if (device_counted(cache)) return 0;
  if (cache->n_q + cache->r == 0) return 0;
  const int sms = device_sms();
  if (sms <= 0) return 0;
  DecodeArgs a;
  a.D = cache->dims.D;
  a.bits = cache->dims.bits;
  a.gq = Hq / cache->dims.Hkv;
  a.dtype = cache->dims.dtype;
  a.meta = cache->dims.meta;
  int occ = 0;
  if (kivi::decode_tc_ctas_per_sm(a, &occ) != cudaSuccess) return 0;
  StreamPlan sp;
  plan_stream(cache, sms, occ, ws_splits(cache->dims, sms), &sp);
  return sp.max_seg;
}

const char* kivi_status_string(int status) {
  switch (status) {
    case KIVI_OK: return "KIVI_OK";
    case KIVI_ERR_ARG: return "KIVI_ERR_ARG: invalid argument";
    case KIVI_ERR_UNSUPPORTED: return "KIVI_ERR_UNSUPPORTED: shape or format not built";
    case KIVI_ERR_STATE: return "KIVI_ERR_STATE: cache state does not allow this call";
    case KIVI_ERR_CAPACITY: return "KIVI_ERR_CAPACITY: tokens exceed the cache capacity";
    case KIVI_ERR_WORKSPACE: return "KIVI_ERR_WORKSPACE: workspace missing, small or misaligned";
    case KIVI_ERR_CUDA: return "KIVI_ERR_CUDA: CUDA launch or query failed";
    case KIVI_ERR_SCRATCH_LIMIT:
      return "KIVI_ERR_SCRATCH_LIMIT: request exceeds the fixed scratch of the no-allocation call";
  }
  return "unknown kivi status";
}

}  // extern "C"
