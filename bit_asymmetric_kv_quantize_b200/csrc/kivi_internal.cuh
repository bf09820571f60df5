// kivi_internal.cuh -- device-side view of a KIVI cache and small helpers
// shared by the kernels of libkivi.so (not part of the public ABI).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kivi {

constexpr int kG = 32;        // key group: tokens per (group, channel) scale
constexpr int kGv = 32;       // value group: channels per (token, group) scale
constexpr int kTile = 32;     // tokens per quantize tile (= kG, a multiple of E)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxOut = 4;    // dense-and-sparse variant: kept entries per group, at most

// Device view of one cache; per-unit strides follow the ABI layout.  The
// scales and zeros are binary32 (meta 0) or binary16 (meta 1) elements.
struct CacheView {
  uint32_t* k_codes;
  void* k_scale;
  void* k_zero;
  uint32_t* v_codes;
  void* v_scale;
  void* v_zero;
  void* k_res;
  void* v_res;
  long long Tq;  // quantized-store capacity per unit, tokens
  int R;         // residual window
  int meta;      // 0: binary32 scales and zeros, 1: binary16
  // paged store (bt != null): the quantized store of sequence b is pages of
  // R tokens, page l at pool slot bt[b * pps + l]; the arrays hold n_pages
  // slots of Hkv units of R tokens (contiguous stores: bt null, a unit's
  // arrays span Tq tokens)
  const int* bt;
  int pps;
  long long n_pages;
  int Hkv;
  // dense-and-sparse variant: entries kept exactly per key / value group
  // (0: none) and their lists, [unit][Tq/G][D][k_out] and [unit][Tq][D/Gv][v_out]
  int k_out;
  int v_out;
  int* k_oi;
  float* k_ov;
  int* v_oi;
  float* v_ov;
  __host__ __device__ float* k_scale_f() const { return static_cast<float*>(k_scale); }
  __host__ __device__ float* k_zero_f() const { return static_cast<float*>(k_zero); }
  __host__ __device__ float* v_scale_f() const { return static_cast<float*>(v_scale); }
  __host__ __device__ float* v_zero_f() const { return static_cast<float*>(v_zero); }
};

// Tokens per unit slot of the store arrays (the per-unit stride).
__host__ __device__ inline long long store_tokens(const CacheView& c) {
  return c.bt ? (long long)c.R : c.Tq;
}
// Slot of 32-token tile t of unit u in the store arrays: the array unit su
// and the tile st within it.  Paged: the sequence's page t / (R/32) through
// the block table; false when that page is past the table or its id outside
// the pool (nothing may be read or written then).
__host__ __device__ inline bool store_tile(const CacheView& c, long long u, long long t,
                                           long long* su, long long* st) {
  if (c.bt == nullptr) {
    *su = u;
    *st = t;
    return true;
  }
  const long long tpp = c.R / kTile;
  const long long lp = t / tpp;
  if (t < 0 || lp >= c.pps) return false;
  const long long b = u / c.Hkv;
  const long long pg = c.bt[b * c.pps + lp];
  if (pg < 0 || pg >= c.n_pages) return false;
  *su = pg * c.Hkv + u % c.Hkv;
  *st = t % tpp;
  return true;
}

// Codes come in blocks of E codes held in WB 32-bit words: E = 32/b codes
// in one word (code i at bits [b i, b i + b)) for b = 1, 2, 4; at 3 bits,
// which do not divide 32, E = 32 codes as three bit planes (word p holds bit
// p of code i at bit i).  Keys: a token's blocks run along its channels;
// values: a channel's blocks run along tokens (block tb of channel d in
// rows tb*WB .. tb*WB + WB-1 of the [.][D] value-code array).
template <int D, int BITS>
struct Layout {
  static constexpr int E = BITS == 3 ? 32 : 32 / BITS;  // codes per block
  static constexpr int WB = BITS == 3 ? 3 : 1;          // words per block
  static constexpr int WK = D / E * WB;     // key words per token
  static constexpr int NJ = D / kGv;        // value groups per token
  static constexpr uint32_t MASK = (1u << BITS) - 1u;
  static constexpr int L = (1 << BITS) - 1;  // top code
  __host__ __device__ static long long k_codes_unit(long long Tq) { return Tq * WK; }
  __host__ __device__ static long long k_meta_unit(long long Tq) { return (Tq / kG) * D; }
  __host__ __device__ static long long v_codes_unit(long long Tq) { return (Tq / E) * WB * D; }
  __host__ __device__ static long long v_meta_unit(long long Tq) { return Tq * NJ; }
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

// A scale or zero as stored: binary32 unchanged, or rounded to binary16 (to
// nearest, ties to even; the format variant with binary16 metadata).
template <typename M>
__device__ __forceinline__ float round_meta(float x);
template <>
__device__ __forceinline__ float round_meta<float>(float x) { return x; }
template <>
__device__ __forceinline__ float round_meta<__half>(float x) {
  return __half2float(__float2half_rn(x));
}

// N consecutive scales or zeros (N in {1, 2, 4}) from an address aligned to
// N elements, widened to float.
template <int N>
__device__ __forceinline__ void load_meta(const float* p, float (&o)[N]) {
  if constexpr (N == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  } else if constexpr (N == 2) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    o[0] = v.x; o[1] = v.y;
  } else {
    o[0] = p[0];
  }
}
template <int N>
__device__ __forceinline__ void load_meta(const __half* p, float (&o)[N]) {
  if constexpr (N == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
    o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
  } else if constexpr (N == 2) {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(p));
    o[0] = a.x; o[1] = a.y;
  } else {
    o[0] = __half2float(p[0]);
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Launchers (host), implemented in the .cu files.  Each returns a
// cudaError_t from the launch.
cudaError_t launch_prefill(const CacheView& c, int units, int D, int bits, int dtype,
                           const void* K, const void* V, long long T, long long n_q, int r,
                           cudaStream_t s);
cudaError_t launch_append(const CacheView& c, int units, int D, int bits, int dtype,
                          const void* k, const void* v, long long n_q, int slot, bool flush,
                          cudaStream_t s);

// Device-resident counters of one cache (layout of kivi_dev_state).
struct DevState {
  long long n_q;
  int r;
  int status;  // 0, or 1 once an append found no room (nothing written)
};
// Append reading (n_q, r) from `st` on the device (flush when r == R);
// the counters themselves are advanced by the decode that follows.
cudaError_t launch_append_dev(const CacheView& c, int units, int D, int bits, int dtype,
                              const void* k, const void* v, const DevState* st, cudaStream_t s);
// Ragged batch: st holds one DevState per sequence (Hkv units each); every
// sequence appends one token and flushes on its own when its r == R.
cudaError_t launch_append_ragged(const CacheView& c, int units, int Hkv, int D, int bits,
                                 int dtype, const void* k, const void* v, const DevState* st,
                                 cudaStream_t s);
// After launch_append_ragged: advance the B sequences that took their token.
cudaError_t launch_advance_ragged(DevState* st, long long B, long long Tq, int R, cudaStream_t s);
// Ragged prefill: K, V [units][T_max][D]; sequence b has lens[b] tokens
// (device); writes st[b] = {n_q, r, 0}, or {0, 0, 1} for a length outside
// [1, capacity] (nothing else written for it).
cudaError_t launch_prefill_ragged(const CacheView& c, int units, int Hkv, int D, int bits,
                                  int dtype, const void* K, const void* V, long long T_max,
                                  const long long* lens, DevState* st, cudaStream_t s);
cudaError_t launch_set_state(DevState* st, long long n_q, int r, cudaStream_t s);

// ---- stream-K plan of the tensor-core decode (host and device) -----------
// Every unit is laid out as n_q/32 work indices (its quantized tiles)
// followed by kWinWeight * ceil(r/32) + kMergeWeight indices standing for its
// residual window and its end-of-unit merge; the units' indices end to end
// are cut into equal ranges of W >= 12, one per CTA.  Measured on B200
// (per-CTA timelines): a 32-token window tile costs about two quantized tiles
// (fp16, tensor cores) or three (fp32, CUDA cores) and the end of a unit
// segment (partial write, arrival, merge) about eight, so a CTA whose range
// crosses a unit boundary gets correspondingly fewer tiles.
constexpr int kWinWeight = 3;     // fp32 window tile, CUDA cores
constexpr int kWinWeightF16 = 2;  // fp16 window tile, tensor cores
constexpr int kMergeWeight = 8;   // one unit end
struct StreamPlan {
  int n_cta;
  long long W;
  int max_seg;
  int win_weight;
};
// P: CTAs that run at once; seg_cap: partial slots per unit in the workspace.
__host__ __device__ inline StreamPlan plan_stream_core(long long units, long long n_q, int r,
                                                       bool f16, long long P, int seg_cap) {
  StreamPlan p;
  const long long n_qt = n_q / kTile;
  const int wtw = f16 ? kWinWeightF16 : kWinWeight;
  const int ww = (r > 0 ? wtw * (int)((r + kTile - 1) / kTile) : 1) + kMergeWeight;
  const long long UP = n_qt + ww;
  const long long total = units * UP;
  long long W = (total + P - 1) / P;
  if (W < 12) W = 12;  // at least one full stage per CTA
  if (seg_cap <= 1) {
    W = UP;  // one CTA per unit: ranges align with the units
  } else if ((n_qt + 1 + W - 1) / W + 1 > seg_cap) {
    W = (n_qt + 1 + seg_cap - 2) / (seg_cap - 1);
  }
  p.W = W;
  p.win_weight = ww;
  p.n_cta = (int)((total + W - 1) / W);
  p.max_seg = (W % UP == 0) ? 1 : (int)((n_qt + 1 + W - 1) / W + 1);
  return p;
}

// ---- ragged batches: per-sequence lengths in device memory ---------------
// Lengths (n_q, r) of one sequence as a decode sees them: after the append
// that the same step made when `pending`, else as stored.  ok = false for a
// sequence the append refused (status set) or whose counters are not a valid
// fill of the cache; such a sequence is decoded as empty (NaN output).
struct SeqLen {
  long long n_q;
  int r;
  bool ok;
};
__host__ __device__ inline SeqLen seq_len(const DevState& s, bool pending, long long Tq, int R) {
  SeqLen o;
  o.n_q = 0;
  o.r = 0;
  o.ok = false;
  if (s.status != 0 || s.n_q < 0 || s.n_q > Tq || s.n_q % R != 0 || s.r < 0 || s.r > R) return o;
  if (pending) {
    if (s.n_q + s.r + 1 > Tq + R) return o;
    const bool fl = s.r == R;
    o.n_q = fl ? s.n_q + R : s.n_q;
    o.r = fl ? 1 : s.r + 1;
  } else {
    o.n_q = s.n_q;
    o.r = s.r;
  }
  o.ok = true;
  return o;
}
// Work indices of one unit in the stream-K plan (as plan_stream_core).
__host__ __device__ inline long long unit_work(long long n_q, int r, bool f16) {
  const int wtw = f16 ? kWinWeightF16 : kWinWeight;
  return n_q / kTile + (r > 0 ? wtw * (int)((r + kTile - 1) / kTile) : 1) + kMergeWeight;
}
// Stream-K range length W for a ragged batch: total work indices over P
// CTAs, at least 12, and long enough that no unit of n_qt_max tiles spans
// more than seg_cap CTA segments (seg_cap >= 2).  Returns W; *max_seg gets
// the segment bound floor(n_qt_max / W) + 2.
__host__ __device__ inline long long plan_ragged_w(long long total, long long n_qt_max, long long P,
                                                   int seg_cap, int* max_seg) {
  long long W = (total + P - 1) / P;
  if (W < 12) W = 12;
  if ((n_qt_max + 1 + W - 1) / W + 1 > seg_cap) W = (n_qt_max + 1 + seg_cap - 2) / (seg_cap - 1);
  *max_seg = (int)((n_qt_max + 1 + W - 1) / W + 1);
  return W;
}

struct DecodeArgs {
  CacheView c;
  const void* q;   // [B][Hq][D]
  void* out;       // [B][Hq][D]
  float* ws;       // partials [B*Hq][n_split][D + 2]
  int units;       // B * Hkv
  int Hkv;
  int gq;          // Hq / Hkv
  int D;
  int bits;
  int dtype;
  int meta;        // element type of the scales and zeros (as CacheView::meta)
  long long n_q;
  int r;
  float qscale;    // softmax_scale * log2(e)
  int n_split;          // splits per unit (the tensor-core kernel's last one
                        // holds only the residual window when r > 0)
  int tiles_per_split;  // 32-token quantized tiles per split
  unsigned long long* ctr;  // per-unit arrival counters (in the workspace)
  unsigned int epoch;       // tag of this call in the counters (never 0)
  // tensor-core kernel (persistent, stream-K): each unit occupies
  // n_q/32 + win_weight consecutive work indices (its quantized tiles, then
  // its residual window weighted as win_weight tiles); CTA c owns indices
  // [c * tiles_per_cta, (c + 1) * tiles_per_cta); partials are
  // [units][max_seg][GQ][D + 2]
  int n_cta;
  long long tiles_per_cta;
  int max_seg;
  int win_weight;
  // fused append (tensor-core kernel only): when new_k is non-null the call
  // first writes token new_k/new_v ([B][Hkv][D]) into window slot new_slot
  // (r above already counts it)
  const void* new_k;
  const void* new_v;
  int new_slot;
  // device-counter mode (tensor-core kernel): when dev_state is non-null the
  // kernel reads (n_q, r) before the append from it, decodes over the cache
  // after the append (which an earlier launch performed), plans the split on
  // the device over its gridDim.x CTAs with seg_cap partial slots, writes
  // the new counters back, and counts arrivals in self-resetting counters
  // (the workspace's counter block must start zeroed)
  DevState* dev_state;
  int seg_cap;
  // ragged batch (tensor-core kernel, device-counter mode): dev_state holds
  // one DevState per sequence (units / Hkv of them); the plan follows each
  // sequence's own lengths, and when `pending` the state is the one before
  // this step's append and the last CTA advances every valid sequence
  int ragged;
  int pending;
  // uniform batches, fused append (new_k set): the window is full and is
  // quantized into the store by this launch before the decode reads it (the
  // host sets it; in device-counter mode the kernel decides from the
  // counters).  n_q above already counts the flushed tokens.
  int flush;
};

constexpr float kNaN = __builtin_nanf("");

// Arrival of one CTA at a unit's counter: a 64-bit word holding the call's
// epoch in the high half and the arrivals in the low half; a counter left by
// an earlier call is restarted, so no zeroing is needed.  One thread calls
// this after a CTA barrier that follows the CTA's partial writes: the
// compare-and-swap is acquire-release at GPU scope, so those writes are
// visible to the CTA that arrives last, and after its next CTA barrier that
// CTA sees every earlier arrival's partials.  Lock-free, bounded retries.
// Returns 1 for the n-th arrival, 0 for an earlier one, -1 if retries ran out.
__device__ __forceinline__ int arrive_unit(unsigned long long* ctr, unsigned int epoch,
                                           long long n) {
  const unsigned long long ep = (unsigned long long)epoch << 32;
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ctr) : "memory");
  for (int it = 0; it < 4096; ++it) {
    const unsigned long long nv = ((v >> 32) == epoch) ? v + 1ull : (ep | 1ull);
    unsigned long long old;
    asm volatile("atom.acq_rel.gpu.global.cas.b64 %0, [%1], %2, %3;"
                 : "=l"(old)
                 : "l"(ctr), "l"(v), "l"(nv)
                 : "memory");
    if (old == v) return ((long long)(nv & 0xffffffffull) == n) ? 1 : 0;
    v = old;
  }
  return -1;
}

// Merge of one output element over a unit's n partials P_s = (m_s, l_s,
// acc_s[D]) (P_s at P0 + s * stride): sum_s 2^(m_s - M) acc_s[d] /
// sum_s 2^(m_s - M) l_s with M = max_s m_s.  The partials are read in
// batches of 8 whose loads are all issued before any is used (one L2 round
// trip per batch); empty partials (m_s = -inf) are skipped.
__device__ __forceinline__ float merge_partials(const float* P0, long long stride, int n, int d) {
  constexpr int kB = 8;
  float M = -__builtin_huge_valf(), num = 0.f, den = 0.f;
  for (int s0 = 0; s0 < n; s0 += kB) {
    float m[kB], l[kB], v[kB];
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      m[k] = -__builtin_huge_valf();
      l[k] = 0.f;
      v[k] = 0.f;
      if (s0 + k < n) {
        const float* P = P0 + (long long)(s0 + k) * stride;
        m[k] = __ldcg(P);
        l[k] = __ldcg(P + 1);
        v[k] = __ldcg(P + 2 + d);
      }
    }
    float Mb = M;
#pragma unroll
    for (int k = 0; k < kB; ++k) Mb = fmaxf(Mb, m[k]);
    if (Mb == -__builtin_huge_valf()) continue;
    const float sc = exp2f(M - Mb);  // 0 while M = -inf
    num *= sc;
    den *= sc;
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      if (m[k] == -__builtin_huge_valf()) continue;
      const float e = exp2f(m[k] - Mb);
      num = fmaf(e, v[k], num);
      den = fmaf(e, l[k], den);
    }
    M = Mb;
  }
  return num / den;
}

// Arrival at a counter that starts at zero and is reset to zero by the n-th
// arrival (device-counter mode, where launches replay with the same
// arguments and cannot tag counters with a per-call epoch).  Same memory
// ordering as arrive_unit.  Returns 1 for the n-th arrival, else 0.
__device__ __forceinline__ int arrive_unit_reset(unsigned long long* ctr, long long n) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], 1;" : "=l"(old) : "l"(ctr) : "memory");
  if ((long long)old + 1 != n) return 0;
  asm volatile("st.relaxed.gpu.global.u64 [%0], 0;" ::"l"(ctr) : "memory");
  return 1;
}

// Grid-wide barrier of one launch whose CTAs are all resident at once (the
// persistent decode grid): thread 0 of each of the n CTAs arrives at *ctr and
// waits (acquire, bounded by ~2 s of clock cycles) until all have.  epoch != 0:
// the word carries the call's epoch in its high half, like arrive_unit, so a
// count left by an earlier call restarts: a CTA that finds a stale word tries
// once to swap in (epoch, 1); every other arrival is a fetch-and-add, since
// only this launch's CTAs write the word once it holds this epoch (hundreds
// of CTAs retrying compare-and-swaps on one word would serialize for many
// microseconds).  epoch == 0: a plain count that starts at zero and that the
// caller resets once every CTA is past it.  Returns false if the wait ran out.
__device__ __forceinline__ bool grid_barrier(unsigned long long* ctr, unsigned int epoch,
                                             long long n) {
  if (epoch != 0) {
    const unsigned long long ep = (unsigned long long)epoch << 32;
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ctr) : "memory");
    bool counted = false;
    for (int it = 0; it < 64 && (v >> 32) != epoch; ++it) {
      unsigned long long old;
      asm volatile("atom.acq_rel.gpu.global.cas.b64 %0, [%1], %2, %3;"
                   : "=l"(old)
                   : "l"(ctr), "l"(v), "l"(ep | 1ull)
                   : "memory");
      if (old == v) {
        counted = true;
        break;
      }
      v = old;
    }
    if (!counted) {
      if ((v >> 32) != epoch) return false;
      asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(ctr) : "memory");
    }
  } else {
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(ctr) : "memory");
  }
  const long long t0 = clock64();
  for (;;) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ctr) : "memory");
    const bool done = epoch != 0 ? ((v >> 32) == epoch && (long long)(v & 0xffffffffull) >= n)
                                 : (long long)v >= n;
    if (done) return true;
    if (clock64() - t0 > (1LL << 32)) return false;
    asm volatile("nanosleep.u32 64;" ::: "memory");
  }
}

// End of a split CTA, after it wrote its (m, l, acc[D]) partials: the last CTA
// of the unit to arrive merges all splits of the unit into out.
// out[b][kv*GQ + h][d] = sum_s 2^(m_s - M) acc_s[d] / sum_s 2^(m_s - M) l_s.
template <int D, int GQ, typename T>
__device__ __forceinline__ void finish_unit(const DecodeArgs& a, long long b, int kv,
                                            int* flag) {
  __syncthreads();
  if (threadIdx.x == 0) *flag = arrive_unit(a.ctr + (b * a.Hkv + kv), a.epoch, a.n_split);
  __syncthreads();
  const int last = *flag;
  if (last == 0) return;
  const int Hq = a.Hkv * GQ;
  T* out = reinterpret_cast<T*>(a.out);
  for (int idx = threadIdx.x; idx < GQ * D; idx += blockDim.x) {
    const int h = idx / D, d = idx % D;
    const long long row = b * Hq + (long long)kv * GQ + h;
    float res = kNaN;
    if (last > 0) res = merge_partials(a.ws + row * a.n_split * (D + 2), D + 2, a.n_split, d);
    out[row * D + d] = from_f32<T>(res);
  }
}

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t s, cudaEvent_t ev0,
                               cudaEvent_t ev1);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t s, cudaEvent_t ev0,
                             cudaEvent_t ev1);
// Resident CTAs per SM of the tensor-core kernel instance that `a` selects
// (uses a.D, a.bits, a.gq, a.dtype, a.meta).
cudaError_t decode_tc_ctas_per_sm(const DecodeArgs& a, int* ctas_per_sm);
// The tensor-core instances with binary16 scales and zeros (fp16 caches),
// and the ragged-batch instances (binary32, binary16 metadata); occ
// non-null: return the resident CTAs per SM instead of launching.
cudaError_t tc_dispatch_meta16(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                               cudaEvent_t e1, int* occ);
cudaError_t tc_dispatch_ragged(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                               cudaEvent_t e1, int* occ);
cudaError_t tc_dispatch_ragged_meta16(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                                      cudaEvent_t e1, int* occ);
// The dense-and-sparse instances (binary32 metadata; 1, 2, 4 bits).
cudaError_t tc_dispatch_sparse(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1,
                               int* occ);
// The 3-bit (bit-plane) instances, uniform and ragged batches.
cudaError_t tc_dispatch_3bit(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1,
                             int* occ);
cudaError_t tc_dispatch_3bit_ragged(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                                    cudaEvent_t e1, int* occ);

}  // namespace kivi
