// kivi_quantize.cu -- prefill, append and flush kernels of the KIVI cache.
//
// Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache".
// Keys are quantized per channel over groups of kG consecutive tokens and
// values per token over groups of kGv consecutive channels (mlsanity.com
// index page, "Abstract (arXiv)"; study.space summary: key groups span
// tokens).  Each group gets an asymmetric binary32 scale and zero
// (study.space summary: asymmetric quantizer).  Recent tokens stay in a
// full-precision window of R tokens that is quantized as a block when full
// (study.space summary: grouped and residual parts; scholarfeed.org "KIVI"
// page, third quote: fixed-length residual buffer).
//
// Bit-exactness: every group is reduced by one thread in element order with
// strict compares (first occurrence kept among equal values, which fixes the
// sign of a zero minimum); the scale uses the IEEE round-to-nearest
// intrinsics __fsub_rn / __fdiv_rn, and each code comes from code_of
// (kivi_codes.cuh): the product fl(d * fl(1/s)) decides the code when it lies
// more than 4e-6 from a half-integer, else the IEEE division __fdiv_rn does,
// rounded half to even (__float2int_rn) and clamped.  That equals
// clamp(round_half_even(fl(d / s)), 0, L) for every input (host build of the
// rule checked against true division in tests/test_code_rule.py).  No
// contraction.
//
// Format variant with binary16 scales and zeros (M = __half, fp16 caches):
// the binary32 scale and minimum are rounded to binary16 (nearest, ties to
// even) and the codes are chosen against the rounded pair, so that the
// stored scale and zero reproduce them as closely as the code grid allows.
#include "kivi_internal.cuh"
#include "kivi_quantize_tile.cuh"

namespace kivi {
namespace {

// (quantize_tile: kivi_quantize_tile.cuh; code_of and recip_rn: kivi_codes.cuh)

// grid (n_q / kTile + 1, units); the last x-block copies the r window tokens.
// Ragged (lens != null): grid (T_len / kTile + 1, units); sequence b = unit /
// Hkv has lens[b] tokens, split as r = ((lens - 1) mod R) + 1 and
// n_q = lens - r; the last x-block of the sequence's first unit writes st[b].
// A length outside [1, Tq + R] writes st[b] = {0, 0, 1} and nothing else.
template <int D, int BITS, typename T, typename M>
__global__ void __launch_bounds__(D) prefill_kernel(CacheView c, const T* __restrict__ K,
                                                    const T* __restrict__ V, long long T_len,
                                                    long long n_q, int r,
                                                    const long long* __restrict__ lens,
                                                    DevState* st, int Hkv) {
  __shared__ uint8_t ck[kTile * D];
  __shared__ uint8_t cv[kTile * D];
  const long long unit = blockIdx.y;
  const long long tile = blockIdx.x;
  const T* Ku = K + unit * T_len * D;
  const T* Vu = V + unit * T_len * D;
  if (lens != nullptr) {
    const long long b = unit / Hkv;
    const long long n = lens[b];
    bool ok = n >= 1 && n <= T_len && n <= c.Tq + c.R;
    r = ok ? (int)((n - 1) % c.R) + 1 : 0;
    n_q = ok ? n - r : 0;
    if (ok && c.bt != nullptr) {  // every page the prompt fills must be in the pool
      for (long long l = 0; l < n_q / c.R; ++l) {
        const int pg = c.bt[b * c.pps + l];
        ok = ok && pg >= 0 && pg < c.n_pages;
      }
      if (!ok) {
        r = 0;
        n_q = 0;
      }
    }
    if (tile == gridDim.x - 1 && unit == b * Hkv && threadIdx.x == 0) {
      DevState v;
      v.n_q = n_q;
      v.r = r;
      v.status = ok ? 0 : 1;
      st[b] = v;
    }
    if (!ok) return;
  }
  if (tile < n_q / kTile) {
    quantize_tile<D, BITS, T, M, 0>(c, unit, Ku + tile * kTile * D, Vu + tile * kTile * D,
                                 tile * kTile, ck, cv);
  } else if (tile == gridDim.x - 1) {
    T* kr = reinterpret_cast<T*>(c.k_res) + unit * c.R * D;
    T* vr = reinterpret_cast<T*>(c.v_res) + unit * c.R * D;
    for (int i = threadIdx.x; i < r * D; i += D) {
      kr[i] = Ku[n_q * D + i];
      vr[i] = Vu[n_q * D + i];
    }
  }
}

// grid (tiles, units) with tiles = R/32 when a flush may be due, else 1.
// If `flush`, block x quantizes window tile x (tokens 32x..32x+31) into store
// positions n_q + 32x..; block 0 then writes the new token into window
// `slot` (its own tile has been read by then).  Device mode (st != null):
// n_q and r come from st -- flush when r == R, slot = flush ? 0 : r -- and a
// full cache is left alone with st->status = 1.  Ragged (Hkv > 0): st holds
// one state per sequence b = unit / Hkv, each handled as above on its own.
template <int D, int BITS, typename T, typename M>
__global__ void __launch_bounds__(D) append_kernel(CacheView c, const T* __restrict__ k,
                                                   const T* __restrict__ v, long long n_q,
                                                   int slot, int flush, DevState* st, int Hkv) {
  __shared__ uint8_t ck[kTile * D];
  __shared__ uint8_t cv[kTile * D];
  if (st != nullptr) {
    const long long sb = Hkv > 0 ? (long long)blockIdx.y / Hkv : 0;
    DevState* ss = st + sb;
    const DevState s0 = *ss;
    const long long nq = s0.n_q;
    const int r = s0.r;
    // counters that are not a valid fill of the cache are refused too
    bool bad = s0.status != 0 || nq < 0 || nq > c.Tq || nq % c.R != 0 || r < 0 || r > c.R ||
               nq + r + 1 > c.Tq + c.R;
    if (!bad && c.bt != nullptr && r == c.R) {  // the flush fills page nq / R
      const long long pg = c.bt[sb * c.pps + nq / c.R];
      bad = pg < 0 || pg >= c.n_pages;
    }
    if (bad) {
      if (blockIdx.x == 0 && blockIdx.y == sb * (Hkv > 0 ? Hkv : 1) && threadIdx.x == 0)
        ss->status = 1;
      return;
    }
    flush = r == c.R;
    n_q = nq;
    slot = flush ? 0 : r;
  }
  const long long unit = blockIdx.y;
  const int tile = blockIdx.x;
  T* kr = reinterpret_cast<T*>(c.k_res) + unit * c.R * D;
  T* vr = reinterpret_cast<T*>(c.v_res) + unit * c.R * D;
  if (flush)
    quantize_tile<D, BITS, T, M, 0>(c, unit, kr + tile * kTile * D, vr + tile * kTile * D,
                                 n_q + tile * kTile, ck, cv);
  if (tile == 0) {
    kr[(long long)slot * D + threadIdx.x] = k[unit * D + threadIdx.x];
    vr[(long long)slot * D + threadIdx.x] = v[unit * D + threadIdx.x];
  }
}

__global__ void set_state_kernel(DevState* st, long long n_q, int r) {
  st->n_q = n_q;
  st->r = r;
  st->status = 0;
}

// After a ragged append launch: advance every sequence that took its token.
__global__ void advance_ragged_kernel(DevState* st, long long B, long long Tq, int R) {
  for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < B;
       b += (long long)gridDim.x * blockDim.x) {
    const SeqLen L = seq_len(st[b], true, Tq, R);
    if (L.ok) {
      st[b].n_q = L.n_q;
      st[b].r = L.r;
    }
  }
}

// lens != null: ragged prefill over T_len padded tokens per unit
template <int D, int BITS, typename T, typename M>
cudaError_t prefill_t(const CacheView& c, int units, const void* K, const void* V,
                      long long T_len, long long n_q, int r, const long long* lens, DevState* st,
                      int Hkv, cudaStream_t s) {
  dim3 grid((unsigned)((lens ? T_len : n_q) / kTile + 1), (unsigned)units);
  prefill_kernel<D, BITS, T, M><<<grid, D, 0, s>>>(c, (const T*)K, (const T*)V, T_len, n_q, r,
                                                   lens, st, Hkv);
  return cudaGetLastError();
}

template <int D, int BITS, typename T, typename M>
cudaError_t append_t(const CacheView& c, int units, const void* k, const void* v, long long n_q,
                     int slot, bool flush, DevState* st, int Hkv, cudaStream_t s) {
  const dim3 grid((unsigned)((flush || st) ? c.R / kTile : 1), (unsigned)units);
  append_kernel<D, BITS, T, M><<<grid, D, 0, s>>>(c, (const T*)k, (const T*)v, n_q, slot,
                                                  flush ? 1 : 0, st, Hkv);
  return cudaGetLastError();
}

template <int BITS, typename T, typename M>
cudaError_t prefill_d(int D, const CacheView& c, int units, const void* K, const void* V,
                      long long T_len, long long n_q, int r, const long long* lens, DevState* st,
                      int Hkv, cudaStream_t s) {
  switch (D) {
    case 32: return prefill_t<32, BITS, T, M>(c, units, K, V, T_len, n_q, r, lens, st, Hkv, s);
    case 64: return prefill_t<64, BITS, T, M>(c, units, K, V, T_len, n_q, r, lens, st, Hkv, s);
    case 128: return prefill_t<128, BITS, T, M>(c, units, K, V, T_len, n_q, r, lens, st, Hkv, s);
  }
  return cudaErrorInvalidValue;
}

template <int BITS, typename T, typename M>
cudaError_t append_d(int D, const CacheView& c, int units, const void* k, const void* v,
                     long long n_q, int slot, bool flush, DevState* st, int Hkv, cudaStream_t s) {
  switch (D) {
    case 32: return append_t<32, BITS, T, M>(c, units, k, v, n_q, slot, flush, st, Hkv, s);
    case 64: return append_t<64, BITS, T, M>(c, units, k, v, n_q, slot, flush, st, Hkv, s);
    case 128: return append_t<128, BITS, T, M>(c, units, k, v, n_q, slot, flush, st, Hkv, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t append_any(const CacheView& c, int units, int D, int bits, int dtype, const void* k,
                       const void* v, long long n_q, int slot, bool flush, DevState* st, int Hkv,
                       cudaStream_t s) {
  if (c.meta == 1) {  // binary16 scales and zeros: fp16 caches only
    if (dtype != 0) return cudaErrorInvalidValue;
    if (bits == 1) return append_d<1, __half, __half>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
    if (bits == 2) return append_d<2, __half, __half>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
    if (bits == 3) return append_d<3, __half, __half>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
    if (bits == 4) return append_d<4, __half, __half>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
    return cudaErrorInvalidValue;
  }
  if (c.meta != 0) return cudaErrorInvalidValue;
  if (bits == 1 && dtype == 0) return append_d<1, __half, float>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
  if (bits == 1 && dtype == 1) return append_d<1, float, float>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
  if (bits == 2 && dtype == 0) return append_d<2, __half, float>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
  if (bits == 3 && dtype == 0) return append_d<3, __half, float>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
  if (bits == 2 && dtype == 1) return append_d<2, float, float>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
  if (bits == 3 && dtype == 1) return append_d<3, float, float>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
  if (bits == 4 && dtype == 0) return append_d<4, __half, float>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
  if (bits == 4 && dtype == 1) return append_d<4, float, float>(D, c, units, k, v, n_q, slot, flush, st, Hkv, s);
  return cudaErrorInvalidValue;
}

cudaError_t prefill_any(const CacheView& c, int units, int D, int bits, int dtype, const void* K,
                        const void* V, long long T, long long n_q, int r, const long long* lens,
                        DevState* st, int Hkv, cudaStream_t s) {
  if (c.meta == 1) {  // binary16 scales and zeros: fp16 caches only
    if (dtype != 0) return cudaErrorInvalidValue;
    if (bits == 1) return prefill_d<1, __half, __half>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
    if (bits == 2) return prefill_d<2, __half, __half>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
    if (bits == 3) return prefill_d<3, __half, __half>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
    if (bits == 4) return prefill_d<4, __half, __half>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
    return cudaErrorInvalidValue;
  }
  if (c.meta != 0) return cudaErrorInvalidValue;
  if (bits == 1 && dtype == 0) return prefill_d<1, __half, float>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
  if (bits == 1 && dtype == 1) return prefill_d<1, float, float>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
  if (bits == 2 && dtype == 0) return prefill_d<2, __half, float>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
  if (bits == 3 && dtype == 0) return prefill_d<3, __half, float>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
  if (bits == 2 && dtype == 1) return prefill_d<2, float, float>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
  if (bits == 3 && dtype == 1) return prefill_d<3, float, float>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
  if (bits == 4 && dtype == 0) return prefill_d<4, __half, float>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
  if (bits == 4 && dtype == 1) return prefill_d<4, float, float>(D, c, units, K, V, T, n_q, r, lens, st, Hkv, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prefill(const CacheView& c, int units, int D, int bits, int dtype,
                           const void* K, const void* V, long long T, long long n_q, int r,
                           cudaStream_t s) {
  return prefill_any(c, units, D, bits, dtype, K, V, T, n_q, r, nullptr, nullptr, 0, s);
}

cudaError_t launch_prefill_ragged(const CacheView& c, int units, int Hkv, int D, int bits,
                                  int dtype, const void* K, const void* V, long long T_max,
                                  const long long* lens, DevState* st, cudaStream_t s) {
  return prefill_any(c, units, D, bits, dtype, K, V, T_max, 0, 0, lens, st, Hkv, s);
}

cudaError_t launch_append(const CacheView& c, int units, int D, int bits, int dtype,
                          const void* k, const void* v, long long n_q, int slot, bool flush,
                          cudaStream_t s) {
  return append_any(c, units, D, bits, dtype, k, v, n_q, slot, flush, nullptr, 0, s);
}

cudaError_t launch_append_dev(const CacheView& c, int units, int D, int bits, int dtype,
                              const void* k, const void* v, const DevState* st, cudaStream_t s) {
  return append_any(c, units, D, bits, dtype, k, v, 0, 0, false, const_cast<DevState*>(st), 0, s);
}

cudaError_t launch_append_ragged(const CacheView& c, int units, int Hkv, int D, int bits,
                                 int dtype, const void* k, const void* v, const DevState* st,
                                 cudaStream_t s) {
  return append_any(c, units, D, bits, dtype, k, v, 0, 0, false, const_cast<DevState*>(st), Hkv,
                    s);
}

cudaError_t launch_advance_ragged(DevState* st, long long B, long long Tq, int R,
                                  cudaStream_t s) {
  const long long blocks = (B + 255) / 256;
  advance_ragged_kernel<<<(unsigned)(blocks < 1024 ? blocks : 1024), 256, 0, s>>>(st, B, Tq, R);
  return cudaGetLastError();
}

cudaError_t launch_set_state(DevState* st, long long n_q, int r, cudaStream_t s) {
  set_state_kernel<<<1, 1, 0, s>>>(st, n_q, r);
  return cudaGetLastError();
}

}  // namespace kivi
