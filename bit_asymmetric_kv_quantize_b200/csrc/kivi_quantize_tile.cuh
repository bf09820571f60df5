// kivi_quantize_tile.cuh -- quantization of one 32-token tile of one unit
// into the KIVI store, shared by the prefill / append kernels and the decode
// kernel (which folds a due window flush into its launch).
//
// Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache".
// Keys are quantized per channel over the tile's tokens and values per token
// over groups of kGv channels (mlsanity.com index page, "Abstract (arXiv)";
// study.space summary: key groups span tokens), each group with an
// asymmetric scale and zero (study.space summary).
#pragma once

#include <type_traits>

#include "kivi_codes.cuh"
#include "kivi_internal.cuh"
#include "kivi_sparse.cuh"

namespace kivi {
namespace {

template <int D, int BAR>
__device__ __forceinline__ void tile_sync() {
  if constexpr (BAR == 0) {
    __syncthreads();
  } else {
    asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(D) : "memory");
  }
}

// Quantize one tile of kTile tokens (= one key group) of one unit.
//   Ksrc, Vsrc: the tile's first token row; rows are D elements apart.
//   t0: token position of the tile in the quantized store (multiple of kTile).
// blockDim.x == D.  Thread d reduces key channel d over the tile's tokens;
// thread i reduces value group (token i / NJ, group i % NJ) over kGv channels.
// Codes go through shared memory (ck, cv: kTile * D bytes each) and are
// packed by the same threads.  BAR = 0: the block is exactly these D threads
// and synchronizes with __syncthreads; BAR > 0: threads 0 .. D-1 of a larger
// block call this and synchronize on named barrier BAR (the others must not).
// Paged stores: the tile goes to its page's slot (a page outside the block
// table or the pool writes nothing; the callers have refused such a
// sequence already).  REG: outlier-list groups take quantize_group_sparse_reg
// (same output, the group kept in registers) instead of quantize_group_sparse.
template <int D, int BITS, typename T, typename M, int BAR, bool REG = false>
__device__ __forceinline__ void quantize_tile(const CacheView& c, long long unit,
                                              const T* __restrict__ Ksrc,
                                              const T* __restrict__ Vsrc, long long t0,
                                              uint8_t* ck, uint8_t* cv) {
  using Lt = Layout<D, BITS>;
  constexpr int E = Lt::E, WK = Lt::WK, NJ = Lt::NJ;
  const float Lf = (float)Lt::L;
  const int tid = threadIdx.x;
  const long long Ts = store_tokens(c);
  {
    long long su, stl;
    if (!store_tile(c, unit, t0 / kTile, &su, &stl)) return;  // same for the whole block
    unit = su;
    t0 = stl * kTile;
  }

  // ---- keys: channel tid over kTile tokens
  {
    float x[kTile];
#pragma unroll
    for (int t = 0; t < kTile; ++t) x[t] = to_f32(Ksrc[(long long)t * D + tid]);
    const long long g = t0 / kG;
    bool done = false;
    if constexpr (std::is_same<M, float>::value) {
      if (c.k_out > 0) {
        // dense-and-sparse variant: the group's k_out largest magnitudes are
        // kept exactly (listed in index order, dense code 0), the rest quantized
        float s, z, ov[kMaxOut];
        int codes[kTile], oi[kMaxOut];
        if constexpr (REG)
          quantize_group_sparse_reg<kTile, kMaxOut>(x, c.k_out, BITS, &s, &z, codes, oi, ov);
        else
          quantize_group_sparse<kTile, kMaxOut>(x, c.k_out, BITS, &s, &z, codes, oi, ov);
        c.k_scale_f()[unit * Lt::k_meta_unit(Ts) + g * D + tid] = s;
        c.k_zero_f()[unit * Lt::k_meta_unit(Ts) + g * D + tid] = z;
#pragma unroll
        for (int t = 0; t < kTile; ++t) ck[t * D + tid] = (uint8_t)codes[t];
        const long long lo = ((unit * (Ts / kG) + g) * D + tid) * c.k_out;
        for (int m = 0; m < c.k_out; ++m) {
          c.k_oi[lo + m] = oi[m];
          c.k_ov[lo + m] = ov[m];
        }
        done = true;
      }
    }
    if (!done) {
      float mn = x[0], mx = x[0];
#pragma unroll
      for (int t = 1; t < kTile; ++t) {
        if (x[t] < mn) mn = x[t];
        if (x[t] > mx) mx = x[t];
      }
      const float s = round_meta<M>(__fdiv_rn(__fsub_rn(mx, mn), Lf));
      const float z = round_meta<M>(mn);
      reinterpret_cast<M*>(c.k_scale)[unit * Lt::k_meta_unit(Ts) + g * D + tid] = from_f32<M>(s);
      reinterpret_cast<M*>(c.k_zero)[unit * Lt::k_meta_unit(Ts) + g * D + tid] = from_f32<M>(z);
      const float rs = recip_rn(s);
#pragma unroll
      for (int t = 0; t < kTile; ++t) {
        int code = 0;
        if (s != 0.0f) code = code_of(__fsub_rn(x[t], z), s, rs, Lt::L);
        ck[t * D + tid] = (uint8_t)code;
      }
    }
  }
  // ---- values: token tid / NJ, channel group tid % NJ
  {
    const int t = tid / NJ, j = tid % NJ;
    const T* src = Vsrc + (long long)t * D + j * kGv;
    float x[kGv];
#pragma unroll
    for (int i = 0; i < kGv; ++i) x[i] = to_f32(src[i]);
    const long long mo = unit * Lt::v_meta_unit(Ts) + (t0 + t) * NJ + j;
    bool done = false;
    if constexpr (std::is_same<M, float>::value) {
      if (c.v_out > 0) {
        float s, z, ov[kMaxOut];
        int codes[kGv], oi[kMaxOut];
        if constexpr (REG)
          quantize_group_sparse_reg<kGv, kMaxOut>(x, c.v_out, BITS, &s, &z, codes, oi, ov);
        else
          quantize_group_sparse<kGv, kMaxOut>(x, c.v_out, BITS, &s, &z, codes, oi, ov);
        c.v_scale_f()[mo] = s;
        c.v_zero_f()[mo] = z;
#pragma unroll
        for (int i = 0; i < kGv; ++i) cv[t * D + j * kGv + i] = (uint8_t)codes[i];
        const long long lo = mo * c.v_out;  // [unit][token][group][v_out]
        for (int m = 0; m < c.v_out; ++m) {
          c.v_oi[lo + m] = oi[m];
          c.v_ov[lo + m] = ov[m];
        }
        done = true;
      }
    }
    if (!done) {
      float mn = x[0], mx = x[0];
#pragma unroll
      for (int i = 1; i < kGv; ++i) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
      }
      const float s = round_meta<M>(__fdiv_rn(__fsub_rn(mx, mn), Lf));
      const float z = round_meta<M>(mn);
      reinterpret_cast<M*>(c.v_scale)[mo] = from_f32<M>(s);
      reinterpret_cast<M*>(c.v_zero)[mo] = from_f32<M>(z);
      const float rs = recip_rn(s);
#pragma unroll
      for (int i = 0; i < kGv; ++i) {
        int code = 0;
        if (s != 0.0f) code = code_of(__fsub_rn(x[i], z), s, rs, Lt::L);
        cv[t * D + j * kGv + i] = (uint8_t)code;
      }
    }
  }
  tile_sync<D, BAR>();
  // ---- pack: keys along channels, values along tokens; D*BITS words each
  constexpr int NW = kTile * WK;  // == (kTile / E) * WB * D == D * BITS
  uint32_t* kdst = c.k_codes + unit * Lt::k_codes_unit(Ts) + t0 * WK;
  uint32_t* vdst = c.v_codes + unit * Lt::v_codes_unit(Ts) + (t0 / E) * Lt::WB * D;
  if constexpr (BITS == 3) {
    // bit planes: lane i of a warp holds code i of a block; plane p is the
    // ballot of bit p (bit i of the word = bit p of code i)
    const int lane = tid & 31, wp = tid >> 5;
    constexpr int NWP = D / 32;  // warps
    for (int pb = wp; pb < kTile * (D / 32); pb += NWP) {  // keys: (token, block)
      const int t = pb / (D / 32), w = pb % (D / 32);
      const uint32_t cd = ck[t * D + w * 32 + lane];
      const uint32_t p0 = __ballot_sync(0xffffffffu, cd & 1u);
      const uint32_t p1 = __ballot_sync(0xffffffffu, cd & 2u);
      const uint32_t p2 = __ballot_sync(0xffffffffu, cd & 4u);
      if (lane < 3) kdst[t * WK + 3 * w + lane] = lane == 0 ? p0 : (lane == 1 ? p1 : p2);
    }
    for (int d = wp; d < D; d += NWP) {  // values: channel d, the tile's 32 tokens
      const uint32_t cd = cv[lane * D + d];
      const uint32_t p0 = __ballot_sync(0xffffffffu, cd & 1u);
      const uint32_t p1 = __ballot_sync(0xffffffffu, cd & 2u);
      const uint32_t p2 = __ballot_sync(0xffffffffu, cd & 4u);
      if (lane < 3) vdst[lane * D + d] = lane == 0 ? p0 : (lane == 1 ? p1 : p2);
    }
  } else {
#pragma unroll
    for (int k = tid; k < NW; k += D) {
      const int t = k / WK, w = k % WK;
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < E; ++i) word |= (uint32_t)ck[t * D + w * E + i] << (BITS * i);
      kdst[k] = word;
    }
#pragma unroll
    for (int k = tid; k < NW; k += D) {
      const int tb = k / D, d = k % D;
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < E; ++i) word |= (uint32_t)cv[(tb * E + i) * D + d] << (BITS * i);
      vdst[k] = word;
    }
  }
  tile_sync<D, BAR>();
}

}  // namespace
}  // namespace kivi
