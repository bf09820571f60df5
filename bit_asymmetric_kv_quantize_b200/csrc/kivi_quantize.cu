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
// Bit-exactness: a group's min and max are those of a strict-compare scan in
// element order (first occurrence kept among equal values, which fixes the
// sign of a zero minimum): the general path scans so, the staged path takes
// order-free min/max and then gives a zero result the sign of the group's
// first zero.  The scale uses the IEEE round-to-nearest intrinsics
// __fsub_rn / __fdiv_rn.  Each code comes from code_of (kivi_codes.cuh: the
// product fl(d * fl(1/s)) decides the code when it lies more than 4e-6 from a
// half-integer, else the IEEE division does, rounded half to even and
// clamped), or in the staged path from code_bits, whose group check hands
// any such element to code_of.  Both equal clamp(round_half_even(fl(d / s)),
// 0, L) for every finite input (host builds of both rules checked against
// true division in tests/test_code_rule.py).  No contraction.
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

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}

// E consecutive byte codes (16-byte aligned, E = 32 / BITS) packed into one
// word, code i at bits [BITS i, BITS i + BITS).
template <int BITS>
__device__ __forceinline__ uint32_t pack_bytes(const uint8_t* p) {
  if constexpr (BITS == 2) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    auto c4 = [](uint32_t x) {  // 4 byte codes < 4 -> 8 bits
      x |= x >> 6;
      return (x | (x >> 12)) & 0xFFu;
    };
    return c4(u.x) | (c4(u.y) << 8) | (c4(u.z) << 16) | (c4(u.w) << 24);
  } else if constexpr (BITS == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    auto c4 = [](uint32_t x) {  // 4 byte codes < 16 -> 16 bits
      x = (x | (x >> 4)) & 0x00FF00FFu;
      return (x | (x >> 8)) & 0xFFFFu;
    };
    return c4(u.x) | (c4(u.y) << 16);
  } else {
    static_assert(BITS == 1, "bit widths 1, 2, 4");
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint4 b = *reinterpret_cast<const uint4*>(p + 16);
    // 4 byte codes < 2 -> 4 bits: byte i lands on bit 21 + i of the product
    auto c4 = [](uint32_t x) { return ((x * 0x204081u) >> 21) & 0xFu; };
    return c4(a.x) | (c4(a.y) << 4) | (c4(a.z) << 8) | (c4(a.w) << 12) | (c4(b.x) << 16) |
           (c4(b.y) << 20) | (c4(b.z) << 24) | (c4(b.w) << 28);
  }
}

// Smallest and largest of a group that the elementwise strict-compare scan
// (first occurrence kept) would return: min and max commute except for the
// sign of a zero result, which the first zero of the group in element order
// decides.  `at(i)` yields element i.
template <int N, typename F>
__device__ __forceinline__ void zero_sign_fix(float* mn, float* mx, F at) {
  if (*mn == 0.0f || *mx == 0.0f) {
    float fz = 0.0f;
    for (int i = 0; i < N; ++i) {
      const float v = at(i);
      if (v == 0.0f) {
        fz = v;
        break;
      }
    }
    if (*mn == 0.0f) *mn = fz;
    if (*mx == 0.0f) *mx = fz;
  }
}

// Sum over i < n of 0x4B400000 << (bits i), mod 2^32: what n code_bits
// encodings added at those shifts carry beyond the packed codes.
__host__ __device__ constexpr uint32_t code_bias(int bits, int n) {
  uint32_t b = 0;
  for (int i = 0; i < n && bits * i < 32; ++i) b += 0x4B400000u << (bits * i);
  return b;
}

// Two binary32 lanes per instruction (the packed .f32x2 arithmetic of
// sm_100), each lane rounded to nearest even like its scalar counterpart.
struct F2 {
  unsigned long long v;
};
__device__ __forceinline__ F2 f2(float a, float b) {
  F2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 un(F2 a) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(a.v));
  return r;
}
__device__ __forceinline__ F2 add2(F2 a, F2 b) {
  F2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ F2 sub2(F2 a, F2 b) {
  F2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ F2 mul2(F2 a, F2 b) {
  F2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}

// code_bits (kivi_codes.cuh) on two lanes: x - z, times rq, clamped to
// [0, L] where the zero is rounded (binary16 metadata: an element may lie
// below it, or a quotient above L); with binary32 metadata x >= z = the
// group minimum and q stays below L + 1e-6 for finite s and 1/s, so no clamp
// is needed.  Returns the sums' encodings (0x4B400000 + code per lane).
template <typename M>
__device__ __forceinline__ uint2 code_bits2(F2 x, F2 z, F2 rq, float Lf, float* ae) {
  const F2 kRound = f2(12582912.0f, 12582912.0f);
  F2 q = mul2(sub2(x, z), rq);
  if constexpr (!std::is_same<M, float>::value) {
    const float2 u = un(q);
    q = f2(fminf(fmaxf(u.x, 0.0f), Lf), fminf(fmaxf(u.y, 0.0f), Lf));
  }
  const F2 m = add2(q, kRound);
  const float2 e = un(sub2(q, sub2(m, kRound)));
  *ae = fmaxf(*ae, fmaxf(fabsf(e.x), fabsf(e.y)));
  const float2 mm = un(m);
  return make_uint2(__float_as_uint(mm.x), __float_as_uint(mm.y));
}

template <typename T>
__device__ __forceinline__ F2 load2(const T* p);  // two adjacent elements, widened
template <>
__device__ __forceinline__ F2 load2<__half>(const __half* p) {
  const __half2 h = *reinterpret_cast<const __half2*>(p);
  return f2(__low2float(h), __high2float(h));
}
template <>
__device__ __forceinline__ F2 load2<float>(const float* p) {
  const float2 h = *reinterpret_cast<const float2*>(p);
  return f2(h.x, h.y);
}

// Element (t, d) of a staged tile: half-precision tiles of D >= 64 channels
// keep tokens 16 .. 31 with the 32-element halves of each 64-element block
// swapped.
template <int D, typename T>
__device__ __forceinline__ int stage_idx(int t, int d) {
  return t * D + ((D >= 64 && sizeof(T) == 2) ? (d ^ (((t >> 4) & 1) << 5)) : d);
}

// Issue the asynchronous 16-byte copies of one tile of K and V (kTile rows of
// D elements from Ksrc, Vsrc, 16-byte aligned) into Ks, Vs (stage_idx order),
// as one group.
template <int D, typename T>
__device__ __forceinline__ void stage_tile(T* Ks, T* Vs, const T* __restrict__ Ksrc,
                                           const T* __restrict__ Vsrc) {
  constexpr int EPC = 16 / (int)sizeof(T);  // elements per 16-byte chunk
  constexpr int NCH = kTile * D / EPC;      // chunks per tile
#pragma unroll
  for (int i = threadIdx.x; i < NCH; i += D) {
    const int t = i / (D / EPC), d = (i % (D / EPC)) * EPC;
    cp_async16(Ks + stage_idx<D, T>(t, d), Ksrc + i * EPC);
    cp_async16(Vs + stage_idx<D, T>(t, d), Vsrc + i * EPC);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// One 32-token tile of one unit quantized from its staged copy (stage_tile,
// complete and visible to the block): the prefill's fast path (no outlier
// lists).  blockDim.x == D; vbad[0 .. NJ) must be 0 on entry.  Lane l of warp w
// owns channels d0 = 32 w + 2 (l % 16), d0 + 1 and tokens 16 (l / 16) ..
// + 15: it reduces its two key channels over those tokens (the lane l ^ 16
// holds the other half) and codes them, writing byte codes (ck) that are
// then packed along channels; thread i reduces value group (token i / NJ,
// group i % NJ) into vz / vs; then the same lane/channel split codes the
// values, whose group (= warp) metadata is one broadcast per token, and packs
// them along tokens in registers.  Codes come from code_bits in .f32x2 pairs,
// one check per lane deciding whether code_of must redo its codes
// (kivi_codes.cuh).  Half-precision tiles (stage_idx) and the byte codes of
// tokens 16 .. 31 are stored with 32-element halves swapped, so that the two
// halves of a warp read and write different banks.  Codes, scales and zeros
// equal those of quantize_tile bit for bit.
template <int D, int BITS, typename T, typename M>
__device__ __forceinline__ void quantize_tile_staged(const CacheView& c, long long unit,
                                                     long long t0, const T* Ks, const T* Vs,
                                                     uint8_t* ck, float4* vz, float2* vs,
                                                     int* vbad) {
  using Lt = Layout<D, BITS>;
  constexpr int E = Lt::E, WK = Lt::WK, NJ = Lt::NJ;
  constexpr int EPC = 16 / (int)sizeof(T);  // elements per 16-byte chunk
  constexpr bool SW = D >= 64;
  const float Lf = (float)Lt::L;
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const long long Ts = store_tokens(c);
  {
    long long su, stl;
    if (!store_tile(c, unit, t0 / kTile, &su, &stl)) return;  // same for the whole block
    unit = su;
    t0 = stl * kTile;
  }
  auto xi = [](int t, int d) { return stage_idx<D, T>(t, d); };
  // byte (t, d) of ck (the same swap at every element size)
  auto ci = [](int t, int d) { return t * D + (SW ? (d ^ (((t >> 4) & 1) << 5)) : d); };

  const int h = lane >> 4;                   // token half
  const int d0 = 32 * wp + 2 * (lane & 15);  // channel pair
  const int tb0 = 16 * h;
  // ---- keys: channels d0, d0 + 1 over the tile's tokens
  {
    float mn0, mx0, mn1, mx1;
    if constexpr (sizeof(T) == 2) {
      __half2 lo = *reinterpret_cast<const __half2*>(Ks + xi(tb0, d0)), hi = lo;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        const __half2 v = *reinterpret_cast<const __half2*>(Ks + xi(tb0 + i, d0));
        lo = __hmin2(lo, v);
        hi = __hmax2(hi, v);
      }
      const uint32_t plo = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t*>(&lo), 16);
      const uint32_t phi = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t*>(&hi), 16);
      lo = __hmin2(lo, *reinterpret_cast<const __half2*>(&plo));
      hi = __hmax2(hi, *reinterpret_cast<const __half2*>(&phi));
      mn0 = __low2float(lo);
      mn1 = __high2float(lo);
      mx0 = __low2float(hi);
      mx1 = __high2float(hi);
    } else {
      float2 lo = *reinterpret_cast<const float2*>(Ks + xi(tb0, d0)), hi = lo;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        const float2 v = *reinterpret_cast<const float2*>(Ks + xi(tb0 + i, d0));
        lo = make_float2(fminf(lo.x, v.x), fminf(lo.y, v.y));
        hi = make_float2(fmaxf(hi.x, v.x), fmaxf(hi.y, v.y));
      }
      mn0 = fminf(lo.x, __shfl_xor_sync(0xffffffffu, lo.x, 16));
      mn1 = fminf(lo.y, __shfl_xor_sync(0xffffffffu, lo.y, 16));
      mx0 = fmaxf(hi.x, __shfl_xor_sync(0xffffffffu, hi.x, 16));
      mx1 = fmaxf(hi.y, __shfl_xor_sync(0xffffffffu, hi.y, 16));
    }
    zero_sign_fix<kTile>(&mn0, &mx0, [&](int t) { return to_f32(Ks[xi(t, d0)]); });
    zero_sign_fix<kTile>(&mn1, &mx1, [&](int t) { return to_f32(Ks[xi(t, d0 + 1)]); });
    const float s0 = round_meta<M>(__fdiv_rn(__fsub_rn(mx0, mn0), Lf));
    const float s1 = round_meta<M>(__fdiv_rn(__fsub_rn(mx1, mn1), Lf));
    const float z0 = round_meta<M>(mn0), z1 = round_meta<M>(mn1);
    if (h == 0) {
      const long long mo = unit * Lt::k_meta_unit(Ts) + (t0 / kG) * D + d0;
      reinterpret_cast<M*>(c.k_scale)[mo] = from_f32<M>(s0);
      reinterpret_cast<M*>(c.k_scale)[mo + 1] = from_f32<M>(s1);
      reinterpret_cast<M*>(c.k_zero)[mo] = from_f32<M>(z0);
      reinterpret_cast<M*>(c.k_zero)[mo + 1] = from_f32<M>(z1);
    }
    const float rs0 = recip_rn(s0), rs1 = recip_rn(s1);
    const F2 z2 = f2(z0, z1);
    const F2 rq2 = f2(s0 != 0.0f ? rs0 : 0.0f, s1 != 0.0f ? rs1 : 0.0f);  // constant: code 0
    float ae = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {  // the low byte of code_bits is the code
      const int t = tb0 + i;
      const uint2 b = code_bits2<M>(load2(Ks + xi(t, d0)), z2, rq2, Lf, &ae);
      *reinterpret_cast<uint16_t*>(ck + ci(t, d0)) = (uint16_t)__byte_perm(b.x, b.y, 0x40);
    }
    const bool x0 = s0 != 0.0f && (codes_need_exact(ae, rs0) || !(s0 <= 3.0e38f));
    const bool x1 = s1 != 0.0f && (codes_need_exact(ae, rs1) || !(s1 <= 3.0e38f));
    if (x0 || x1) {
      for (int i = 0; i < 16; ++i) {
        const int t = tb0 + i;
        if (x0) ck[ci(t, d0)] = (uint8_t)code_of(__fsub_rn(to_f32(Ks[xi(t, d0)]), z0), s0, rs0, Lt::L);
        if (x1)
          ck[ci(t, d0 + 1)] =
              (uint8_t)code_of(__fsub_rn(to_f32(Ks[xi(t, d0 + 1)]), z1), s1, rs1, Lt::L);
      }
    }
  }
  // ---- value groups: token tid / NJ, group tid % NJ (min and max only;
  // chunks read in a rotated order that keeps the shared loads conflict-free)
  {
    const int t = tid / NJ, j = tid % NJ;
    float mn, mx;
    if constexpr (sizeof(T) == 2) {
      __half2 lo = __float2half2_rn(0.0f), hi = lo;
#pragma unroll
      for (int cc = 0; cc < kGv / EPC; ++cc) {
        const int ch = (cc + j + t) & (kGv / EPC - 1);
        const uint4 u = *reinterpret_cast<const uint4*>(Vs + xi(t, j * kGv + ch * EPC));
        const __half2 a = *reinterpret_cast<const __half2*>(&u.x);
        const __half2 b = *reinterpret_cast<const __half2*>(&u.y);
        const __half2 e = *reinterpret_cast<const __half2*>(&u.z);
        const __half2 f = *reinterpret_cast<const __half2*>(&u.w);
        const __half2 m1 = __hmin2(__hmin2(a, b), __hmin2(e, f));
        const __half2 m2 = __hmax2(__hmax2(a, b), __hmax2(e, f));
        lo = cc == 0 ? m1 : __hmin2(lo, m1);
        hi = cc == 0 ? m2 : __hmax2(hi, m2);
      }
      mn = fminf(__low2float(lo), __high2float(lo));
      mx = fmaxf(__low2float(hi), __high2float(hi));
    } else {
      mn = Vs[xi(t, j * kGv)];
      mx = mn;
#pragma unroll
      for (int cc = 0; cc < kGv / EPC; ++cc) {
        const int ch = (cc + j + t) & (kGv / EPC - 1);
        const float4 u = *reinterpret_cast<const float4*>(Vs + xi(t, j * kGv + ch * EPC));
        mn = fminf(fminf(mn, fminf(u.x, u.y)), fminf(u.z, u.w));
        mx = fmaxf(fmaxf(mx, fmaxf(u.x, u.y)), fmaxf(u.z, u.w));
      }
    }
    zero_sign_fix<kGv>(&mn, &mx, [&](int i) { return to_f32(Vs[xi(t, j * kGv + i)]); });
    const float s = round_meta<M>(__fdiv_rn(__fsub_rn(mx, mn), Lf));
    const float z = round_meta<M>(mn);
    const long long mo = unit * Lt::v_meta_unit(Ts) + (t0 + t) * NJ + j;
    reinterpret_cast<M*>(c.v_scale)[mo] = from_f32<M>(s);
    reinterpret_cast<M*>(c.v_zero)[mo] = from_f32<M>(z);
    const float rs = recip_rn(s);
    const float rq = s != 0.0f ? rs : 0.0f;  // a constant group codes to 0
    vz[t * NJ + j] = make_float4(z, z, rq, rq);
    vs[t * NJ + j] = make_float2(s, rs);
    if (s != 0.0f && (!(rs <= 3.0e38f) || !(s <= 3.0e38f))) atomicOr(&vbad[j], 1);
  }
  __syncthreads();
  // ---- value codes: channels d0, d0 + 1 over tokens tb0 .. tb0 + 15, packed
  // along tokens (a word holds E tokens; at E = 32 the lane l ^ 16 holds the
  // other half of each word)
  {
    const int j = d0 / kGv;  // the warp's group
    constexpr int EH = E < 16 ? E : 16;  // codes per word part held by a lane
    constexpr int NP = 16 / EH;          // word parts per lane and channel
    constexpr uint32_t kBias = code_bias(BITS, EH);
    float ae = 0.0f;
    // word parts (BITS != 3) or bit-plane halves (BITS == 3) of both channels
    uint32_t pa[BITS == 3 ? 3 : NP], pb[BITS == 3 ? 3 : NP];
    auto accumulate = [&](auto code_pair) {
#pragma unroll
      for (int p = 0; p < (BITS == 3 ? 3 : NP); ++p) pa[p] = pb[p] = 0u;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint2 b = code_pair(tb0 + i);  // encodings, 0x4B400000 + code
        if constexpr (BITS == 3) {
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            pa[k] |= ((b.x >> k) & 1u) << i;
            pb[k] |= ((b.y >> k) & 1u) << i;
          }
        } else {
          pa[i / EH] += b.x << (BITS * (i % EH));
          pb[i / EH] += b.y << (BITS * (i % EH));
        }
      }
      if constexpr (BITS != 3) {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          pa[p] -= kBias;
          pb[p] -= kBias;
        }
      }
    };
    accumulate([&](int t) {
      const float4 m = vz[t * NJ + j];
      return code_bits2<M>(load2(Vs + xi(t, d0)), f2(m.x, m.y), f2(m.z, m.w), Lf, &ae);
    });
    if (codes_need_exact(ae, 0.0f) || vbad[j] != 0) {
      accumulate([&](int t) {
        const float4 m = vz[t * NJ + j];
        const float2 sr = vs[t * NJ + j];
        uint32_t a = 0x4B400000u, b = 0x4B400000u;
        if (sr.x != 0.0f) {
          a += code_of(__fsub_rn(to_f32(Vs[xi(t, d0)]), m.x), sr.x, sr.y, Lt::L);
          b += code_of(__fsub_rn(to_f32(Vs[xi(t, d0 + 1)]), m.x), sr.x, sr.y, Lt::L);
        }
        return make_uint2(a, b);
      });
    }
    uint32_t* vdst = c.v_codes + unit * Lt::v_codes_unit(Ts) + (t0 / E) * Lt::WB * D;
    if constexpr (E == 32) {
      // whole words: lane h = 0 writes channel d0, lane h = 1 channel d0 + 1,
      // each taking the other half from its partner
      constexpr int NWD = BITS == 3 ? 3 : 1;
#pragma unroll
      for (int k = 0; k < NWD; ++k) {
        const uint32_t give = h == 0 ? pb[k] : pa[k];
        const uint32_t got = __shfl_xor_sync(0xffffffffu, give, 16);
        const uint32_t w = h == 0 ? (pa[k] | (got << 16)) : (got | (pb[k] << 16));
        vdst[k * D + d0 + h] = w;
      }
    } else {
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int tb = h * NP + p;  // token block of E tokens
        *reinterpret_cast<uint2*>(vdst + tb * D + d0) = make_uint2(pa[p], pb[p]);
      }
    }
  }
  // ---- key codes: packed along channels from the byte codes
  uint32_t* kdst = c.k_codes + unit * Lt::k_codes_unit(Ts) + t0 * WK;
  if constexpr (BITS == 3) {
    constexpr int NWP = D / 32;
    for (int pb = wp; pb < kTile * (D / 32); pb += NWP) {  // (token, 32-channel block)
      const int t = pb / (D / 32), w = pb % (D / 32);
      const uint32_t cd = ck[ci(t, w * 32 + lane)];
      const uint32_t p0 = __ballot_sync(0xffffffffu, cd & 1u);
      const uint32_t p1 = __ballot_sync(0xffffffffu, cd & 2u);
      const uint32_t p2 = __ballot_sync(0xffffffffu, cd & 4u);
      if (lane < 3) kdst[t * WK + 3 * w + lane] = lane == 0 ? p0 : (lane == 1 ? p1 : p2);
    }
  } else {
#pragma unroll
    for (int k = tid; k < kTile * WK; k += D) {
      const int t = k / WK, w = k % WK;
      kdst[k] = pack_bytes<BITS>(ck + ci(t, w * E));
    }
  }
}

// The span of unit `unit` in a ragged prefill: sequence unit / Hkv has
// lens[.] tokens, split as r = ((lens - 1) mod R) + 1 and n_q = lens - r.  A
// length outside [1, min(T_len, Tq + R)], or (paged) a page the prompt fills
// outside the block table's pool, gives ok = false and n_q = r = 0.
__device__ __forceinline__ bool ragged_span(const CacheView& c, const long long* lens,
                                            long long unit, long long T_len, int Hkv,
                                            long long* n_q, int* r) {
  const long long b = unit / Hkv;
  const long long n = lens[b];
  bool ok = n >= 1 && n <= T_len && n <= c.Tq + c.R;
  *r = ok ? (int)((n - 1) % c.R) + 1 : 0;
  *n_q = ok ? n - *r : 0;
  if (ok && c.bt != nullptr) {  // every page the prompt fills must be in the pool
    for (long long l = 0; l < *n_q / c.R; ++l) {
      const int pg = c.bt[b * c.pps + l];
      ok = ok && pg >= 0 && pg < c.n_pages;
    }
    if (!ok) {
      *r = 0;
      *n_q = 0;
    }
  }
  return ok;
}

// General path (outlier lists, or K, V or a window not 16-byte aligned):
// grid (n_q / kTile + 1, units); the last x-block copies the r window tokens.
// Ragged (lens != null): grid (T_len / kTile + 1, units), each unit's span
// from ragged_span; the last x-block of the sequence's first unit writes st[b]
// ({0, 0, 1} for a refused sequence, which writes nothing else).
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
    const bool ok = ragged_span(c, lens, unit, T_len, Hkv, &n_q, &r);
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
    quantize_tile<D, BITS, T, M, 0, true>(c, unit, Ku + tile * kTile * D, Vu + tile * kTile * D,
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

// Dynamic shared memory of prefill_staged_kernel: the K and V tiles, the
// key byte codes, the value groups' metadata and flags.
template <int D, typename T>
struct StagedSmem {
  static constexpr int TILE_B = kTile * D * (int)sizeof(T);
  static constexpr int O_CK = 2 * TILE_B;
  static constexpr int O_VZ = O_CK + kTile * D;
  static constexpr int O_VS = O_VZ + kTile * (D / kGv) * 16;
  static constexpr int O_BAD = O_VS + kTile * (D / kGv) * 8;
  static constexpr int BYTES = O_BAD + 16;
};

// Fast path (no outlier lists; K, V and the windows 16-byte aligned): the
// grid of prefill_kernel, each CTA staging its tile by asynchronous copies
// and quantizing it with quantize_tile_staged; the window tokens move in
// 16-byte chunks.  At most 64 registers a thread, so that eight CTAs share
// an SM and hide each other's load latency (measured against 5 CTAs at 82
// registers: 7B prompt 283 -> 217 us).
template <int D, int BITS, typename T, typename M>
__global__ void __launch_bounds__(D, 8) prefill_staged_kernel(CacheView c, const T* __restrict__ K,
                                                              const T* __restrict__ V,
                                                              long long T_len, long long n_q, int r,
                                                              const long long* __restrict__ lens,
                                                              DevState* st, int Hkv) {
  using SM = StagedSmem<D, T>;
  extern __shared__ __align__(16) unsigned char smem[];
  T* Ks = reinterpret_cast<T*>(smem);
  T* Vs = reinterpret_cast<T*>(smem + SM::TILE_B);
  const long long unit = blockIdx.y;
  const long long tile = blockIdx.x;
  const int tid = threadIdx.x;
  const T* Ku = K + unit * T_len * D;
  const T* Vu = V + unit * T_len * D;
  if (lens != nullptr) {
    const long long b = unit / Hkv;
    const bool ok = ragged_span(c, lens, unit, T_len, Hkv, &n_q, &r);
    if (tile == gridDim.x - 1 && unit == b * Hkv && tid == 0) {
      DevState v;
      v.n_q = n_q;
      v.r = r;
      v.status = ok ? 0 : 1;
      st[b] = v;
    }
    if (!ok) return;
  }
  if (tile < n_q / kTile) {
    int* vbad = reinterpret_cast<int*>(smem + SM::O_BAD);
    if (tid < D / kGv) vbad[tid] = 0;
    stage_tile<D, T>(Ks, Vs, Ku + tile * kTile * D, Vu + tile * kTile * D);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    quantize_tile_staged<D, BITS, T, M>(c, unit, tile * kTile, Ks, Vs, smem + SM::O_CK,
                                        reinterpret_cast<float4*>(smem + SM::O_VZ),
                                        reinterpret_cast<float2*>(smem + SM::O_VS), vbad);
  } else if (tile == gridDim.x - 1) {  // rows of D elements are whole 16-byte chunks
    constexpr int EPC = 16 / (int)sizeof(T);
    const uint4* ks = reinterpret_cast<const uint4*>(Ku + n_q * D);
    const uint4* vs = reinterpret_cast<const uint4*>(Vu + n_q * D);
    uint4* kr = reinterpret_cast<uint4*>(reinterpret_cast<T*>(c.k_res) + unit * c.R * D);
    uint4* vr = reinterpret_cast<uint4*>(reinterpret_cast<T*>(c.v_res) + unit * c.R * D);
    for (int i = tid; i < r * D / EPC; i += D) {
      kr[i] = ks[i];
      vr[i] = vs[i];
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
// STAGED (no outlier lists, 16-byte aligned windows): the window tile is
// staged and quantized as the prompt's tiles are (quantize_tile_staged, the
// StagedSmem layout in dynamic shared memory).
template <int D, int BITS, typename T, typename M, bool STAGED>
__global__ void __launch_bounds__(D, STAGED ? 8 : 1)
    append_kernel(CacheView c, const T* __restrict__ k, const T* __restrict__ v, long long n_q,
                  int slot, int flush, DevState* st, int Hkv) {
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ uint8_t ck[STAGED ? 1 : kTile * D];
  __shared__ uint8_t cv[STAGED ? 1 : kTile * D];
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
  if (flush) {
    if constexpr (STAGED) {
      using SM = StagedSmem<D, T>;
      T* Ks = reinterpret_cast<T*>(dsm);
      T* Vs = reinterpret_cast<T*>(dsm + SM::TILE_B);
      int* vbad = reinterpret_cast<int*>(dsm + SM::O_BAD);
      if (threadIdx.x < D / kGv) vbad[threadIdx.x] = 0;
      stage_tile<D, T>(Ks, Vs, kr + tile * kTile * D, vr + tile * kTile * D);
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncthreads();
      quantize_tile_staged<D, BITS, T, M>(c, unit, n_q + tile * kTile, Ks, Vs, dsm + SM::O_CK,
                                          reinterpret_cast<float4*>(dsm + SM::O_VZ),
                                          reinterpret_cast<float2*>(dsm + SM::O_VS), vbad);
    } else {
      quantize_tile<D, BITS, T, M, 0, true>(c, unit, kr + tile * kTile * D, vr + tile * kTile * D,
                                   n_q + tile * kTile, ck, cv);
    }
  }
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
  const bool aligned = (((uintptr_t)K | (uintptr_t)V | (uintptr_t)c.k_res | (uintptr_t)c.v_res) &
                        15u) == 0;
  dim3 grid((unsigned)((lens ? T_len : n_q) / kTile + 1), (unsigned)units);
  if (aligned && c.k_out == 0 && c.v_out == 0) {
    static_assert(StagedSmem<D, T>::BYTES <= 48 * 1024, "no opt-in needed");
    prefill_staged_kernel<D, BITS, T, M><<<grid, D, StagedSmem<D, T>::BYTES, s>>>(
        c, (const T*)K, (const T*)V, T_len, n_q, r, lens, st, Hkv);
  } else {
    prefill_kernel<D, BITS, T, M><<<grid, D, 0, s>>>(c, (const T*)K, (const T*)V, T_len, n_q, r,
                                                     lens, st, Hkv);
  }
  return cudaGetLastError();
}

template <int D, int BITS, typename T, typename M>
cudaError_t append_t(const CacheView& c, int units, const void* k, const void* v, long long n_q,
                     int slot, bool flush, DevState* st, int Hkv, cudaStream_t s) {
  const dim3 grid((unsigned)((flush || st) ? c.R / kTile : 1), (unsigned)units);
  const bool aligned = (((uintptr_t)c.k_res | (uintptr_t)c.v_res) & 15u) == 0;
  if (aligned && c.k_out == 0 && c.v_out == 0 && (flush || st))
    append_kernel<D, BITS, T, M, true><<<grid, D, StagedSmem<D, T>::BYTES, s>>>(
        c, (const T*)k, (const T*)v, n_q, slot, flush ? 1 : 0, st, Hkv);
  else
    append_kernel<D, BITS, T, M, false><<<grid, D, 0, s>>>(c, (const T*)k, (const T*)v, n_q, slot,
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
