// kivi_decode_simt.cu -- split-context decode attention over the packed
// KIVI cache on CUDA cores (SIMT); the split merge is fused in (finish_unit).
//
// Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache",
// study.space summary: decode attention is computed over the quantized
// ("grouped") part and combined with the full-precision residual part.
// Here both parts enter one online softmax (flash-decoding style): each CTA
// owns a contiguous range of 32-token tiles of one (batch, KV head) unit for
// all query heads of the GQA group, keeps a running max m, sum l and
// unnormalised accumulator per head, and writes (m, l, acc[D]) to the
// workspace; the last CTA of the unit rescales the splits to a common max.
//
// Keys use the factored form  q.khat = sum_d (q_d s_gd) c_td + sum_d q_d z_gd
// (scale and zero are per key group and channel); values are dequantized as
// fmaf(c, s, z) per element.  Scores are kept in log2 units
// (q pre-multiplied by softmax_scale * log2 e) and exponentiated with exp2f.
#include "kivi_internal.cuh"

namespace kivi {
namespace {

constexpr int kWarps = 4;
constexpr float kNegInf = -__builtin_huge_valf();

template <int N>
struct Words;
template <>
struct Words<1> { static __device__ __forceinline__ void load(const uint32_t* p, uint32_t* w) { w[0] = p[0]; } };
template <>
struct Words<2> {
  static __device__ __forceinline__ void load(const uint32_t* p, uint32_t* w) {
    uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  }
};
template <>
struct Words<4> {
  static __device__ __forceinline__ void load(const uint32_t* p, uint32_t* w) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
};

template <int D, int BITS, int GQ, typename T, typename MT>
__global__ void __launch_bounds__(kWarps * 32) decode_split_simt(DecodeArgs a) {
  using Lt = Layout<D, BITS>;
  constexpr int E = Lt::E, WK = Lt::WK, NJ = Lt::NJ;
  constexpr int CPL = D / 32;  // value channels per lane
  constexpr int TB = kTile / E;  // value words per channel per tile
  __shared__ float qs[GQ][D];
  __shared__ float qk[kWarps][GQ][D];
  __shared__ float vs[kWarps][kTile][NJ];
  __shared__ float vz[kWarps][kTile][NJ];
  __shared__ float red_m[kWarps][GQ], red_l[kWarps][GQ];
  __shared__ float red_acc[kWarps][GQ][D];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long unit = blockIdx.y;
  const int split = blockIdx.x;
  const long long b = unit / a.Hkv;
  const int kv = (int)(unit % a.Hkv);
  const int Hq = a.Hkv * GQ;
  const CacheView& c = a.c;

  const T* q = reinterpret_cast<const T*>(a.q) + (b * Hq + (long long)kv * GQ) * D;
  for (int i = threadIdx.x; i < GQ * D; i += kWarps * 32) (&qs[0][0])[i] = to_f32(q[i]) * a.qscale;
  __syncthreads();

  const long long n_qt = a.n_q / kTile;
  const long long total = n_qt + (a.r + kTile - 1) / kTile;
  const long long first = (long long)split * a.tiles_per_split;
  const long long last = min(total, first + a.tiles_per_split);

  const uint32_t* kc = c.k_codes + unit * Lt::k_codes_unit(c.Tq);
  const MT* ksc = reinterpret_cast<const MT*>(c.k_scale) + unit * Lt::k_meta_unit(c.Tq);
  const MT* kze = reinterpret_cast<const MT*>(c.k_zero) + unit * Lt::k_meta_unit(c.Tq);
  const uint32_t* vc = c.v_codes + unit * Lt::v_codes_unit(c.Tq);
  const MT* vsc = reinterpret_cast<const MT*>(c.v_scale) + unit * Lt::v_meta_unit(c.Tq);
  const MT* vze = reinterpret_cast<const MT*>(c.v_zero) + unit * Lt::v_meta_unit(c.Tq);
  const T* kr = reinterpret_cast<const T*>(c.k_res) + unit * c.R * D;
  const T* vr = reinterpret_cast<const T*>(c.v_res) + unit * c.R * D;

  const int d0 = lane * CPL;  // this lane's value channels d0..d0+CPL-1
  const int jl = d0 / kGv;    // their value group
  float m[GQ], l[GQ], acc[GQ][CPL];
#pragma unroll
  for (int h = 0; h < GQ; ++h) {
    m[h] = kNegInf;
    l[h] = 0.f;
#pragma unroll
    for (int k = 0; k < CPL; ++k) acc[h][k] = 0.f;
  }

  for (long long tile = first + warp; tile < last; tile += kWarps) {
    float lg[GQ];
    const bool quant = tile < n_qt;
    const long long tok0 = tile * kTile;
    if (quant) {
      // q' = q * s (this key group), bias = q . z
      float bias[GQ];
#pragma unroll
      for (int h = 0; h < GQ; ++h) bias[h] = 0.f;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const int d = lane + 32 * i;
        const float s = to_f32(ksc[tile * D + d]), z = to_f32(kze[tile * D + d]);
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          qk[warp][h][d] = qs[h][d] * s;
          bias[h] = fmaf(qs[h][d], z, bias[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < GQ; ++h) lg[h] = warp_sum(bias[h]);
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        vs[warp][lane][j] = to_f32(vsc[(tok0 + lane) * NJ + j]);
        vz[warp][lane][j] = to_f32(vze[(tok0 + lane) * NJ + j]);
      }
      __syncwarp();
      // scores: lane = token tok0 + lane
      const uint32_t* row = kc + (tok0 + lane) * WK;
#pragma unroll
      for (int w0 = 0; w0 < WK; w0 += (WK >= 4 ? 4 : WK)) {
        constexpr int NV = WK >= 4 ? 4 : WK;
        uint32_t wv[NV];
        Words<NV>::load(row + w0, wv);
#pragma unroll
        for (int u = 0; u < NV; ++u) {
#pragma unroll
          for (int i = 0; i < E; ++i) {
            const float cf = (float)((wv[u] >> (BITS * i)) & Lt::MASK);
            const int d = (w0 + u) * E + i;
#pragma unroll
            for (int h = 0; h < GQ; ++h) lg[h] = fmaf(qk[warp][h][d], cf, lg[h]);
          }
        }
      }
    } else {
      const int t_in = (int)(tile - n_qt) * kTile + lane;
      if (t_in < a.r) {
#pragma unroll
        for (int h = 0; h < GQ; ++h) lg[h] = 0.f;
        const T* row = kr + (long long)t_in * D;
#pragma unroll 8
        for (int d = 0; d < D; ++d) {
          const float kf = to_f32(row[d]);
#pragma unroll
          for (int h = 0; h < GQ; ++h) lg[h] = fmaf(qs[h][d], kf, lg[h]);
        }
      } else {
#pragma unroll
        for (int h = 0; h < GQ; ++h) lg[h] = kNegInf;
      }
    }
    // online softmax update (log2 units)
    float p[GQ];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
      const float mt = warp_max(lg[h]);
      const float mn = fmaxf(m[h], mt);
      const float alpha = exp2f(m[h] - mn);
      p[h] = exp2f(lg[h] - mn);
      l[h] = fmaf(l[h], alpha, p[h]);
#pragma unroll
      for (int k = 0; k < CPL; ++k) acc[h][k] *= alpha;
      m[h] = mn;
    }
    // P.V
    if (quant) {
      uint32_t vw[TB][CPL];
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) Words<CPL>::load(vc + (tok0 / E + tb) * D + d0, vw[tb]);
#pragma unroll
      for (int t = 0; t < kTile; ++t) {
        const float sv = vs[warp][t][jl], zv = vz[warp][t][jl];
        float pt[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) pt[h] = __shfl_sync(0xffffffffu, p[h], t);
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
          const float cf = (float)((vw[t / E][k] >> (BITS * (t % E))) & Lt::MASK);
          const float vh = fmaf(cf, sv, zv);
#pragma unroll
          for (int h = 0; h < GQ; ++h) acc[h][k] = fmaf(pt[h], vh, acc[h][k]);
        }
      }
    } else {
      const int tbase = (int)(tile - n_qt) * kTile;
      const int nt = min(kTile, a.r - tbase);
      for (int t = 0; t < nt; ++t) {
        float pt[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) pt[h] = __shfl_sync(0xffffffffu, p[h], t);
        const T* row = vr + (long long)(tbase + t) * D + d0;
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
          const float vh = to_f32(row[k]);
#pragma unroll
          for (int h = 0; h < GQ; ++h) acc[h][k] = fmaf(pt[h], vh, acc[h][k]);
        }
      }
    }
    __syncwarp();
  }

  // merge the warps of this CTA, write the split's partial
#pragma unroll
  for (int h = 0; h < GQ; ++h) {
    const float lt = warp_sum(l[h]);
    if (lane == 0) {
      red_m[warp][h] = m[h];
      red_l[warp][h] = lt;
    }
#pragma unroll
    for (int k = 0; k < CPL; ++k) red_acc[warp][h][d0 + k] = acc[h][k];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < GQ * D; idx += kWarps * 32) {
    const int h = idx / D, d = idx % D;
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w][h]);
    float num = 0.f, den = 0.f;
    if (M != kNegInf) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        if (red_m[w][h] == kNegInf) continue;
        const float sc = exp2f(red_m[w][h] - M);
        num = fmaf(sc, red_acc[w][h][d], num);
        den = fmaf(sc, red_l[w][h], den);
      }
    }
    float* P = a.ws + ((b * Hq + (long long)kv * GQ + h) * a.n_split + split) * (D + 2);
    if (d == 0) {
      P[0] = M;
      P[1] = den;
    }
    P[2 + d] = num;
  }
  __shared__ int last_flag;
  finish_unit<D, GQ, T>(a, b, kv, &last_flag);
}

template <int D, int BITS, int GQ, typename T, typename MT>
cudaError_t simt_t(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1) {
  dim3 grid((unsigned)a.n_split, (unsigned)a.units);
  if (e0) cudaEventRecord(e0, s);
  decode_split_simt<D, BITS, GQ, T, MT><<<grid, kWarps * 32, 0, s>>>(a);
  cudaError_t err = cudaGetLastError();
  if (e1) cudaEventRecord(e1, s);
  return err;
}

template <int D, int BITS, typename T, typename M>
cudaError_t simt_g(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1) {
  switch (a.gq) {
    case 1: return simt_t<D, BITS, 1, T, M>(a, s, e0, e1);
    case 2: return simt_t<D, BITS, 2, T, M>(a, s, e0, e1);
    case 4: return simt_t<D, BITS, 4, T, M>(a, s, e0, e1);
    case 8: return simt_t<D, BITS, 8, T, M>(a, s, e0, e1);
  }
  return cudaErrorInvalidValue;
}

template <int BITS, typename T, typename M>
cudaError_t simt_d(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1) {
  switch (a.D) {
    case 32: return simt_g<32, BITS, T, M>(a, s, e0, e1);
    case 64: return simt_g<64, BITS, T, M>(a, s, e0, e1);
    case 128: return simt_g<128, BITS, T, M>(a, s, e0, e1);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                               cudaEvent_t e1) {
  if (a.meta == 1) {  // binary16 scales and zeros: fp16 caches only
    if (a.dtype != 0) return cudaErrorInvalidValue;
    if (a.bits == 1) return simt_d<1, __half, __half>(a, s, e0, e1);
    if (a.bits == 2) return simt_d<2, __half, __half>(a, s, e0, e1);
    if (a.bits == 4) return simt_d<4, __half, __half>(a, s, e0, e1);
    return cudaErrorInvalidValue;
  }
  if (a.meta != 0) return cudaErrorInvalidValue;
  if (a.bits == 1 && a.dtype == 0) return simt_d<1, __half, float>(a, s, e0, e1);
  if (a.bits == 1 && a.dtype == 1) return simt_d<1, float, float>(a, s, e0, e1);
  if (a.bits == 2 && a.dtype == 0) return simt_d<2, __half, float>(a, s, e0, e1);
  if (a.bits == 2 && a.dtype == 1) return simt_d<2, float, float>(a, s, e0, e1);
  if (a.bits == 4 && a.dtype == 0) return simt_d<4, __half, float>(a, s, e0, e1);
  if (a.bits == 4 && a.dtype == 1) return simt_d<4, float, float>(a, s, e0, e1);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
