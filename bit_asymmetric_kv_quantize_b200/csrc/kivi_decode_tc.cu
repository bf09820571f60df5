// kivi_decode_tc.cu -- split-context decode attention over the packed KIVI
// cache with the two contractions on tensor cores (mma.sync, fp16 operands,
// fp32 accumulation).
//
// Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache",
// study.space summary: decode attention runs over the quantized ("grouped")
// part and is combined with the full-precision residual part; mlsanity.com
// index page, "Abstract (arXiv)": loading the cache bounds decode.  Both parts
// enter one online softmax; each CTA writes (m, l, acc[D]) per query head to
// the workspace and decode_combine merges the splits.
//
// Per CTA: one (batch, KV head) unit and a contiguous range of 32-token tiles
// (one key group each), all query heads of the GQA group.  The last split of
// a unit owns the residual window and runs on CUDA cores; every other split
// streams its tiles:
//   * memory: one thread issues 1-D bulk copies (cp.async.bulk, completion
//     on an mbarrier) of each stage -- 4 tiles of key codes, key scales, key
//     zeros, value codes, value scales, value zeros, six contiguous ranges --
//     into a ring of shared-memory stages; the four warps take one tile each.
//   * scores: S = q' K^T on tensor cores, q'_{h,d} = q_{h,d} s_{g,d} split
//     into fp16 hi + lo rows (A, 16 x 16 per channel slice), key codes as
//     the B operand (16 channels x 8 tokens), taken from one 32-bit word by a
//     shift and a mask: a 2-bit code c placed in the low mantissa bits of an
//     fp16 is the exact value c * 2^-24, so no conversion is needed and the
//     2^24 is restored on the fp32 result.  score = 2^24 S + sum_d q_d z_{g,d}.
//   * softmax: running max and sum in log2 units (q pre-scaled by
//     softmax_scale * log2 e, exp2f).
//   * values: O += V^T p' on tensor cores, value codes as the A operand
//     (16 channels x 16 tokens, same shift-and-mask), p'_{t,h} =
//     p_{t,h} s_{t,j} split into hi + lo columns of B; the zero enters as
//     sum_t p_t z_{t,j} per value group.
// The q' and p' fragments are built cooperatively (each lane converts a few
// values and stores them in fragment order in per-warp shared memory).
// The channel (key) and token (value) order inside an mma k-slice follows
// the bit order of the words, and the score columns are assigned to tokens
// so that each lane already holds the probabilities its P.V fragment needs.
#include "kivi_internal.cuh"

namespace kivi {
namespace {

constexpr int kW = 4;           // warps per CTA
constexpr int kStage = 4;       // tiles per pipeline stage (one per warp)
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kTwo24 = 16777216.0f;
constexpr long long kWaitCycles = 1LL << 32;  // ~2 s: bounded wait on our own copies

template <int D, int BITS, int GQ>
struct Geo {
  static constexpr int E = 32 / BITS;
  static constexpr int WK = D / E;       // key words per token
  static constexpr int NJ = D / kGv;     // value groups per token
  static constexpr int KSL = D / 16;     // k-slices of the score product
  static constexpr int KC_B = kTile * WK * 4;
  static constexpr int KM_B = D * 4;
  static constexpr int VC_B = (kTile / E) * D * 4;
  static constexpr int VM_B = kTile * NJ * 4;
  static constexpr int TILE_B = KC_B + 2 * KM_B + VC_B + 2 * VM_B;
  static constexpr int O_KC = 0;
  static constexpr int O_KS = O_KC + kStage * KC_B;
  static constexpr int O_KZ = O_KS + kStage * KM_B;
  static constexpr int O_VC = O_KZ + kStage * KM_B;
  static constexpr int O_VS = O_VC + kStage * VC_B;
  static constexpr int O_VZ = O_VS + kStage * VM_B;
  static constexpr int STAGE_B = O_VZ + kStage * VM_B;
  static constexpr int NSTAGE = BITS == 2 ? 4 : 3;
  static constexpr int NPB = GQ == 8 ? 2 : 1;          // p' B operands (hi/lo split)
  // per-warp scratch (bytes)
  static constexpr int QA_B = KSL * 32 * 16;           // q' A fragments
  static constexpr int PB_B = NPB * NJ * 2 * 32 * 8;   // p' B fragments
  static constexpr int PBUF_B = GQ * kTile * 4;        // p per head and token
  static constexpr int WARP_B = QA_B + PB_B + PBUF_B;
  // whole CTA
  static constexpr int O_WARP = NSTAGE * STAGE_B;
  static constexpr int O_QS = O_WARP + kW * WARP_B;    // q (fp32, scaled) for the window path
  static constexpr int O_BAR = O_QS + GQ * D * 4;
  static constexpr int SMEM_B = O_BAR + NSTAGE * 8;
  // end-of-CTA merge buffers, placed over the stage ring
  static constexpr int MERGE_B = kW * GQ * (D + 2) * 4;
  static_assert(MERGE_B <= NSTAGE * STAGE_B, "merge buffers must fit in the stage ring");
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for a stage; gives up (returns false) after kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Position of element i (0..15) of a k-slice inside an mma fragment:
// lane group `tq` (threadID_in_group), k-pair `kp` (0: k = 2tq,2tq+1;
// 1: k = 2tq+8, 2tq+9) and half `hf` of the 32-bit register.  It mirrors the
// shift-and-mask extraction: 2-bit words give pairs (i, i+8) and
// (i+4, i+12), 4-bit word pairs give (i, i+4) and (i+8, i+12).
template <int BITS>
__device__ __forceinline__ void slot_of(int i, int& tq, int& kp, int& hf) {
  tq = i & 3;
  if (BITS == 2) {
    kp = (i >> 2) & 1;
    hf = i >> 3;
  } else {
    kp = i >> 3;
    hf = (i >> 2) & 1;
  }
}

// Token (0..31) held by score column `col` (0..7) of n-tile nt (0..3).
template <int BITS>
__device__ __forceinline__ int score_token(int nt, int col) {
  const int a = col >> 1, e = col & 1, H = nt >> 1, sub = nt & 1;
  return 16 * H + (BITS == 2 ? a + 4 * sub + 8 * e : a + 8 * sub + 4 * e);
}

// Two fp16 codes (as exact subnormals c * 2^-24) per register: k-pairs tq and tq+4.
template <int BITS>
__device__ __forceinline__ void codes_pair(uint32_t w_lo, uint32_t w_hi, int tq, uint32_t& kp0,
                                           uint32_t& kp1) {
  if (BITS == 2) {
    const uint32_t w1 = w_lo >> (2 * tq);
    kp0 = w1 & 0x00030003u;
    kp1 = (w1 >> 8) & 0x00030003u;
  } else {
    kp0 = (w_lo >> (4 * tq)) & 0x000F000Fu;
    kp1 = (w_hi >> (4 * tq)) & 0x000F000Fu;
  }
}

__device__ __forceinline__ void split_f16(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

template <int D, int BITS, int GQ, typename T>
__global__ void __launch_bounds__(kW * 32, 2) decode_split_tc(DecodeArgs a) {
  using G = Geo<D, BITS, GQ>;
  using Lt = Layout<D, BITS>;
  constexpr int E = G::E, WK = G::WK, NJ = G::NJ, KSL = G::KSL;
  constexpr int NM = D / 16;  // value m-tiles (16 channels each)
  extern __shared__ __align__(128) unsigned char smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const long long unit = blockIdx.y;
  const int split = blockIdx.x;
  const long long b = unit / a.Hkv;
  const int kv = (int)(unit % a.Hkv);
  const int Hq = a.Hkv * GQ;
  const CacheView& c = a.c;
  const T* qg = reinterpret_cast<const T*>(a.q) + (b * Hq + (long long)kv * GQ) * D;

  unsigned char* wbase = smem + G::O_WARP + warp * G::WARP_B;
  uint32_t* qA = reinterpret_cast<uint32_t*>(wbase);
  __half* qAh = reinterpret_cast<__half*>(wbase);
  uint32_t* pB = reinterpret_cast<uint32_t*>(wbase + G::QA_B);
  __half* pBh = reinterpret_cast<__half*>(wbase + G::QA_B);
  float* pbuf = reinterpret_cast<float*>(wbase + G::QA_B + G::PB_B);
  float* qs = reinterpret_cast<float*>(smem + G::O_QS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::O_BAR);

  // zero the fragment scratch (rows / columns without a head stay zero)
  for (int i = lane; i < (G::QA_B + G::PB_B) / 4; i += 32) qA[i] = 0u;
  for (int i = tid; i < GQ * D; i += kW * 32) qs[i] = to_f32(qg[i]) * a.qscale;

  const bool window_cta = a.r > 0 && split == a.n_split - 1;
  const long long n_qt = a.n_q / kTile;
  const long long first = (long long)split * a.tiles_per_split;
  const long long last = window_cta ? first : min(n_qt, first + a.tiles_per_split);
  const long long ntiles = last > first ? last - first : 0;
  const long long nstages = (ntiles + kStage - 1) / kStage;

  if (tid == 0) {
    for (int s = 0; s < G::NSTAGE; ++s) mbar_init(&bars[s]);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const uint32_t* kc_u = c.k_codes + unit * Lt::k_codes_unit(c.Tq);
  const float* ks_u = c.k_scale + unit * Lt::k_meta_unit(c.Tq);
  const float* kz_u = c.k_zero + unit * Lt::k_meta_unit(c.Tq);
  const uint32_t* vc_u = c.v_codes + unit * Lt::v_codes_unit(c.Tq);
  const float* vs_u = c.v_scale + unit * Lt::v_meta_unit(c.Tq);
  const float* vz_u = c.v_zero + unit * Lt::v_meta_unit(c.Tq);

  auto issue = [&](long long st) {
    unsigned char* buf = smem + (int)(st % G::NSTAGE) * G::STAGE_B;
    uint64_t* bar = &bars[st % G::NSTAGE];
    const long long t0 = first + st * kStage;
    const int n = (int)min((long long)kStage, last - t0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_expect_tx(bar, (uint32_t)(n * G::TILE_B));
    bulk_copy(buf + G::O_KC, kc_u + t0 * kTile * WK, n * G::KC_B, bar);
    bulk_copy(buf + G::O_KS, ks_u + t0 * D, n * G::KM_B, bar);
    bulk_copy(buf + G::O_KZ, kz_u + t0 * D, n * G::KM_B, bar);
    bulk_copy(buf + G::O_VC, vc_u + t0 * (kTile / E) * D, n * G::VC_B, bar);
    bulk_copy(buf + G::O_VS, vs_u + t0 * kTile * NJ, n * G::VM_B, bar);
    bulk_copy(buf + G::O_VZ, vz_u + t0 * kTile * NJ, n * G::VM_B, bar);
  };
  if (tid == 0) {
    for (long long st = 0; st < nstages && st < G::NSTAGE; ++st) issue(st);
  }

  // ---- per-lane state
  // q for the cooperative q' build: lane owns channels lane + 32 i
  float qv[GQ][NJ];
#pragma unroll
  for (int h = 0; h < GQ; ++h)
#pragma unroll
    for (int i = 0; i < NJ; ++i) qv[h][i] = to_f32(qg[h * D + lane + 32 * i]) * a.qscale;
  const bool hv = g < GQ;            // this lane's score row is a real head
  float m_run = kNegInf, l_part = 0.f;
  float bv[GQ][NJ];                  // sum_t p z per (head, value group), lane partial
  float acc[G::NPB][NM][4];          // P.V accumulators (fragment layout)
#pragma unroll
  for (int h = 0; h < GQ; ++h)
#pragma unroll
    for (int j = 0; j < NJ; ++j) bv[h][j] = 0.f;
#pragma unroll
  for (int p = 0; p < G::NPB; ++p)
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[p][m][e] = 0.f;
  __syncwarp();

  bool failed = false;
  long long fail_st = 0;
  for (long long st = 0; st < nstages; ++st) {
    const bool ok = mbar_wait(&bars[st % G::NSTAGE], (uint32_t)((st / G::NSTAGE) & 1));
    if (__syncthreads_or(!ok)) {
      failed = true;
      fail_st = st;
      break;
    }
    const unsigned char* buf = smem + (int)(st % G::NSTAGE) * G::STAGE_B;
    const long long tile = first + st * kStage + warp;
    if (tile < last) {
      const uint32_t* kc = reinterpret_cast<const uint32_t*>(buf + G::O_KC) + warp * kTile * WK;
      const float* ks = reinterpret_cast<const float*>(buf + G::O_KS) + warp * D;
      const float* kz = reinterpret_cast<const float*>(buf + G::O_KZ) + warp * D;
      const uint32_t* vc = reinterpret_cast<const uint32_t*>(buf + G::O_VC) + warp * (kTile / E) * D;
      const float* vs = reinterpret_cast<const float*>(buf + G::O_VS) + warp * kTile * NJ;
      const float* vz = reinterpret_cast<const float*>(buf + G::O_VZ) + warp * kTile * NJ;

      // -- q' = q * s for this key group (hi/lo fp16 in fragment order), bias = q . z
      float bk[GQ];
#pragma unroll
      for (int h = 0; h < GQ; ++h) bk[h] = 0.f;
#pragma unroll
      for (int i = 0; i < NJ; ++i) {
        const int ch = lane + 32 * i;
        const float s = ks[ch], z = kz[ch];
        int t4, kp, hf;
        slot_of<BITS>(ch & 15, t4, kp, hf);
        const int sl = ch >> 4;
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          bk[h] = fmaf(qv[h][i], z, bk[h]);
          __half hi, lo;
          split_f16(qv[h][i] * s, hi, lo);
          const int base = ((sl * 32 + h * 4 + t4) * 4 + kp * 2) * 2 + hf;
          qAh[base] = hi;      // row h
          qAh[base + 2] = lo;  // row h + 8
        }
      }
      float mybk = 0.f;
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        bk[h] = warp_sum(bk[h]);
        if (g == h) mybk = bk[h];
      }
      __syncwarp();

      // -- scores: 4 n-tiles of 8 tokens, KSL k-slices of 16 channels
      float dq[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const uint32_t* row = kc + score_token<BITS>(nt, g) * WK;
        uint32_t wv[WK];
#pragma unroll
        for (int w4 = 0; w4 < WK; w4 += 2) {
          const uint2 v2 = *reinterpret_cast<const uint2*>(row + w4);
          wv[w4] = v2.x;
          wv[w4 + 1] = v2.y;
        }
#pragma unroll
        for (int sl = 0; sl < KSL; ++sl) {
          const uint4 af = *reinterpret_cast<const uint4*>(qA + (sl * 32 + lane) * 4);
          const uint32_t A[4] = {af.x, af.y, af.z, af.w};
          uint32_t b0, b1;
          if (BITS == 2)
            codes_pair<2>(wv[sl], 0u, tq, b0, b1);
          else
            codes_pair<4>(wv[2 * sl], wv[2 * sl + 1], tq, b0, b1);
          mma16816(dq[nt], A, b0, b1);
        }
      }

      // -- online softmax for head g over this tile (log2 units)
      float lg[8];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        lg[2 * nt] = fmaf(dq[nt][0] + dq[nt][2], kTwo24, mybk);
        lg[2 * nt + 1] = fmaf(dq[nt][1] + dq[nt][3], kTwo24, mybk);
      }
      float tmax = kNegInf;
#pragma unroll
      for (int i = 0; i < 8; ++i) tmax = fmaxf(tmax, lg[i]);
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
      float alpha = 1.f;
      float p[8];
      if (hv) {
        const float mn = fmaxf(m_run, tmax);
        alpha = exp2f(m_run - mn);
        float ps = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          p[i] = exp2f(lg[i] - mn);
          ps += p[i];
        }
        l_part = fmaf(l_part, alpha, ps);
        m_run = mn;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          pbuf[g * kTile + score_token<BITS>(nt, 2 * tq)] = p[2 * nt];
          pbuf[g * kTile + score_token<BITS>(nt, 2 * tq + 1)] = p[2 * nt + 1];
        }
      }
      __syncwarp();

      // -- p' = p * s_v (hi/lo, fragment order); bias_v += p * z_v; rescale partials
      float al[GQ];
#pragma unroll
      for (int h = 0; h < GQ; ++h) al[h] = __shfl_sync(0xffffffffu, alpha, h * 4);
      {
        const int t = lane;  // this lane's token
        int t4, kp, hf;
        slot_of<BITS>(t & 15, t4, kp, hf);
        const int Hs = t >> 4;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float s = vs[t * NJ + j], z = vz[t * NJ + j];
#pragma unroll
          for (int h = 0; h < GQ; ++h) {
            const float ph = pbuf[h * kTile + t];
            bv[h][j] = fmaf(ph, z, bv[h][j] * al[h]);
            __half hi, lo;
            split_f16(ph * s, hi, lo);
            if (GQ == 8) {
              const int base = (((j * 2 + Hs) * 32 + h * 4 + t4) * 2 + kp) * 2 + hf;
              pBh[base] = hi;
              pBh[base + NJ * 2 * 32 * 2 * 2] = lo;
            } else {
              const int bhi = (((j * 2 + Hs) * 32 + h * 4 + t4) * 2 + kp) * 2 + hf;
              const int blo = (((j * 2 + Hs) * 32 + (4 + h) * 4 + t4) * 2 + kp) * 2 + hf;
              pBh[bhi] = hi;
              pBh[blo] = lo;
            }
          }
        }
      }
      // rescale the P.V accumulators: columns 2tq, 2tq+1 hold heads
      // (GQ <= 4: col n is hi of head n for n < 4, lo of head n-4 after)
      {
        const int c0 = 2 * tq, c1 = 2 * tq + 1;
        const int h0 = GQ == 8 ? c0 : (c0 & 3), h1 = GQ == 8 ? c1 : (c1 & 3);
        float a0 = 1.f, a1 = 1.f;
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          if (h0 == h) a0 = al[h];
          if (h1 == h) a1 = al[h];
        }
#pragma unroll
        for (int p2 = 0; p2 < G::NPB; ++p2)
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            acc[p2][m][0] *= a0;
            acc[p2][m][1] *= a1;
            acc[p2][m][2] *= a0;
            acc[p2][m][3] *= a1;
          }
      }
      __syncwarp();

      // -- P.V: per value group j, m-tiles 2j (channels 32j+4g, +1) and 2j+1 (+2, +3)
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
#pragma unroll
        for (int Hs = 0; Hs < 2; ++Hs) {
          uint32_t A0[4], A1[4];
          if (BITS == 2) {
            const uint4 w = *reinterpret_cast<const uint4*>(vc + Hs * D + 32 * j + 4 * g);
            codes_pair<2>(w.x, 0u, tq, A0[0], A0[2]);
            codes_pair<2>(w.y, 0u, tq, A0[1], A0[3]);
            codes_pair<2>(w.z, 0u, tq, A1[0], A1[2]);
            codes_pair<2>(w.w, 0u, tq, A1[1], A1[3]);
          } else {
            const uint4 w0 = *reinterpret_cast<const uint4*>(vc + (2 * Hs) * D + 32 * j + 4 * g);
            const uint4 w1 = *reinterpret_cast<const uint4*>(vc + (2 * Hs + 1) * D + 32 * j + 4 * g);
            codes_pair<4>(w0.x, w1.x, tq, A0[0], A0[2]);
            codes_pair<4>(w0.y, w1.y, tq, A0[1], A0[3]);
            codes_pair<4>(w0.z, w1.z, tq, A1[0], A1[2]);
            codes_pair<4>(w0.w, w1.w, tq, A1[1], A1[3]);
          }
#pragma unroll
          for (int p2 = 0; p2 < G::NPB; ++p2) {
            const uint2 bb = *reinterpret_cast<const uint2*>(
                pB + p2 * (NJ * 2 * 32 * 2) + ((j * 2 + Hs) * 32 + lane) * 2);
            mma16816(acc[p2][2 * j], A0, bb.x, bb.y);
            mma16816(acc[p2][2 * j + 1], A1, bb.x, bb.y);
          }
        }
      }
    }
    __syncthreads();
    if (tid == 0 && st + G::NSTAGE < nstages) issue(st + G::NSTAGE);
  }

  // ---- this warp's state -> shared memory, then merge the warps
  float* mg_m = reinterpret_cast<float*>(smem);              // [kW][GQ]
  float* mg_l = mg_m + kW * GQ;                               // [kW][GQ]
  float* mg_acc = mg_l + kW * GQ;                             // [kW][GQ][D]
  if (failed) {
    // a stage did not arrive in time: wait (bounded) for the copies that are
    // still in flight, then publish NaN so that the merged output is NaN
    if (tid == 0) {
      for (long long s2 = fail_st; s2 < nstages && s2 < fail_st + G::NSTAGE; ++s2)
        (void)mbar_wait(&bars[s2 % G::NSTAGE], (uint32_t)((s2 / G::NSTAGE) & 1));
    }
    __syncthreads();
    for (int i = tid; i < GQ * (D + 2); i += kW * 32) {
      const int h = i / (D + 2), d = i % (D + 2);
      float* P = a.ws + ((b * Hq + (long long)kv * GQ + h) * a.n_split + split) * (D + 2);
      P[d] = d == 0 ? 0.f : __int_as_float(0x7fc00000);
    }
    return;
  }

  if (window_cta) {
    // ---- residual window on CUDA cores: warp w takes window tiles w, w+4, ...
    constexpr int CPL = D / 32;
    const T* kr = reinterpret_cast<const T*>(c.k_res) + unit * c.R * D;
    const T* vr = reinterpret_cast<const T*>(c.v_res) + unit * c.R * D;
    const int d0 = lane * CPL;
    float wm[GQ], wl[GQ], wacc[GQ][CPL];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
      wm[h] = kNegInf;
      wl[h] = 0.f;
#pragma unroll
      for (int k = 0; k < CPL; ++k) wacc[h][k] = 0.f;
    }
    const int nwt = (a.r + kTile - 1) / kTile;
    for (int wt = warp; wt < nwt; wt += kW) {
      const int t_in = wt * kTile + lane;
      float lg[GQ];
      if (t_in < a.r) {
#pragma unroll
        for (int h = 0; h < GQ; ++h) lg[h] = 0.f;
        const T* row = kr + (long long)t_in * D;
#pragma unroll 8
        for (int d = 0; d < D; ++d) {
          const float kf = to_f32(row[d]);
#pragma unroll
          for (int h = 0; h < GQ; ++h) lg[h] = fmaf(qs[h * D + d], kf, lg[h]);
        }
      } else {
#pragma unroll
        for (int h = 0; h < GQ; ++h) lg[h] = kNegInf;
      }
      float p[GQ];
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        const float mt = warp_max(lg[h]);
        const float mn = fmaxf(wm[h], mt);
        const float al = exp2f(wm[h] - mn);
        p[h] = exp2f(lg[h] - mn);
        wl[h] = fmaf(wl[h], al, p[h]);
#pragma unroll
        for (int k = 0; k < CPL; ++k) wacc[h][k] *= al;
        wm[h] = mn;
      }
      const int nt = min(kTile, a.r - wt * kTile);
      for (int t = 0; t < nt; ++t) {
        const T* row = vr + (long long)(wt * kTile + t) * D + d0;
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          const float pt = __shfl_sync(0xffffffffu, p[h], t);
#pragma unroll
          for (int k = 0; k < CPL; ++k) wacc[h][k] = fmaf(pt, to_f32(row[k]), wacc[h][k]);
        }
      }
    }
    __syncthreads();  // stage ring is free: reuse it for the merge
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
      const float lt = warp_sum(wl[h]);
      if (lane == 0) {
        mg_m[warp * GQ + h] = wm[h];
        mg_l[warp * GQ + h] = lt;
      }
#pragma unroll
      for (int k = 0; k < CPL; ++k) mg_acc[(warp * GQ + h) * D + d0 + k] = wacc[h][k];
    }
  } else {
    __syncthreads();  // all stages consumed: reuse the ring for the merge
    // l: sum over the quad of head g; bias_v: sum over the warp
    const float lq = l_part + __shfl_xor_sync(0xffffffffu, l_part, 1);
    const float lt = lq + __shfl_xor_sync(0xffffffffu, lq, 2);
#pragma unroll
    for (int h = 0; h < GQ; ++h)
#pragma unroll
      for (int j = 0; j < NJ; ++j) bv[h][j] = warp_sum(bv[h][j]);
    if (hv && tq == 0) {
      mg_m[warp * GQ + g] = m_run;
      mg_l[warp * GQ + g] = lt;
    }
    // accumulators: m-tile 2j+mm, row g -> channel 32j+4g+2mm, row g+8 -> +1;
    // columns 2tq, 2tq+1.  GQ <= 4: hi columns (tq < 2) get the lo columns
    // (tq + 2) added; GQ == 8: hi and lo are in the same lane.
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      const int j = m >> 1, mm = m & 1;
      const int ch0 = 32 * j + 4 * g + 2 * mm;
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[e] = acc[0][m][e];
        if (G::NPB == 2) v[e] += acc[G::NPB - 1][m][e];
        else v[e] += __shfl_xor_sync(0xffffffffu, v[e], 2);
      }
      if (GQ == 8 || tq < 2) {
        const int hc0 = 2 * tq, hc1 = 2 * tq + 1;  // heads of columns 0/1 of this lane
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = (e & 1) ? hc1 : hc0;
          const int ch = ch0 + (e >> 1);
          if (h < GQ) {
            float bias = 0.f;
#pragma unroll
            for (int hh = 0; hh < GQ; ++hh)
              if (hh == h) bias = bv[hh][j];
            mg_acc[(warp * GQ + h) * D + ch] = fmaf(v[e], kTwo24, bias);
          }
        }
      }
    }
    // warps that had no tile publish an empty state
    if (first + warp >= last) {
      for (int h = lane; h < GQ; h += 32) {
        mg_m[warp * GQ + h] = kNegInf;
        mg_l[warp * GQ + h] = 0.f;
      }
      for (int i = lane; i < GQ * D; i += 32) mg_acc[warp * GQ * D + i] = 0.f;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < GQ * D; idx += kW * 32) {
    const int h = idx / D, d = idx % D;
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kW; ++w) M = fmaxf(M, mg_m[w * GQ + h]);
    float num = 0.f, den = 0.f;
    if (M != kNegInf) {
#pragma unroll
      for (int w = 0; w < kW; ++w) {
        const float mw = mg_m[w * GQ + h];
        if (mw == kNegInf) continue;
        const float sc = exp2f(mw - M);
        num = fmaf(sc, mg_acc[(w * GQ + h) * D + d], num);
        den = fmaf(sc, mg_l[w * GQ + h], den);
      }
    }
    float* P = a.ws + ((b * Hq + (long long)kv * GQ + h) * a.n_split + split) * (D + 2);
    if (d == 0) {
      P[0] = M;
      P[1] = den;
    }
    P[2 + d] = num;
  }
}

template <int D, int BITS, int GQ, typename T>
cudaError_t tc_t(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1) {
  using G = Geo<D, BITS, GQ>;
  static bool configured[128] = {};  // dynamic shared memory opt-in, once per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128 || !configured[dev]) {
    e = cudaFuncSetAttribute(decode_split_tc<D, BITS, GQ, T>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_B);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 128) configured[dev] = true;
  }
  dim3 grid((unsigned)a.n_split, (unsigned)a.units);
  if (e0) cudaEventRecord(e0, s);
  decode_split_tc<D, BITS, GQ, T><<<grid, kW * 32, G::SMEM_B, s>>>(a);
  cudaError_t err = cudaGetLastError();
  if (e1) cudaEventRecord(e1, s);
  return err;
}

template <int D, int BITS, typename T>
cudaError_t tc_g(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1) {
  switch (a.gq) {
    case 1: return tc_t<D, BITS, 1, T>(a, s, e0, e1);
    case 2: return tc_t<D, BITS, 2, T>(a, s, e0, e1);
    case 4: return tc_t<D, BITS, 4, T>(a, s, e0, e1);
    case 8: return tc_t<D, BITS, 8, T>(a, s, e0, e1);
  }
  return cudaErrorInvalidValue;
}

template <int BITS, typename T>
cudaError_t tc_d(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1) {
  switch (a.D) {
    case 32: return tc_g<32, BITS, T>(a, s, e0, e1);
    case 64: return tc_g<64, BITS, T>(a, s, e0, e1);
    case 128: return tc_g<128, BITS, T>(a, s, e0, e1);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                             cudaEvent_t e1) {
  if (a.bits == 2 && a.dtype == 0) return tc_d<2, __half>(a, s, e0, e1);
  if (a.bits == 2 && a.dtype == 1) return tc_d<2, float>(a, s, e0, e1);
  if (a.bits == 4 && a.dtype == 0) return tc_d<4, __half>(a, s, e0, e1);
  if (a.bits == 4 && a.dtype == 1) return tc_d<4, float>(a, s, e0, e1);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
