// kivi_decode_tc.cu -- split-context decode attention over the packed KIVI
// cache with both contractions on tensor cores (mma.sync, fp16 operands,
// fp32 accumulation), the split merge fused in.
//
// Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache",
// study.space summary: decode attention runs over the quantized ("grouped")
// part and is combined with the full-precision residual part; mlsanity.com
// index page, "Abstract (arXiv)": loading the cache bounds decode.  Both parts
// enter one online softmax; each CTA writes (m, l, acc[D]) per query head to
// the workspace and the last CTA of the unit merges the splits.
//
// Per CTA: one (batch, KV head) unit and a contiguous range of 32-token tiles
// (one key group each), all query heads of the GQA group.  The last split of
// a unit owns the residual window and runs on CUDA cores; every other split
// streams its tiles:
//   * memory: a producer warp issues 1-D bulk copies (cp.async.bulk,
//     completion on a "full" mbarrier) of each stage -- NW tiles of key
//     codes, key scales, key zeros, value codes, value scales, value zeros,
//     six contiguous ranges -- into a ring of shared-memory stages; NW
//     consumer warps take one tile each and release the stage on an "empty"
//     mbarrier.  No CTA-wide barrier in the streaming loop.  The grid is
//     exactly the CTAs that fit at once (persistent).
//   * scores: S = K q'^T on tensor cores: key codes as the A operand
//     (16 tokens x 16 channels per mma), taken from one 32-bit word per token
//     by a shift and a mask -- a code c in the low mantissa bits of an fp16
//     is the exact subnormal c * 2^-24, so no conversion is needed and 2^24
//     is restored on the fp32 result; q'_{h,d} = q_{h,d} s_{g,d} split into
//     fp16 hi and lo columns of B.  score = 2^24 S + sum_d q_d z_{g,d}.
//   * softmax: running max and sum in log2 units (q pre-scaled by
//     softmax_scale * log2 e, exp2f).
//   * values: O += V^T p' on tensor cores, value codes as the A operand
//     (16 channels x 16 tokens, same shift-and-mask), p'_{t,h} =
//     p_{t,h} s_{t,j} split into hi and lo columns of B; the zero enters as
//     sum_t p_t z_{t,j} per value group.
// The q' and p' fragments are built cooperatively (each lane converts a few
// values and stores them in fragment order in per-warp shared memory).  The
// channel (key) and token (value) order inside an mma k-slice follows the
// bit order of the words.
#include "kivi_internal.cuh"

namespace kivi {
namespace {

constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kTwo24 = 16777216.0f;
constexpr long long kWaitCycles = 1LL << 32;  // ~2 s: bounded wait on our own copies

// NW consumer warps (one 32-token tile each per stage) and one producer warp
// per CTA.  Measured on B200: one query head per KV head runs best as three
// 4-warp CTAs per SM (124 registers); grouped heads need ~160 registers per
// thread and run best as one CTA per SM with 11 (GQ 2, 4) or 7 (GQ 8)
// consumer warps sharing one ring.
template <int D, int BITS, int GQ>
struct Geo {
  static constexpr int NW = GQ == 1 ? 4 : (GQ == 8 ? 7 : 11);
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr int kStage = NW;             // tiles per pipeline stage
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
  static constexpr int NSTAGE = NW == 4 ? (BITS == 2 ? 3 : 2) : 2;
  static constexpr int NPB = GQ == 8 ? 2 : 1;          // hi/lo in separate B operands
  // per-warp scratch (bytes)
  static constexpr int QB_B = NPB * KSL * 32 * 8;      // q' B fragments (score product)
  static constexpr int PB_B = NPB * NJ * 2 * 32 * 8;   // p' B fragments (value product)
  static constexpr int PBUF_B = GQ * kTile * 4;        // p per head and token
  static constexpr int WARP_B = QB_B + PB_B + PBUF_B;
  // whole CTA
  static constexpr int O_WARP = NSTAGE * STAGE_B;
  static constexpr int O_QS = O_WARP + NW * WARP_B;    // q (fp32, scaled) for the window path
  static constexpr int O_MG = O_QS + GQ * D * 4;       // per-warp (m, l, acc[D]) for the merge
  static constexpr int O_BAR = O_MG + NW * GQ * (D + 2) * 4;  // full[NSTAGE], empty[NSTAGE]
  static constexpr int O_FLAG = O_BAR + 2 * NSTAGE * 8;
  static constexpr int SMEM_B = O_FLAG + 16;
  static_assert(SMEM_B <= 227 * 1024, "shared memory per CTA");
  static constexpr int MIN_CTAS = NW == 4 ? 3 : 1;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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
// Wait for a phase; gives up (returns false) after kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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

// Two fp16 codes (exact subnormals c * 2^-24) per register: k-pairs tq, tq+4.
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

// Column of the fragment B operands (q' and p') that holds the hi or lo part
// of head h: GQ <= 4 packs hi in columns 0..3 and lo in 4..7 of one
// operand; GQ == 8 uses two operands (hi, lo) with column h each.
template <int GQ>
__device__ __forceinline__ int col_of(int h, int lo) { return GQ == 8 ? h : h + 4 * lo; }

// Consumer-only barrier (the producer warp keeps streaming meanwhile).
template <int NW>
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
}

template <int D, int BITS, int GQ, typename T>
__global__ void __launch_bounds__(Geo<D, BITS, GQ>::THREADS, Geo<D, BITS, GQ>::MIN_CTAS)
    decode_stream_tc(DecodeArgs a) {
  using G = Geo<D, BITS, GQ>;
  constexpr int kW = G::NW;
  constexpr int kThreads = G::THREADS;
  constexpr int kStage = G::kStage;
  (void)kThreads;
  using Lt = Layout<D, BITS>;
  constexpr int E = G::E, WK = G::WK, NJ = G::NJ, KSL = G::KSL;
  constexpr int NM = D / 16;  // value m-tiles (16 channels each)
  constexpr int NPB = G::NPB;
  constexpr int CPL = D / 32;  // window path: channels per lane
  extern __shared__ __align__(128) unsigned char smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int cta = blockIdx.x;
  const int Hq = a.Hkv * GQ;
  const CacheView& c = a.c;

  float* qs = reinterpret_cast<float*>(smem + G::O_QS);
  float* mg_m = reinterpret_cast<float*>(smem + G::O_MG);  // [kW][GQ]
  float* mg_l = mg_m + kW * GQ;                              // [kW][GQ]
  float* mg_acc = mg_l + kW * GQ;                            // [kW][GQ][D]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::O_BAR);
  uint64_t* empty = full + G::NSTAGE;
  int* flag = reinterpret_cast<int*>(smem + G::O_FLAG);  // [0] abort, [1] merge flag

  const long long n_qt = a.n_q / kTile;
  const long long UP = n_qt + a.win_weight;  // work indices per unit
  const long long total = (long long)a.units * UP;
  const long long W = a.tiles_per_cta;
  const long long G0 = (long long)cta * W;
  const long long G1 = min(total, G0 + W);

  if (tid == 0) {
    for (int s = 0; s < G::NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kW);
    }
    flag[0] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp < kW) {
    unsigned char* wb = smem + G::O_WARP + warp * G::WARP_B;
    for (int i = lane; i < (G::QB_B + G::PB_B) / 4; i += 32) reinterpret_cast<uint32_t*>(wb)[i] = 0u;
  }
  __syncthreads();

  if (warp == kW) {
    // ---------------- producer warp: one thread streams this CTA's stages
    if (lane == 0 && G0 < G1) {
      long long st = 0;
      for (long long u = G0 / UP; u <= (G1 - 1) / UP; ++u) {
        const long long base = u * UP;
        if (cta < base / W || cta > (base + n_qt) / W) continue;  // no work of u here
        const long long t_end = min(G1 - base, n_qt);
        const uint32_t* kc_u = c.k_codes + u * Lt::k_codes_unit(c.Tq);
        const float* ks_u = c.k_scale + u * Lt::k_meta_unit(c.Tq);
        const float* kz_u = c.k_zero + u * Lt::k_meta_unit(c.Tq);
        const uint32_t* vc_u = c.v_codes + u * Lt::v_codes_unit(c.Tq);
        const float* vs_u = c.v_scale + u * Lt::v_meta_unit(c.Tq);
        const float* vz_u = c.v_zero + u * Lt::v_meta_unit(c.Tq);
        for (long long t0 = max(G0 - base, 0ll); t0 < t_end; t0 += kStage, ++st) {
          const int s = (int)(st % G::NSTAGE);
          if (st >= G::NSTAGE &&
              !mbar_wait(&empty[s], (uint32_t)(((st / G::NSTAGE) - 1) & 1))) {
            atomicExch(&flag[0], 1);
            break;
          }
          if (*(volatile int*)&flag[0]) break;
          unsigned char* buf = smem + s * G::STAGE_B;
          const int n = (int)min((long long)kStage, t_end - t0);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_expect_tx(&full[s], (uint32_t)(n * G::TILE_B));
          bulk_copy(buf + G::O_KC, kc_u + t0 * kTile * WK, n * G::KC_B, &full[s]);
          bulk_copy(buf + G::O_KS, ks_u + t0 * D, n * G::KM_B, &full[s]);
          bulk_copy(buf + G::O_KZ, kz_u + t0 * D, n * G::KM_B, &full[s]);
          bulk_copy(buf + G::O_VC, vc_u + t0 * (kTile / E) * D, n * G::VC_B, &full[s]);
          bulk_copy(buf + G::O_VS, vs_u + t0 * kTile * NJ, n * G::VM_B, &full[s]);
          bulk_copy(buf + G::O_VZ, vz_u + t0 * kTile * NJ, n * G::VM_B, &full[s]);
        }
        if (*(volatile int*)&flag[0]) break;
        if (a.r > 0 && cta == (base + n_qt) / W) {
          // this CTA owns the unit's residual window: pull it into L2 while
          // the consumers work through the unit's last stages
          const uint32_t wbytes = (uint32_t)((size_t)a.r * D * sizeof(T));
          const T* kr = reinterpret_cast<const T*>(c.k_res) + u * c.R * D;
          const T* vr = reinterpret_cast<const T*>(c.v_res) + u * c.R * D;
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(kr), "r"(wbytes) : "memory");
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(vr), "r"(wbytes) : "memory");
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- consumer warps
    unsigned char* wb = smem + G::O_WARP + warp * G::WARP_B;
    uint32_t* qB = reinterpret_cast<uint32_t*>(wb);
    __half* qBh = reinterpret_cast<__half*>(wb);
    uint32_t* pB = reinterpret_cast<uint32_t*>(wb + G::QB_B);
    __half* pBh = reinterpret_cast<__half*>(wb + G::QB_B);
    float* pbuf = reinterpret_cast<float*>(wb + G::QB_B + G::PB_B);

    // score-side head pair of this lane: hA = 2*(tq & 1) (GQ <= 4) or 2*tq
    // (GQ == 8), and hA + 1; the P.V accumulator columns 2tq, 2tq+1 hold the
    // same two heads (hi or lo part)
    const int hA = GQ == 8 ? 2 * tq : 2 * (tq & 1);
    const int hB = hA + 1;
    const bool vA = hA < GQ, vB = hB < GQ;
    const bool owner = (GQ == 8 || tq < 2);  // lanes whose columns are the hi parts
    constexpr float kCodeScale = kTwo24;  // codes enter the mma as c * 2^-24

    long long st = 0;  // ring position, in step with the producer
    for (long long u = G0 / UP; G0 < G1 && u <= (G1 - 1) / UP; ++u) {
      const long long base = u * UP;
      // CTAs f_cta..l_cta cover the unit's tiles and its window start index;
      // l_cta owns the window
      const long long f_cta = base / W;
      const long long l_cta = (base + n_qt) / W;
      if (cta < f_cta || cta > l_cta) continue;
      const long long b = u / a.Hkv;
      const int kv = (int)(u % a.Hkv);
      const T* qg = reinterpret_cast<const T*>(a.q) + (b * Hq + (long long)kv * GQ) * D;
      const long long t_beg = max(G0 - base, 0ll);
      const long long t_end = min(G1 - base, n_qt);
      const int slot = (int)(cta - f_cta);
      const int n_seg = (int)(l_cta - f_cta + 1);
      const bool window_owner = a.r > 0 && cta == l_cta;

      float qv[GQ][NJ];  // q for the cooperative q' build: channels lane + 32 i
#pragma unroll
      for (int h = 0; h < GQ; ++h)
#pragma unroll
        for (int i = 0; i < NJ; ++i) qv[h][i] = to_f32(qg[h * D + lane + 32 * i]) * a.qscale;
      if (window_owner)
        for (int i = tid; i < GQ * D; i += kW * 32) qs[i] = to_f32(qg[i]) * a.qscale;

      float m_run[2] = {kNegInf, kNegInf}, l_part[2] = {0.f, 0.f};
      float bv[GQ][NJ];  // sum_t p z per (head, value group), lane partial (token = lane)
      float acc[NPB][NM][4];
#pragma unroll
      for (int h = 0; h < GQ; ++h)
#pragma unroll
        for (int j = 0; j < NJ; ++j) bv[h][j] = 0.f;
#pragma unroll
      for (int p = 0; p < NPB; ++p)
#pragma unroll
        for (int m = 0; m < NM; ++m)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[p][m][e] = 0.f;

      for (long long t0 = t_beg; t0 < t_end; t0 += kStage, ++st) {
        const int s = (int)(st % G::NSTAGE);
        const bool ok = mbar_wait(&full[s], (uint32_t)((st / G::NSTAGE) & 1));
        if (!__all_sync(0xffffffffu, ok) || *(volatile int*)&flag[0]) {
          if (lane == 0) atomicExch(&flag[0], 1);
          break;
        }
        const unsigned char* buf = smem + s * G::STAGE_B;
        if (t0 + warp < t_end) {
          const uint32_t* kc = reinterpret_cast<const uint32_t*>(buf + G::O_KC) + warp * kTile * WK;
          const float* ks = reinterpret_cast<const float*>(buf + G::O_KS) + warp * D;
          const float* kz = reinterpret_cast<const float*>(buf + G::O_KZ) + warp * D;
          const uint32_t* vc =
              reinterpret_cast<const uint32_t*>(buf + G::O_VC) + warp * (kTile / E) * D;
          const float* vs = reinterpret_cast<const float*>(buf + G::O_VS) + warp * kTile * NJ;
          const float* vz = reinterpret_cast<const float*>(buf + G::O_VZ) + warp * kTile * NJ;

          // -- q' = q * s (this key group): hi/lo fp16 in B-fragment order; bias = q . z
          float bk[GQ];
#pragma unroll
          for (int h = 0; h < GQ; ++h) bk[h] = 0.f;
#pragma unroll
          for (int i = 0; i < NJ; ++i) {
            const int ch = lane + 32 * i;
            const float sv = ks[ch], zv = kz[ch];
            int t4, kp, hf;
            slot_of<BITS>(ch & 15, t4, kp, hf);
            const int sl = ch >> 4;
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
              bk[h] = fmaf(qv[h][i], zv, bk[h]);
              __half hi, lo;
              split_f16(qv[h][i] * sv, hi, lo);
              const int ih = ((sl * 32 + col_of<GQ>(h, 0) * 4 + t4) * 2 + kp) * 2 + hf;
              const int il = ((sl * 32 + col_of<GQ>(h, 1) * 4 + t4) * 2 + kp) * 2 + hf;
              qBh[ih] = hi;
              qBh[il + (NPB == 2 ? KSL * 32 * 4 : 0)] = lo;
            }
          }
          float bkA = 0.f, bkB = 0.f;
#pragma unroll
          for (int h = 0; h < GQ; ++h) {
            bk[h] = warp_sum(bk[h]);
            if (h == hA) bkA = bk[h];
            if (h == hB) bkB = bk[h];
          }
          __syncwarp();

          // -- scores: 2 m-tiles of 16 tokens (rows g, g+8), KSL k-slices
          float dq[NPB][2][4];
#pragma unroll
          for (int p = 0; p < NPB; ++p)
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
              for (int e = 0; e < 4; ++e) dq[p][mt][e] = 0.f;
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const uint32_t* r0 = kc + (16 * mt + g) * WK;
            const uint32_t* r1 = kc + (16 * mt + g + 8) * WK;
            uint32_t w0[WK], w1[WK];
#pragma unroll
            for (int w = 0; w < WK; w += 2) {
              const uint2 x0 = *reinterpret_cast<const uint2*>(r0 + w);
              const uint2 x1 = *reinterpret_cast<const uint2*>(r1 + w);
              w0[w] = x0.x;
              w0[w + 1] = x0.y;
              w1[w] = x1.x;
              w1[w + 1] = x1.y;
            }
#pragma unroll
            for (int sl = 0; sl < KSL; ++sl) {
              uint32_t a0, a1, a2, a3;
              if (BITS == 2) {
                codes_pair<2>(w0[sl], 0u, tq, a0, a2);
                codes_pair<2>(w1[sl], 0u, tq, a1, a3);
              } else {
                codes_pair<4>(w0[2 * sl], w0[2 * sl + 1], tq, a0, a2);
                codes_pair<4>(w1[2 * sl], w1[2 * sl + 1], tq, a1, a3);
              }
#pragma unroll
              for (int p = 0; p < NPB; ++p) {
                const uint2 bb =
                    *reinterpret_cast<const uint2*>(qB + p * KSL * 32 * 2 + (sl * 32 + lane) * 2);
                mma16816(dq[p][mt], a0, a1, a2, a3, bb.x, bb.y);
              }
            }
          }

          // -- hi + lo, bias: lane holds heads hA (col 2tq) and hB (col 2tq+1)
          // for tokens 16mt + g (e = 0,1) and 16mt + g + 8 (e = 2,3)
          float sc[2][4];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float v = dq[0][mt][e];
              if (NPB == 2) v += dq[NPB - 1][mt][e];
              else v += __shfl_xor_sync(0xffffffffu, v, 2);
              const int hh = e & 1, ti = mt * 2 + (e >> 1);
              sc[hh][ti] = fmaf(v, kCodeScale, hh ? bkB : bkA);
            }
          // -- online softmax per head over the tile's 32 tokens (8 lanes x 4)
          float alpha[2], p[2][4];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float tm = fmaxf(fmaxf(sc[hh][0], sc[hh][1]), fmaxf(sc[hh][2], sc[hh][3]));
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
            const float mn = fmaxf(m_run[hh], tm);
            alpha[hh] = exp2f(m_run[hh] - mn);
            float ps = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              p[hh][i] = exp2f(sc[hh][i] - mn);
              ps += p[hh][i];
            }
            l_part[hh] = fmaf(l_part[hh], alpha[hh], ps);
            m_run[hh] = mn;
          }
          if (owner) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int tok = 16 * (i >> 1) + g + 8 * (i & 1);
              if (vA) pbuf[hA * kTile + tok] = p[0][i];
              if (vB) pbuf[hB * kTile + tok] = p[1][i];
            }
          }
          // rescale the P.V accumulators only if a running max moved
          if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
            for (int q2 = 0; q2 < NPB; ++q2)
#pragma unroll
              for (int m = 0; m < NM; ++m) {
                acc[q2][m][0] *= alpha[0];
                acc[q2][m][1] *= alpha[1];
                acc[q2][m][2] *= alpha[0];
                acc[q2][m][3] *= alpha[1];
              }
          }
          // per-head alpha for the lane-partial value bias (heads live in lanes 0..3)
          float al[GQ];
#pragma unroll
          for (int h = 0; h < GQ; ++h)
            al[h] = __shfl_sync(0xffffffffu, (h & 1) ? alpha[1] : alpha[0], h >> 1);
          __syncwarp();

          // -- p' = p * s_v (hi/lo, B-fragment order); bias_v += p * z_v
          {
            const int t = lane;
            int t4, kp, hf;
            slot_of<BITS>(t & 15, t4, kp, hf);
            const int Hs = t >> 4;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
              const float sv = vs[t * NJ + j], zv = vz[t * NJ + j];
#pragma unroll
              for (int h = 0; h < GQ; ++h) {
                const float ph = pbuf[h * kTile + t];
                bv[h][j] = fmaf(ph, zv, bv[h][j] * al[h]);
                __half hi, lo;
                split_f16(ph * sv, hi, lo);
                const int ih = (((j * 2 + Hs) * 32 + col_of<GQ>(h, 0) * 4 + t4) * 2 + kp) * 2 + hf;
                const int il = (((j * 2 + Hs) * 32 + col_of<GQ>(h, 1) * 4 + t4) * 2 + kp) * 2 + hf;
                pBh[ih] = hi;
                pBh[il + (NPB == 2 ? NJ * 2 * 32 * 4 : 0)] = lo;
              }
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
                const uint4 x0 = *reinterpret_cast<const uint4*>(vc + (2 * Hs) * D + 32 * j + 4 * g);
                const uint4 x1 =
                    *reinterpret_cast<const uint4*>(vc + (2 * Hs + 1) * D + 32 * j + 4 * g);
                codes_pair<4>(x0.x, x1.x, tq, A0[0], A0[2]);
                codes_pair<4>(x0.y, x1.y, tq, A0[1], A0[3]);
                codes_pair<4>(x0.z, x1.z, tq, A1[0], A1[2]);
                codes_pair<4>(x0.w, x1.w, tq, A1[1], A1[3]);
              }
#pragma unroll
              for (int q2 = 0; q2 < NPB; ++q2) {
                const uint2 bb = *reinterpret_cast<const uint2*>(
                    pB + q2 * (NJ * 2 * 32 * 2) + ((j * 2 + Hs) * 32 + lane) * 2);
                mma16816(acc[q2][2 * j], A0[0], A0[1], A0[2], A0[3], bb.x, bb.y);
                mma16816(acc[q2][2 * j + 1], A1[0], A1[1], A1[2], A1[3], bb.x, bb.y);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      const bool failed = *(volatile int*)&flag[0] != 0;

      // ---- this warp's streamed state -> mg slot `warp`
      {
        float lt[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v = l_part[hh];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          lt[hh] = v;
        }
#pragma unroll
        for (int h = 0; h < GQ; ++h)
#pragma unroll
          for (int j = 0; j < NJ; ++j) bv[h][j] = warp_sum(bv[h][j]);
        if (g == 0 && owner) {
          if (vA) {
            mg_m[warp * GQ + hA] = m_run[0];
            mg_l[warp * GQ + hA] = lt[0];
          }
          if (vB) {
            mg_m[warp * GQ + hB] = m_run[1];
            mg_l[warp * GQ + hB] = lt[1];
          }
        }
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const int j = m >> 1, mm = m & 1;
          const int ch0 = 32 * j + 4 * g + 2 * mm;
          float v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[e] = acc[0][m][e];
            if (NPB == 2) v[e] += acc[NPB - 1][m][e];
            else v[e] += __shfl_xor_sync(0xffffffffu, v[e], 2);
          }
          if (owner) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int h = (e & 1) ? hB : hA;
              const int ch = ch0 + (e >> 1);
              if (h < GQ) {
                float bias = 0.f;
#pragma unroll
                for (int hh = 0; hh < GQ; ++hh)
                  if (hh == h) bias = bv[hh][j];
                mg_acc[(warp * GQ + h) * D + ch] = fmaf(v[e], kCodeScale, bias);
              }
            }
          }
        }
      }
      __syncwarp();

      // ---- residual window (CTA that ends the unit): warp w takes window
      // tiles w, w+4, ... on CUDA cores, folded into its mg slot
      if (window_owner && !failed) {
        consumers_sync<kW>();  // qs written by all consumer threads
        const T* kr = reinterpret_cast<const T*>(c.k_res) + u * c.R * D;
        const T* vr = reinterpret_cast<const T*>(c.v_res) + u * c.R * D;
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
        constexpr int VEC = 16 / (int)sizeof(T);  // elements per 16-byte load
        for (int wt = warp; wt < nwt; wt += kW) {
          const int t_in = wt * kTile + lane;
          const int nt = min(kTile, a.r - wt * kTile);
          float lg[GQ];
#pragma unroll
          for (int h = 0; h < GQ; ++h) lg[h] = 0.f;
          if (t_in < a.r) {
            // lane = token: its key row, 16 bytes per load, 8 loads in flight
            const uint4* row = reinterpret_cast<const uint4*>(kr + (long long)t_in * D);
            constexpr int NV = D / VEC;
            constexpr int CH = NV < 8 ? NV : 8;
#pragma unroll
            for (int v0 = 0; v0 < NV; v0 += CH) {
              uint4 raw[CH];
#pragma unroll
              for (int v = 0; v < CH; ++v) raw[v] = row[v0 + v];
#pragma unroll
              for (int v = 0; v < CH; ++v) {
                const T* e = reinterpret_cast<const T*>(&raw[v]);
#pragma unroll
                for (int x4 = 0; x4 < VEC; x4 += 4) {
#pragma unroll
                  for (int h = 0; h < GQ; ++h) {
                    const float4 q4 = *reinterpret_cast<const float4*>(&qs[h * D + (v0 + v) * VEC + x4]);
                    lg[h] = fmaf(q4.x, to_f32(e[x4]), lg[h]);
                    lg[h] = fmaf(q4.y, to_f32(e[x4 + 1]), lg[h]);
                    lg[h] = fmaf(q4.z, to_f32(e[x4 + 2]), lg[h]);
                    lg[h] = fmaf(q4.w, to_f32(e[x4 + 3]), lg[h]);
                  }
                }
              }
            }
          } else {
#pragma unroll
            for (int h = 0; h < GQ; ++h) lg[h] = kNegInf;
          }
          float pw[GQ];
#pragma unroll
          for (int h = 0; h < GQ; ++h) {
            const float mt = warp_max(lg[h]);
            const float mn = fmaxf(wm[h], mt);
            const float al = exp2f(wm[h] - mn);
            pw[h] = exp2f(lg[h] - mn);
            wl[h] = fmaf(wl[h], al, pw[h]);
#pragma unroll
            for (int k = 0; k < CPL; ++k) wacc[h][k] *= al;
            wm[h] = mn;
          }
          // lane = channels d0..d0+CPL-1; NX token rows in flight
          constexpr int NX = GQ >= 4 ? 4 : 8;
          for (int t8 = 0; t8 < nt; t8 += NX) {
            float vf[NX][CPL];
#pragma unroll
            for (int x = 0; x < NX; ++x) {
              const int t = t8 + x;
              const T* row = vr + (long long)(wt * kTile + min(t, nt - 1)) * D + d0;
              if (CPL * sizeof(T) == 16) {
                const uint4 raw = *reinterpret_cast<const uint4*>(row);
                const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
                for (int k = 0; k < CPL; ++k) vf[x][k] = to_f32(e[k]);
              } else if (CPL * sizeof(T) == 8) {
                const uint2 raw = *reinterpret_cast<const uint2*>(row);
                const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
                for (int k = 0; k < CPL; ++k) vf[x][k] = to_f32(e[k]);
              } else {
#pragma unroll
                for (int k = 0; k < CPL; ++k) vf[x][k] = to_f32(row[k]);
              }
            }
#pragma unroll
            for (int x = 0; x < NX; ++x) {
#pragma unroll
              for (int h = 0; h < GQ; ++h) {
                const float pt = __shfl_sync(0xffffffffu, pw[h], (t8 + x) & 31);
                if (t8 + x < nt) {
#pragma unroll
                  for (int k = 0; k < CPL; ++k) wacc[h][k] = fmaf(pt, vf[x][k], wacc[h][k]);
                }
              }
            }
          }
        }
        // fold the window state into this warp's slot (same warp wrote it)
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          const float lw = warp_sum(wl[h]);
          const float m1 = mg_m[warp * GQ + h];
          const float mn = fmaxf(m1, wm[h]);
          const float s1 = m1 == kNegInf ? 0.f : exp2f(m1 - mn);
          const float s2 = wm[h] == kNegInf ? 0.f : exp2f(wm[h] - mn);
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            float* x = &mg_acc[(warp * GQ + h) * D + d0 + k];
            *x = *x * s1 + wacc[h][k] * s2;
          }
          __syncwarp();
          if (lane == 0) {
            mg_l[warp * GQ + h] = mg_l[warp * GQ + h] * s1 + lw * s2;
            mg_m[warp * GQ + h] = mn;
          }
          __syncwarp();
        }
      }
      consumers_sync<kW>();

      // ---- merge the warps, write this CTA's partial for unit u
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
            const float s2 = exp2f(mw - M);
            num = fmaf(s2, mg_acc[(w * GQ + h) * D + d], num);
            den = fmaf(s2, mg_l[w * GQ + h], den);
          }
        }
        float* P = a.ws + ((u * a.max_seg + slot) * GQ + h) * (D + 2);
        if (failed) {
          M = 0.f;
          den = kNaN;
          num = kNaN;
        }
        if (d == 0) {
          P[0] = M;
          P[1] = den;
        }
        P[2 + d] = num;
      }
      // ---- arrival; the last segment of the unit merges all its partials
      __threadfence();
      consumers_sync<kW>();
      if (tid == 0) {
        unsigned long long* ctr = a.ctr + u;
        const unsigned long long ep = (unsigned long long)a.epoch << 32;
        unsigned long long v = atomicAdd(ctr, 0ull);
        int last = -1;
        for (int it = 0; it < 4096; ++it) {
          const unsigned long long nv = ((v >> 32) == a.epoch) ? v + 1ull : (ep | 1ull);
          const unsigned long long old = atomicCAS(ctr, v, nv);
          if (old == v) {
            last = ((long long)(nv & 0xffffffffull) == (long long)n_seg) ? 1 : 0;
            break;
          }
          v = old;
        }
        flag[1] = last;
      }
      consumers_sync<kW>();
      const int last = flag[1];
      if (last != 0) {
        __threadfence();
        T* out = reinterpret_cast<T*>(a.out);
        for (int idx = tid; idx < GQ * D; idx += kW * 32) {
          const int h = idx / D, d = idx % D;
          const long long row = b * Hq + (long long)kv * GQ + h;
          float res = kNaN;
          if (last > 0) {
            float M = kNegInf;
            for (int sg = 0; sg < n_seg; ++sg)
              M = fmaxf(M, __ldcg(a.ws + ((u * a.max_seg + sg) * GQ + h) * (D + 2)));
            float num = 0.f, den = 0.f;
            for (int sg = 0; sg < n_seg; ++sg) {
              const float* P = a.ws + ((u * a.max_seg + sg) * GQ + h) * (D + 2);
              const float ms = __ldcg(P);
              if (ms == kNegInf) continue;
              const float s2 = exp2f(ms - M);
              num = fmaf(s2, __ldcg(P + 2 + d), num);
              den = fmaf(s2, __ldcg(P + 1), den);
            }
            res = num / den;
          }
          out[row * D + d] = from_f32<T>(res);
        }
      }
      consumers_sync<kW>();  // mg buffers and flag[1] are reused by the next unit
      if (failed) break;
    }
  }
  __syncthreads();
}

// Opt in to the kernel's dynamic shared memory and return how many of its
// CTAs fit on one SM (both once per device).
template <int D, int BITS, int GQ, typename T>
cudaError_t tc_setup(int* ctas_per_sm) {
  using G = Geo<D, BITS, GQ>;
  static int occ[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 128 && occ[dev] > 0) {
    *ctas_per_sm = occ[dev];
    return cudaSuccess;
  }
  e = cudaFuncSetAttribute(decode_stream_tc<D, BITS, GQ, T>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_B);
  if (e != cudaSuccess) return e;
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_stream_tc<D, BITS, GQ, T>,
                                                    G::THREADS, G::SMEM_B);
  if (e != cudaSuccess) return e;
  if (n < 1) return cudaErrorInvalidConfiguration;
  if (dev >= 0 && dev < 128) occ[dev] = n;
  *ctas_per_sm = n;
  return cudaSuccess;
}

template <int D, int BITS, int GQ, typename T>
cudaError_t tc_t(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1,
                 int* ctas_per_sm) {
  using G = Geo<D, BITS, GQ>;
  if (ctas_per_sm) return tc_setup<D, BITS, GQ, T>(ctas_per_sm);
  int occ = 0;
  cudaError_t e = tc_setup<D, BITS, GQ, T>(&occ);
  if (e != cudaSuccess) return e;
  if (e0) cudaEventRecord(e0, s);
  decode_stream_tc<D, BITS, GQ, T><<<a.n_cta, G::THREADS, G::SMEM_B, s>>>(a);
  cudaError_t err = cudaGetLastError();
  if (e1) cudaEventRecord(e1, s);
  return err;
}

template <int D, int BITS, typename T>
cudaError_t tc_g(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1, int* occ) {
  switch (a.gq) {
    case 1: return tc_t<D, BITS, 1, T>(a, s, e0, e1, occ);
    case 2: return tc_t<D, BITS, 2, T>(a, s, e0, e1, occ);
    case 4: return tc_t<D, BITS, 4, T>(a, s, e0, e1, occ);
    case 8: return tc_t<D, BITS, 8, T>(a, s, e0, e1, occ);
  }
  return cudaErrorInvalidValue;
}

template <int BITS, typename T>
cudaError_t tc_d(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1, int* occ) {
  switch (a.D) {
    case 32: return tc_g<32, BITS, T>(a, s, e0, e1, occ);
    case 64: return tc_g<64, BITS, T>(a, s, e0, e1, occ);
    case 128: return tc_g<128, BITS, T>(a, s, e0, e1, occ);
  }
  return cudaErrorInvalidValue;
}

cudaError_t tc_dispatch(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1,
                        int* occ) {
  if (a.bits == 2 && a.dtype == 0) return tc_d<2, __half>(a, s, e0, e1, occ);
  if (a.bits == 2 && a.dtype == 1) return tc_d<2, float>(a, s, e0, e1, occ);
  if (a.bits == 4 && a.dtype == 0) return tc_d<4, __half>(a, s, e0, e1, occ);
  if (a.bits == 4 && a.dtype == 1) return tc_d<4, float>(a, s, e0, e1, occ);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                             cudaEvent_t e1) {
  return tc_dispatch(a, s, e0, e1, nullptr);
}

cudaError_t decode_tc_ctas_per_sm(const DecodeArgs& a, int* ctas_per_sm) {
  return tc_dispatch(a, nullptr, nullptr, nullptr, ctas_per_sm);
}

}  // namespace kivi
