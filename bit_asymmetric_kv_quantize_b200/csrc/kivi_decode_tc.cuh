// kivi_decode_tc.cuh -- split-context decode attention over the packed KIVI
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
// Per CTA: a contiguous range of work indices over (unit, 32-token tile)
// pairs (persistent, stream-K), all query heads of the GQA group.  The CTA
// that ends a unit also folds in the unit's residual window (CUDA cores).
//   * memory: a producer warp issues 1-D bulk copies (cp.async.bulk,
//     completion on a "full" mbarrier) of each stage -- NW tiles of key
//     codes, key scales, key zeros, value codes, value scales, value zeros,
//     six contiguous ranges -- into a ring of shared-memory stages; NW
//     consumer warps take one tile each and release the stage on an "empty"
//     mbarrier.  No CTA-wide barrier in the streaming loop.
//   * codes as fp16 operands: a 2-bit word holds code i at bits 2i, a 4-bit
//     word code i at bits 4i.  A "pair" (two codes, one per 16-bit half) is
//     taken out with a mask after at most one shift, which leaves each code
//     at some bit e < 10 of its half: read as fp16 that is the exact
//     subnormal c * 2^(e - 24).  The other operand's row for that k carries
//     the factor 2^(S - e), so every product is c * x * 2^(S - 24) and the
//     fp32 result is rescaled once by 2^(24 - S).
//   * scores: S = K q'^T, key codes as the A operand (16 tokens x 16
//     channels per mma; lane tq of a row owns the code pairs
//     [tq*D/8, (tq+1)*D/8) of the token), q'_{h,d} = q_{h,d} s_{g,d} split
//     into fp16 hi and lo; head h uses columns 2(h%4) (hi) and 2(h%4)+1 (lo)
//     of n-tile h/4, so each lane's accumulator pair is one head.
//     score = sum_d q'_d c_d + sum_d q_d z_{g,d}.
//   * softmax: running max and sum in log2 units (q pre-scaled by
//     softmax_scale * log2 e, exp2f); the cross-lane max is formed only when
//     some score exceeds the running max (a warp vote), so p <= 1 always.
//   * values: O += V^T p' on tensor cores, value codes as the A operand
//     (16 channels x 16 tokens), p'_{t,h} = p_{t,h} s_{t,j} split into hi and
//     lo columns as above; the zero enters as sum_t p_t z_{t,j}.
// The q' and p' fragments are built cooperatively (each lane converts a few
// values and stores them in fragment order, XOR-swizzled, in per-warp shared
// memory).
// Scales and zeros (template type MT) are binary32, or binary16 in the
// format variant with binary16 metadata; the ring holds them as stored and
// they are widened to fp32 where the q' and p' fragments are built.
#pragma once

#include <cuda.h>
#include <string.h>

#include <mutex>

#include "kivi_internal.cuh"
#include "kivi_quantize_tile.cuh"

namespace kivi {
namespace {

constexpr float kNegInf = -__builtin_huge_valf();
constexpr long long kWaitCycles = 1LL << 32;  // ~2 s: bounded wait on our own copies
constexpr int kSuspendNs = 1000;  // a waiting thread sleeps up to this long per try

// Code pairs of one 32-bit word.  1-bit: pair i (i < 16) = codes i and
// i + 16; 2-bit: pair i (i < 8) = codes i and i + 8; 4-bit: pair i (i < 4) =
// codes i and i + 4.  (w >> shift(i)) & mask(i) puts the pair's codes at bit
// e(i) of the low and the high half.
template <int BITS>
struct Pairs;
template <>
struct Pairs<1> {
  static constexpr int PPW = 16;  // pairs per word
  static constexpr int EMAX = 9;  // largest e
  __host__ __device__ static constexpr int e(int i) { return i < 10 ? i : i - 10; }
  __host__ __device__ static constexpr int shift(int i) { return i < 10 ? 0 : 10; }
  __host__ __device__ static constexpr uint32_t mask(int i) { return 0x00010001u << e(i); }
};
template <>
struct Pairs<2> {
  static constexpr int PPW = 8;   // pairs per word
  static constexpr int EMAX = 8;  // largest e
  __host__ __device__ static constexpr int e(int i) { return i < 5 ? 2 * i : 2 * (i - 5); }
  __host__ __device__ static constexpr int shift(int i) { return i < 5 ? 0 : 10; }
  __host__ __device__ static constexpr uint32_t mask(int i) { return 0x00030003u << e(i); }
};
// 3 bits: a block of 32 codes is three bit-plane words; pair i (i < 16) =
// codes i and i + 16, taken from each plane by the 1-bit rule but with e
// kept below 8 (a shift by 8 for i >= 8), so that the three planes' bits of
// a code land at bits e, e + 1, e + 2 of its half: the exact subnormal
// c 2^(e - 24), c < 8.
template <>
struct Pairs<3> {
  static constexpr int PPW = 16;  // pairs per block
  static constexpr int EMAX = 7;
  __host__ __device__ static constexpr int e(int i) { return i & 7; }
  __host__ __device__ static constexpr int shift(int i) { return i < 8 ? 0 : 8; }
  __host__ __device__ static constexpr uint32_t mask(int i) { return 0x00010001u << e(i); }
};
// The code pair of three bit planes p0, p1, p2 after a right shift by sh,
// placed at bit e of each half by mask m = 0x00010001 << e.
__device__ __forceinline__ uint32_t planes3(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t sh,
                                            uint32_t m) {
  return ((p0 >> sh) & m) | (((p1 >> sh) << 1) & (m << 1)) | (((p2 >> sh) << 2) & (m << 2));
}
template <>
struct Pairs<4> {
  static constexpr int PPW = 4;
  static constexpr int EMAX = 4;
  __host__ __device__ static constexpr int e(int i) { return 4 * (i & 1); }
  __host__ __device__ static constexpr int shift(int i) { return i < 2 ? 0 : 8; }
  __host__ __device__ static constexpr uint32_t mask(int i) { return 0x000F000Fu << e(i); }
};

// NW consumer warps (TPW 32-token tiles each per stage) and one producer
// warp per CTA.  Measured on B200: one query head per KV head runs best as
// 4-warp CTAs, two tiles per warp at 2-bit (two CTAs per SM) and one at 4-bit
// (three per SM); grouped heads run best as one CTA per SM with 11 (GQ 2, 4)
// or 7 (GQ 8) consumer warps sharing one ring.
// SP: the dense-and-sparse variant (kept entries per group; their lists
// ride in the ring beside the codes): four consumer warps, one tile each.
template <int D, int BITS, int GQ, int MB, bool SP = false>
struct Geo {
  static constexpr int NW = SP ? 4 : (GQ == 1 ? 4 : (GQ == 8 ? 7 : 11));
  // tiles per warp and stage (1-bit MHA also needs two to fit a window tile in a stage)
  static constexpr int TPW = (!SP && GQ == 1 && BITS <= 2) ? 2 : 1;
  static constexpr int WB = Layout<D, BITS>::WB;  // words per code block (3: bit planes)
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr int kStage = NW * TPW;       // tiles per pipeline stage
  static constexpr int E = Layout<D, BITS>::E;   // codes per block
  static constexpr int WK = Layout<D, BITS>::WK;  // key words per token
  static constexpr int NJ = D / kGv;     // value groups per token
  static constexpr int KSL = D / 16;     // k-slices of the score product
  static constexpr int NSL = kTile / 16;  // k-slices of the value product
  static constexpr int KC_B = kTile * WK * 4;
  static constexpr int KM_B = D * MB;  // MB: bytes per scale or zero
  static constexpr int VC_B = (kTile / E) * WB * D * 4;
  static constexpr int VM_B = kTile * NJ * MB;
  static constexpr int TILE_B = KC_B + 2 * KM_B + VC_B + 2 * VM_B;
  static constexpr int O_KC = 0;
  static constexpr int O_KS = O_KC + kStage * KC_B;
  static constexpr int O_KZ = O_KS + kStage * KM_B;
  static constexpr int O_VC = O_KZ + kStage * KM_B;
  static constexpr int O_VS = O_VC + kStage * VC_B;
  static constexpr int O_VZ = O_VS + kStage * VM_B;
  // dense-and-sparse lists per tile, slots sized for kMaxOut entries per
  // group: key (token, value) per channel, value (channel, value) per
  // token and value group
  static constexpr int KOI_B = SP ? D * kMaxOut * 4 : 0;
  static constexpr int VOI_B = SP ? kTile * NJ * kMaxOut * 4 : 0;
  static constexpr int O_KOI = O_VZ + kStage * VM_B;
  static constexpr int O_KOV = O_KOI + kStage * KOI_B;
  static constexpr int O_VOI = O_KOV + kStage * KOI_B;
  static constexpr int O_VOV = O_VOI + kStage * VOI_B;
  static constexpr int O_CODE_END = O_VOV + kStage * VOI_B;
  // fp16 residual window through the ring: a window stage holds WT tokens of
  // K, then of V, as 2-D tensor-copy boxes of BW columns (rows of RB bytes)
  // in the hardware's 128-byte (64-byte when D = 32) swizzle
  static constexpr int WT = kTile;
  static constexpr int BW = D < 64 ? D : 64;
  static constexpr int NBX = D / BW;
  static constexpr int RB = BW * 2;
  static constexpr int BOX_B = WT * RB;
  static constexpr int WTILE_B = 2 * NBX * BOX_B;     // one 32-token window tile (K, V)
  // a stage holds kStage code tiles, and at least one window tile
  static constexpr int CODE_STAGE_B = (O_CODE_END + 1023) / 1024 * 1024;
  static constexpr int STAGE_B = CODE_STAGE_B < WTILE_B ? WTILE_B : CODE_STAGE_B;
  static constexpr int MIN_CTAS =
      SP ? ((GQ == 1 && BITS <= 2) ? 2 : 1) : (NW == 4 ? (TPW == 2 ? 2 : 3) : 1);
  static constexpr int NPB = GQ == 8 ? 2 : 1;  // n-tiles of 8 columns (4 heads x hi, lo)
  static constexpr int PST = TPW * kTile + 8;  // p buffer stride per head (floats)
  // B fragment blocks: only the lanes whose column carries a head are kept
  // (fragment column n = lane / 4; GQ heads use columns 0 .. 2 GQ - 1): NLB
  // lanes x 2 words per block, and the swizzle XORs lane bits 2.. with
  // (k-slice & S3M) so that it stays inside the block
  static constexpr int NLB = GQ == 1 ? 8 : (GQ == 2 ? 16 : 32);
  static constexpr int BLKW = 2 * NLB;           // words per block
  static constexpr int S3M = GQ == 1 ? 1 : 3;
  // per-warp scratch (bytes)
  static constexpr int QB_B = NPB * KSL * BLKW * 4;       // q' B fragments (score product)
  static constexpr int PB_B = NPB * NJ * NSL * BLKW * 4;  // p' B fragments (value product)
  static constexpr int PBUF_B = GQ * PST * 4;         // p per head and token
  // dense-and-sparse: score corrections per head and token of the warp's
  // tiles, and the value corrections per head and channel of its unit
  static constexpr int CORR_B = SP ? TPW * GQ * kTile * 4 : 0;
  static constexpr int VCORR_B = SP ? GQ * D * 4 : 0;
  static constexpr int WARP_B = TPW * (QB_B + PB_B) + PBUF_B + CORR_B + VCORR_B;
  // ring depth: three stages where they fit beside MIN_CTAS - 1 other CTAs
  // (228 KB of shared memory per SM, 1 KB of it reserved per CTA), else two:
  // the bytes in flight per SM bound the achieved bandwidth
  static constexpr int REST_B = NW * WARP_B + GQ * D * 4 + NW * GQ * (D + 2) * 4 + 6 * 8 + 16;
  static constexpr int SMEM_LIMIT = 228 * 1024 / MIN_CTAS - 1024;
  static constexpr int NSTAGE = 3 * STAGE_B + REST_B <= SMEM_LIMIT ? 3 : 2;
  // whole CTA
  static constexpr int O_WARP = NSTAGE * STAGE_B;
  static constexpr int O_QS = O_WARP + NW * WARP_B;    // q (fp32, scaled) for the window path
  static constexpr int O_MG = O_QS + GQ * D * 4;       // per-warp (m, l, acc[D]) for the merge
  static constexpr int O_BAR = O_MG + NW * GQ * (D + 2) * 4;  // full[NSTAGE], empty[NSTAGE]
  static constexpr int O_FLAG = O_BAR + 2 * NSTAGE * 8;
  static constexpr int SMEM_B = O_FLAG + 16;
  static_assert(SMEM_B <= 227 * 1024, "shared memory per CTA");
  static_assert(O_BAR % 8 == 0 && WARP_B % 16 == 0, "alignment");
  static_assert(SMEM_B <= SMEM_LIMIT, "MIN_CTAS CTAs fit one SM");
  // key operand: code pairs per lane and row, words a lane loads per row
  static constexpr int PPL = D / 8;
  static constexpr int PPW = Pairs<BITS>::PPW;
  static constexpr bool WHOLE = PPL >= PPW;  // a lane's pairs fill whole words
  static constexpr int NWL = WHOLE ? PPL / PPW : 1;
  // operand scale offsets: the factor 2^(S - e) lies in [2^-S, 2^S]
  static constexpr int SK = Pairs<BITS>::EMAX / 2;
  static constexpr int SV = BITS == 2 ? 3 : 2;  // value e: 1, 3-bit 0..3; 2-bit 0,2,4,6; 4-bit 0,4
  static constexpr int WPS = STAGE_B / WTILE_B;       // window tiles per stage
  static_assert(WPS >= 1, "a window tile fits one ring slot");
  static_assert(WTILE_B % 1024 == 0, "window tiles keep the 1024-byte alignment");
  static_assert(STAGE_B % 1024 == 0, "swizzled boxes start on 1024-byte boundaries");
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
// 2-D tensor copy (no multicast) of one box at element coordinates (x, y)
// into shared memory, completion on an mbarrier.
__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int x, int y,
                                       uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendNs)
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

// D (16x8, fp32) += A (16x16, fp16, row) * B (16x8, fp16, col).  Not volatile:
// no side effects, so the compiler may schedule independent chains together.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 fp16 matrices from shared memory; lanes 8i..8i+7 give the row
// addresses of matrix i.  .trans delivers each matrix transposed.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p))
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p))
               : "memory");
}

__device__ __forceinline__ float load1(const float* p) { return *p; }
__device__ __forceinline__ float load1(const __half* p) { return __half2float(*p); }

__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}

// x = hi + lo in fp16 for two values at once (low half: a, high half: b).
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 f = __half22float2(h);
  hi = h2_bits(h);
  lo = h2_bits(__floats2half2_rn(a - f.x, b - f.y));
}

// Word offset of fragment slot `lane2` (= 4 n + tq) in a B block for k-slice
// `sl`: an XOR swizzle (of lane2's column bits with sl & S3M) that spreads the
// cooperative fragment stores over the banks while each lane still reads a
// contiguous 8 bytes.
template <int S3M>
__device__ __forceinline__ int frag_word(int lane2, int sl) { return 2 * (lane2 ^ (4 * (sl & S3M))); }

// x / y for non-negative x and positive y, by a 32-bit division when both fit
// (the usual case: a few instructions instead of the 64-bit division routine).
__device__ __forceinline__ long long div_ll(long long x, long long y) {
  if (((unsigned long long)x | (unsigned long long)y) >> 32 == 0)
    return (long long)((unsigned)x / (unsigned)y);
  return x / y;
}

// ---- the units of a CTA's work range ---------------------------------------
// A cursor over consecutive units: unit u occupies work indices
// [base, base + up), its quantized tiles first (n_qt of them), then its
// window of r tokens and its end-of-unit weight.  Uniform batches: every unit
// has the same n_qt and r and base = u * up.  Ragged batches: the lengths of
// sequence b (units b * Hkv .. b * Hkv + Hkv - 1) come from its DevState.
struct UnitCur {
  long long u, base, n_qt, up;
  int r;
};

__device__ __forceinline__ SeqLen ragged_len(const DecodeArgs& a, long long b) {
  return seq_len(a.dev_state[b], a.pending != 0, a.c.Tq, a.c.R);
}

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ long long warp_max_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Ragged plan (every lane of the calling warp, same result in every warp):
// total work indices over all units and the stream-K range length W for P
// CTAs (plan_ragged_w).
__device__ __forceinline__ long long ragged_plan(const DecodeArgs& a, bool f16, long long P,
                                                 long long* total, int* max_seg) {
  const int lane = threadIdx.x & 31;
  const long long B = a.units / a.Hkv;
  long long tot = 0, mx = 0;
  for (long long b0 = 0; b0 < B; b0 += 32) {
    if (b0 + lane < B) {
      const SeqLen L = ragged_len(a, b0 + lane);
      tot += unit_work(L.n_q, L.r, f16) * a.Hkv;
      mx = max(mx, L.n_q / kTile);
    }
  }
  tot = warp_sum_ll(tot);
  mx = warp_max_ll(mx);
  *total = tot;
  return plan_ragged_w(tot, mx, P, a.seg_cap, max_seg);
}

// The unit holding work index G0 (every lane of the calling warp).  Returns
// u = units when G0 is past the last unit.
template <bool RAG>
__device__ __forceinline__ UnitCur cur_first(const DecodeArgs& a, bool f16, long long G0,
                                             long long UP, long long n_qt) {
  UnitCur c;
  if constexpr (!RAG) {
    c.u = div_ll(G0, UP);
    c.base = c.u * UP;
    c.n_qt = n_qt;
    c.up = UP;
    c.r = a.r;
    return c;
  } else {
  const int lane = threadIdx.x & 31;
  const long long B = a.units / a.Hkv;
  long long pre = 0;  // work indices of the sequences before this chunk
  for (long long b0 = 0; b0 < B; b0 += 32) {
    const long long b = b0 + lane;
    SeqLen L;
    L.n_q = 0;
    L.r = 0;
    long long w = 0;
    if (b < B) {
      L = ragged_len(a, b);
      w = unit_work(L.n_q, L.r, f16) * a.Hkv;
    }
    long long inc = w;  // inclusive scan over the chunk
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, b < B && G0 < pre + inc);
    if (hit != 0u) {  // the first such lane's sequence holds G0
      const int l = __ffs(hit) - 1;
      const long long e = __shfl_sync(0xffffffffu, pre + inc - w, l);
      const long long nq = __shfl_sync(0xffffffffu, L.n_q, l);
      const int r = __shfl_sync(0xffffffffu, L.r, l);
      c.up = unit_work(nq, r, f16);
      const long long h = (G0 - e) / c.up;
      c.u = (b0 + l) * a.Hkv + h;
      c.base = e + h * c.up;
      c.n_qt = nq / kTile;
      c.r = r;
      return c;
    }
    pre = __shfl_sync(0xffffffffu, pre + inc, 31);
  }
  c.u = a.units;
  c.base = pre;
  c.n_qt = 0;
  c.up = 1;
  c.r = 0;
  return c;
  }
}

// Step to the next unit (any thread; ragged: reads the next sequence's
// lengths at a sequence boundary).
template <bool RAG>
__device__ __forceinline__ void cur_next(const DecodeArgs& a, bool f16, UnitCur& c) {
  c.base += c.up;
  ++c.u;
  if (RAG && c.u < a.units && c.u % a.Hkv == 0) {
    const SeqLen L = ragged_len(a, c.u / a.Hkv);
    c.n_qt = L.n_q / kTile;
    c.r = L.r;
    c.up = unit_work(L.n_q, L.r, f16);
  }
}

// Consumer-only barrier (the producer warp keeps streaming meanwhile).
template <int NW>
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
}

// RAG: ragged batch (per-sequence lengths in dev_state; device-counter mode)
template <int D, int BITS, int GQ, typename T, typename MT, bool RAG, bool SP = false>
__global__ void __launch_bounds__(Geo<D, BITS, GQ, sizeof(MT), SP>::THREADS,
                                  Geo<D, BITS, GQ, sizeof(MT), SP>::MIN_CTAS)
    decode_stream_tc(const DecodeArgs args, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV) {
  using G = Geo<D, BITS, GQ, sizeof(MT), SP>;
  using PR = Pairs<BITS>;
  constexpr int kW = G::NW;
  constexpr int kStage = G::kStage;
  using Lt = Layout<D, BITS>;
  constexpr int E = G::E, WK = G::WK, NJ = G::NJ, KSL = G::KSL, NSL = G::NSL;
  constexpr int NM = D / 16;  // value m-tiles (16 channels each)
  constexpr int NPB = G::NPB;
  constexpr int PST = G::PST;
  constexpr int TPW = G::TPW;
  constexpr int CPL = D / 32;  // window path: channels per lane
  constexpr int BLKW = G::BLKW;  // words per B fragment block
  constexpr int S3M = G::S3M;
  auto fw = [](int lane2, int sl) { return frag_word<S3M>(lane2, sl); };
  constexpr float kKeyOut = (float)(1 << (24 - G::SK));
  constexpr float kValOut = (float)(1 << (24 - G::SV));
  extern __shared__ __align__(1024) unsigned char smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int cta = blockIdx.x;

  // launched with programmatic stream serialization: the CTAs may start
  // while the preceding grid drains; every thread waits for it to complete
  // (and its writes to be visible) before touching global memory, and the
  // next grid may be scheduled as soon as SM room frees up.  Uniform batches
  // with host counters read nothing from global memory to plan, so they set
  // up shared memory first and wait just before the first global access.
  const bool early = !RAG && args.dev_state == nullptr;
  if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  DecodeArgs a = args;
  const bool dev = args.dev_state != nullptr;
  constexpr bool kF16 = sizeof(T) == 2;
  long long total_ragged = 0;
  if constexpr (RAG) {
    // ragged batch: every warp plans from the sequences' own lengths
    int ms = 0;
    a.tiles_per_cta = ragged_plan(a, kF16, gridDim.x, &total_ragged, &ms);
    a.max_seg = ms;
    a.n_split = ms;
    a.win_weight = 1;
    a.n_q = 0;
    a.r = 0;
    a.new_k = nullptr;
  } else if (dev) {
    // device counters as they stand before this step's append; decode the
    // cache after it (a flush first when r was R).  With new_k set this
    // launch performs the append itself (the flush below, the token into
    // window slot r, or slot 0 after a flush); else an earlier launch did.
    const DevState st0 = *args.dev_state;
    if (st0.status != 0 || st0.n_q + st0.r + 1 > args.c.Tq + args.c.R) {
      // cache full: nothing is written and the state says so
      if (args.new_k != nullptr && cta == 0 && threadIdx.x == 0) args.dev_state->status = 1;
      return;
    }
    const bool fl = st0.r == args.c.R;
    a.n_q = fl ? st0.n_q + args.c.R : st0.n_q;
    a.r = fl ? 1 : st0.r + 1;
    a.flush = (fl && args.new_k != nullptr) ? 1 : 0;
    a.new_slot = fl ? 0 : st0.r;
    const StreamPlan pl =
        plan_stream_core(args.units, a.n_q, a.r, sizeof(T) == 2, gridDim.x, args.seg_cap);
    a.tiles_per_cta = pl.W;
    a.win_weight = pl.win_weight;
    a.max_seg = pl.max_seg;
    a.n_split = pl.max_seg;
  }
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
  const long long UP = n_qt + a.win_weight;  // work indices per unit (uniform batches)
  const long long total = RAG ? total_ragged : (long long)a.units * UP;
  const long long W = a.tiles_per_cta;
  const long long G0 = (long long)cta * W;
  const long long G1 = min(total, G0 + W);

  if (tid == 0) {
    for (int s = 0; s < G::NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kW);
    }
    // swizzled window boxes need 1024-byte aligned stages: refuse (abort
    // flag, NaN outputs) rather than read a mis-swizzled layout
    flag[0] = (sizeof(T) == 2 && (smem_u32(smem) & 1023u) != 0) ? 1 : 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (early) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (!RAG && a.flush) {
    // a due window flush folded into this launch: every unit's R window
    // tokens are quantized into the store at positions n_q - R .. n_q - 1
    // (n_q counts them already), the tiles spread over all CTAs and taken by
    // threads 0 .. D-1 of each in the ring's shared memory, which is not in
    // use yet; then a grid barrier (the persistent grid's CTAs are all
    // resident), after which the stream reads those tiles like any other
    uint8_t* ck = smem;
    uint8_t* cv = smem + kTile * D;
    const int wt = c.R / kTile;
    const long long nft = (long long)a.units * wt;
    for (long long f = cta; f < nft; f += gridDim.x) {
      if (tid < D) {
        const long long u = f / wt;
        const int x = (int)(f - u * wt);
        const T* kr = reinterpret_cast<const T*>(c.k_res) + (u * c.R + x * kTile) * D;
        const T* vr = reinterpret_cast<const T*>(c.v_res) + (u * c.R + x * kTile) * D;
        quantize_tile<D, BITS, T, MT, 2>(c, u, kr, vr, a.n_q - c.R + x * kTile, ck, cv);
      }
    }
    // the store's new tiles are read by bulk copies (the async proxy)
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncthreads();
    if (tid == 0 && !grid_barrier(a.ctr + a.units + 1, dev ? 0u : a.epoch, gridDim.x))
      atomicExch(&flag[0], 1);
    __syncthreads();
  }
  if (sizeof(T) == 4 && a.new_k != nullptr) {
    // fused append, fp32 window (read by generic loads after the barrier
    // below): the CTA that owns a unit's window writes the unit's new token
    // into window slot new_slot.  (fp16: the warp that takes the window tile
    // holding the slot patches the token into shared memory and the cache.)
    for (long long u = G0 / UP; G0 < G1 && u <= (G1 - 1) / UP; ++u) {
      if (cta != (u * UP + n_qt) / W) continue;
      T* kr = reinterpret_cast<T*>(c.k_res) + (u * c.R + a.new_slot) * D;
      T* vr = reinterpret_cast<T*>(c.v_res) + (u * c.R + a.new_slot) * D;
      const T* kn = reinterpret_cast<const T*>(a.new_k) + u * D;
      const T* vn = reinterpret_cast<const T*>(a.new_v) + u * D;
      for (int i = tid; i < D; i += G::THREADS) {
        kr[i] = kn[i];
        vr[i] = vn[i];
      }
    }
  }
  __syncthreads();

  if (warp == kW) {
    // ---------------- producer warp: one thread streams this CTA's stages
    const UnitCur cu0 = cur_first<RAG>(a, kF16, G0, UP, n_qt);
    if (lane == 0 && G0 < G1) {
      // ring position: slot rs, its fill round's parity rph; a slot is
      // refilled once the consumers released its previous fill
      int rs = 0;
      uint32_t rph = 0;
      bool rwrap = false;
      auto adv = [&]() {
        if (++rs == G::NSTAGE) {
          rs = 0;
          rph ^= 1u;
          rwrap = true;
        }
      };
      for (UnitCur cu = cu0; cu.u < a.units && cu.base < G1; cur_next<RAG>(a, kF16, cu)) {
        const long long u = cu.u, base = cu.base, n_qt_u = cu.n_qt;
        const int r_u = cu.r;
        const long long f_cta = div_ll(base, W), l_cta = div_ll(base + n_qt_u, W);
        if (cta < f_cta || cta > l_cta) continue;  // no work of u here
        if (l_cta - f_cta + 1 > a.max_seg) {  // (cannot happen: plan bound)
          atomicExch(&flag[0], 1);
          break;
        }
        const long long t_end = min(G1 - base, n_qt_u);
        const long long Ts = store_tokens(c);  // tokens per unit slot of the arrays
        const uint32_t* kc_u = c.k_codes + u * Lt::k_codes_unit(Ts);
        const MT* ks_u = reinterpret_cast<const MT*>(c.k_scale) + u * Lt::k_meta_unit(Ts);
        const MT* kz_u = reinterpret_cast<const MT*>(c.k_zero) + u * Lt::k_meta_unit(Ts);
        const uint32_t* vc_u = c.v_codes + u * Lt::v_codes_unit(Ts);
        const MT* vs_u = reinterpret_cast<const MT*>(c.v_scale) + u * Lt::v_meta_unit(Ts);
        const MT* vz_u = reinterpret_cast<const MT*>(c.v_zero) + u * Lt::v_meta_unit(Ts);
        // paged store: this unit's row of the block table and its head
        const int* pg_row = nullptr;
        int pg_head = 0;
        if constexpr (RAG) {
          if (c.bt != nullptr) {
            pg_row = c.bt + (u / c.Hkv) * c.pps;
            pg_head = (int)(u % c.Hkv);
          }
        }
        for (int t0 = (int)max(G0 - base, 0ll); t0 < (int)t_end; t0 += kStage, adv()) {
          const int s = rs;
          const int n = min(kStage, (int)t_end - t0);
          if (rwrap && !mbar_wait(&empty[s], rph ^ 1u)) {
            atomicExch(&flag[0], 1);
            break;
          }
          if (*(volatile int*)&flag[0]) break;
          unsigned char* buf = smem + s * G::STAGE_B;
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          // dense-and-sparse lists of the stage's tiles (index and value each)
          const uint32_t kl_b = SP ? (uint32_t)(D * c.k_out * 4) : 0u;
          const uint32_t vl_b = SP ? (uint32_t)(kTile * NJ * c.v_out * 4) : 0u;
          mbar_expect_tx(&full[s], (uint32_t)(n * (G::TILE_B + 2 * kl_b + 2 * vl_b)));
          if constexpr (SP) {
            if (kl_b > 0) {
              const long long kl = (u * (Ts / kG) + t0) * D * c.k_out;
              bulk_copy(buf + G::O_KOI, c.k_oi + kl, n * kl_b, &full[s]);
              bulk_copy(buf + G::O_KOV, c.k_ov + kl, n * kl_b, &full[s]);
            }
            if (vl_b > 0) {
              const long long vl = (u * Ts + (long long)t0 * kTile) * NJ * c.v_out;
              bulk_copy(buf + G::O_VOI, c.v_oi + vl, n * vl_b, &full[s]);
              bulk_copy(buf + G::O_VOV, c.v_ov + vl, n * vl_b, &full[s]);
            }
          }
          if (!RAG || c.bt == nullptr) {
            bulk_copy(buf + G::O_KC, kc_u + (long long)t0 * kTile * WK, n * G::KC_B, &full[s]);
            bulk_copy(buf + G::O_KS, ks_u + (long long)t0 * D, n * G::KM_B, &full[s]);
            bulk_copy(buf + G::O_KZ, kz_u + (long long)t0 * D, n * G::KM_B, &full[s]);
            bulk_copy(buf + G::O_VC, vc_u + (long long)t0 * (kTile / E) * G::WB * D, n * G::VC_B,
                      &full[s]);
            bulk_copy(buf + G::O_VS, vs_u + (long long)t0 * kTile * NJ, n * G::VM_B, &full[s]);
            bulk_copy(buf + G::O_VZ, vz_u + (long long)t0 * kTile * NJ, n * G::VM_B, &full[s]);
          } else {
            // paged store: one run of copies per page the stage touches (the
            // single producer thread is on the critical path: one 32-bit
            // division per stage, pages stepped from there)
            const int tpp = c.R / kTile;  // tiles per page
            int lp = (int)t0 / tpp;
            int stl = (int)t0 - lp * tpp;
            for (int o = 0; o < n;) {
              const int pg = lp < c.pps ? pg_row[lp] : -1;
              if (pg < 0 || pg >= c.n_pages) {  // page outside the table or pool
                atomicExch(&flag[0], 1);
                break;
              }
              const long long su = (long long)pg * c.Hkv + pg_head;
              const int run = min(n - o, tpp - stl);
              const uint32_t* kc = c.k_codes + su * Lt::k_codes_unit(Ts);
              const MT* ks = reinterpret_cast<const MT*>(c.k_scale) + su * Lt::k_meta_unit(Ts);
              const MT* kz = reinterpret_cast<const MT*>(c.k_zero) + su * Lt::k_meta_unit(Ts);
              const uint32_t* vc = c.v_codes + su * Lt::v_codes_unit(Ts);
              const MT* vs = reinterpret_cast<const MT*>(c.v_scale) + su * Lt::v_meta_unit(Ts);
              const MT* vz = reinterpret_cast<const MT*>(c.v_zero) + su * Lt::v_meta_unit(Ts);
              bulk_copy(buf + G::O_KC + o * G::KC_B, kc + stl * kTile * WK, run * G::KC_B, &full[s]);
              bulk_copy(buf + G::O_KS + o * G::KM_B, ks + stl * D, run * G::KM_B, &full[s]);
              bulk_copy(buf + G::O_KZ + o * G::KM_B, kz + stl * D, run * G::KM_B, &full[s]);
              bulk_copy(buf + G::O_VC + o * G::VC_B, vc + stl * (kTile / E) * G::WB * D, run * G::VC_B,
                        &full[s]);
              bulk_copy(buf + G::O_VS + o * G::VM_B, vs + stl * kTile * NJ, run * G::VM_B, &full[s]);
              bulk_copy(buf + G::O_VZ + o * G::VM_B, vz + stl * kTile * NJ, run * G::VM_B, &full[s]);
              o += run;
              ++lp;
              stl = 0;
            }
            if (*(volatile int*)&flag[0]) break;
          }
        }
        if (*(volatile int*)&flag[0]) break;
        if (r_u > 0 && cta == l_cta) {
          const T* kr = reinterpret_cast<const T*>(c.k_res) + u * c.R * D;
          const T* vr = reinterpret_cast<const T*>(c.v_res) + u * c.R * D;
          if constexpr (sizeof(T) == 2) {
            // this CTA owns the unit's residual window: stream it through
            // the ring, WT tokens of K and of V per stage
            for (int w0 = 0; w0 < r_u; w0 += G::WT * G::WPS, adv()) {
              const int s = rs;
              if (rwrap && !mbar_wait(&empty[s], rph ^ 1u)) {
                atomicExch(&flag[0], 1);
                break;
              }
              if (*(volatile int*)&flag[0]) break;
              unsigned char* buf = smem + s * G::STAGE_B;
              const int ntile = min(G::WPS, (r_u - w0 + G::WT - 1) / G::WT);
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              mbar_expect_tx(&full[s], (uint32_t)(ntile * G::WTILE_B));
              for (int j = 0; j < ntile; ++j) {
                unsigned char* tb = buf + j * G::WTILE_B;
                const int y = (int)(u * c.R + w0 + j * G::WT);  // row of the [units * R][D] window
#pragma unroll
                for (int bx = 0; bx < G::NBX; ++bx) {
                  tma_2d(tb + bx * G::BOX_B, &tmK, bx * G::BW, y, &full[s]);
                  tma_2d(tb + (G::NBX + bx) * G::BOX_B, &tmV, bx * G::BW, y, &full[s]);
                }
              }
            }
          } else {
            // fp32 window (CUDA-core path): pull it into L2 while the
            // consumers work through the unit's last stages
            const uint32_t wbytes = (uint32_t)((size_t)r_u * D * sizeof(T));
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(kr), "r"(wbytes) : "memory");
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(vr), "r"(wbytes) : "memory");
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- consumer warps
    unsigned char* wb = smem + G::O_WARP + warp * G::WARP_B;
    // fragment columns of absent heads stay zero (after the CTA barrier, so
    // that the producer starts streaming meanwhile)
    for (int i = lane; i < TPW * (G::QB_B + G::PB_B) / 4; i += 32) reinterpret_cast<uint32_t*>(wb)[i] = 0u;
    // dense-and-sparse corrections start at zero (and are left at zero)
    float* corr = reinterpret_cast<float*>(wb + TPW * (G::QB_B + G::PB_B) + G::PBUF_B);  // [TPW][GQ][32]
    float* vcorr = corr + TPW * GQ * kTile;                                               // [GQ][D]
    if constexpr (SP) {
      for (int i = lane; i < (G::CORR_B + G::VCORR_B) / 4; i += 32) corr[i] = 0.f;
    }
    __syncwarp();
    uint32_t* qB = reinterpret_cast<uint32_t*>(wb);                     // [TPW][NPB][KSL][BLKW]
    uint32_t* pB = reinterpret_cast<uint32_t*>(wb + TPW * G::QB_B);     // [TPW][NPB][NJ][NSL][BLKW]
    __half* pBh = reinterpret_cast<__half*>(pB);
    float* pbuf = reinterpret_cast<float*>(wb + TPW * (G::QB_B + G::PB_B));  // [GQ][PST]

    // -- q' build: lane classes.  Head class hc = lane % GL builds heads
    // hc + GL x; within a class, lane index jl = lane / GL takes the
    // "couples" (two adjacent pairs of one owner lane: B registers b0, b1 of
    // k-slice sl for owner tq_o) with tq_o = jl & 3, sl = (jl >> 2) + (8/GL) m.
    constexpr int GL = GQ < 4 ? GQ : 4;
    constexpr int HX = GQ / GL;
    constexpr int MC = (KSL * GL + 7) / 8;
    const int hc = lane % GL, jl = lane / GL;
    int cp_ch[MC];       // first channel c0 of the couple (pairs: c0, c0+1 | c0+PPW, c0+PPW+1)
    int cp_w[MC];        // word offset of the owner's slot for column 0 in block sl
    int cp_s3[MC];       // sl & 3 (swizzle)
    float cp_f0[MC], cp_f1[MC];  // 2^(SK - e) of the two pairs
    bool cp_ok[MC];
#pragma unroll
    for (int m = 0; m < MC; ++m) {
      const int tq_o = jl & 3, sl = (jl >> 2) + (8 / GL) * m;
      cp_ok[m] = sl < KSL;
      const int slc = cp_ok[m] ? sl : 0;
      const int pidx0 = tq_o * G::PPL + 2 * slc;
      const int wd = pidx0 / G::PPW, i0 = pidx0 % G::PPW;
      cp_ch[m] = wd * E + i0;
      cp_s3[m] = slc & S3M;
      cp_w[m] = slc * BLKW + 2 * tq_o;
      cp_f0[m] = __int_as_float((127 + G::SK - PR::e(i0)) << 23);
      cp_f1[m] = __int_as_float((127 + G::SK - PR::e(i0 + 1)) << 23);
    }
    // -- key operand when a lane's PPL pairs are part of one word (2-bit
    // D = 32, 1-bit D = 32, 64): they sit in word tq PPL / PPW, pairs
    // (tq PPL) % PPW + jj -- shifts and masks differ per lane
    constexpr int NKS = G::WHOLE ? 1 : G::PPL;
    uint32_t kS[NKS], kM[NKS];
#pragma unroll
    for (int jj = 0; jj < NKS; ++jj) {
      const int i = (tq * G::PPL) % G::PPW + jj;
      kS[jj] = (uint32_t)PR::shift(i);
      kM[jj] = PR::mask(i);
    }
    // -- value operand: lane tq takes the pairs at e = 2 tq (2-bit) or
    // 4 (tq & 1) (4-bit) of its word; a0 / a1 unshifted, a2 / a3 after >> 8.
    // 1-bit: one word holds the tile's 32 tokens (low half 0..15, high half
    // 16..31); k-slice sl takes tokens 8 sl .. 8 sl + 7 and their +16
    // partners, lane tq the pair at bit tq after a shift by 8 sl (a0 / a1)
    // or 8 sl + 4 (a2 / a3)
    const uint32_t vM = (BITS == 1 || BITS == 3) ? (0x00010001u << tq)
                        : BITS == 2 ? (0x00030003u << (2 * tq))
                                    : ((tq & 1) ? 0x00F000F0u : 0x000F000Fu);
    const int vtw = BITS == 4 ? (tq >> 1) : 0;  // token-word offset of this lane
    // -- p' build, lane = token t: its k-slice, owner slot and e
    int pt_sl, pt_tq, pt_kp, pt_hf, pt_e;
    if (BITS == 1 || BITS == 3) {
      const int i = lane & 15;
      pt_hf = lane >> 4; pt_sl = i >> 3; pt_kp = (i >> 2) & 1; pt_tq = i & 3; pt_e = pt_tq;
    } else if (BITS == 2) {
      const int i = lane & 15;
      pt_sl = lane >> 4; pt_tq = i & 3; pt_kp = (i >> 2) & 1; pt_hf = (i >> 3) & 1; pt_e = 2 * pt_tq;
    } else {
      const int tw = lane >> 3, i = lane & 7;
      pt_sl = tw >> 1; pt_tq = 2 * (tw & 1) + (i & 1); pt_kp = (i >> 1) & 1; pt_hf = (i >> 2) & 1;
      pt_e = 4 * (i & 1);
    }
    const float pt_f = __int_as_float((127 + G::SV - pt_e) << 23);
    const int pt_base = pt_sl * 2 * BLKW + 2 * pt_kp + pt_hf;  // halves, block (0, 0, pt_sl)
    const int pt_s3 = pt_sl & S3M;

    // B-fragment column n = g of this lane carries a head (hi or lo part);
    // lanes of absent heads' columns use zeros without loading them
    const bool bcol = GQ >= 4 || g < 2 * GQ;
    bool vh[NPB];  // this lane's score / accumulator head tq + 4p exists
#pragma unroll
    for (int p = 0; p < NPB; ++p) vh[p] = tq + 4 * p < GQ;

    // ring position, in step with the producer: slot rs, fill parity rph
    int rs = 0;
    uint32_t rph = 0;
    auto adv = [&]() {
      if (++rs == G::NSTAGE) {
        rs = 0;
        rph ^= 1u;
      }
    };
    const UnitCur cu0 = cur_first<RAG>(a, kF16, G0, UP, n_qt);
    for (UnitCur cu = cu0; G0 < G1 && cu.u < a.units && cu.base < G1; cur_next<RAG>(a, kF16, cu)) {
      const long long u = cu.u, base = cu.base, n_qt_u = cu.n_qt;
      const int r_u = cu.r;
      // CTAs f_cta..l_cta cover the unit's tiles and its window start index;
      // l_cta owns the window
      const long long f_cta = div_ll(base, W);
      const long long l_cta = div_ll(base + n_qt_u, W);
      if (cta < f_cta || cta > l_cta) continue;
      if (l_cta - f_cta + 1 > a.max_seg) break;  // (cannot happen: plan bound; producer aborts)
      const long long b = u / a.Hkv;
      const int kv = (int)(u % a.Hkv);
      const T* qg = reinterpret_cast<const T*>(a.q) + (b * Hq + (long long)kv * GQ) * D;
      const long long t_beg = max(G0 - base, 0ll);
      const long long t_end = min(G1 - base, n_qt_u);
      const int slot = (int)(cta - f_cta);
      const int n_seg = (int)(l_cta - f_cta + 1);
      const bool window_owner = r_u > 0 && cta == l_cta;

      // q (scaled by softmax_scale log2 e) at this lane's couple channels,
      // order c0, c0+PPW, c0+1, c0+PPW+1 (b0 low, b0 high, b1 low, b1 high)
      float qf[HX][MC][4];
#pragma unroll
      for (int x = 0; x < HX; ++x)
#pragma unroll
        for (int m = 0; m < MC; ++m) {
          const T* qh = qg + (hc + GL * x) * D + cp_ch[m];
          qf[x][m][0] = to_f32(qh[0]) * a.qscale;
          qf[x][m][1] = to_f32(qh[G::PPW]) * a.qscale;
          qf[x][m][2] = to_f32(qh[1]) * a.qscale;
          qf[x][m][3] = to_f32(qh[G::PPW + 1]) * a.qscale;
        }
      if (window_owner || SP) {
        // (dense-and-sparse: the key corrections read q at any channel)
        for (int i = tid; i < GQ * D; i += kW * 32) qs[i] = to_f32(qg[i]) * a.qscale;
        consumers_sync<kW>();  // qs is read by whichever warps take the window
      }

      float m_run[NPB], l_part[NPB];
      float acc[NPB][NM][4];
      float bv[GQ][NJ];  // sum_t p z per (head, value group), lane partial (lane = token)
#pragma unroll
      for (int p = 0; p < NPB; ++p) {
        m_run[p] = kNegInf;
        l_part[p] = 0.f;
#pragma unroll
        for (int m = 0; m < NM; ++m)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[p][m][e] = 0.f;
      }
#pragma unroll
      for (int h = 0; h < GQ; ++h)
#pragma unroll
        for (int j = 0; j < NJ; ++j) bv[h][j] = 0.f;

      for (int t0 = (int)t_beg; t0 < (int)t_end; t0 += kStage, adv()) {
        if (*(volatile int*)&flag[0]) break;
        const int s = rs;
        const bool ok = mbar_wait(&full[s], rph);
        if (!__all_sync(0xffffffffu, ok) || *(volatile int*)&flag[0]) {
          if (lane == 0) atomicExch(&flag[0], 1);
          break;
        }
        const unsigned char* buf = smem + s * G::STAGE_B;
        const int tw0 = t0 + warp * TPW;  // this warp's first tile
        if (tw0 < (int)t_end) {
          // this warp's TPW tiles; a tile past the end of the segment reuses
          // tile 0's data and is masked out (its scores are -inf, so p = 0)
          bool tv[TPW];
          const uint32_t* kc[TPW];
          const MT* ks[TPW];
          const MT* kz[TPW];
          const uint32_t* vc[TPW];
          const MT* vs[TPW];
          const MT* vz[TPW];
#pragma unroll
          for (int tt = 0; tt < TPW; ++tt) {
            tv[tt] = tw0 + tt < (int)t_end;
            const int ti = warp * TPW + (tv[tt] ? tt : 0);
            kc[tt] = reinterpret_cast<const uint32_t*>(buf + G::O_KC) + ti * kTile * WK;
            ks[tt] = reinterpret_cast<const MT*>(buf + G::O_KS) + ti * D;
            kz[tt] = reinterpret_cast<const MT*>(buf + G::O_KZ) + ti * D;
            vc[tt] = reinterpret_cast<const uint32_t*>(buf + G::O_VC) + ti * (kTile / E) * G::WB * D;
            vs[tt] = reinterpret_cast<const MT*>(buf + G::O_VS) + ti * kTile * NJ;
            vz[tt] = reinterpret_cast<const MT*>(buf + G::O_VZ) + ti * kTile * NJ;
          }

          // -- q' = q s 2^(SK - e) (hi, lo) into the B fragments; bias = q . z
          float bk[TPW][HX];
#pragma unroll
          for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
            for (int x = 0; x < HX; ++x) bk[tt][x] = 0.f;
#pragma unroll
          for (int m = 0; m < MC; ++m) {
            if (!cp_ok[m]) continue;
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
              float sA[2], sB[2], zA[2], zB[2];
              load_meta<2>(ks[tt] + cp_ch[m], sA);
              load_meta<2>(ks[tt] + cp_ch[m] + G::PPW, sB);
              load_meta<2>(kz[tt] + cp_ch[m], zA);
              load_meta<2>(kz[tt] + cp_ch[m] + G::PPW, zB);
              const float s0 = sA[0] * cp_f0[m], s1 = sB[0] * cp_f0[m];
              const float s2 = sA[1] * cp_f1[m], s3 = sB[1] * cp_f1[m];
#pragma unroll
              for (int x = 0; x < HX; ++x) {
                const int h = hc + GL * x;
                uint2 hi, lo;
                split2(qf[x][m][0] * s0, qf[x][m][1] * s1, hi.x, lo.x);
                split2(qf[x][m][2] * s2, qf[x][m][3] * s3, hi.y, lo.y);
                uint32_t* blk = qB + tt * (G::QB_B / 4) + (h >> 2) * KSL * BLKW + cp_w[m];
                const int nh = 2 * (h & 3);
                *reinterpret_cast<uint2*>(blk + 8 * (nh ^ cp_s3[m])) = hi;
                *reinterpret_cast<uint2*>(blk + 8 * ((nh + 1) ^ cp_s3[m])) = lo;
                float t = bk[tt][x];
                t = fmaf(qf[x][m][0], zA[0], t);
                t = fmaf(qf[x][m][1], zB[0], t);
                t = fmaf(qf[x][m][2], zA[1], t);
                t = fmaf(qf[x][m][3], zB[1], t);
                bk[tt][x] = t;
              }
            }
          }
          // sum over the lanes of a head class; lane tq then holds head tq + 4p
#pragma unroll
          for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
            for (int x = 0; x < HX; ++x)
#pragma unroll
              for (int o = GL; o < 32; o <<= 1)
                bk[tt][x] += __shfl_xor_sync(0xffffffffu, bk[tt][x], o);
          __syncwarp();

          // -- scores: per tile 2 m-tiles of 16 tokens (rows g, g+8), KSL k-slices
          uint32_t kw[TPW][2][2][G::NWL * G::WB];
#pragma unroll
          for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                const uint32_t* row = kc[tt] + (16 * mt + 8 * r + g) * WK +
                                      G::WB * (G::WHOLE ? tq * G::NWL : (tq * G::PPL) / G::PPW);
                if constexpr (BITS == 3) {
#pragma unroll
                  for (int x = 0; x < G::NWL * 3; ++x) kw[tt][mt][r][x] = row[x];
                } else if constexpr (G::NWL == 4) {
                  const uint4 v = *reinterpret_cast<const uint4*>(row);
                  kw[tt][mt][r][0] = v.x; kw[tt][mt][r][1] = v.y;
                  kw[tt][mt][r][2] = v.z; kw[tt][mt][r][3] = v.w;
                } else if constexpr (G::NWL == 2) {
                  const uint2 v = *reinterpret_cast<const uint2*>(row);
                  kw[tt][mt][r][0] = v.x; kw[tt][mt][r][1] = v.y;
                } else {
                  kw[tt][mt][r][0] = row[0];
                }
              }
          auto key_reg = [&](const uint32_t (&w)[G::NWL * G::WB], int jj) -> uint32_t {
            if constexpr (BITS == 3) {
              if constexpr (G::WHOLE) {
                const int i = jj % G::PPW, bk = 3 * (jj / G::PPW);
                return planes3(w[bk], w[bk + 1], w[bk + 2], PR::shift(i), PR::mask(i));
              } else {
                return planes3(w[0], w[1], w[2], kS[jj], kM[jj]);
              }
            } else if constexpr (G::WHOLE) {
              const int i = jj % G::PPW;
              return (w[jj / G::PPW] >> PR::shift(i)) & PR::mask(i);
            } else {
              return (w[0] >> kS[jj]) & kM[jj];
            }
          };
          float dq[TPW][NPB][2][4];
#pragma unroll
          for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
            for (int p = 0; p < NPB; ++p)
#pragma unroll
              for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) dq[tt][p][mt][e] = 0.f;
#pragma unroll
          for (int sl = 0; sl < KSL; ++sl) {
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
              uint2 bq[NPB];
#pragma unroll
              for (int p = 0; p < NPB; ++p)
                bq[p] = bcol ? *reinterpret_cast<const uint2*>(qB + tt * (G::QB_B / 4) +
                                                               (p * KSL + sl) * BLKW + fw(lane, sl))
                             : make_uint2(0u, 0u);
#pragma unroll
              for (int mt = 0; mt < 2; ++mt) {
                const uint32_t a0 = key_reg(kw[tt][mt][0], 2 * sl);
                const uint32_t a2 = key_reg(kw[tt][mt][0], 2 * sl + 1);
                const uint32_t a1 = key_reg(kw[tt][mt][1], 2 * sl);
                const uint32_t a3 = key_reg(kw[tt][mt][1], 2 * sl + 1);
#pragma unroll
                for (int p = 0; p < NPB; ++p)
                  mma16816(dq[tt][p][mt], a0, a1, a2, a3, bq[p].x, bq[p].y);
              }
            }
          }

          // -- scores of head tq + 4p for tokens 32 tt + {g, g+8, 16+g, 24+g}
          float sc[NPB][4 * TPW];
#pragma unroll
          for (int p = 0; p < NPB; ++p)
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
              const float bias = bk[tt][HX > 1 ? p : 0];
#pragma unroll
              for (int mt = 0; mt < 2; ++mt) {
                const float v0 = fmaf(dq[tt][p][mt][0] + dq[tt][p][mt][1], kKeyOut, bias);
                const float v1 = fmaf(dq[tt][p][mt][2] + dq[tt][p][mt][3], kKeyOut, bias);
                sc[p][4 * tt + 2 * mt] = tv[tt] ? v0 : kNegInf;
                sc[p][4 * tt + 2 * mt + 1] = tv[tt] ? v1 : kNegInf;
              }
            }
          if constexpr (SP) {
            // dense-and-sparse keys: a kept entry (token t, channel d, value x)
            // was reconstructed by the codes as z_{g,d} (code 0); add
            // q_d (x - z_{g,d}) to token t's score, for every head
            if (c.k_out > 0) {
              const int nk = D * c.k_out;
#pragma unroll
              for (int tt = 0; tt < TPW; ++tt) {
                const int ti = warp * TPW + (tv[tt] ? tt : 0);
                const int* oi = reinterpret_cast<const int*>(buf + G::O_KOI) + ti * nk;
                const float* ov = reinterpret_cast<const float*>(buf + G::O_KOV) + ti * nk;
                for (int e = lane; e < nk; e += 32) {
                  const int d = e / c.k_out;
                  const float dx = ov[e] - load1(kz[tt] + d);
                  const int tok = oi[e] & (kTile - 1);
#pragma unroll
                  for (int h = 0; h < GQ; ++h) atomicAdd(&corr[(tt * GQ + h) * kTile + tok], qs[h * D + d] * dx);
                }
              }
              __syncwarp();
#pragma unroll
              for (int p = 0; p < NPB; ++p) {
                if (!vh[p]) continue;
                const int h = tq + 4 * p;
#pragma unroll
                for (int i = 0; i < 4 * TPW; ++i) {
                  const int tt = i >> 2, tok = 16 * ((i >> 1) & 1) + 8 * (i & 1) + g;
                  float* cp = &corr[(tt * GQ + h) * kTile + tok];
                  sc[p][i] += *cp;
                  *cp = 0.f;
                }
              }
              __syncwarp();
            }
          }
          // -- online softmax: the running max moves only when a score exceeds it
          float lm[NPB];
          bool need = false;
#pragma unroll
          for (int p = 0; p < NPB; ++p) {
            float v = sc[p][0];
#pragma unroll
            for (int i = 1; i < 4 * TPW; ++i) v = fmaxf(v, sc[p][i]);
            lm[p] = v;
            need |= vh[p] && v > m_run[p];
          }
          if (__any_sync(0xffffffffu, need)) {
            float al[NPB];
#pragma unroll
            for (int p = 0; p < NPB; ++p) {
              float tm = lm[p];
              tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
              tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
              tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
              const float mn = fmaxf(m_run[p], tm);
              al[p] = exp2f(m_run[p] - mn);
              m_run[p] = mn;
              l_part[p] *= al[p];
#pragma unroll
              for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[p][m][e] *= al[p];
            }
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
              const float ah = __shfl_sync(0xffffffffu, al[h >> 2], h & 3);
#pragma unroll
              for (int j = 0; j < NJ; ++j) bv[h][j] *= ah;
              if constexpr (SP) {
                for (int d = lane; d < D; d += 32) vcorr[h * D + d] *= ah;
              }
            }
          }
#pragma unroll
          for (int p = 0; p < NPB; ++p) {
            float ps = 0.f;
#pragma unroll
            for (int i = 0; i < 4 * TPW; ++i) {
              const float pv = exp2f(sc[p][i] - m_run[p]);
              ps += pv;
              const int tok = 32 * (i >> 2) + 16 * ((i >> 1) & 1) + 8 * (i & 1) + g;
              if (vh[p]) pbuf[(tq + 4 * p) * PST + tok] = pv;
            }
            l_part[p] += ps;
          }
          __syncwarp();

          if constexpr (SP) {
            // dense-and-sparse values: a kept entry (token t, channel c, value
            // x) was reconstructed as z_{t,j} (code 0); add p_t (x - z_{t,j})
            // to channel c of the unit's value corrections, every head
            if (c.v_out > 0) {
              const int nv = kTile * NJ * c.v_out;
#pragma unroll
              for (int tt = 0; tt < TPW; ++tt) {
                if (!tv[tt]) continue;
                const int ti = warp * TPW + tt;
                const int* oi = reinterpret_cast<const int*>(buf + G::O_VOI) + ti * nv;
                const float* ov = reinterpret_cast<const float*>(buf + G::O_VOV) + ti * nv;
                for (int e = lane; e < nv; e += 32) {
                  const int tj = e / c.v_out;  // token * NJ + group
                  const int t = tj / NJ, j = tj - t * NJ;
                  const float dx = ov[e] - load1(vz[tt] + tj);
                  const int ch = j * kGv + (oi[e] & (kGv - 1));
#pragma unroll
                  for (int h = 0; h < GQ; ++h)
                    atomicAdd(&vcorr[h * D + ch], pbuf[h * PST + 32 * tt + t] * dx);
                }
              }
              __syncwarp();
            }
          }
          // -- p' = p s_v 2^(SV - e) (hi, lo) into the B fragments; bias_v += p z_v
#pragma unroll
          for (int tt = 0; tt < TPW; ++tt) {
            float sv[NJ], zv[NJ];
            load_meta<NJ>(vs[tt] + lane * NJ, sv);
            load_meta<NJ>(vz[tt] + lane * NJ, zv);
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
              const float ph = pbuf[h * PST + 32 * tt + lane];
              const float phf = ph * pt_f;
              const int nh = 2 * (h & 3);
              const int o_hi = pt_base + 4 * (4 * (nh ^ pt_s3) + pt_tq);
              const int o_lo = pt_base + 4 * (4 * ((nh + 1) ^ pt_s3) + pt_tq);
#pragma unroll
              for (int j = 0; j < NJ; ++j) {
                bv[h][j] = fmaf(ph, zv[j], bv[h][j]);
                const float x = phf * sv[j];
                const __half hi = __float2half_rn(x);
                const __half lo = __float2half_rn(x - __half2float(hi));
                __half* blk = pBh + tt * (G::PB_B / 2) + ((h >> 2) * NJ + j) * NSL * 2 * BLKW;
                blk[o_hi] = hi;
                blk[o_lo] = lo;
              }
            }
          }
          __syncwarp();

          // -- P.V: per tile, k-slice sl and value group j, m-tiles 2j
          // (channels 32j+4g, +1) and 2j+1 (+2, +3)
#pragma unroll
          for (int tt = 0; tt < TPW; ++tt) {
#pragma unroll
            for (int sl = 0; sl < NSL; ++sl) {
              const int tw = (BITS == 1 || BITS == 3) ? 0 : BITS == 2 ? sl : 2 * sl + vtw;
              constexpr int SH = BITS == 1 ? 4 : 8;  // shift to the a2 / a3 pairs
              const int s0 = BITS == 1 ? 8 * sl : 0;  // 1-bit: this slice's byte
#pragma unroll
              for (int j = 0; j < NJ; ++j) {
                uint32_t x0, x1, x2, x3, y0, y1, y2, y3;
                if constexpr (BITS == 3) {
                  // three bit-plane rows of the tile, each word a channel's 32
                  // tokens (the 1-bit token order)
                  const uint32_t* vr = vc[tt] + 32 * j + 4 * g;
                  const uint4 p0 = *reinterpret_cast<const uint4*>(vr);
                  const uint4 p1 = *reinterpret_cast<const uint4*>(vr + D);
                  const uint4 p2 = *reinterpret_cast<const uint4*>(vr + 2 * D);
                  const uint32_t sa = 8 * sl, sb = 8 * sl + 4;
                  x0 = planes3(p0.x, p1.x, p2.x, sa, vM); x2 = planes3(p0.x, p1.x, p2.x, sb, vM);
                  x1 = planes3(p0.y, p1.y, p2.y, sa, vM); x3 = planes3(p0.y, p1.y, p2.y, sb, vM);
                  y0 = planes3(p0.z, p1.z, p2.z, sa, vM); y2 = planes3(p0.z, p1.z, p2.z, sb, vM);
                  y1 = planes3(p0.w, p1.w, p2.w, sa, vM); y3 = planes3(p0.w, p1.w, p2.w, sb, vM);
                } else {
                  uint4 w = *reinterpret_cast<const uint4*>(vc[tt] + tw * D + 32 * j + 4 * g);
                  if (BITS == 1) {
                    w.x >>= s0; w.y >>= s0; w.z >>= s0; w.w >>= s0;
                  }
                  x0 = w.x & vM; x2 = (w.x >> SH) & vM;
                  x1 = w.y & vM; x3 = (w.y >> SH) & vM;
                  y0 = w.z & vM; y2 = (w.z >> SH) & vM;
                  y1 = w.w & vM; y3 = (w.w >> SH) & vM;
                }
#pragma unroll
                for (int p = 0; p < NPB; ++p) {
                  const uint2 bb = bcol ? *reinterpret_cast<const uint2*>(
                                              pB + tt * (G::PB_B / 4) + ((p * NJ + j) * NSL + sl) * BLKW +
                                              fw(lane, sl))
                                        : make_uint2(0u, 0u);
                  mma16816(acc[p][2 * j], x0, x1, x2, x3, bb.x, bb.y);
                  mma16816(acc[p][2 * j + 1], y0, y1, y2, y3, bb.x, bb.y);
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // ---- one fp16 window stage of nt tokens on tensor cores: S = K q
      // (K rows by ldmatrix), the same online softmax, O += V^T p (V^T by
      // ldmatrix.trans); rows past nt read row 0 and are masked out
      auto window_tile = [&](unsigned char* wbuf, int nt, int tw0) {
        unsigned char* Kw = wbuf;
        unsigned char* Vw = wbuf + G::NBX * G::BOX_B;
        // address of 16-byte chunk cc (channels 8 cc .. 8 cc + 7) of row tok:
        // the swizzle XORs the chunk index with address bits 7.. of the row
        auto chunk = [&](unsigned char* base, int tok, int cc) -> unsigned char* {
          constexpr int CPR = G::RB / 16;  // chunks per box row
          unsigned char* row = base + (cc / CPR) * G::BOX_B + tok * G::RB;
          const uint32_t ra = smem_u32(row);
          const int x = G::RB == 128 ? (int)((ra >> 7) & 7u) : (int)((ra >> 7) & 3u);
          return row + (((cc % CPR) ^ x) << 4);
        };
        if (a.new_k != nullptr && a.new_slot >= tw0 && a.new_slot < tw0 + G::WT) {
          // fused append: the copies brought the window before this call's
          // token; put the token into its row here and into the cache for
          // later calls (16 bytes per lane, K then V)
          constexpr int NC = D * 2 / 16;  // 16-byte chunks per row
          const int row = a.new_slot - tw0;
          if (lane < 2 * NC) {
            const int cc = lane % NC;
            const bool isv = lane >= NC;
            const uint4 x = reinterpret_cast<const uint4*>(
                reinterpret_cast<const T*>(isv ? a.new_v : a.new_k) + u * D)[cc];
            *reinterpret_cast<uint4*>(chunk(isv ? Vw : Kw, row, cc)) = x;
            T* dst = reinterpret_cast<T*>(isv ? c.v_res : c.k_res) + (u * c.R + a.new_slot) * D;
            reinterpret_cast<uint4*>(dst)[cc] = x;
          }
          __syncwarp();
        }
        float dq[NPB][2][4];
#pragma unroll
        for (int p = 0; p < NPB; ++p)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) dq[p][mt][e] = 0.f;
#pragma unroll
        for (int sl = 0; sl < KSL; ++sl) {
          uint2 bq[NPB];
#pragma unroll
          for (int p = 0; p < NPB; ++p)
            bq[p] = bcol ? *reinterpret_cast<const uint2*>(qB + (p * KSL + sl) * BLKW + fw(lane, sl))
                         : make_uint2(0u, 0u);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const int tok = 16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1);
            uint32_t af[4];
            ldsm_x4(af, chunk(Kw, tok < nt ? tok : 0, 2 * sl + (lane >> 4)));
#pragma unroll
            for (int p = 0; p < NPB; ++p) mma16816(dq[p][mt], af[0], af[1], af[2], af[3], bq[p].x, bq[p].y);
          }
        }
        float sc[NPB][4];
#pragma unroll
        for (int p = 0; p < NPB; ++p)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const float v = dq[p][mt][2 * r] + dq[p][mt][2 * r + 1];
              sc[p][2 * mt + r] = (16 * mt + 8 * r + g < nt) ? v : kNegInf;
            }
        float lm[NPB];
        bool need = false;
#pragma unroll
        for (int p = 0; p < NPB; ++p) {
          lm[p] = fmaxf(fmaxf(sc[p][0], sc[p][1]), fmaxf(sc[p][2], sc[p][3]));
          need |= vh[p] && lm[p] > m_run[p];
        }
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int p = 0; p < NPB; ++p) {
            float tm = lm[p];
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
            const float mn = fmaxf(m_run[p], tm);
            const float al = exp2f(m_run[p] - mn);
            m_run[p] = mn;
            l_part[p] *= al;
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[p][m][e] *= al;
          }
        }
#pragma unroll
        for (int p = 0; p < NPB; ++p) {
          float ps = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float pv = exp2f(sc[p][i] - m_run[p]);
            ps += pv;
            if (vh[p]) pbuf[(tq + 4 * p) * PST + 16 * (i >> 1) + 8 * (i & 1) + g] = pv;
          }
          l_part[p] += ps;
        }
        __syncwarp();
        // p (hi, lo) into the value B fragments, tokens in natural order
        {
          const int slp = lane >> 4, kk = lane & 15;
          const int tqk = (kk & 7) >> 1, kp = kk >> 3, hf = kk & 1;
#pragma unroll
          for (int h = 0; h < GQ; ++h) {
            const float x = pbuf[h * PST + lane];
            const __half hi = __float2half_rn(x);
            const __half lo = __float2half_rn(x - __half2float(hi));
            __half* blk = pBh + ((h >> 2) * NJ * NSL + slp) * 2 * BLKW + 2 * kp + hf;
            const int nh = 2 * (h & 3);
            blk[2 * fw(4 * nh + tqk, slp)] = hi;
            blk[2 * fw(4 * (nh + 1) + tqk, slp)] = lo;
          }
        }
        __syncwarp();
#pragma unroll
        for (int sl = 0; sl < NSL; ++sl) {
          uint2 bb[NPB];
#pragma unroll
          for (int p = 0; p < NPB; ++p)
            bb[p] = bcol ? *reinterpret_cast<const uint2*>(pB + (p * NJ * NSL + sl) * BLKW + fw(lane, sl))
                         : make_uint2(0u, 0u);
          const int tok = 16 * sl + (lane & 7) + 8 * (lane >> 4);
          const int tr = tok < nt ? tok : 0;
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            uint32_t af[4];
            ldsm_x4_t(af, chunk(Vw, tr, 2 * m + ((lane >> 3) & 1)));
#pragma unroll
            for (int p = 0; p < NPB; ++p) mma16816(acc[p][m], af[0], af[1], af[2], af[3], bb[p].x, bb[p].y);
          }
        }
      };

      // ---- this warp's quantized-tile state (m, l, acc + value zeros) -> mg slot
      auto flush_code = [&]() {
        float lt[NPB];
#pragma unroll
        for (int p = 0; p < NPB; ++p) {
          float v = l_part[p];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          lt[p] = v;
        }
#pragma unroll
        for (int h = 0; h < GQ; ++h)
#pragma unroll
          for (int j = 0; j < NJ; ++j) bv[h][j] = warp_sum(bv[h][j]);
#pragma unroll
        for (int p = 0; p < NPB; ++p) {
          if (!vh[p]) continue;
          const int h = tq + 4 * p;
          if (g == 0) {
            mg_m[warp * GQ + h] = m_run[p];
            mg_l[warp * GQ + h] = lt[p];
          }
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int j = m >> 1;
            const int ch = 32 * j + 4 * g + 2 * (m & 1);
            float bias = 0.f;
#pragma unroll
            for (int hh = 0; hh < GQ; ++hh)
              if (hh == h) bias = bv[hh][j];
            float* dst = mg_acc + (warp * GQ + h) * D + ch;
            dst[0] = fmaf(acc[p][m][0] + acc[p][m][1], kValOut, bias);
            dst[1] = fmaf(acc[p][m][2] + acc[p][m][3], kValOut, bias);
          }
        }
        if constexpr (SP) {
          // the unit's dense-and-sparse value corrections (same softmax state)
          __syncwarp();
#pragma unroll
          for (int h = 0; h < GQ; ++h)
            for (int d = lane; d < D; d += 32) {
              mg_acc[(warp * GQ + h) * D + d] += vcorr[h * D + d];
              vcorr[h * D + d] = 0.f;
            }
          __syncwarp();
        }
      };

      // ---- fp16 residual window on tensor cores: window tile k (WPS per
      // stage) goes to warp k % kW, which first flushes its quantized-tile
      // state and then keeps a separate softmax state for the window (plain q
      // and p, scale 1)
      bool wmode = false;
      if constexpr (sizeof(T) == 2) {
        if (window_owner) {
          int k = 0;
          for (int w0 = 0; w0 < r_u; w0 += G::WT * G::WPS, adv()) {
            if (*(volatile int*)&flag[0]) break;
            const int s = rs;
            const bool ok = mbar_wait(&full[s], rph);
            if (!__all_sync(0xffffffffu, ok) || *(volatile int*)&flag[0]) {
              if (lane == 0) atomicExch(&flag[0], 1);
              break;
            }
            for (int j = 0; j < G::WPS; ++j, ++k) {
            const int tw0 = w0 + j * G::WT;
            if (tw0 >= r_u) break;
            if (k % kW == warp) {
              if (!wmode) {
                flush_code();
                __syncwarp();
                wmode = true;
#pragma unroll
                for (int p = 0; p < NPB; ++p) {
                  m_run[p] = kNegInf;
                  l_part[p] = 0.f;
#pragma unroll
                  for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[p][m][e] = 0.f;
                }
                // B fragments of plain q (hi, lo), channels in natural order:
                // k-slice sl, k = channel - 16 sl; lane takes channel pairs
#pragma unroll
                for (int cp0 = 0; cp0 < D / 2; cp0 += 32) {
                  const int cpr = cp0 + lane;  // channels 2 cpr, 2 cpr + 1
                  if (cpr < D / 2) {
                    const int sl = cpr >> 3, kk = 2 * (cpr & 7);
                    const int tqk = (kk & 7) >> 1, kp = kk >> 3;
#pragma unroll
                    for (int h = 0; h < GQ; ++h) {
                      const float2 x = *reinterpret_cast<const float2*>(qs + h * D + 2 * cpr);
                      uint32_t hi, lo;
                      split2(x.x, x.y, hi, lo);
                      uint32_t* blk = qB + ((h >> 2) * KSL + sl) * BLKW + kp;
                      const int nh = 2 * (h & 3);
                      blk[fw(4 * nh + tqk, sl)] = hi;
                      blk[fw(4 * (nh + 1) + tqk, sl)] = lo;
                    }
                  }
                }
                __syncwarp();
              }
              window_tile(smem + s * G::STAGE_B + j * G::WTILE_B, min(G::WT, r_u - tw0), tw0);
            }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
          }
        }
      }
      const bool failed = *(volatile int*)&flag[0] != 0;
      if (!wmode) {
        flush_code();
      } else {
        // fold the window state into this warp's slot (quantized-tile state)
        float lt[NPB], m1[NPB], l1[NPB];
#pragma unroll
        for (int p = 0; p < NPB; ++p) {
          float v = l_part[p];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          lt[p] = v;
          const int h = tq + 4 * p;
          m1[p] = vh[p] ? mg_m[warp * GQ + h] : kNegInf;
          l1[p] = vh[p] ? mg_l[warp * GQ + h] : 0.f;
        }
        __syncwarp();
#pragma unroll
        for (int p = 0; p < NPB; ++p) {
          if (!vh[p]) continue;
          const int h = tq + 4 * p;
          const float mn = fmaxf(m1[p], m_run[p]);
          const float s1 = m1[p] == kNegInf ? 0.f : exp2f(m1[p] - mn);
          const float s2 = m_run[p] == kNegInf ? 0.f : exp2f(m_run[p] - mn);
          float* dst = mg_acc + (warp * GQ + h) * D;
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int ch = 16 * m + g;
            dst[ch] = fmaf(dst[ch], s1, (acc[p][m][0] + acc[p][m][1]) * s2);
            dst[ch + 8] = fmaf(dst[ch + 8], s1, (acc[p][m][2] + acc[p][m][3]) * s2);
          }
          if (g == 0) {
            mg_m[warp * GQ + h] = mn;
            mg_l[warp * GQ + h] = fmaf(l1[p], s1, lt[p] * s2);
          }
        }
      }
      __syncwarp();
      // ---- residual window (CTA that ends the unit): warp w takes window
      // tiles w, w+4, ... on CUDA cores, folded into its mg slot
      if (sizeof(T) == 4 && window_owner && !failed) {
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
        const int nwt = (r_u + kTile - 1) / kTile;
        constexpr int VEC = 16 / (int)sizeof(T);  // elements per 16-byte load
        for (int wt = warp; wt < nwt; wt += kW) {
          const int t_in = wt * kTile + lane;
          const int nt = min(kTile, r_u - wt * kTile);
          float lg[GQ];
#pragma unroll
          for (int h = 0; h < GQ; ++h) lg[h] = 0.f;
          if (t_in < r_u) {
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
      consumers_sync<kW>();
      if (tid == 0) {
        if (dev) {
          flag[1] = arrive_unit_reset(a.ctr + u, n_seg);
        } else {
          flag[1] = arrive_unit(a.ctr + u, a.epoch, n_seg);
        }
      }
      consumers_sync<kW>();
      const int last = flag[1];
      if (last != 0) {
        T* out = reinterpret_cast<T*>(a.out);
        for (int idx = tid; idx < GQ * D; idx += kW * 32) {
          const int h = idx / D, d = idx % D;
          const long long row = b * Hq + (long long)kv * GQ + h;
          float res = kNaN;
          if (last > 0)
            res = merge_partials(a.ws + (u * a.max_seg * GQ + h) * (D + 2), (long long)GQ * (D + 2),
                                 n_seg, d);
          out[row * D + d] = from_f32<T>(res);
        }
      }
      consumers_sync<kW>();  // mg buffers and flag[1] are reused by the next unit
      if (failed) break;
    }
  }
  __syncthreads();
  if (!RAG && dev && tid == 0 && arrive_unit_reset(a.ctr + a.units, gridDim.x) == 1) {
    // the last CTA to finish advances the device counters (and clears the
    // flush barrier's count: every CTA is past it)
    args.dev_state->n_q = a.n_q;
    args.dev_state->r = a.r;
    if (a.flush) asm volatile("st.relaxed.gpu.global.u64 [%0], 0;" ::"l"(a.ctr + a.units + 1) : "memory");
  }
  if (RAG && a.pending) {
    // the last CTA to finish advances every sequence that took its token
    if (tid == 0) flag[1] = arrive_unit_reset(a.ctr + a.units, gridDim.x);
    __syncthreads();
    if (flag[1] == 1) {
      for (long long b = tid; b < a.units / a.Hkv; b += G::THREADS) {
        const SeqLen L = ragged_len(a, b);
        if (L.ok) {
          args.dev_state[b].n_q = L.n_q;
          args.dev_state[b].r = L.r;
        }
      }
    }
  }
}

// Opt in to the kernel's dynamic shared memory and return how many of its
// CTAs fit on one SM (both once per device).
template <int D, int BITS, int GQ, typename T, typename MT, bool RAG, bool SP>
cudaError_t tc_setup(int* ctas_per_sm) {
  using G = Geo<D, BITS, GQ, sizeof(MT), SP>;
  static int occ[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 128 && occ[dev] > 0) {
    *ctas_per_sm = occ[dev];
    return cudaSuccess;
  }
  e = cudaFuncSetAttribute(decode_stream_tc<D, BITS, GQ, T, MT, RAG, SP>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_B);
  if (e != cudaSuccess) return e;
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_stream_tc<D, BITS, GQ, T, MT, RAG, SP>,
                                                    G::THREADS, G::SMEM_B);
  if (e != cudaSuccess) return e;
  if (n < 1) return cudaErrorInvalidConfiguration;
  if (dev >= 0 && dev < 128) occ[dev] = n;
  *ctas_per_sm = n;
  return cudaSuccess;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library), looked up once.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// Tensor map of one fp16 residual buffer viewed as [units * R][D]: boxes of
// 32 rows x min(D, 64) columns, swizzled (128-byte rows: 128B, 64-byte: 64B).
cudaError_t window_map(CUtensorMap* m, const void* base, long long rows, int D) {
  const EncodeTiledFn fn = encode_tiled();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {(cuuint32_t)(D < 64 ? D : 64), (cuuint32_t)kTile};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                        box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        D < 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The two window tensor maps of a cache, encoded once and kept: they depend
// only on the window buffers, the row count and D, which a cache never
// changes, so steady decode calls skip the encoding.  A small table per
// process (guarded by a mutex), replaced round-robin.
cudaError_t window_maps(const void* k_res, const void* v_res, long long rows, int D,
                        CUtensorMap* mk, CUtensorMap* mv) {
  struct Entry {
    const void* k;
    const void* v;
    long long rows;
    int D;
    int dev;
    CUtensorMap mk, mv;
  };
  constexpr int kN = 32;
  static std::mutex mu;
  static Entry table[kN];
  static int used = 0, next = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i) {
      const Entry& x = table[i];
      if (x.k == k_res && x.v == v_res && x.rows == rows && x.D == D && x.dev == dev) {
        *mk = x.mk;
        *mv = x.mv;
        return cudaSuccess;
      }
    }
  }
  e = window_map(mk, k_res, rows, D);
  if (e == cudaSuccess) e = window_map(mv, v_res, rows, D);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  Entry& x = table[next];
  x.k = k_res;
  x.v = v_res;
  x.rows = rows;
  x.D = D;
  x.dev = dev;
  x.mk = *mk;
  x.mv = *mv;
  next = (next + 1) % kN;
  if (used < kN) ++used;
  return cudaSuccess;
}

template <int D, int BITS, int GQ, typename T, typename MT, bool RAG, bool SP>
cudaError_t tc_t(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1,
                 int* ctas_per_sm) {
  using G = Geo<D, BITS, GQ, sizeof(MT), SP>;
  if (ctas_per_sm) return tc_setup<D, BITS, GQ, T, MT, RAG, SP>(ctas_per_sm);
  int occ = 0;
  cudaError_t e = tc_setup<D, BITS, GQ, T, MT, RAG, SP>(&occ);
  if (e != cudaSuccess) return e;
  CUtensorMap tmK, tmV;
  memset(&tmK, 0, sizeof(tmK));
  memset(&tmV, 0, sizeof(tmV));
  if (sizeof(T) == 2 && a.r > 0) {
    const long long rows = (long long)a.units * a.c.R;
    if (rows >= (1LL << 31)) return cudaErrorInvalidValue;  // 32-bit box coordinates
    e = window_maps(a.c.k_res, a.c.v_res, rows, D, &tmK, &tmV);
    if (e != cudaSuccess) return e;
  }
  if (e0) cudaEventRecord(e0, s);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)a.n_cta);
  cfg.blockDim = dim3(G::THREADS);
  cfg.dynamicSmemBytes = G::SMEM_B;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err =
      cudaLaunchKernelEx(&cfg, decode_stream_tc<D, BITS, GQ, T, MT, RAG, SP>, a, tmK, tmV);
  if (err == cudaSuccess) err = cudaGetLastError();
  if (e1) cudaEventRecord(e1, s);
  return err;
}

template <int D, int BITS, typename T, typename MT, bool RAG, bool SP>
cudaError_t tc_g(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1, int* occ) {
  switch (a.gq) {
    case 1: return tc_t<D, BITS, 1, T, MT, RAG, SP>(a, s, e0, e1, occ);
    case 2: return tc_t<D, BITS, 2, T, MT, RAG, SP>(a, s, e0, e1, occ);
    case 4: return tc_t<D, BITS, 4, T, MT, RAG, SP>(a, s, e0, e1, occ);
    case 8: return tc_t<D, BITS, 8, T, MT, RAG, SP>(a, s, e0, e1, occ);
  }
  return cudaErrorInvalidValue;
}

template <int BITS, typename T, typename MT, bool RAG, bool SP = false>
cudaError_t tc_d(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1, int* occ) {
  switch (a.D) {
    case 32: return tc_g<32, BITS, T, MT, RAG, SP>(a, s, e0, e1, occ);
    case 64: return tc_g<64, BITS, T, MT, RAG, SP>(a, s, e0, e1, occ);
    case 128: return tc_g<128, BITS, T, MT, RAG, SP>(a, s, e0, e1, occ);
  }
  return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace kivi
