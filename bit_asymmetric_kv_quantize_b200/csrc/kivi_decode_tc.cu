// kivi_decode_tc.cu -- instances of the tensor-core decode kernel
// (kivi_decode_tc.cuh) with binary32 scales and zeros for uniform batches,
// and the entry points that select an instance.
#include "kivi_decode_tc.cuh"

namespace kivi {
namespace {

cudaError_t tc_dispatch(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1,
                        int* occ) {
  if (a.c.k_out > 0 || a.c.v_out > 0) return tc_dispatch_sparse(a, s, e0, e1, occ);
  if (a.bits == 3) return a.ragged ? tc_dispatch_3bit_ragged(a, s, e0, e1, occ)
                                   : tc_dispatch_3bit(a, s, e0, e1, occ);
  if (a.ragged) {
    if (a.meta == 1) return tc_dispatch_ragged_meta16(a, s, e0, e1, occ);
    if (a.meta != 0) return cudaErrorInvalidValue;
    return tc_dispatch_ragged(a, s, e0, e1, occ);
  }
  if (a.meta == 1) return tc_dispatch_meta16(a, s, e0, e1, occ);
  if (a.meta != 0) return cudaErrorInvalidValue;
  if (a.bits == 1 && a.dtype == 0) return tc_d<1, __half, float, false>(a, s, e0, e1, occ);
  if (a.bits == 1 && a.dtype == 1) return tc_d<1, float, float, false>(a, s, e0, e1, occ);
  if (a.bits == 2 && a.dtype == 0) return tc_d<2, __half, float, false>(a, s, e0, e1, occ);
  if (a.bits == 2 && a.dtype == 1) return tc_d<2, float, float, false>(a, s, e0, e1, occ);
  if (a.bits == 4 && a.dtype == 0) return tc_d<4, __half, float, false>(a, s, e0, e1, occ);
  if (a.bits == 4 && a.dtype == 1) return tc_d<4, float, float, false>(a, s, e0, e1, occ);
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
