// kivi_decode_tc_sparse.cu -- instances of the tensor-core decode kernel
// (kivi_decode_tc.cuh) for the dense-and-sparse variant (each group's
// largest magnitudes kept exactly in side lists; binary32 scales and zeros;
// 1, 2 or 4 bits), uniform and ragged batches.
#include "kivi_decode_tc.cuh"

namespace kivi {

cudaError_t tc_dispatch_sparse(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1,
                               int* occ) {
  if (a.meta != 0) return cudaErrorInvalidValue;
  if (a.ragged) {
    if (a.bits == 1 && a.dtype == 0) return tc_d<1, __half, float, true, true>(a, s, e0, e1, occ);
    if (a.bits == 1 && a.dtype == 1) return tc_d<1, float, float, true, true>(a, s, e0, e1, occ);
    if (a.bits == 2 && a.dtype == 0) return tc_d<2, __half, float, true, true>(a, s, e0, e1, occ);
    if (a.bits == 2 && a.dtype == 1) return tc_d<2, float, float, true, true>(a, s, e0, e1, occ);
    if (a.bits == 4 && a.dtype == 0) return tc_d<4, __half, float, true, true>(a, s, e0, e1, occ);
    if (a.bits == 4 && a.dtype == 1) return tc_d<4, float, float, true, true>(a, s, e0, e1, occ);
    return cudaErrorInvalidValue;
  }
  if (a.bits == 1 && a.dtype == 0) return tc_d<1, __half, float, false, true>(a, s, e0, e1, occ);
  if (a.bits == 1 && a.dtype == 1) return tc_d<1, float, float, false, true>(a, s, e0, e1, occ);
  if (a.bits == 2 && a.dtype == 0) return tc_d<2, __half, float, false, true>(a, s, e0, e1, occ);
  if (a.bits == 2 && a.dtype == 1) return tc_d<2, float, float, false, true>(a, s, e0, e1, occ);
  if (a.bits == 4 && a.dtype == 0) return tc_d<4, __half, float, false, true>(a, s, e0, e1, occ);
  if (a.bits == 4 && a.dtype == 1) return tc_d<4, float, float, false, true>(a, s, e0, e1, occ);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
