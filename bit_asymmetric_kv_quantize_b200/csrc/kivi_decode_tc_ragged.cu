// kivi_decode_tc_ragged.cu -- instances of the tensor-core decode kernel
// (kivi_decode_tc.cuh) for ragged batches (per-sequence lengths held in
// device memory) with binary32 scales and zeros.
#include "kivi_decode_tc.cuh"

namespace kivi {

cudaError_t tc_dispatch_ragged(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                               cudaEvent_t e1, int* occ) {
  if (a.bits == 1 && a.dtype == 0) return tc_d<1, __half, float, true>(a, s, e0, e1, occ);
  if (a.bits == 1 && a.dtype == 1) return tc_d<1, float, float, true>(a, s, e0, e1, occ);
  if (a.bits == 2 && a.dtype == 0) return tc_d<2, __half, float, true>(a, s, e0, e1, occ);
  if (a.bits == 2 && a.dtype == 1) return tc_d<2, float, float, true>(a, s, e0, e1, occ);
  if (a.bits == 4 && a.dtype == 0) return tc_d<4, __half, float, true>(a, s, e0, e1, occ);
  if (a.bits == 4 && a.dtype == 1) return tc_d<4, float, float, true>(a, s, e0, e1, occ);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
