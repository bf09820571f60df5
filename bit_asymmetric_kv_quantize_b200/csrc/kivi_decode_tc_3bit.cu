// kivi_decode_tc_3bit.cu -- instances of the tensor-core decode kernel
// (kivi_decode_tc.cuh) for the 3-bit format variant (codes as three bit
// planes per block of 32), uniform batches, binary32 or binary16 scales and
// zeros.  Kept apart from the other widths so the build compiles them in
// parallel.
#include "kivi_decode_tc.cuh"

namespace kivi {

cudaError_t tc_dispatch_3bit(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0, cudaEvent_t e1,
                             int* occ) {
  if (a.bits != 3) return cudaErrorInvalidValue;
  if (a.meta == 1) {
    if (a.dtype != 0) return cudaErrorInvalidValue;
    return tc_d<3, __half, __half, false>(a, s, e0, e1, occ);
  }
  if (a.meta != 0) return cudaErrorInvalidValue;
  if (a.dtype == 0) return tc_d<3, __half, float, false>(a, s, e0, e1, occ);
  if (a.dtype == 1) return tc_d<3, float, float, false>(a, s, e0, e1, occ);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
