// kivi_decode_tc_3bit_ragged.cu -- instances of the tensor-core decode
// kernel (kivi_decode_tc.cuh) for the 3-bit format variant, ragged batches
// (per-sequence lengths held in device memory).
#include "kivi_decode_tc.cuh"

namespace kivi {

cudaError_t tc_dispatch_3bit_ragged(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                                    cudaEvent_t e1, int* occ) {
  if (a.bits != 3) return cudaErrorInvalidValue;
  if (a.meta == 1) {
    if (a.dtype != 0) return cudaErrorInvalidValue;
    return tc_d<3, __half, __half, true>(a, s, e0, e1, occ);
  }
  if (a.meta != 0) return cudaErrorInvalidValue;
  if (a.dtype == 0) return tc_d<3, __half, float, true>(a, s, e0, e1, occ);
  if (a.dtype == 1) return tc_d<3, float, float, true>(a, s, e0, e1, occ);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
