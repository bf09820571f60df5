// kivi_decode_tc_ragged_meta16.cu -- instances of the tensor-core decode
// kernel (kivi_decode_tc.cuh) for ragged batches with binary16 scales and
// zeros (fp16 caches only).
#include "kivi_decode_tc.cuh"

namespace kivi {

cudaError_t tc_dispatch_ragged_meta16(const DecodeArgs& a, cudaStream_t s, cudaEvent_t e0,
                                      cudaEvent_t e1, int* occ) {
  if (a.dtype != 0) return cudaErrorInvalidValue;
  if (a.bits == 1) return tc_d<1, __half, __half, true>(a, s, e0, e1, occ);
  if (a.bits == 2) return tc_d<2, __half, __half, true>(a, s, e0, e1, occ);
  if (a.bits == 4) return tc_d<4, __half, __half, true>(a, s, e0, e1, occ);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
