// Tensor-core decode kernel (placeholder until the fragment-level kernel lands).
#include "kvq_internal.cuh"

namespace kvq {

bool decode_mma_supported(const Dims&) { return false; }

cudaError_t launch_decode_mma(const Dims&, const CacheBufs&, const DecodeWork&, const __half*,
                              const Partials&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kvq
