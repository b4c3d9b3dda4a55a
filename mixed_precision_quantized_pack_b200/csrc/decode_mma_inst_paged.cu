// Tensor-core decode instances for paged caches (see decode_mma_instances.h).
#include "decode_mma.cuh"
#include "decode_mma_instances.h"

namespace kvq {
namespace mma {

#define KVQ_INST_P(KB, VB, DK, NREP, GV, GK)                                                     \
  template cudaError_t launch<KB, VB, DK, NREP, GV, GK, true, 0, 4, true>(                    \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,         \
      cudaStream_t);
KVQ_MMA_PAGED_INSTANCES(KVQ_INST_P)

}  // namespace mma
}  // namespace kvq
