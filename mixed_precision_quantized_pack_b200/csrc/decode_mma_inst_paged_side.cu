// Tensor-core decode instances for paged caches with a side code (see decode_mma_instances.h).
#include "decode_mma.cuh"
#include "decode_mma_instances.h"

namespace kvq {
namespace mma {

#define KVQ_INST_T(KB, VB, DK, NREP, GV, GK, SR, SQ)                                          \
  template cudaError_t launch<KB, VB, DK, NREP, GV, GK, true, SR, SQ, true>(                \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,       \
      cudaStream_t);
KVQ_MMA_PAGED_SIDE_INSTANCES(KVQ_INST_T)

}  // namespace mma
}  // namespace kvq
