// Tensor-core decode instances with a side code (see decode_mma_instances.h).
#include "decode_mma.cuh"
#include "decode_mma_instances.h"

namespace kvq {
namespace mma {

#define KVQ_INST_S(KB, VB, DK, NREP, GV, GK, SR, SQ)                                          \
  template cudaError_t launch<KB, VB, DK, NREP, GV, GK, true, SR, SQ>(                      \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,       \
      cudaStream_t);
KVQ_MMA_SIDE_INSTANCES(KVQ_INST_S)

}  // namespace mma
}  // namespace kvq
