// Tensor-core decode instances for unquantized fp16 caches (see decode_mma_instances.h).
#include "decode_mma.cuh"
#include "decode_mma_instances.h"

namespace kvq {
namespace mma {

#define KVQ_INST_F(DK, NREP)                                                                   \
  template cudaError_t launch<4, 2, DK, NREP, 64, 64, false>(const Dims&, const CacheBufs&,    \
                                                            const DecodeWork&, const __half*,  \
                                                            const Partials&, cudaStream_t);
KVQ_MMA_FP16_INSTANCES(KVQ_INST_F)

}  // namespace mma
}  // namespace kvq
