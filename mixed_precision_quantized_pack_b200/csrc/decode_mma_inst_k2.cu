// Tensor-core decode instances with 2-bit keys (see decode_mma_instances.h).
#include "decode_mma.cuh"
#include "decode_mma_instances.h"

namespace kvq {
namespace mma {

#define KVQ_INST_Q(KB, VB, DK, NREP, GV, GK)                                                     \
  template cudaError_t launch<KB, VB, DK, NREP, GV, GK, true>(                                \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,         \
      cudaStream_t);
#define KVQ_PICK(KB, VB, DK, NREP, GV, GK) KVQ_PICK_##KB(KB, VB, DK, NREP, GV, GK)
#define KVQ_PICK_2(KB, VB, DK, NREP, GV, GK) KVQ_INST_Q(KB, VB, DK, NREP, GV, GK)
#define KVQ_PICK_4(...)
#define KVQ_PICK_8(...)
KVQ_MMA_QUANT_INSTANCES(KVQ_PICK)

}  // namespace mma
}  // namespace kvq
