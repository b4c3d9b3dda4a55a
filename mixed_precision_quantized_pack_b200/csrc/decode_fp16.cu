// mma.sync decode instances for the fp16 rows (see decode_instances.h).
#include "decode_instances.h"
#include "decode_mma.cuh"

namespace kvq {
namespace mma {

#define KVQ_INST_F(DK, NREP)                                                                  \
  template cudaError_t launch_fp16<DK, NREP>(const Dims&, const CacheBufs&, const DecodeWork&, \
                                             const __half*, const Partials&, cudaStream_t);
KVQ_FP16_INSTANCES(KVQ_INST_F)

}  // namespace mma
}  // namespace kvq
