// Width-map decode instances with value groups of 16 channels (see decode_var.cuh).
#include "decode_var.cuh"

namespace kvq {
namespace var {

#define KVQ_VAR_INST(NREP, GK)                                                                  \
  template cudaError_t launch_var<NREP, 16, GK>(const Dims&, const CacheBufs&, const DecodeWork&,   \
                                                 const VarPlan&, const __half*, const Partials&,  \
                                                 cudaStream_t);
KVQ_VAR_INST(1, 16)
KVQ_VAR_INST(1, 32)
KVQ_VAR_INST(1, 64)
KVQ_VAR_INST(1, 128)
KVQ_VAR_INST(4, 16)
KVQ_VAR_INST(4, 32)
KVQ_VAR_INST(4, 64)
KVQ_VAR_INST(4, 128)

}  // namespace var
}  // namespace kvq
