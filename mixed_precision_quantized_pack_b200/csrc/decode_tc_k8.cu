// tcgen05 decode instances with 8-bit keys (see decode_instances.h).
#include "decode_instances.h"
#include "decode_tc.cuh"

namespace kvq {
namespace tc {

#define KVQ_INST_Q(KB, VB, DK, NREP, GV, GK)                                                     \
  template cudaError_t launch<KB, VB, DK, NREP, GV, GK>(const Dims&, const CacheBufs&,        \
                                                        const DecodeWork&, const __half*,      \
                                                        const Partials&, cudaStream_t);
#define KVQ_PICK(KB, VB, DK, NREP, GV, GK) KVQ_PICK_##KB(KB, VB, DK, NREP, GV, GK)
#define KVQ_PICK_2(...)
#define KVQ_PICK_4(...)
#define KVQ_PICK_8(...) KVQ_INST_Q(__VA_ARGS__)
KVQ_TC_INSTANCES(KVQ_PICK)

}  // namespace tc
}  // namespace kvq
