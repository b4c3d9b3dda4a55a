// Width-map decode instances for the maps known at build time (see decode_var.cuh).
#include "decode_var.cuh"

namespace kvq {
namespace var {

template cudaError_t launch_var<4, 32, 64, MapK3V2>(const Dims&, const CacheBufs&, const DecodeWork&,
                                                     const VarPlan&, const __half*, const Partials&, cudaStream_t);
template cudaError_t launch_var<4, 64, 64, MapK8K2>(const Dims&, const CacheBufs&, const DecodeWork&,
                                                     const VarPlan&, const __half*, const Partials&, cudaStream_t);

}  // namespace var
}  // namespace kvq
