// Dispatch of the fast decode path: the tcgen05 kernel over the quantized groups and
// the mma.sync kernel over the fp16 rows, from tables of the built instances.
#include "decode_instances.h"
#include "decode_mma.cuh"
#include "decode_tc.cuh"

namespace kvq {
namespace tc {
#define KVQ_DECL_Q(KB, VB, DK, NREP, GV, GK)                                                  \
  extern template cudaError_t launch<KB, VB, DK, NREP, GV, GK>(                              \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,       \
      cudaStream_t);
KVQ_TC_INSTANCES(KVQ_DECL_Q)
}  // namespace tc
namespace mma {
#define KVQ_DECL_F(DK, NREP)                                                                   \
  extern template cudaError_t launch_fp16<DK, NREP>(const Dims&, const CacheBufs&,            \
                                                    const DecodeWork&, const __half*,          \
                                                    const Partials&, cudaStream_t);
KVQ_FP16_INSTANCES(KVQ_DECL_F)
}  // namespace mma

namespace {

using LaunchFn = cudaError_t (*)(const Dims&, const CacheBufs&, const DecodeWork&, const __half*,
                                 const Partials&, cudaStream_t);
struct QEntry {
  int kb, vb, dk, nrep, gv, gk;
  LaunchFn fn;
};
struct FEntry {
  int dk, nrep;
  LaunchFn fn;
};

#define KVQ_ENTRY_Q(KB, VB, DK, NREP, GV, GK) {KB, VB, DK, NREP, GV, GK, &tc::launch<KB, VB, DK, NREP, GV, GK>},
#define KVQ_ENTRY_F(DK, NREP) {DK, NREP, &mma::launch_fp16<DK, NREP>},
const QEntry kQTable[] = {KVQ_TC_INSTANCES(KVQ_ENTRY_Q)};
const FEntry kFTable[] = {KVQ_FP16_INSTANCES(KVQ_ENTRY_F)};

LaunchFn find_fp16(const Dims& d) {
  if (d.dv != 128) return nullptr;
  for (const FEntry& e : kFTable)
    if (e.dk == d.dk && e.nrep == d.n_rep) return e.fn;
  return nullptr;
}

LaunchFn find_quant(const Dims& d) {
  if (d.dv != 128) return nullptr;
  for (const QEntry& e : kQTable)
    if (e.kb == d.kb && e.vb == d.vb && e.dk == d.dk && e.nrep == d.n_rep && e.gv == d.gv &&
        e.gk == d.gk)
      return e.fn;
  return nullptr;
}

}  // namespace

bool decode_mma_supported(const Dims& d) {
  return find_fp16(d) != nullptr && (!d.quantized() || find_quant(d) != nullptr);
}

cudaError_t launch_decode_mma(const Dims& d, const CacheBufs& c, const DecodeWork& w,
                              const __half* q, const Partials& p, cudaStream_t s) {
  if (!decode_mma_supported(d)) return cudaErrorNotSupported;
  if (w.splits_q > 0) {
    const cudaError_t e = find_quant(d)(d, c, w, q, p, s);
    if (e != cudaSuccess) return e;
  }
  if (w.splits_f > 0) return find_fp16(d)(d, c, w, q, p, s);
  return cudaSuccess;
}

}  // namespace kvq
