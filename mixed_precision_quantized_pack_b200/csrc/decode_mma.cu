// Dispatch of the tensor-core decode kernel: a table of the built instances.
#include "decode_mma.cuh"
#include "decode_mma_instances.h"

namespace kvq {
namespace mma {
#define KVQ_DECL_Q(KB, VB, DK, NREP, GV, GK)                                                 \
  extern template cudaError_t launch<KB, VB, DK, NREP, GV, GK, true>(                    \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,     \
      cudaStream_t);
#define KVQ_DECL_F(DK, NREP)                                                                 \
  extern template cudaError_t launch<4, 2, DK, NREP, 64, 64, false>(                     \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,     \
      cudaStream_t);
#define KVQ_DECL_S(KB, VB, DK, NREP, GV, GK, SR, SQ)                                       \
  extern template cudaError_t launch<KB, VB, DK, NREP, GV, GK, true, SR, SQ>(              \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,     \
      cudaStream_t);
#define KVQ_DECL_P(KB, VB, DK, NREP, GV, GK)                                                 \
  extern template cudaError_t launch<KB, VB, DK, NREP, GV, GK, true, 0, 4, true>(        \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,     \
      cudaStream_t);
#define KVQ_DECL_T(KB, VB, DK, NREP, GV, GK, SR, SQ)                                       \
  extern template cudaError_t launch<KB, VB, DK, NREP, GV, GK, true, SR, SQ, true>(        \
      const Dims&, const CacheBufs&, const DecodeWork&, const __half*, const Partials&,     \
      cudaStream_t);
KVQ_MMA_QUANT_INSTANCES(KVQ_DECL_Q)
KVQ_MMA_PAGED_INSTANCES(KVQ_DECL_P)
KVQ_MMA_PAGED_SIDE_INSTANCES(KVQ_DECL_T)
KVQ_MMA_SIDE_INSTANCES(KVQ_DECL_S)
KVQ_MMA_FP16_INSTANCES(KVQ_DECL_F)
}  // namespace mma

namespace {

using LaunchFn = cudaError_t (*)(const Dims&, const CacheBufs&, const DecodeWork&, const __half*,
                                 const Partials&, cudaStream_t);
struct Entry {
  int kb, vb, dk, nrep, gv, gk, sr, sq, paged;
  LaunchFn fn;
};

#define KVQ_ENTRY_Q(KB, VB, DK, NREP, GV, GK) \
  {KB, VB, DK, NREP, GV, GK, 0, 0, 0, &mma::launch<KB, VB, DK, NREP, GV, GK, true>},
#define KVQ_ENTRY_S(KB, VB, DK, NREP, GV, GK, SR, SQ) \
  {KB, VB, DK, NREP, GV, GK, SR, SQ, 0, &mma::launch<KB, VB, DK, NREP, GV, GK, true, SR, SQ>},
#define KVQ_ENTRY_F(DK, NREP) {16, 16, DK, NREP, 0, 0, 0, 0, 0, &mma::launch<4, 2, DK, NREP, 64, 64, false>},
#define KVQ_ENTRY_P(KB, VB, DK, NREP, GV, GK) \
  {KB, VB, DK, NREP, GV, GK, 0, 0, 1, &mma::launch<KB, VB, DK, NREP, GV, GK, true, 0, 4, true>},
#define KVQ_ENTRY_T(KB, VB, DK, NREP, GV, GK, SR, SQ) \
  {KB, VB, DK, NREP, GV, GK, SR, SQ, 1, &mma::launch<KB, VB, DK, NREP, GV, GK, true, SR, SQ, true>},
const Entry kTable[] = {KVQ_MMA_QUANT_INSTANCES(KVQ_ENTRY_Q) KVQ_MMA_SIDE_INSTANCES(KVQ_ENTRY_S)
                            KVQ_MMA_FP16_INSTANCES(KVQ_ENTRY_F) KVQ_MMA_PAGED_INSTANCES(KVQ_ENTRY_P)
                                KVQ_MMA_PAGED_SIDE_INSTANCES(KVQ_ENTRY_T)};

LaunchFn find(const Dims& d) {
  if (d.dv != 128) return nullptr;
  const int gv = d.quantized() ? d.gv : 0;
  const int gk = d.quantized() ? d.gk : 0;
  for (const Entry& e : kTable)
    if (e.kb == d.kb && e.vb == d.vb && e.dk == d.dk && e.nrep == d.n_rep && e.gv == gv &&
        e.gk == gk && e.sr == d.sr && (d.sr == 0 || e.sq == d.sq) && e.paged == d.paged)
      return e.fn;
  return nullptr;
}

}  // namespace

bool decode_mma_supported(const Dims& d) { return find(d) != nullptr; }

cudaError_t launch_decode_mma(const Dims& d, const CacheBufs& c, const DecodeWork& w,
                              const __half* q, const Partials& p, cudaStream_t s) {
  LaunchFn fn = find(d);
  if (!fn) return cudaErrorNotSupported;
  return fn(d, c, w, q, p, s);
}

}  // namespace kvq
