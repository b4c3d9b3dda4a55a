// The decode kernel instances this library is built with, as X-macros:
//   Q(KB, VB, DK, NREP, GV, GK)  quantized groups on tcgen05 (decode_tc.cuh), d_v = 128
//   F(DK, NREP)                  fp16 rows on mma.sync (decode_mma.cuh), d_v = 128
// decode_dispatch.cu builds its dispatch table from the same lists; each
// decode_tc_k*.cu file instantiates the entries whose KB it owns.  Shapes not
// listed here run on the generic CUDA-core kernel.
#pragma once

#define KVQ_TC_INSTANCES(Q)                                                                     \
  Q(4, 2, 128, 4, 64, 64) Q(4, 2, 128, 1, 64, 64) Q(4, 2, 128, 4, 32, 32) Q(4, 2, 128, 1, 32, 32) \
  Q(4, 2, 32, 4, 32, 32) Q(4, 2, 32, 1, 32, 32) Q(4, 2, 32, 4, 64, 64) Q(4, 2, 32, 1, 64, 64)     \
  Q(4, 4, 128, 4, 64, 64) Q(4, 4, 128, 1, 64, 64) Q(4, 4, 32, 4, 64, 64) Q(4, 4, 32, 1, 64, 64)   \
  Q(8, 4, 128, 4, 64, 64) Q(8, 4, 128, 1, 64, 64) Q(8, 4, 128, 4, 32, 32) Q(8, 4, 128, 1, 32, 32) \
  Q(8, 4, 32, 4, 64, 64) Q(8, 4, 32, 1, 64, 64)                                                 \
  Q(2, 2, 128, 4, 64, 64) Q(2, 2, 128, 1, 64, 64) Q(2, 2, 128, 4, 32, 32) Q(2, 2, 128, 1, 32, 32)

#define KVQ_FP16_INSTANCES(F) F(128, 4) F(128, 1) F(32, 4) F(32, 1)
