// The tensor-core decode instances this library is built with, as an X-macro:
//   Q(KB, VB, DK, NREP, GV, GK)          quantized caches (value head dim 128)
//   S(KB, VB, DK, NREP, GV, GK, SR, SQ)  quantized caches with a rank-SR, SQ-bit side code
//   F(DK, NREP)                          unquantized fp16 caches (value head dim 128)
//   P(KB, VB, DK, NREP, GV, GK)          quantized paged caches (groups found through a block table)
//   T(KB, VB, DK, NREP, GV, GK, SR, SQ)  paged caches with a side code
// decode_mma.cu builds its dispatch table from the same lists; each
// decode_mma_inst_k*.cu file instantiates the Q entries whose KB it owns,
// decode_mma_inst_side.cu the S entries, decode_mma_inst_paged.cu the P entries and
// decode_mma_inst_paged_side.cu the T entries.
// Shapes not listed here run on the generic CUDA-core kernel.
#pragma once

#define KVQ_MMA_QUANT_INSTANCES(Q)                                                              \
  Q(4, 2, 128, 4, 64, 64) Q(4, 2, 128, 1, 64, 64) Q(4, 2, 128, 4, 32, 32) Q(4, 2, 128, 1, 32, 32) \
  Q(4, 2, 32, 4, 32, 32) Q(4, 2, 32, 1, 32, 32) Q(4, 2, 32, 4, 64, 64) Q(4, 2, 32, 1, 64, 64)     \
  Q(4, 4, 128, 4, 64, 64) Q(4, 4, 128, 1, 64, 64) Q(4, 4, 32, 4, 64, 64) Q(4, 4, 32, 1, 64, 64)   \
  Q(8, 4, 128, 4, 64, 64) Q(8, 4, 128, 1, 64, 64) Q(8, 4, 128, 4, 32, 32) Q(8, 4, 128, 1, 32, 32) \
  Q(8, 4, 32, 4, 64, 64) Q(8, 4, 32, 1, 64, 64)                                                 \
  Q(2, 2, 128, 4, 64, 64) Q(2, 2, 128, 1, 64, 64) Q(2, 2, 128, 4, 32, 32) Q(2, 2, 128, 1, 32, 32)

#define KVQ_MMA_FP16_INSTANCES(F) F(128, 4) F(128, 1) F(32, 4) F(32, 1)

#define KVQ_MMA_SIDE_INSTANCES(S)                                                               \
  S(4, 2, 128, 4, 64, 64, 4, 4) S(4, 2, 128, 4, 64, 64, 4, 8) S(4, 2, 128, 4, 64, 64, 8, 4)      \
  S(2, 2, 128, 4, 64, 64, 4, 4) S(2, 2, 128, 4, 64, 64, 4, 8) S(2, 2, 128, 4, 64, 64, 8, 4)

#define KVQ_MMA_PAGED_INSTANCES(P)                                                              \
  P(4, 2, 128, 4, 64, 64) P(4, 2, 128, 1, 64, 64) P(4, 4, 128, 4, 64, 64) P(8, 4, 128, 4, 64, 64) \
  P(2, 2, 128, 4, 64, 64)

#define KVQ_MMA_PAGED_SIDE_INSTANCES(T)                                                         \
  T(4, 2, 128, 4, 64, 64, 4, 4) T(4, 2, 128, 4, 64, 64, 4, 8) T(4, 2, 128, 4, 64, 64, 8, 4)      \
  T(2, 2, 128, 4, 64, 64, 4, 4) T(2, 2, 128, 4, 64, 64, 4, 8) T(2, 2, 128, 4, 64, 64, 8, 4)
