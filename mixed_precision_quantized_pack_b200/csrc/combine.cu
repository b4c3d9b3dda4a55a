// Merge of the split partials of a decode (flash-decoding log-sum-exp merge).
// Each split s of row (b, hq) left m_s (running max of log2-scaled scores),
// l_s = sum_j 2^(s_j - m_s) and o_s = sum_j 2^(s_j - m_s) v_j.  The output is
//   o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s,
// in fp32, rounded once to fp16.  Splits that saw no token carry m = -inf, l = 0
// and are skipped.  Token order does not matter ("LogQuant: Log-Distributed
// 2-Bit Quantization of KV Cache", §4), so the splits may cover any partition.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

__global__ void combine_kernel(const float2* __restrict__ ml, const float* __restrict__ o,
                               int splits, int dv, __half* __restrict__ out) {
  const int row = blockIdx.x;
  const float2* mlr = ml + static_cast<size_t>(row) * splits;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, mlr[s].x);
  const float* orow = o + static_cast<size_t>(row) * splits * dv;
  for (int c = threadIdx.x; c < dv; c += blockDim.x) {
    float num = 0.0f, den = 0.0f;
    for (int s = 0; s < splits; ++s) {
      const float2 v = mlr[s];
      if (v.x == -INFINITY) continue;
      const float w = exp2f(v.x - M);
      num = fmaf(w, orow[static_cast<size_t>(s) * dv + c], num);
      den = fmaf(w, v.y, den);
    }
    out[static_cast<size_t>(row) * dv + c] = __float2half_rn(num / den);
  }
}

}  // namespace

cudaError_t launch_combine(const Dims& d, const DecodeWork& w, const Partials& p, __half* out,
                           cudaStream_t s) {
  const int rows = d.B * d.Hq;
  const int threads = d.dv < 128 ? d.dv : 128;
  combine_kernel<<<rows, threads, 0, s>>>(p.ml, p.o, w.splits, d.dv, out);
  return cudaGetLastError();
}

}  // namespace kvq
