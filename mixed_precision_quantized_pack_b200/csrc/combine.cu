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

// One warp per row (b, hq): lane s < splits holds split s's (m, l); the warp reduces the
// maximum and the weighted sum of l with shuffles, then every lane merges 4 channels
// (dv / 4 <= 32 * 4) of all splits with independent 16-byte loads.
constexpr int kRowsPerBlock = 4;

__global__ void __launch_bounds__(32 * kRowsPerBlock)
combine_kernel(const float2* __restrict__ ml, const float* __restrict__ o, int rows, int splits, int dv,
               __half* __restrict__ out) {
  // launched as a programmatic dependent of the decode kernel: wait until that grid has
  // completed and its partials are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  if (row >= rows) return;                                    // uniform per warp
  const float2* mlr = ml + static_cast<size_t>(row) * splits;
  const float* orow = o + static_cast<size_t>(row) * splits * dv;
  float M = -INFINITY;
  for (int s = lane; s < splits; s += 32) M = fmaxf(M, mlr[s].x);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float den = 0.0f;
  for (int s = lane; s < splits; s += 32) {
    const float2 v = mlr[s];
    if (v.x != -INFINITY) den = fmaf(exp2f(v.x - M), v.y, den);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  // every lane runs every iteration (the shuffles need the whole warp); lanes past d_v
  // only skip their loads and stores
  for (int c0 = 0; c0 < dv; c0 += 128) {
    const int c = c0 + 4 * lane;
    const bool mine = c < dv;
    float4 num = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int s0 = 0; s0 < splits; s0 += 32) {
      // weight of split s0 + j, held by lane j
      const int sj = s0 + lane;
      float wj = 0.0f;
      if (sj < splits) {
        const float mj = mlr[sj].x;
        wj = mj == -INFINITY ? 0.0f : exp2f(mj - M);
      }
      const int n = min(32, splits - s0);
      for (int j = 0; j < n; ++j) {
        const float w = __shfl_sync(0xffffffffu, wj, j);
        if (w == 0.0f || !mine) continue;
        const float4 x = *reinterpret_cast<const float4*>(orow + static_cast<size_t>(s0 + j) * dv + c);
        num.x = fmaf(w, x.x, num.x);
        num.y = fmaf(w, x.y, num.y);
        num.z = fmaf(w, x.z, num.z);
        num.w = fmaf(w, x.w, num.w);
      }
    }
    if (mine) {
      const __half2 h0 = __floats2half2_rn(num.x / den, num.y / den);
      const __half2 h1 = __floats2half2_rn(num.z / den, num.w / den);
      uint2 packed;
      packed.x = *reinterpret_cast<const uint32_t*>(&h0);
      packed.y = *reinterpret_cast<const uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(out + static_cast<size_t>(row) * dv + c) = packed;
    }
  }
}

}  // namespace

cudaError_t launch_combine(const Dims& d, const DecodeWork& w, const Partials& p, __half* out,
                           cudaStream_t s) {
  const int rows = d.B * d.Hq;
  // Programmatic dependent launch: the merge may be scheduled while the decode grid drains;
  // it waits (griddepcontrol.wait) for that grid before reading its partials.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((rows + kRowsPerBlock - 1) / kRowsPerBlock);
  cfg.blockDim = dim3(32 * kRowsPerBlock);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, p.ml, static_cast<const float*>(p.o), rows, w.splits,
                            d.dv, out);
}

}  // namespace kvq
