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

// One warp per row (b, hq); lane l merges channels 4l .. 4l+3 of every 128-channel block.  The
// merge is latency-bound (a few kilobytes per row, in L2), so each lane first issues the loads
// of kChunk splits' 16-byte pieces at once, then reads the splits' (m, l) (the same address in
// every lane) for the maximum and the denominator, then weights the pieces it already holds.
constexpr int kRowsPerBlock = 4;
constexpr int kChunk = 8;

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
  float M = -INFINITY, den = 0.0f;
  for (int c0 = 0; c0 < dv; c0 += 128) {
    const int c = c0 + 4 * lane;
    const bool mine = c < dv;
    float4 num = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int s0 = 0; s0 < splits; s0 += kChunk) {
      float4 buf[kChunk];
#pragma unroll
      for (int j = 0; j < kChunk; ++j)
        buf[j] = mine && s0 + j < splits
                     ? *reinterpret_cast<const float4*>(orow + static_cast<size_t>(s0 + j) * dv + c)
                     : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (c0 == 0 && s0 == 0) {
        // splits that saw no token carry m = -inf, l = 0 and are skipped
        for (int s = 0; s < splits; ++s) M = fmaxf(M, mlr[s].x);
        for (int s = 0; s < splits; ++s) {
          const float2 v = mlr[s];
          if (v.x != -INFINITY) den = fmaf(exp2f(v.x - M), v.y, den);
        }
      }
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        if (s0 + j >= splits) break;
        const float mj = mlr[s0 + j].x;
        const float wj = mj == -INFINITY ? 0.0f : exp2f(mj - M);
        num.x = fmaf(wj, buf[j].x, num.x);
        num.y = fmaf(wj, buf[j].y, num.y);
        num.z = fmaf(wj, buf[j].z, num.z);
        num.w = fmaf(wj, buf[j].w, num.w);
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
