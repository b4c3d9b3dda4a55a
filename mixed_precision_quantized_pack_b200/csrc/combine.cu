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
// merge is latency-bound (a few kilobytes per row, in L2).  The lanes first read the splits'
// (m, l) strided over the warp (a split per lane) and reduce M and the denominator by shuffles,
// leaving each split's weight 2^(m_s - M) in shared memory; then each lane issues the loads of
// kChunk splits' 16-byte pieces at once and weights them.
constexpr int kRowsPerBlock = 4;
constexpr int kChunk = 16;
constexpr int kMaxSplits = 512;     // the planner's cap: 256 quantized + 256 fp16 splits of a row

__global__ void __launch_bounds__(32 * kRowsPerBlock)
combine_kernel(const float2* __restrict__ ml, const float* __restrict__ o, int rows, int splits, int dv,
               __half* __restrict__ out) {
  __shared__ float sm_w[kRowsPerBlock][kMaxSplits];
  // launched as a programmatic dependent of the decode kernel: wait until that grid has
  // completed and its partials are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int wr = threadIdx.x >> 5;
  const int row = blockIdx.x * kRowsPerBlock + wr;
  if (row >= rows) return;                                    // uniform per warp
  const float2* mlr = ml + static_cast<size_t>(row) * splits;
  const float* orow = o + static_cast<size_t>(row) * splits * dv;
  float* wts = sm_w[wr];
  // splits that saw no token carry m = -inf, l = 0: weight 0
  float2 v[kMaxSplits / 32];
#pragma unroll
  for (int i = 0; i < kMaxSplits / 32; ++i) {
    const int s = lane + 32 * i;
    v[i] = s < splits ? mlr[s] : make_float2(-INFINITY, 0.0f);
  }
  float M = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxSplits / 32; ++i) M = fmaxf(M, v[i].x);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float den = 0.0f;
#pragma unroll
  for (int i = 0; i < kMaxSplits / 32; ++i) {
    const int s = lane + 32 * i;
    const float wgt = v[i].x == -INFINITY ? 0.0f : exp2f(v[i].x - M);
    if (s < splits) wts[s] = wgt;
    den = fmaf(wgt, v[i].y, den);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  __syncwarp();
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
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        if (s0 + j >= splits) break;
        const float wj = wts[s0 + j];
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
  if (w.splits < 1 || w.splits > kMaxSplits) return cudaErrorInvalidValue;
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
