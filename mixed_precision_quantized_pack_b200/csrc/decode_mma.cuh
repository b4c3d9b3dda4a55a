// Split-K flash-decoding kernel for the fp16 rows of the cache: the retained
// tokens, then the recent window (or, for an unquantized cache, every token).
//
// One CTA = 4 warps = one split of one (b, kv head) over the fp16 list.  The
// quantized groups are read by the tcgen05 kernel (decode_tc.cuh); token order is
// free ("LogQuant: Log-Distributed 2-Bit Quantization of KV Cache", §4), so the
// two kinds of tokens are visited by separate CTAs and merged by the log-sum-exp
// combine.  The fp16 list of a quantized cache is short (window R plus at most 32
// retained tokens), so this path stays on warp-level mma.sync.
//
// Units of 16 list rows go round-robin to the CTA's warps and flow through a
// CTA-wide ring of shared-memory stages filled by 1-D bulk copies (cp.async.bulk)
// that complete on a per-stage mbarrier; the warp that finishes unit k refills
// its stage with unit k + ring.  A per-stage unit tag keeps a waiting warp from
// confusing two phases of the same mbarrier.  Waits are bounded (1 s of
// globaltimer); on timeout the CTA sets KVQ_STATUS_TIMEOUT in the workspace
// status word, waits (again bounded) for its last copies and contributes nothing.
//
// Scores ("HeadQ", §2.1: s_j = q.k_j/sqrt(d); "Thin Keys, Full Values", §2:
// d = d_k) use mma.m16n8k16 with the 16 rows of a unit on M and the GQA query
// heads sharing the kv head on N (column 2h; column 2h+1 stays zero); p.V uses
// the transposed orientation (channels on M, the 16 rows on K) with p split into
// (hi, lo) fp16 halves in columns 2h, 2h+1 so that p keeps about 22 bits.
#pragma once

#include "../../include/kvq.h"
#include "kvq_internal.cuh"
#include "ptx.cuh"

namespace kvq {
namespace mma {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr int kDV = 128;
constexpr int kMaxRing = 8;
constexpr int kMinRing = kWarps + 1;         // fewer stages than warps would idle a warp
constexpr float kLazyRescale = 8.0f;         // see the online-softmax update
constexpr int kSmemPerCta = 57344;           // 228 KB per SM / 4 CTAs, minus 1 KB reserved each

template <int DK>
struct Raw {
  static constexpr int KST = DK * 2 + 16;            // padded row strides in shared memory
  static constexpr int VST = kDV * 2 + 16;
  static constexpr int BYTES = 16 * (KST + VST);
  static constexpr int KSTEPS = DK / 16;
};

// Shared memory of one CTA: R mbarriers, R copy counters, R unit tags and a failure flag,
// then a ring of R stages that the CTA's warps share: unit k lives in stage k % R.  The
// tag of a stage is the unit whose copy was last issued into it: a warp waits for its
// unit's tag before it waits on the stage's mbarrier, so that barrier is never more than
// one phase away from the one the warp's parity names.
struct Smem {
  static constexpr int kBars = 0;
  static constexpr int kIssued = kBars + kMaxRing * 8;
  static constexpr int kTag = kIssued + kMaxRing * 4;
  static constexpr int kFail = kTag + kMaxRing * 4;
  static constexpr int kStages = 256;
  static_assert(kFail + 4 <= kStages, "header overflow");
};

template <int DK>
constexpr int stage_bytes() {
  return (Raw<DK>::BYTES + 127) / 128 * 128;
}

template <int DK>
constexpr int ring_stages() {
  const int r = (kSmemPerCta - Smem::kStages) / stage_bytes<DK>();
  return r < kMinRing ? kMinRing : (r > kMaxRing ? kMaxRing : r);
}

template <int DK, int NREP>
__global__ void __launch_bounds__(kThreads, 4)
decode_fp16_kernel(Dims d, CacheBufs cb, DecodeWork w, const __half* __restrict__ q, Partials part) {
  using R = Raw<DK>;
  constexpr int KSTEPS = DK / 16;
  constexpr int STAGE = stage_bytes<DK>();
  constexpr int RING = ring_stages<DK>();
  extern __shared__ __align__(128) unsigned char smem[];

  // the fp16 CTAs' partials follow those of the quantized groups
  const int split = w.splits_q + blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * d.Hkv + h;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = lane & 3;          // quad index: C columns 2qi, 2qi+1 = head qi (hi, lo)
  const int qr = lane >> 2;         // row group: A rows qr, qr+8; B column qr
  const int bhead = qr >> 1;        // head of this thread's B column
  const bool blo = (qr & 1) != 0;   // B column holds the lo half
  const bool bvalid = bhead < NREP;
  const bool cvalid = qi < NREP;    // lanes of padding columns compute values nobody reads

  int* sm_issued = reinterpret_cast<int*>(smem + Smem::kIssued);
  volatile int* sm_tag = reinterpret_cast<volatile int*>(smem + Smem::kTag);
  int* sm_fail = reinterpret_cast<int*>(smem + Smem::kFail);
  const uint32_t bar0 = ptx::smem_addr(smem + Smem::kBars);
  unsigned char* stages = smem + Smem::kStages;
  const uint32_t stages_s = ptx::smem_addr(stages);

  if (threadIdx.x == 0) {
    for (int s = 0; s < RING; ++s) {
      ptx::mbar_init(bar0 + 8 * s, 1);
      sm_issued[s] = 0;
      sm_tag[s] = -1;
    }
    *sm_fail = 0;
    ptx::fence_barrier_init();
  }
  const __half* qrow = q + (static_cast<size_t>(b) * d.Hq + h * NREP + (bvalid ? bhead : 0)) * DK;

  // this CTA's rows of the fp16 list, in units of 16
  const int f = blockIdx.x;
  const int list_begin = static_cast<int>(static_cast<long long>(f) * w.n_fp16 / w.splits_f);
  const int list_end = static_cast<int>(static_cast<long long>(f + 1) * w.n_fp16 / w.splits_f);
  const int n_units = (list_end - list_begin + 15) / 16;

  // running softmax state of head qi over this warp's rows
  float m_run = -INFINITY, l_run = 0.0f;
  float co[8][4];
#pragma unroll
  for (int mv = 0; mv < 8; ++mv)
#pragma unroll
    for (int e = 0; e < 4; ++e) co[mv][e] = 0.0f;
  bool failed = false;
  const float alpha = w.score_scale;                       // log2(e) / sqrt(d_k)

  uint32_t qn[KSTEPS][2];
#pragma unroll
  for (int s = 0; s < KSTEPS; ++s)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = 16 * s + 2 * qi + 8 * j;
      qn[s][j] = (bvalid && !blo) ? ptx::h2_as_u32(__halves2half2(qrow[c], qrow[c + 1])) : 0u;
    }
  // stale shared memory must hold finite values: masked rows multiply p = 0
  for (int i = threadIdx.x; i < RING * STAGE / 16; i += kThreads)
    reinterpret_cast<uint4*>(stages)[i] = make_uint4(0, 0, 0, 0);
  ptx::fence_proxy_async_smem();
  __syncthreads();

  // the 32 lanes of one warp copy the up to 16 key and 16 value rows of unit k
  auto issue = [&](int k) {
    const int st = k % RING;
    const uint32_t bar = bar0 + 8 * st;
    const uint32_t dst = stages_s + st * STAGE;
    const int e0 = list_begin + 16 * k;
    const int nvalid = min(16, list_end - e0);
    if (lane == 0) {
      sm_issued[st] += 1;
      sm_tag[st] = k;
      ptx::mbar_arrive_expect_tx(bar, nvalid * (DK + kDV) * 2);
    }
    __syncwarp();
    const int row = lane & 15;
    if (row < nvalid) {
      const int e = e0 + row;
      size_t slot;
      const __half* base_k;
      const __half* base_v;
      if (e < w.ret.n) {
        slot = static_cast<size_t>(bh) * kMaxRetained + e;
        base_k = cb.ret_k;
        base_v = cb.ret_v;
      } else {
        const int pos = w.Q + (e - w.ret.n);
        slot = static_cast<size_t>(bh) * d.cap + pos % d.cap;
        base_k = cb.win_k;
        base_v = cb.win_v;
      }
      if (lane < 16)
        ptx::bulk_g2s(dst + row * R::KST, base_k + slot * DK, DK * 2, bar);
      else
        ptx::bulk_g2s(dst + 16 * R::KST + row * R::VST, base_v + slot * kDV, kDV * 2, bar);
    }
  };

  if (warp == 0)
    for (int k = 0; k < RING && k < n_units; ++k) issue(k);
  for (int k = warp; k < n_units; k += kWarps) {
    const int st = k % RING;
    const bool ok = ptx::wait_equal_bounded(sm_tag + st, k, kWaitLimitNs) &&
                    ptx::mbar_wait_bounded(bar0 + 8 * st, (k / RING) & 1, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) {
      failed = true;
      break;
    }
    const uint32_t S = stages_s + st * STAGE;
    const int nvalid = min(16, list_end - (list_begin + 16 * k));
    // scores: A = 16 key rows via ldmatrix, B = q (hi columns only)
    float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int mi = lane >> 3;                         // which 8x8 matrix this lane addresses
    const int arow = (mi & 1) * 8 + (lane & 7);
#pragma unroll
    for (int s = 0; s < KSTEPS; ++s) {
      uint32_t a0, a1, a2, a3;
      ptx::ldmatrix_x4(S + arow * R::KST + (16 * s + (mi >> 1) * 8) * 2, a0, a1, a2, a3);
      ptx::mma_16816(cs, a0, a1, a2, a3, qn[s][0], qn[s][1]);
    }
    float s0 = (cs[0] + cs[1]) * alpha;
    float s1 = (cs[2] + cs[3]) * alpha;
    if (qr >= nvalid) s0 = -INFINITY;
    if (qr + 8 >= nvalid) s1 = -INFINITY;
    float gmax = fmaxf(s0, s1);
    gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 4));
    gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 8));
    gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 16));
    // The reference maximum moves only when a score exceeds it by more than
    // kLazyRescale (log2 units): weights then stay below 2^kLazyRescale and the
    // accumulators are rescaled rarely.
    const float m_new = fmaxf(m_run, gmax);
    if (__any_sync(0xffffffffu, m_new > m_run + kLazyRescale)) {
      const float a = (m_new == -INFINITY) ? 1.0f : ptx::ex2(m_run - m_new);
      l_run *= a;
#pragma unroll
      for (int mv = 0; mv < 8; ++mv)
#pragma unroll
        for (int e = 0; e < 4; ++e) co[mv][e] *= a;
      m_run = m_new;
    }
    const float m_use = m_run == -INFINITY ? 0.0f : m_run;
    const float p0 = ptx::ex2(s0 - m_use);
    const float p1 = ptx::ex2(s1 - m_use);
    l_run += p0 + p1;
    uint32_t x0, x1;
    ptx::split_hi_lo_pair(p0, p1, x0, x1);
    const uint32_t bp0 = ptx::movmatrix_trans(x0);
    const uint32_t bp1 = ptx::movmatrix_trans(x1);
    // p.V: A = V^T tiles via ldmatrix.trans (rows = tokens in shared memory)
    const int vrow = (mi >> 1) * 8 + (lane & 7);
#pragma unroll
    for (int mv = 0; mv < 8; ++mv) {
      uint32_t a0, a1, a2, a3;
      ptx::ldmatrix_x4_trans(S + 16 * R::KST + vrow * R::VST + (16 * mv + (mi & 1) * 8) * 2, a0, a1,
                             a2, a3);
      ptx::mma_16816(co[mv], a0, a1, a2, a3, bp0, bp1);
    }
    __syncwarp();
    if (k + RING < n_units) {
      if (lane == 0) ptx::fence_proxy_async_smem();
      issue(k + RING);
    }
  }

  // A bounded wait gave up: flag it, then wait (bounded) for the last copy issued into
  // every stage so that no copy lands in shared memory after the CTA has exited.
  if (failed && lane == 0) {
    atomicOr(part.status, KVQ_STATUS_TIMEOUT);
    atomicOr(sm_fail, 1);
  }
  __syncthreads();
  if (*sm_fail) {
    if (threadIdx.x < RING && sm_issued[threadIdx.x] > 0)
      ptx::mbar_wait_bounded(bar0 + 8 * threadIdx.x, (sm_issued[threadIdx.x] - 1) & 1, kWaitLimitNs);
    failed = true;     // the CTA's partial is dropped as a whole
  }

  // ---------------- warp totals, then the CTA merge ----------------
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 4);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
  if (failed) {
    m_run = -INFINITY;
    l_run = 0.0f;
  }
  __syncthreads();   // every warp is done with the stages: reuse them for the merge
  float* sm_o = reinterpret_cast<float*>(smem + Smem::kStages);      // [kWarps][NREP][kDV]
  float* sm_ml = sm_o + kWarps * NREP * kDV;                         // [kWarps][NREP][2]
  if (cvalid) {
    float* dst = sm_o + (warp * NREP + qi) * kDV;
#pragma unroll
    for (int mv = 0; mv < 8; ++mv) {
      float o0 = co[mv][0] + co[mv][1];
      float o1 = co[mv][2] + co[mv][3];
      if (failed) o0 = o1 = 0.0f;
      dst[16 * mv + qr] = o0;
      dst[16 * mv + qr + 8] = o1;
    }
    if (qr == 0) {
      sm_ml[(warp * NREP + qi) * 2] = m_run;
      sm_ml[(warp * NREP + qi) * 2 + 1] = l_run;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < NREP * kDV; idx += kThreads) {
    const int r = idx / kDV, c = idx % kDV;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, sm_ml[(ww * NREP + r) * 2]);
    float acc = 0.0f, lsum = 0.0f;
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) {
      const float mw = sm_ml[(ww * NREP + r) * 2];
      const float wt = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
      acc = fmaf(wt, sm_o[(ww * NREP + r) * kDV + c], acc);
      lsum = fmaf(wt, sm_ml[(ww * NREP + r) * 2 + 1], lsum);
    }
    const size_t pi = (static_cast<size_t>(b) * d.Hq + h * NREP + r) * w.splits + split;
    part.o[pi * kDV + c] = acc;
    if (c == 0) part.ml[pi] = make_float2(M, lsum);
  }
}

// Launches the fp16-list CTAs: grid.x = w.splits_f, writing partials splits_q .. splits-1.
template <int DK, int NREP>
cudaError_t launch_fp16(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                        const Partials& p, cudaStream_t s) {
  constexpr int stage = stage_bytes<DK>();
  constexpr int ring = ring_stages<DK>();
  int smem = Smem::kStages + ring * stage;
  const int merge = kWarps * NREP * kDV * 4 + kWarps * NREP * 8;
  if (Smem::kStages + merge > smem) smem = Smem::kStages + merge;
  auto kern = decode_fp16_kernel<DK, NREP>;
  static int configured = 0;
  if (configured < smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  dim3 grid(w.splits_f, d.Hkv, d.B);
  kern<<<grid, kThreads, smem, s>>>(d, c, w, q, p);
  return cudaGetLastError();
}

}  // namespace mma
}  // namespace kvq
