// Fused dequant + split-K flash-decoding kernel on the tensor cores (sm_100a).
//
// One CTA = 4 warps = one split of one (b, kv head).  Splits [0, splits_q) cover
// whole key groups of the quantized prefix; splits [splits_q, splits) cover the
// fp16 list (retained tokens, then the window).  Token order is free
// ("LogQuant: Log-Distributed 2-Bit Quantization of KV Cache", §4), so the two
// kinds of tokens are visited separately and merged by the log-sum-exp combine.
//
// A CTA's units (key groups, or tiles of 16 fp16 rows) go round-robin to its warps
// and flow through a CTA-wide ring of shared-memory stages (as many as keep four
// CTAs per SM), each filled by 1-D bulk copies (cp.async.bulk) that complete on a
// per-stage mbarrier; the warp that finishes unit k refills its stage with unit
// k + ring.  Waits are bounded (1 s of globaltimer); on timeout the CTA sets
// KVQ_STATUS_TIMEOUT in the workspace status word, waits (again bounded) for its
// last copies and contributes nothing.
//
// Scores ("HeadQ", §2.1: s_j = q.k_j/sqrt(d); "Thin Keys, Full Values", §2: d = d_k)
// use mma.m16n8k16 with the tokens of a 16-token tile on M and, on N, the GQA
// query heads sharing the kv head, each twice: column 2h holds hi(q'_h), column
// 2h+1 holds lo(q'_h), where q'_c = q_c * s_{g,c} folds the per-channel key scale
// into the query once per group and hi/lo are the two fp16 halves of the exact
// fp32 product (hi + lo == q'_c).  The key codes enter the MMA unconverted: a
// b-bit field masked in place inside a 16-bit lane is an fp16 subnormal of value
// code * 2^(p-24), p its bit offset (p + b <= 8 after at most one byte shift), so
// unpacking is one AND per two codes; the factor 2^-p goes into q' and the common
// 2^-24 into the softmax scale.  The zero points add sum_c q_c z_{g,c} per group,
// computed by one more MMA per k-step with z in A and q in B.  A group's key
// (scale, zero) block lists, per packed word, the channel pairs of its registers,
// so the B pairs (s_c, s_c+16/b) and the A pairs (z_c, z_c+16/b) are plain loads;
// the words' blocks are quarter-interleaved so that the four quads of a warp, which
// read the four quarters of a key row, load neighbouring blocks.
//
// With a side code ("HeadQ: Distortion visible par le modele et correction dans
// l'espace des scores pour la quantification du cache KV", §3, step 3) each 16-token
// tile gets one more MMA (m16n8k8) into the same score accumulator: A = the side
// codes of the tile's tokens (r coordinates on K, masked as subnormals like the key
// codes), B = (hi, lo) of (U_h^T q)_i * s_i per head, and the side zeros add
// sum_i (U_h^T q)_i z_i to the group's bias.  U_h^T q is formed once per CTA.
//
// p.V uses the transposed orientation: channels on M, the 16 tokens on K, and on
// N again (hi, lo) pairs, now of p_j * s_{j,g} (per-token value scale), moved from
// the score accumulator layout to the B layout with movmatrix.  Value codes are
// masked as subnormals too; their 2^(p-24) factors are per output channel and are
// removed once at the end, where sum_j p_j z_{j,g} is added.
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
constexpr int kMaxRing = 8;                  // stages of a CTA-wide copy ring, at most
constexpr int kMinRing = kWarps + 1;         // fewer stages than warps would idle a warp
constexpr float kLazyRescale = 8.0f;         // see the online-softmax update
constexpr int kCtasPerSm = 4;
constexpr int kSmemPerCta = 233472 / kCtasPerSm - 1024;   // 228 KB per SM, 1 KB reserved per CTA

// ---------------------------------------------------------------- geometry ----
template <int KB, int VB, int DK, int GV>
struct Quant {
  static constexpr int KW = DK * KB / 32;            // u32 words per key row
  static constexpr int VW = kDV * VB / 32;           // u32 words per value row
  static constexpr int WPT = KW / 4;                 // key words per thread (a quad shares a row)
  static constexpr int KSTEPS = DK / 16;
  static constexpr int RPW = 16 / KB;                // A registers per key word
  static constexpr int KSPW = RPW / 2;               // k-steps per key word
  static constexpr int CPW = 32 / KB;                // channels per key word
  static constexpr int NVG = kDV / GV;               // value groups per token
  static constexpr int MPG = GV / 16;                // value m-tiles per value group
  static constexpr int CPG = GV / 8;                 // channels a thread owns per value group
  static constexpr int RUN = CPG * VB;               // bits of that run in a value row
  static constexpr int KBYTES_ROW = DK * KB / 8;
  static constexpr int VBYTES_ROW = kDV * VB / 8;
  static_assert(WPT >= 1 && KSTEPS == WPT * KSPW, "key row too short for the fragment mapping");
  static_assert(RUN == 8 || RUN == 16 || RUN == 32, "value run must be 8, 16 or 32 bits");
  static_assert(MPG >= 1, "value group below 16 channels");
};

// Side-code geometry: SR coordinates of SQ bits per token, one row of ZB bytes.  Quad qi
// (lanes with lane % 4 == qi) holds k-slots (2qi, 2qi+1) of the m16n8k8 side MMA, i.e.
// coordinates (qi, qi + SR/2) for qi < SR/2; its A register of a row is
// (row >> shift(qi)) & mask(qi), a pair of subnormals with factor 2^(p(qi)-24).
template <int SR, int SQ>
struct Side {
  static constexpr int ZB = SR * SQ / 8;
  static constexpr int NQ = SR / 2;            // quads that hold coordinates
  static_assert(SR == 0 || (SR * SQ == 16 || SR * SQ == 32), "side row of 16 or 32 bits");
  __host__ __device__ static constexpr int shift(int qi) {
    return SR == 8 ? 8 * (qi >> 1) : (SQ == 8 ? 8 * qi : 0);
  }
  __host__ __device__ static constexpr int pos(int qi) {   // bit offset of the field in its half
    return SR == 8 ? 4 * (qi & 1) : (SQ == 8 ? 0 : 4 * qi);
  }
  __host__ __device__ static constexpr uint32_t mask(int qi) {
    return qi >= NQ ? 0u : (SQ == 8 ? 0x00FF00FFu : (0x000F000Fu << pos(qi)));
  }
};

template <int DK>
struct Raw {
  static constexpr int KST = DK * 2 + 16;            // padded row strides in shared memory
  static constexpr int VST = kDV * 2 + 16;
  static constexpr int BYTES = 16 * (KST + VST);
  static constexpr int KSTEPS = DK / 16;
};

// fp16 mantissa-field masks: the `bits`-wide field at bit `pos` of both 16-bit halves.
template <int BITS, int POS>
struct Mask {
  static constexpr uint32_t v = (((1u << BITS) - 1u) << POS) * 0x00010001u;
};

// Register rho of a key word: the pair (channel c, channel c + 16/KB) as subnormals
// with factor 2^(p-24), p = (KB * rho) mod 8.
template <int KB>
__device__ __forceinline__ void unpack_key_word(uint32_t w, uint32_t (&r)[16 / KB]) {
  if constexpr (KB == 4) {
    const uint32_t u = w >> 8;
    r[0] = w & Mask<4, 0>::v;
    r[1] = w & Mask<4, 4>::v;
    r[2] = u & Mask<4, 0>::v;
    r[3] = u & Mask<4, 4>::v;
  } else if constexpr (KB == 2) {
    const uint32_t u = w >> 8;
    r[0] = w & Mask<2, 0>::v;
    r[1] = w & Mask<2, 2>::v;
    r[2] = w & Mask<2, 4>::v;
    r[3] = w & Mask<2, 6>::v;
    r[4] = u & Mask<2, 0>::v;
    r[5] = u & Mask<2, 2>::v;
    r[6] = u & Mask<2, 4>::v;
    r[7] = u & Mask<2, 6>::v;
  } else {
    r[0] = w & Mask<8, 0>::v;
    r[1] = (w >> 8) & Mask<8, 0>::v;
  }
}

template <int KB>
__host__ __device__ constexpr int key_reg_shift(int rho) { return (KB * rho) % 8; }

// The codes of one 16-bit piece (token a in the low half, token b in the high
// half), as subnormal pairs; code e' sits at bit VB*e' of the piece.
template <int VB>
__device__ __forceinline__ void unpack_value_piece16(uint32_t x, uint32_t* r) {
  const uint32_t u = x >> 8;
  if constexpr (VB == 2) {
    r[0] = x & Mask<2, 0>::v;
    r[1] = x & Mask<2, 2>::v;
    r[2] = x & Mask<2, 4>::v;
    r[3] = x & Mask<2, 6>::v;
    r[4] = u & Mask<2, 0>::v;
    r[5] = u & Mask<2, 2>::v;
    r[6] = u & Mask<2, 4>::v;
    r[7] = u & Mask<2, 6>::v;
  } else if constexpr (VB == 4) {
    r[0] = x & Mask<4, 0>::v;
    r[1] = x & Mask<4, 4>::v;
    r[2] = u & Mask<4, 0>::v;
    r[3] = u & Mask<4, 4>::v;
  } else {
    r[0] = x & Mask<8, 0>::v;
    r[1] = u & Mask<8, 0>::v;
  }
}

template <int VB>
__device__ __forceinline__ void unpack_value_piece8(uint32_t x, uint32_t* r) {
  static_assert(VB == 2 || VB == 4 || VB == 8, "");
  if constexpr (VB == 2) {
    r[0] = x & Mask<2, 0>::v;
    r[1] = x & Mask<2, 2>::v;
    r[2] = x & Mask<2, 4>::v;
    r[3] = x & Mask<2, 6>::v;
  } else if constexpr (VB == 4) {
    r[0] = x & Mask<4, 0>::v;
    r[1] = x & Mask<4, 4>::v;
  } else {
    r[0] = x & Mask<8, 0>::v;
  }
}

// Bit offset (within its fp16 lane) of code e of a thread's value run.
template <int VB, int RUN>
__host__ __device__ constexpr int value_code_shift(int e) {
  return RUN == 8 ? (VB * e) % 8 : (VB * (e % (16 / VB))) % 8;
}

// N consecutive u32 from shared memory at an address aligned to min(4N, 16) bytes.
template <int N>
__device__ __forceinline__ void load_words(const uint32_t* p, uint32_t* out) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(p + i);
      out[i] = v.x;
      out[i + 1] = v.y;
      out[i + 2] = v.z;
      out[i + 3] = v.w;
    }
  } else if constexpr (N == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    out[0] = v.x;
    out[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = p[i];
  }
}

// The zero-point MMA's copy of q in shared memory: entry e of lane l, grouped four
// entries per lane so that a lane reads its consecutive entries with one 128-bit load.
__device__ __forceinline__ int qb_index(int e, int lane) { return ((e >> 2) * 32 + lane) * 4 + (e & 3); }

// --------------------------------------------------------------- the kernel ----
// Shared memory of one CTA: the query for the zero-point MMA and the query scaled for the
// score MMA (each u32 [2*KSTEPS][32 lanes]),
// then R mbarriers, R copy counters, R unit tags and a failure flag, then a ring of R
// stages that the CTA's warps share: unit k (a key group or 16 fp16 rows) lives in stage
// k % R.  The tag of a stage is the unit whose copy was last issued into it: a warp
// waits for its unit's tag before it waits on the stage's mbarrier, so that barrier is
// never more than one phase away from the one the warp's parity names.
template <int KSTEPS, int SR = 0>
struct Smem {
  static constexpr int kQb = 0;
  static constexpr int kQf = kQb + 2 * KSTEPS * 32 * 4;     // q scaled by 2^-p, same layout
  static constexpr int kBars = kQf + 2 * KSTEPS * 32 * 4;
  static constexpr int kIssued = kBars + kMaxRing * 8;
  static constexpr int kTag = kIssued + kMaxRing * 4;
  static constexpr int kFail = kTag + kMaxRing * 4;
  static constexpr int kPage = kFail + 16;                   // per warp: the next unit's page
  static constexpr int kQt = kPage + 16;                     // U_h^T q: fp32 [4 heads][SR]
  static constexpr int kStages = kBars + (SR ? 512 : 256);
  static_assert(kQt + 4 * SR * 4 <= kStages, "header overflow");
};

struct StageLayout {
  int k_off, kmeta_off, v_off, vmeta_off, z_off, zmeta_off, bytes;
};

__host__ __device__ inline StageLayout quant_stage_layout(int gk, int dk, int kb, int vb, int nvg,
                                                          int zb = 0, int sr = 0) {
  StageLayout s;
  s.k_off = 0;
  s.kmeta_off = gk * dk * kb / 8;
  s.v_off = s.kmeta_off + dk * 4;
  s.vmeta_off = s.v_off + gk * kDV * vb / 8;
  s.z_off = s.vmeta_off + gk * nvg * 4;
  s.zmeta_off = s.z_off + gk * zb;
  s.bytes = s.zmeta_off + sr * 4;
  return s;
}

// Bytes of one stage, rounded to 128: a whole key group for the quantized splits, 16 padded
// fp16 rows for the fp16 splits.  Each kind of split has its own ring over the same shared
// memory, with as many stages as keep a CTA within its share of the SM (kCtasPerSm CTAs).
template <int KB, int VB, int DK, int GV, int GK, int SR, int SQ>
constexpr int quant_stage_bytes() {
  return (GK * DK * KB / 8 + DK * 4 + GK * kDV * VB / 8 + GK * (kDV / GV) * 4 + GK * Side<SR, SQ>::ZB +
          SR * 4 + 127) / 128 * 128;
}

template <int DK>
constexpr int raw_stage_bytes() { return (Raw<DK>::BYTES + 127) / 128 * 128; }

constexpr int ring_for(int avail, int stage, int lo) {
  return avail / stage < lo ? lo : (avail / stage > kMaxRing ? kMaxRing : avail / stage);
}

template <int KB, int VB, int DK, int GV, int GK, bool QUANT, int SR, int SQ>
struct Rings {
  static constexpr int HDR = Smem<DK / 16, SR>::kStages;
  static constexpr int STAGE_Q = QUANT ? quant_stage_bytes<KB, VB, DK, GV, GK, SR, SQ>() : 128;
  static constexpr int STAGE_F = raw_stage_bytes<DK>();
  static constexpr int RING_Q = QUANT ? ring_for(kSmemPerCta - HDR, STAGE_Q, kMinRing) : 0;
  static constexpr int RING_F = ring_for(kSmemPerCta - HDR, STAGE_F, kWarps);
  static constexpr int BYTES = HDR + (RING_Q * STAGE_Q > RING_F * STAGE_F ? RING_Q * STAGE_Q
                                                                          : RING_F * STAGE_F);
};

template <int KB, int VB, int DK, int NREP, int GV, int GK, bool QUANT, int SR = 0, int SQ = 4,
          bool PAGED = false, bool CENTER = false>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
decode_mma_kernel(Dims d, CacheBufs cb, DecodeWork w, const __half* __restrict__ q, Partials part) {
  using G = Quant<(QUANT ? KB : 4), (QUANT ? VB : 2), (QUANT ? DK : 128), (QUANT ? GV : 64)>;
  using R = Raw<DK>;
  using Z = Side<SR, SQ>;
  constexpr int KSTEPS = DK / 16;
  using RG = Rings<KB, VB, DK, GV, GK, QUANT, SR, SQ>;
  using SM = Smem<KSTEPS, SR>;
  extern __shared__ __align__(128) unsigned char smem[];

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * d.Hkv + h;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = lane & 3;          // quad index: C columns 2qi, 2qi+1 = head qi (hi, lo)
  const int qr = lane >> 2;         // row group: A rows qr, qr+8; B column qr
  const int bhead = qr >> 1;        // head of this thread's B column
  const bool blo = (qr & 1) != 0;   // B column holds the lo half
  const bool bvalid = bhead < NREP;
  const bool cvalid = qi < NREP;   // lanes of padding columns compute values nobody reads

  uint32_t* sm_qb = reinterpret_cast<uint32_t*>(smem + SM::kQb);
  uint32_t* sm_qf = reinterpret_cast<uint32_t*>(smem + SM::kQf);
  int* sm_issued = reinterpret_cast<int*>(smem + SM::kIssued);
  volatile int* sm_tag = reinterpret_cast<volatile int*>(smem + SM::kTag);
  int* sm_fail = reinterpret_cast<int*>(smem + SM::kFail);
  const uint32_t bar0 = ptx::smem_addr(smem + SM::kBars);
  unsigned char* stages = smem + SM::kStages;
  const uint32_t stages_s = ptx::smem_addr(stages);

  const bool quant = QUANT && split < w.splits_q;
  const int ring = quant ? RG::RING_Q : RG::RING_F;     // stages of this CTA's ring
  if (threadIdx.x == 0) {
    for (int s = 0; s < ring; ++s) {
      ptx::mbar_init(bar0 + 8 * s, 1);
      sm_issued[s] = 0;
      sm_tag[s] = -1;
    }
    *sm_fail = 0;
    ptx::fence_barrier_init();
  }
  // the query rows of this CTA's heads (head j at qbase + j * DK); with key rotation, their
  // rotations, written by warp j into the stage area before the ring uses it
  const __half* qbase = q + (static_cast<size_t>(b) * d.Hq + h * NREP) * DK;
  if (d.rot) {
    __half* qr_s = reinterpret_cast<__half*>(stages);
    if (warp < NREP) {
      float x[DK / 32];
#pragma unroll
      for (int m = 0; m < DK / 32; ++m) x[m] = __half2float(qbase[warp * DK + lane + 32 * m]);
      rotate_row_warp<DK / 32>(x, DK / 32, d.rot_signs, d.rot_inv_cq, lane);
#pragma unroll
      for (int m = 0; m < DK / 32; ++m) qr_s[warp * DK + lane + 32 * m] = __float2half_rn(x[m]);
    }
    __syncthreads();
    qbase = qr_s;
  }
  const __half* qrow = qbase + (bvalid ? bhead : 0) * DK;

  // ---------------- work list of this warp ----------------
  const SeqWork sw = seq_work(w, b, QUANT ? GK : 1, QUANT ? d.log_retain : 0);   // this sequence's lengths
  int unit_begin, unit_end;      // quantized: groups; fp16: tiles of 16 list entries
  int list_begin = 0, list_end = 0;
  if (quant) {
    unit_begin = static_cast<int>(static_cast<long long>(split) * sw.n_groups / w.splits_q);
    unit_end = static_cast<int>(static_cast<long long>(split + 1) * sw.n_groups / w.splits_q);
  } else {
    const int f = split - (QUANT ? w.splits_q : 0);
    list_begin = static_cast<int>(static_cast<long long>(f) * sw.n_fp16 / w.splits_f);
    list_end = static_cast<int>(static_cast<long long>(f + 1) * sw.n_fp16 / w.splits_f);
    unit_begin = 0;
    unit_end = (list_end - list_begin + 15) / 16;
  }
  // unit k of this CTA (k < n_units) is processed by warp k % kWarps, in stage k % ring
  const int n_units = unit_end - unit_begin;

  // running softmax state of head qi over this warp's tokens
  float m_run = -INFINITY, l_run = 0.0f;
  float zsum[G::NVG];               // sum_j p_j z_{j,g}, lane-partial
#pragma unroll
  for (int g = 0; g < G::NVG; ++g) zsum[g] = 0.0f;
  float co[8][4];
#pragma unroll
  for (int mv = 0; mv < 8; ++mv)
#pragma unroll
    for (int e = 0; e < 4; ++e) co[mv][e] = 0.0f;
  bool failed = false;

  const float alpha = w.score_scale;                       // log2(e) / sqrt(d_k)
  constexpr float kMid = static_cast<float>(1 << ((QUANT ? VB : 2) - 1));   // centre of the value codes
  const float alpha24 = w.score_scale * 16777216.0f;       // undoes the 2^-24 of subnormal codes

  if (quant) {
    if constexpr (QUANT) {
      // B operands: q (scaled by 2^-p per k-slot) in registers, plain q in shared memory
#pragma unroll
      for (int s = 0; s < KSTEPS; ++s)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int omega = qi * G::WPT + s / G::KSPW;
          const int rho = 2 * (s % G::KSPW) + j;
          const int c_lo = G::CPW * omega + rho;
          const int c_hi = c_lo + 16 / KB;
          const __half2 pair = bvalid ? __halves2half2(qrow[c_lo], qrow[c_hi]) : __float2half2_rn(0.0f);
          const float f = 1.0f / static_cast<float>(1 << key_reg_shift<KB>(rho));
          if (warp == 0) {
            sm_qf[qb_index(2 * s + j, lane)] = ptx::h2_as_u32(__hmul2(pair, __float2half2_rn(f)));
            sm_qb[qb_index(2 * s + j, lane)] = ptx::h2_as_u32(pair);
          }
        }
      if constexpr (SR > 0) {
        // U_h^T q of head `warp`: each lane sums DK/32 channels, then the warp reduces
        float* sm_qt = reinterpret_cast<float*>(smem + SM::kQt);
        if (warp < NREP) {
          const __half* qw = qbase + warp * DK;
          const float* uh = cb.side_u + static_cast<size_t>(h) * DK * SR;
          float acc[SR];
#pragma unroll
          for (int i = 0; i < SR; ++i) acc[i] = 0.0f;
#pragma unroll
          for (int cc = 0; cc < DK / 32; ++cc) {
            const int c = lane + 32 * cc;
            const float qc = __half2float(qw[c]);
#pragma unroll
            for (int i4 = 0; i4 < SR; i4 += 4) {
              const float4 u4 = *reinterpret_cast<const float4*>(uh + c * SR + i4);
              acc[i4] = fmaf(u4.x, qc, acc[i4]);
              acc[i4 + 1] = fmaf(u4.y, qc, acc[i4 + 1]);
              acc[i4 + 2] = fmaf(u4.z, qc, acc[i4 + 2]);
              acc[i4 + 3] = fmaf(u4.w, qc, acc[i4 + 3]);
            }
          }
#pragma unroll
          for (int i = 0; i < SR; ++i) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
          }
          if (lane < SR) {
            float v = acc[0];
#pragma unroll
            for (int i = 1; i < SR; ++i) v = lane == i ? acc[i] : v;
            sm_qt[warp * SR + lane] = v;
          }
        }
      }
      __syncthreads();

      // retained positions, one per lane (ascending), for masking the quantized tiles
      const int ret_pos = lane < sw.n_ret ? retained_position(sw.Q, lane) : -1;
      const StageLayout L = quant_stage_layout(GK, DK, KB, VB, G::NVG, Z::ZB, SR);
      constexpr int gk = GK;
      constexpr int MT = GK / 16;     // 16-token m-tiles per key group
      // per-lane shuffle selectors for the bank-conflict-free value-row loads
      const bool swap = qi >= 2;
      const uint32_t sel_lo = swap ? 0x1054u : 0x5410u;
      const uint32_t sel_hi = swap ? 0x3276u : 0x7632u;

      constexpr int RING = RG::RING_Q, STAGE = RG::STAGE_Q;
      // Group index of unit k: its (scale, zero) block; its first token row is that times
      // GK.  A paged cache takes the group's page from the block table: a refill reads the
      // entry that its warp's lane 0 fetched (cp.async into the warp's slot) when the warp
      // began the unit before it.
      int* sm_page = reinterpret_cast<int*>(smem + SM::kPage);
      auto table_entry = [&](int k) {
        const int gg = unit_begin + k;
        return cb.table + (b * d.max_groups + (KVQ_IN_BOUNDS(d, kSiteDecTable, gg, d.max_groups) ? gg : 0));
      };
      auto group_of = [&](int k, bool fetched) -> size_t {
        if constexpr (!PAGED) return static_cast<size_t>(bh) * d.max_groups + unit_begin + k;
        int page;
        if (fetched) {
          ptx::cp_async_wait_all();
          page = sm_page[warp];
        } else {
          page = __ldg(table_entry(k));
        }
        return static_cast<size_t>(page) * d.Hkv + h;
      };
      // one lane copies unit k (a whole key group: 4 contiguous runs) into stage k % RING
      auto issue = [&](int k, size_t gi) {
        // (bounds-check builds) a group outside the buffers is replaced by group 0, so that the
        // stage's copies still complete
        if (!KVQ_IN_BOUNDS(d, kSiteDecKCode, static_cast<long long>(gi), quant_groups(d))) gi = 0;
        const int st = k % RING;
        const uint32_t bar = bar0 + 8 * st;
        const uint32_t dst = stages_s + st * STAGE;
        sm_issued[st] += 1;
        sm_tag[st] = k;
        // (test hook) one stage that never completes: its waits run into their bound
        const bool stall = w.stall && k == 0 && split == 0 && h == 0 && b == 0;
        ptx::mbar_arrive_expect_tx(bar, L.bytes + (stall ? 16u : 0u));
        const size_t tok = gi * gk;
        ptx::bulk_g2s(dst + L.k_off, cb.kcode + tok * G::KW, gk * G::KBYTES_ROW, bar);
        ptx::bulk_g2s(dst + L.kmeta_off, cb.ksz + gi * DK, DK * 4, bar);
        ptx::bulk_g2s(dst + L.v_off, cb.vcode + tok * G::VW, gk * G::VBYTES_ROW, bar);
        ptx::bulk_g2s(dst + L.vmeta_off, cb.vsz + tok * G::NVG, gk * G::NVG * 4, bar);
        if constexpr (SR > 0) {
          ptx::bulk_g2s(dst + L.z_off, cb.zcode + tok * Z::ZB, gk * Z::ZB, bar);
          ptx::bulk_g2s(dst + L.zmeta_off, cb.zsz + gi * SR, SR * 4, bar);
        }
      };

      if (threadIdx.x == 0) {
        ptx::fence_proxy_async_smem();     // the rotated query rows were written to the stages
        for (int k = 0; k < RING && k < n_units; ++k) issue(k, group_of(k, false));
      }

      for (int k = warp; k < n_units; k += kWarps) {
        // the page the stage is refilled with after this unit, fetched early
        if (PAGED && lane == 0 && k + RING < n_units)
          ptx::cp_async_4(ptx::smem_addr(sm_page + warp), table_entry(k + RING));
        const int g = unit_begin + k;
        const int st = k % RING;
        const bool ok = ptx::wait_equal_bounded(sm_tag + st, k, kWaitLimitNs) &&
                        ptx::mbar_wait_bounded(bar0 + 8 * st, (k / RING) & 1, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) {
          failed = true;
          break;
        }
        const unsigned char* S = stages + st * STAGE;
        const uint32_t* skc = reinterpret_cast<const uint32_t*>(S + L.k_off);
        const uint32_t* skm = reinterpret_cast<const uint32_t*>(S + L.kmeta_off);
        const uint32_t* svc = reinterpret_cast<const uint32_t*>(S + L.v_off);
        const uint32_t* svm = reinterpret_cast<const uint32_t*>(S + L.vmeta_off);

        // ---- group prologue: B = hi or lo of q*s, and the zero-point bias ----
        uint32_t bq[KSTEPS][2];
        float cbias[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
        for (int u = 0; u < G::WPT; ++u) {
          const int omega = qi * G::WPT + u;
          uint32_t meta[G::CPW];
#pragma unroll
          for (int c4 = 0; c4 < G::CPW; c4 += 4) {
            // word omega = qi * WPT + u: its block is stored at position u * 4 + qi
            const uint4 v4 = *reinterpret_cast<const uint4*>(skm + G::CPW * (u * 4 + qi) + c4);
            meta[c4] = v4.x;
            meta[c4 + 1] = v4.y;
            meta[c4 + 2] = v4.z;
            meta[c4 + 3] = v4.w;
          }
          uint32_t qbx[2 * G::KSPW], qfx[2 * G::KSPW];
          if constexpr (2 * G::KSPW >= 4) {
#pragma unroll
            for (int c4 = 0; c4 < 2 * G::KSPW; c4 += 4) {
              load_words<4>(sm_qb + qb_index(2 * u * G::KSPW + c4, lane), qbx + c4);
              load_words<4>(sm_qf + qb_index(2 * u * G::KSPW + c4, lane), qfx + c4);
            }
          } else {
            load_words<2 * G::KSPW>(sm_qb + qb_index(2 * u * G::KSPW, lane), qbx);
            load_words<2 * G::KSPW>(sm_qf + qb_index(2 * u * G::KSPW, lane), qfx);
          }
#pragma unroll
          for (int ls = 0; ls < G::KSPW; ++ls) {
            const int s = u * G::KSPW + ls;
            uint32_t za[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int rho = 2 * ls + j;
              // the word's block holds (s_c, s_c+16/KB) for each register, then the zeros
              const uint32_t s2 = meta[rho];
              za[j] = meta[G::RPW + rho];
              const __half2 qs = ptx::u32_as_h2(qfx[2 * ls + j]);
              const __half2 sc = ptx::u32_as_h2(s2);
              const __half2 hi = __hmul2(qs, sc);
              bq[s][j] = blo ? ptx::h2_as_u32(__hfma2(qs, sc, __hneg2(hi))) : ptx::h2_as_u32(hi);
            }
            ptx::mma_16816(cbias[s & 1], za[0], za[0], za[1], za[1], qbx[2 * ls], qbx[2 * ls + 1]);
          }
        }
        float side_bias = 0.0f;
        uint32_t bz = 0u;                 // B of the side MMA: (hi or lo) of (U^T q)_i * s_i * 2^-p
        if constexpr (SR > 0) {
          const float* sm_qt = reinterpret_cast<const float*>(smem + SM::kQt);
          const __half2* zm = reinterpret_cast<const __half2*>(S + L.zmeta_off);
          if (qi < Z::NQ) {
            const float f = 1.0f / static_cast<float>(1 << Z::pos(qi));
            const float2 m0 = __half22float2(zm[qi]), m1 = __half22float2(zm[qi + Z::NQ]);
            const int hb = bvalid ? bhead : 0;
            const float x0 = sm_qt[hb * SR + qi] * m0.x * f;
            const float x1 = sm_qt[hb * SR + qi + Z::NQ] * m1.x * f;
            const __half2 p0 = ptx::u32_as_h2(ptx::split_hi_lo_trunc(x0));
            const __half2 p1 = ptx::u32_as_h2(ptx::split_hi_lo_trunc(x1));
            bz = ptx::h2_as_u32(blo ? __highs2half2(p0, p1) : __lows2half2(p0, p1));
          }
          const int hc = cvalid ? qi : 0;
#pragma unroll
          for (int i = 0; i < SR; ++i)
            side_bias = fmaf(sm_qt[hc * SR + i], __high2float(zm[i]), side_bias);
        }
        const float beta = (cbias[0][0] + cbias[1][0] + side_bias) * alpha;

        // ---- scores of the whole group ----
        float sc[MT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          const int t0 = 16 * mt + qr;
          uint32_t w0[G::WPT], w1[G::WPT];
          load_words<G::WPT>(skc + t0 * G::KW + qi * G::WPT, w0);
          load_words<G::WPT>(skc + (t0 + 8) * G::KW + qi * G::WPT, w1);
#pragma unroll
          for (int u = 0; u < G::WPT; ++u) {
            uint32_t r0[G::RPW], r1[G::RPW];
            unpack_key_word<KB>(w0[u], r0);
            unpack_key_word<KB>(w1[u], r1);
#pragma unroll
            for (int ls = 0; ls < G::KSPW; ++ls) {
              const int s = u * G::KSPW + ls;
              ptx::mma_16816(cs, r0[2 * ls], r1[2 * ls], r0[2 * ls + 1], r1[2 * ls + 1], bq[s][0],
                             bq[s][1]);
            }
          }
          if constexpr (SR > 0) {
            const unsigned char* zr = S + L.z_off;
            uint32_t x0, x1;
            if constexpr (Z::ZB == 4) {
              x0 = *reinterpret_cast<const uint32_t*>(zr + t0 * 4);
              x1 = *reinterpret_cast<const uint32_t*>(zr + (t0 + 8) * 4);
            } else {
              // (c0 c1 | c2 c3) of a 16-bit row -> c0 c1 in the low half, c2 c3 in the high half
              x0 = ptx::prmt(*reinterpret_cast<const uint16_t*>(zr + t0 * 2), 0u, 0x0100u);
              x1 = ptx::prmt(*reinterpret_cast<const uint16_t*>(zr + (t0 + 8) * 2), 0u, 0x0100u);
            }
            ptx::mma_1688(cs, (x0 >> Z::shift(qi)) & Z::mask(qi), (x1 >> Z::shift(qi)) & Z::mask(qi), bz);
          }
          sc[mt][0] = fmaf(cs[0] + cs[1], alpha24, beta);
          sc[mt][1] = fmaf(cs[2] + cs[3], alpha24, beta);
        }
        // retained tokens of this group are read from the fp16 list: mask them here
        const int g0 = g * gk;
        unsigned hits = __ballot_sync(0xffffffffu, ret_pos >= g0 && ret_pos < g0 + gk);
        while (hits) {
          const int src = __ffs(hits) - 1;
          hits &= hits - 1;
          const int off = __shfl_sync(0xffffffffu, ret_pos, src) - g0;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            if (off == 16 * mt + qr) sc[mt][0] = -INFINITY;
            if (off == 16 * mt + qr + 8) sc[mt][1] = -INFINITY;
          }
        }
        // ---- online softmax update for the group ----
        float gmax = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) gmax = fmaxf(gmax, fmaxf(sc[mt][0], sc[mt][1]));
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
          for (int gg = 0; gg < G::NVG; ++gg) zsum[gg] *= a;
#pragma unroll
          for (int mv = 0; mv < 8; ++mv)
#pragma unroll
            for (int e = 0; e < 4; ++e) co[mv][e] *= a;
          m_run = m_new;
        }
        const float m_use = m_run == -INFINITY ? 0.0f : m_run;   // all masked: every p is 0

        // ---- p.V over the group ----
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          {
            const int t0 = 16 * mt + qr;
            const float p0 = ptx::ex2(sc[mt][0] - m_use);
            const float p1 = ptx::ex2(sc[mt][1] - m_use);
            l_run += p0 + p1;
            // value (scale, zero) of the two tokens this thread weights
            uint32_t vm0[G::NVG], vm1[G::NVG];
            load_words<G::NVG>(svm + t0 * G::NVG, vm0);
            load_words<G::NVG>(svm + (t0 + 8) * G::NVG, vm1);
            // value words: tokens 2qi, 2qi+1, 2qi+8, 2qi+9 of the tile, swapped for qi >= 2
            const int ta = 16 * mt + 2 * qi + (swap ? 1 : 0);
            const int tb = 16 * mt + 2 * qi + (swap ? 0 : 1);
            // 16-bit runs (a value group's row is 16 bytes): ldmatrix.trans over the rows of
            // tokens 0-7 and 8-15 of the tile hands lane (qr, qi) the pair (token 2qi, token
            // 2qi+1) of 16-bit column qr, i.e. exactly its run of both tokens in one register
            constexpr bool kLdm = G::RUN == 16 && GV * VB / 8 == 16 && G::NVG % 2 == 0;
            uint32_t xv[G::NVG][2];
            if constexpr (kLdm) {
              const int j = lane >> 3, r = lane & 7;
#pragma unroll
              for (int g4 = 0; g4 < G::NVG; g4 += 2)
                ptx::ldmatrix_x4_trans(ptx::smem_addr(svc) + (16 * mt + 8 * (j & 1) + r) * G::VBYTES_ROW +
                                           (g4 + (j >> 1)) * 16,
                                       xv[g4][0], xv[g4][1], xv[g4 + 1][0], xv[g4 + 1][1]);
            }
#pragma unroll
            for (int gg = 0; gg < G::NVG; ++gg) {
              const float2 f0 = __half22float2(ptx::u32_as_h2(vm0[gg]));
              const float2 f1 = __half22float2(ptx::u32_as_h2(vm1[gg]));
              // with centred codes (c - mid) the zero-point sum takes z + mid * s instead of z
              const float zc0 = CENTER ? fmaf(kMid, f0.x, f0.y) : f0.y;
              const float zc1 = CENTER ? fmaf(kMid, f1.x, f1.y) : f1.y;
              zsum[gg] = fmaf(p0, zc0, fmaf(p1, zc1, zsum[gg]));
              const uint32_t x0 = ptx::split_hi_lo_trunc(p0 * f0.x);
              const uint32_t x1 = ptx::split_hi_lo_trunc(p1 * f1.x);
              const uint32_t bp0 = ptx::movmatrix_trans(x0);
              const uint32_t bp1 = ptx::movmatrix_trans(x1);

              const int bit0 = (gg * GV + qr * G::CPG) * VB;
              const int wv = bit0 >> 5;
              const int ob = bit0 & 31;
              uint32_t ra[G::CPG], rb[G::CPG];   // codes of tokens (2qi, 2qi+1) and (2qi+8, 2qi+9)
              if constexpr (kLdm) {
                unpack_value_piece16<VB>(xv[gg][0], ra);
                unpack_value_piece16<VB>(xv[gg][1], rb);
              } else {
                // other run widths: four word loads and a byte permute per pair of tokens
                const uint32_t wa0 = svc[ta * G::VW + wv], wb0 = svc[tb * G::VW + wv];
                const uint32_t wa1 = svc[(ta + 8) * G::VW + wv], wb1 = svc[(tb + 8) * G::VW + wv];
                if constexpr (G::RUN == 8) {
                  const uint32_t bsel = static_cast<uint32_t>(ob >> 3);
                  const uint32_t s8 = swap ? ((4 + bsel) | ((4 + bsel) << 4) | (bsel << 8) | (bsel << 12))
                                           : (bsel | (bsel << 4) | ((4 + bsel) << 8) | ((4 + bsel) << 12));
                  unpack_value_piece8<VB>(ptx::prmt(wa0, wb0, s8), ra);
                  unpack_value_piece8<VB>(ptx::prmt(wa1, wb1, s8), rb);
                } else if constexpr (G::RUN == 16) {
                  const uint32_t s16 = ob ? sel_hi : sel_lo;
                  unpack_value_piece16<VB>(ptx::prmt(wa0, wb0, s16), ra);
                  unpack_value_piece16<VB>(ptx::prmt(wa1, wb1, s16), rb);
                } else {
                  constexpr int n16 = 16 / VB;
                  unpack_value_piece16<VB>(ptx::prmt(wa0, wb0, sel_lo), ra);
                  unpack_value_piece16<VB>(ptx::prmt(wa0, wb0, sel_hi), ra + n16);
                  unpack_value_piece16<VB>(ptx::prmt(wa1, wb1, sel_lo), rb);
                  unpack_value_piece16<VB>(ptx::prmt(wa1, wb1, sel_hi), rb + n16);
                }
              }
              if constexpr (CENTER) {
                // centred codes (c - mid) * 2^(p-24), mid = 2^(VB-1): an exact fp16 subnormal
                // subtraction that keeps the accumulators near zero
#pragma unroll
                for (int e = 0; e < G::CPG; ++e) {
                  const uint32_t mid = (1u << (VB - 1 + value_code_shift<VB, G::RUN>(e))) * 0x00010001u;
                  ra[e] = ptx::h2_as_u32(__hsub2(ptx::u32_as_h2(ra[e]), ptx::u32_as_h2(mid)));
                  rb[e] = ptx::h2_as_u32(__hsub2(ptx::u32_as_h2(rb[e]), ptx::u32_as_h2(mid)));
                }
              }
#pragma unroll
              for (int ml = 0; ml < G::MPG; ++ml)
                ptx::mma_16816(co[gg * G::MPG + ml], ra[ml], ra[ml + G::MPG], rb[ml], rb[ml + G::MPG],
                               bp0, bp1);
            }
          }
        }

        // ---- release the stage: refill it with unit k + RING ----
        __syncwarp();
        if (lane == 0 && k + RING < n_units) {
          ptx::fence_proxy_async_smem();
          issue(k + RING, group_of(k + RING, true));
        }
      }
    }
  } else {
    // ---------------- fp16 rows: retained tokens, then the window ----------------
    constexpr int RING = RG::RING_F, STAGE = RG::STAGE_F;
    uint32_t qn[KSTEPS][2];
#pragma unroll
    for (int s = 0; s < KSTEPS; ++s)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = 16 * s + 2 * qi + 8 * j;
        qn[s][j] = (bvalid && !blo) ? ptx::h2_as_u32(__halves2half2(qrow[c], qrow[c + 1])) : 0u;
      }
    if (d.rot) __syncthreads();          // every warp has read the rotated query rows
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
        const bool stall = w.stall && k == 0 && split == w.splits_q && h == 0 && b == 0;
        ptx::mbar_arrive_expect_tx(bar, nvalid * (DK + kDV) * 2 + (stall ? 16 : 0));
      }
      __syncwarp();
      const int row = lane & 15;
      if (row < nvalid) {
        const int e = e0 + row;
        size_t slot;
        const __half* base_k;
        const __half* base_v;
        if (e < sw.n_ret) {
          slot = static_cast<size_t>(bh) * kMaxRetained + e;
          base_k = cb.ret_k;
          base_v = cb.ret_v;
        } else {
          const int pos = sw.Q + (e - sw.n_ret);
          slot = static_cast<size_t>(bh) * d.cap + pos % d.cap;
          base_k = cb.win_k;
          base_v = cb.win_v;
        }
        if (!KVQ_IN_BOUNDS(d, base_k == cb.ret_k ? kSiteDecRetK : kSiteDecWinK, static_cast<long long>(slot),
                           base_k == cb.ret_k ? ret_rows(d) : win_rows(d)))
          slot = 0;
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
      const uint32_t x0 = ptx::split_hi_lo_trunc(p0);
      const uint32_t x1 = ptx::split_hi_lo_trunc(p1);
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
  }

  // A bounded wait gave up: flag it, then wait (bounded) for the last copy issued into
  // every stage so that no copy lands in shared memory after the CTA has exited.
  if (failed && lane == 0) {
    atomicOr(part.status, KVQ_STATUS_TIMEOUT);
    atomicOr(sm_fail, 1);
  }
  if constexpr (PAGED) ptx::cp_async_wait_all();   // a page fetch of a unit given up on
  __syncthreads();
  if (*sm_fail) {
    if (threadIdx.x < ring && sm_issued[threadIdx.x] > 0)
      ptx::mbar_wait_bounded(bar0 + 8 * threadIdx.x, (sm_issued[threadIdx.x] - 1) & 1, kWaitLimitNs);
    failed = true;     // the CTA's partial is dropped as a whole
  }

  // ---------------- warp totals, then the CTA merge ----------------
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 4);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
#pragma unroll
  for (int gg = 0; gg < G::NVG; ++gg) {
    zsum[gg] += __shfl_xor_sync(0xffffffffu, zsum[gg], 4);
    zsum[gg] += __shfl_xor_sync(0xffffffffu, zsum[gg], 8);
    zsum[gg] += __shfl_xor_sync(0xffffffffu, zsum[gg], 16);
  }
  if (failed) {
    m_run = -INFINITY;
    l_run = 0.0f;
  }
  __syncthreads();   // every warp is done with the stages: reuse them for the merge
  float* sm_o = reinterpret_cast<float*>(smem + SM::kStages);        // [kWarps][NREP][kDV]
  float* sm_ml = sm_o + kWarps * NREP * kDV;                         // [kWarps][NREP][2]
  if (cvalid) {
    float* dst = sm_o + (warp * NREP + qi) * kDV;
#pragma unroll
    for (int mv = 0; mv < 8; ++mv) {
      float o0 = co[mv][0] + co[mv][1];
      float o1 = co[mv][2] + co[mv][3];
      int c0, c1;
      if (quant) {
        const int gg = mv / G::MPG, ml = mv % G::MPG;
        c0 = gg * GV + qr * G::CPG + ml;
        c1 = c0 + G::MPG;
        o0 = fmaf(o0, static_cast<float>(1 << (24 - value_code_shift<VB, G::RUN>(ml))), zsum[gg]);
        o1 = fmaf(o1, static_cast<float>(1 << (24 - value_code_shift<VB, G::RUN>(ml + G::MPG))),
                  zsum[gg]);
      } else {
        c0 = 16 * mv + qr;
        c1 = c0 + 8;
      }
      if (failed) o0 = o1 = 0.0f;
      dst[c0] = o0;
      dst[c1] = o1;
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
    if (!KVQ_IN_BOUNDS(d, kSiteDecPartial, static_cast<long long>(pi), static_cast<long long>(d.B) * d.Hq * w.splits))
      continue;
    part.o[pi * kDV + c] = acc;
    if (c == 0) part.ml[pi] = make_float2(M, lsum);
  }
}

template <int KB, int VB, int DK, int NREP, int GV, int GK, bool QUANT, int SR, int SQ, bool PAGED,
          bool CENTER>
cudaError_t launch_impl(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                        const Partials& p, cudaStream_t s) {
  using RG = Rings<KB, VB, DK, GV, GK, QUANT, SR, SQ>;
  int smem = RG::BYTES;
  const int merge = kWarps * NREP * kDV * 4 + kWarps * NREP * 8;
  if (RG::HDR + merge > smem) smem = RG::HDR + merge;
  auto kern = decode_mma_kernel<KB, VB, DK, NREP, GV, GK, QUANT, SR, SQ, PAGED, CENTER>;
  static int configured = 0;
  if (configured < smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  dim3 grid(w.splits, d.Hkv, d.B);
  kern<<<grid, kThreads, smem, s>>>(d, c, w, q, p);
  return cudaGetLastError();
}

// The kernel instance for a decode: quantized caches take the centred-code instance when the
// plan asks for it (long contexts), so the uncentred instance carries no trace of it.
template <int KB, int VB, int DK, int NREP, int GV, int GK, bool QUANT, int SR = 0, int SQ = 4,
          bool PAGED = false>
cudaError_t launch(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                   const Partials& p, cudaStream_t s) {
  if constexpr (QUANT) {
    if (w.center) return launch_impl<KB, VB, DK, NREP, GV, GK, QUANT, SR, SQ, PAGED, true>(d, c, w, q, p, s);
  }
  return launch_impl<KB, VB, DK, NREP, GV, GK, QUANT, SR, SQ, PAGED, false>(d, c, w, q, p, s);
}

}  // namespace mma
}  // namespace kvq
