// Fused dequant + split-K flash-decoding kernel for the quantized groups of the
// cache, on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// One CTA = one split of one (b, kv head): a run of whole key groups, walked in
// blocks of 128 tokens (the MMA's M).  Warps are specialised:
//
//   control warp (lane 0): refills a ring of shared-memory stages with 1-D bulk
//       copies (cp.async.bulk; one stage = one block), and issues the MMAs:
//       D_S = A_K x B_S + A_one x B_Z once the compute warps have written the
//       block's keys and query operands, D_PV += A_V x B_P once they have written
//       its values and weights.  Each tcgen05.mma costs the issuing thread about
//       50 cycles whatever its N, so a thread of its own issues them.
//   8 compute warps, two per TMEM lane quadrant (warp w owns lanes 32(w%4) ..):
//   (a) keys.    Unpack the key codes of 16 tokens and store them with
//       tcgen05.st into A_K (TMEM; lane = token, 128 x d_k fp16).  A b-bit field
//       masked in place inside a 16-bit lane is an fp16 subnormal of value
//       code * 2^(p-24), p its bit offset, so unpacking is one AND per two codes.
//   (b) query.   Per key group g and channel c the query is scaled by the key
//       scale ("HeadQ", §2.1: s_j = q.k_j / sqrt(d); "Thin Keys, Full Values",
//       §2: d = d_k) and by 2^-p of that channel's code field:
//       B_S[c][h] = q_h,c * 2^-p * s_g,c as an exact (hi, lo) fp16 pair, and the
//       zero-point term B_Z[c][h] = q_h,c * z_g,c likewise; both go to shared
//       memory as MN-major UMMA operands (N = head x {hi, lo} x group).  A_one is
//       2^-24 in every element, so the zero-point sum lands in the codes' scale.
//   (c) values.  Unpack the value codes of 16 channels into A_V (TMEM; lane =
//       channel, K = the block's tokens).  Values are stored channel-major inside
//       each key group, so a thread's codes of one channel are whole words.
//   (d) softmax. Read the scores of the quadrant's 32 tokens for half of the
//       heads from D_S (tcgen05.ld), keep a CTA-wide reference maximum per head
//       that moves only when a score exceeds it by more than kLazyRescale (log2
//       units), and write B_P[token][vg, h] = p_h * s_token,vg * 2^-p' as (hi, lo)
//       fp16, p' the bit offset of that token's value field; sum_j p_j z_j,vg and
//       sum_j p_j are kept per thread.
//
// The compute warps hand work to the control warp through mbarrier arrivals and
// wait for MMA completion on mbarriers the MMAs commit to; the only CTA-wide
// step per block is one named-barrier reduction that decides whether the
// reference maximum moves.  Token order inside a block is free ("LogQuant:
// Log-Distributed 2-Bit Quantization of KV Cache", §4), so tokens are assigned to
// TMEM lanes and K slots in whatever order makes the unpacking cheap; A_K lane l,
// B_P row k and A_V column k all name the same token through one map.
//
// Waits are bounded (1 s of globaltimer); on timeout the CTA sets
// KVQ_STATUS_TIMEOUT, waits (again bounded) for its copies and MMAs in flight,
// frees its tensor memory and contributes nothing.
#pragma once

#include "../../include/kvq.h"
#include "kvq_internal.cuh"
#include "ptx.cuh"

namespace kvq {
namespace tc {

constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 32;   // + the control warp
constexpr int kComputeBar = 1;                   // named barrier of the compute warps
constexpr int kTok = 128;                        // tokens per block
constexpr int kDV = 128;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kLazyRescale = 8.0f;
constexpr uint32_t kTmemCols = 256;              // two CTAs per SM share the 512 columns
constexpr int kColAK = 0, kColAV = 64, kColA1 = 128, kColDS = 160, kColDP = 192;
constexpr int kSmemPerCta = 112 * 1024;          // at most two CTAs per SM
constexpr int kMaxRing = 16;

template <int KB, int VB, int DK, int NREP, int GV, int GK>
struct Geom {
  static constexpr int NG = kTok / GK;            // key groups per block
  static constexpr int KW = DK * KB / 32;         // u32 words per key row
  static constexpr int WPT = KW / 4;              // key words per thread per row
  static constexpr int RPW = 16 / KB;             // registers per key word
  static constexpr int CPW = 32 / KB;             // channels per key word
  static constexpr int KSTEPS = DK / 16;
  static constexpr int NVG = kDV / GV;            // value groups per token
  static constexpr int VRW = GK * VB / 32;        // words of one channel's codes in a group
  static constexpr int RPWV = 16 / VB;            // registers per value word
  static constexpr int CPWV = 32 / VB;            // tokens per value word
  static constexpr int RG = 16 / NG;              // value registers per group, channel and thread
  static constexpr int WS = NREP <= 4 ? 8 : 16;   // columns per key group / per value group
  static constexpr int NS = NG * WS < 16 ? 16 : NG * WS;
  static constexpr int NP = NVG * WS < 16 ? 16 : NVG * WS;
  static constexpr int HP = (NREP + 1) / 2;       // head pairs
  static constexpr int HPW = (HP + 1) / 2;        // head pairs per compute warp
  // one block (NG key groups) per ring stage: key codes of the 128 tokens, key (s, z)
  // of the groups, value codes per group (64 B of padding between groups keeps the
  // two groups' rows in different banks), value (s, z) of the 128 tokens
  static constexpr int KROW = DK * KB / 8;
  static constexpr int S_K = 0;
  static constexpr int S_KM = kTok * KROW;
  static constexpr int VGROUP = kDV * VRW * 4;
  static constexpr int VGS = VGROUP + 64;
  static constexpr int S_V = S_KM + NG * DK * 4;
  static constexpr int S_VM = S_V + NG * VGS;
  static constexpr int STAGE_BYTES = S_VM + kTok * NVG * 4;
  static constexpr int STAGE_STRIDE = (STAGE_BYTES + 127) / 128 * 128;
  // shared memory: barriers and scratch, B_S, B_Z, B_P, ring
  static constexpr int SM_FULL = 0;                             // u64 [kMaxRing]
  static constexpr int SM_KREADY = kMaxRing * 8;
  static constexpr int SM_PREADY = SM_KREADY + 8;
  static constexpr int SM_SDONE = SM_PREADY + 8;
  static constexpr int SM_PDONE = SM_SDONE + 8;
  static constexpr int SM_TMEM = SM_PDONE + 8;
  static constexpr int SM_ISSUED = SM_TMEM + 8;                 // int [kMaxRing]
  static constexpr int SM_WMAX = SM_ISSUED + kMaxRing * 4;      // float [4][8]
  static constexpr int SM_RED = SM_WMAX + 4 * 8 * 4;            // float [8 warps][2 * HPW * (NVG + 1)]
  static constexpr int NRED = 2 * HPW * (NVG + 1);
  static constexpr int SM_BS = (SM_RED + kComputeWarps * NRED * 4 + 127) / 128 * 128;
  static constexpr int SM_BZ = SM_BS + DK * NS * 2;
  static constexpr int SM_BP = SM_BZ + DK * NS * 2;
  static constexpr int SM_RING = (SM_BP + kTok * NP * 2 + 127) / 128 * 128;
  static constexpr int RING_FIT = (kSmemPerCta - SM_RING) / STAGE_STRIDE;
  static constexpr int RING = RING_FIT > kMaxRing ? kMaxRing : RING_FIT;
  static constexpr int SMEM = SM_RING + RING * STAGE_STRIDE;

  static_assert(NG >= 1 && kTok % GK == 0, "group_k must divide 128");
  static_assert(WPT >= 1, "key row too short for the fragment mapping");
  static_assert(DK % 16 == 0 && kComputeThreads % DK == 0 && DK <= 128, "d_k must divide 128");
  static_assert(RG * 2 >= RPWV, "value words too long for the group size");
  static_assert(NS <= 32 && NP <= 32, "TMEM column plan");
  static_assert(RING >= 2, "ring too small");
  static_assert(GV >= 32, "a warp's 32 channels must share one value group");
  static_assert(SMEM <= kSmemPerCta, "shared memory plan");
};

// fp16 mantissa-field masks: the `bits`-wide field at bit `pos` of both 16-bit halves.
template <int BITS, int POS>
struct Mask {
  static constexpr uint32_t v = (((1u << BITS) - 1u) << POS) * 0x00010001u;
};

// The 16/B registers of one packed word: register rho holds the fields rho (low half) and
// rho + 16/B (high half), each at bit offset (B * rho) mod 8 of its 16-bit lane.
template <int B>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t* r) {
  const uint32_t u = w >> 8;
  if constexpr (B == 2) {
    r[0] = w & Mask<2, 0>::v;
    r[1] = w & Mask<2, 2>::v;
    r[2] = w & Mask<2, 4>::v;
    r[3] = w & Mask<2, 6>::v;
    r[4] = u & Mask<2, 0>::v;
    r[5] = u & Mask<2, 2>::v;
    r[6] = u & Mask<2, 4>::v;
    r[7] = u & Mask<2, 6>::v;
  } else if constexpr (B == 4) {
    r[0] = w & Mask<4, 0>::v;
    r[1] = w & Mask<4, 4>::v;
    r[2] = u & Mask<4, 0>::v;
    r[3] = u & Mask<4, 4>::v;
  } else {
    r[0] = w & Mask<8, 0>::v;
    r[1] = u & Mask<8, 0>::v;
  }
}

// Registers [0, 8/B) of a word (the caller passes w >> 8 for the upper ones).
template <int B>
__device__ __forceinline__ void unpack_half_word(uint32_t w, uint32_t* r) {
  if constexpr (B == 2) {
    r[0] = w & Mask<2, 0>::v;
    r[1] = w & Mask<2, 2>::v;
    r[2] = w & Mask<2, 4>::v;
    r[3] = w & Mask<2, 6>::v;
  } else if constexpr (B == 4) {
    r[0] = w & Mask<4, 0>::v;
    r[1] = w & Mask<4, 4>::v;
  } else {
    r[0] = w & Mask<8, 0>::v;
  }
}

template <int N>
__device__ __forceinline__ void lds_words(const unsigned char* p, uint32_t* out) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(p + 4 * i);
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
    out[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

// K slot of TMEM lane l (A_K / D_S row): lanes 8a .. 8a+7 take the slots 8a + (0,2,4,6,1,3,5,7),
// which keeps the key-row loads free of bank conflicts.
__host__ __device__ constexpr int kslot_of_lane(int l) { return (l & ~7) | ((l & 3) << 1) | ((l >> 2) & 1); }

struct TokenSlot {
  int g;     // key group within the block
  int tok;   // token within the group
  int pv;    // bit offset of its value field inside the fp16 lane
};

// The token held by K slot k of A_V (and row k of B_P): slot k is half (k & 1) of TMEM
// column k >> 1, which the value unpacking fills from register m of thread tq (see the
// 16x256b store layout) with the fields of one packed value word.
template <int VB, int GK>
__host__ __device__ constexpr TokenSlot token_of_kslot(int k) {
  constexpr int NG = kTok / GK, RG = 16 / NG, RPWV = 16 / VB, CPWV = 32 / VB;
  const int col = k >> 1, half = k & 1;
  const int j = col >> 3, tq = (col & 7) >> 1, e = col & 1;
  const int m = 2 * j + e;
  const int g = m / RG, mp = m % RG;
  const int G = tq * RG + mp;
  const int wd = G / RPWV, rho = G % RPWV;
  return TokenSlot{g, wd * CPWV + rho + half * (16 / VB), (VB * rho) % 8};
}

// The channel held by K slot k of A_K (row k of B_S / B_Z) and the bit offset of its field.
template <int KB, int DK>
__host__ __device__ constexpr int2 channel_of_kslot(int k) {
  constexpr int KW = DK * KB / 32, WPT = KW / 4, RPW = 16 / KB, CPW = 32 / KB;
  const int col = k >> 1, half = k & 1;
  const int j = col >> 3, tq = (col & 7) >> 1, e = col & 1;
  const int mk = 2 * j + e;
  const int u = mk / RPW, rho = mk % RPW;
  return int2{CPW * (tq * WPT + u) + rho + half * (16 / KB), (KB * rho) % 8};
}

// UMMA shared-memory descriptor of an MN-major operand without swizzle: 8x8 core matrices
// of 128 B, `lbo` bytes apart along K and `sbo` bytes apart along M/N.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(lbo >> 4) << 16) |
         (static_cast<uint64_t>(sbo >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor: kind::f16 with f16 A (K-major) and B (MN-major), f32 D, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
  return (1u << 4) | (1u << 16) | (static_cast<uint32_t>(n >> 3) << 17) | ((128u >> 4) << 24);
}

template <int KB, int VB, int DK, int NREP, int GV, int GK>
__global__ void __launch_bounds__(kThreads, 2)
decode_tc_kernel(Dims d, CacheBufs cb, DecodeWork w, const __half* __restrict__ q, Partials part) {
  using G = Geom<KB, VB, DK, NREP, GV, GK>;
  constexpr int NG = G::NG, RING = G::RING, WS = G::WS, NS = G::NS, NP = G::NP, HP = G::HP,
                HPW = G::HPW;
  extern __shared__ __align__(1024) unsigned char smem[];

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * d.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool control = warp == kComputeWarps;
  const int qd = warp & 3;            // TMEM lane quadrant of a compute warp
  const int hf = (warp >> 2) & 1;     // which 16-lane half / which head pairs
  const int qr = lane >> 2, qi = lane & 3;

  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t bar_full = sbase + G::SM_FULL, bar_kready = sbase + G::SM_KREADY,
                 bar_pready = sbase + G::SM_PREADY, bar_sdone = sbase + G::SM_SDONE,
                 bar_pdone = sbase + G::SM_PDONE;
  int* sm_issued = reinterpret_cast<int*>(smem + G::SM_ISSUED);
  float* sm_wmax = reinterpret_cast<float*>(smem + G::SM_WMAX);
  float* sm_red = reinterpret_cast<float*>(smem + G::SM_RED);
  unsigned char* sBS = smem + G::SM_BS;
  unsigned char* sBZ = smem + G::SM_BZ;
  unsigned char* sBP = smem + G::SM_BP;
  unsigned char* ring = smem + G::SM_RING;
  const uint32_t ring_s = sbase + G::SM_RING;

  // this CTA's key groups
  const int g_begin = static_cast<int>(static_cast<long long>(split) * w.n_groups / w.splits_q);
  const int g_end = static_cast<int>(static_cast<long long>(split + 1) * w.n_groups / w.splits_q);
  const int n_units = g_end - g_begin;
  const int n_blocks = (n_units + NG - 1) / NG;

  if (control) {
    ptx::tmem_alloc(sbase + G::SM_TMEM, kTmemCols);
    ptx::tmem_relinquish();
    if (lane == 0) {
      for (int s = 0; s < RING; ++s) {
        ptx::mbar_init(bar_full + 8 * s, 1);
        sm_issued[s] = 0;
      }
      ptx::mbar_init(bar_kready, kComputeWarps);
      ptx::mbar_init(bar_pready, kComputeWarps);
      ptx::mbar_init(bar_sdone, 1);
      ptx::mbar_init(bar_pdone, 1);
      ptx::fence_barrier_init();
    }
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + G::SM_TMEM);
  bool bad = false;        // this thread saw a bounded wait give up

  if (control) {
    // =============== control warp: bulk copies and MMA issue (lane 0) ===============
    if (lane == 0) {
      // one stage = one block: keys and key (s, z) of its groups, value codes per group,
      // value (s, z) of its tokens
      auto issue = [&](int blk) {
        const int st = blk % RING;
        const uint32_t bar = bar_full + 8 * st;
        const uint32_t dst = ring_s + st * G::STAGE_STRIDE;
        const int g0 = g_begin + blk * NG;
        const int ng = min(NG, g_end - g0);
        sm_issued[st] += 1;
        ptx::mbar_arrive_expect_tx(bar, ng * (GK * G::KROW + DK * 4 + G::VGROUP + GK * G::NVG * 4));
        const size_t grp = static_cast<size_t>(bh) * (d.lcap / GK) + g0;
        const size_t tok = static_cast<size_t>(bh) * d.lcap + static_cast<size_t>(g0) * GK;
        ptx::bulk_g2s(dst + G::S_K, cb.kcode + tok * G::KW, ng * GK * G::KROW, bar);
        ptx::bulk_g2s(dst + G::S_KM, cb.ksz + grp * DK, ng * DK * 4, bar);
        for (int g = 0; g < ng; ++g)
          ptx::bulk_g2s(dst + G::S_V + g * G::VGS, cb.vcode + (grp + g) * (kDV * G::VRW), G::VGROUP, bar);
        ptx::bulk_g2s(dst + G::S_VM, cb.vsz + tok * G::NVG, ng * GK * G::NVG * 4, bar);
      };
      for (int blk = 0; blk < RING && blk < n_blocks; ++blk) issue(blk);

      const uint32_t idesc_s = idesc_f16(NS), idesc_p = idesc_f16(NP);
      constexpr uint32_t LBO_S = (NS / 8) * 128, LBO_P = (NP / 8) * 128;
      const uint32_t bs = ptx::smem_addr(sBS), bz = ptx::smem_addr(sBZ), bp = ptx::smem_addr(sBP);
      int s_commits = 0, p_commits = 0;
      for (int blk = 0; blk < n_blocks; ++blk) {
        if (!ptx::mbar_wait_bounded(bar_kready, blk & 1, kWaitLimitNs)) {
          bad = true;
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int s = 0; s < G::KSTEPS; ++s)
          ptx::mma_f16_ts(tmem + kColDS, tmem + kColAK + 8 * s, smem_desc(bs + 2 * LBO_S * s, LBO_S, 128),
                          idesc_s, s > 0);
#pragma unroll
        for (int s = 0; s < G::KSTEPS; ++s)
          ptx::mma_f16_ts(tmem + kColDS, tmem + kColA1, smem_desc(bz + 2 * LBO_S * s, LBO_S, 128), idesc_s,
                          true);
        ptx::tc_commit(bar_sdone);
        ++s_commits;
        if (!ptx::mbar_wait_bounded(bar_pready, blk & 1, kWaitLimitNs)) {
          bad = true;
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int s = 0; s < kTok / 16; ++s)
          ptx::mma_f16_ts(tmem + kColDP, tmem + kColAV + 8 * s, smem_desc(bp + 2 * LBO_P * s, LBO_P, 128),
                          idesc_p, blk > 0 || s > 0);
        ptx::tc_commit(bar_pdone);
        ++p_commits;
        // the block's stage has been read by every compute warp: refill it
        ptx::fence_proxy_async_smem();
        if (blk + RING < n_blocks) issue(blk + RING);
      }
      if (bad) {
        // wait (bounded) for every copy and MMA this thread started
        for (int s = 0; s < RING; ++s)
          if (sm_issued[s] > 0) ptx::mbar_wait_bounded(bar_full + 8 * s, (sm_issued[s] - 1) & 1, kWaitLimitNs);
        if (s_commits > 0) ptx::mbar_wait_bounded(bar_sdone, (s_commits - 1) & 1, kWaitLimitNs);
        if (p_commits > 0) ptx::mbar_wait_bounded(bar_pdone, (p_commits - 1) & 1, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else {
    // =============== compute warps ===============
    // A_one: 2^-24 (the smallest fp16 subnormal) in both halves of 8 columns
    if (hf == 0) {
      uint32_t one[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) one[i] = 0x00010001u;
      ptx::tmem_st_32x32b<8>(tmem + (static_cast<uint32_t>(32 * qd) << 16) + kColA1, one);
    }
    const uint32_t tq_lanes = static_cast<uint32_t>(32 * qd) << 16;          // my quadrant
    const uint32_t th_lanes = static_cast<uint32_t>(32 * qd + 16 * hf) << 16; // my 16-lane half
    // key rows of lanes 32qd + 16hf + qr + 8e
    int koff[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const TokenSlot t = token_of_kslot<VB, GK>(kslot_of_lane(32 * qd + 16 * hf + qr + 8 * e));
      koff[e] = G::S_K + (t.g * GK + t.tok) * G::KROW + qi * G::WPT * 4;
    }
    // softmax: the token of my TMEM lane, its B_P row and value-field shift
    const int my_k = kslot_of_lane(32 * qd + lane);
    const TokenSlot me = token_of_kslot<VB, GK>(my_k);
    const float my_pv = static_cast<float>(me.pv);
    // query operands: K slot tid % DK of key groups tid / DK, tid / DK + 256 / DK, ...
    const int bk = tid % DK;
    const int2 bch = channel_of_kslot<KB, DK>(bk);
    __half2 q2[HP], qf2[HP];
    {
      const __half* qrow = q + (static_cast<size_t>(b) * d.Hq + h * NREP) * DK + bch.x;
      const __half2 f2 = __float2half2_rn(1.0f / static_cast<float>(1 << bch.y));
#pragma unroll
      for (int i = 0; i < HP; ++i) {
        const __half q0 = qrow[(2 * i) * DK];
        const __half q1 = (2 * i + 1 < NREP) ? qrow[(2 * i + 1) * DK] : __float2half(0.0f);
        q2[i] = __halves2half2(q0, q1);
        qf2[i] = __hmul2(q2[i], f2);
      }
    }
    const int ret_pos = lane < w.ret.n ? w.ret.pos[lane] : -1;
    const float alpha24 = w.score_scale * 16777216.0f;      // undoes the 2^-24 of the codes
    // my head pairs: hf * HPW .. (hf + 1) * HPW - 1 (those < HP)
    float m_reg[2 * HPW], lsum[2 * HPW], zs[G::NVG][2 * HPW];
#pragma unroll
    for (int i = 0; i < 2 * HPW; ++i) {
      m_reg[i] = -INFINITY;
      lsum[i] = 0.0f;
#pragma unroll
      for (int vg = 0; vg < G::NVG; ++vg) zs[vg][i] = 0.0f;
    }
    bool failed = false;

    for (int blk = 0; blk < n_blocks; ++blk) {
      const int st = blk % RING;
      const unsigned char* S = ring + st * G::STAGE_STRIDE;
      const int nvalid = min(NG, n_units - blk * NG);
      if (!ptx::mbar_wait_bounded(bar_full + 8 * st, (blk / RING) & 1, kWaitLimitNs)) bad = true;

      // ---- (a) keys -> A_K (one 16-lane half) ----
      {
        uint32_t regs[4 * G::KSTEPS];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          uint32_t wds[G::WPT];
          lds_words<G::WPT>(S + koff[e], wds);
#pragma unroll
          for (int u = 0; u < G::WPT; ++u) {
            uint32_t r[G::RPW];
            unpack_word<KB>(wds[u], r);
#pragma unroll
            for (int rho = 0; rho < G::RPW; ++rho) {
              const int m = u * G::RPW + rho;
              regs[4 * (m >> 1) + 2 * e + (m & 1)] = r[rho];
            }
          }
        }
        ptx::tmem_st_16x256b<G::KSTEPS>(tmem + th_lanes + kColAK, regs);
      }

      // ---- (b) query scaled per key group -> B_S, B_Z ----
#pragma unroll
      for (int gg0 = 0; gg0 < NG; gg0 += kComputeThreads / DK) {
        const int gg = gg0 + tid / DK;
        if (gg < nvalid) {
          const __half2 sz = *reinterpret_cast<const __half2*>(S + G::S_KM + (gg * DK + bch.x) * 4);
          const __half2 s2 = __low2half2(sz), z2 = __high2half2(sz);
          uint32_t vs[2 * HP], vz[2 * HP];
#pragma unroll
          for (int i = 0; i < HP; ++i) {
            const __half2 hi = __hmul2(qf2[i], s2);
            const __half2 lo = __hfma2(qf2[i], s2, __hneg2(hi));
            const __half2 zh = __hmul2(q2[i], z2);
            const __half2 zl = __hfma2(q2[i], z2, __hneg2(zh));
            vs[2 * i] = ptx::h2_as_u32(hi);
            vs[2 * i + 1] = ptx::h2_as_u32(lo);
            vz[2 * i] = ptx::h2_as_u32(zh);
            vz[2 * i + 1] = ptx::h2_as_u32(zl);
          }
          const int off = ((bk >> 3) * (NS / 8) + gg * (WS / 8)) * 128 + (bk & 7) * 16;
#pragma unroll
          for (int c = 0; c < WS / 8; ++c) {
            const uint32_t x2 = 4 * c + 2 < 2 * HP ? vs[4 * c + 2] : 0u;
            const uint32_t x3 = 4 * c + 3 < 2 * HP ? vs[4 * c + 3] : 0u;
            const uint32_t y2 = 4 * c + 2 < 2 * HP ? vz[4 * c + 2] : 0u;
            const uint32_t y3 = 4 * c + 3 < 2 * HP ? vz[4 * c + 3] : 0u;
            *reinterpret_cast<uint4*>(sBS + off + c * 128) = make_uint4(vs[4 * c], vs[4 * c + 1], x2, x3);
            *reinterpret_cast<uint4*>(sBZ + off + c * 128) = make_uint4(vz[4 * c], vz[4 * c + 1], y2, y3);
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_kready);

      // ---- (c) values -> A_V (one 16-lane half), once the previous p.V MMA is done ----
      if (blk > 0 && !ptx::mbar_wait_bounded(bar_pdone, (blk - 1) & 1, kWaitLimitNs)) bad = true;
      ptx::tc_fence_after();
      {
        uint32_t regs[32];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 32 * qd + 16 * hf + qr + 8 * e;
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            uint32_t r[G::RG];
            const unsigned char* row = S + G::S_V + g * G::VGS + c * (G::VRW * 4);
            if constexpr (G::RG >= G::RPWV) {
              constexpr int NW = G::RG / G::RPWV;
              uint32_t wds[NW];
              lds_words<NW>(row + qi * NW * 4, wds);
#pragma unroll
              for (int wv = 0; wv < NW; ++wv) unpack_word<VB>(wds[wv], r + wv * G::RPWV);
            } else {
              // half a word per thread: registers [0, RPWV/2) of the word, or of the word >> 8
              const uint32_t x = *reinterpret_cast<const uint32_t*>(row + (qi >> 1) * 4);
              unpack_half_word<VB>((qi & 1) ? (x >> 8) : x, r);
            }
#pragma unroll
            for (int mp = 0; mp < G::RG; ++mp) {
              const int m = g * G::RG + mp;
              regs[4 * (m >> 1) + 2 * e + (m & 1)] = g < nvalid ? r[mp] : 0u;
            }
          }
        }
        ptx::tmem_st_16x256b<8>(tmem + th_lanes + kColAV, regs);
      }

      // ---- (d) scores -> softmax -> B_P ----
      if (!ptx::mbar_wait_bounded(bar_sdone, blk & 1, kWaitLimitNs)) bad = true;
      ptx::tc_fence_after();
      float sc[2 * HPW];
      {
        uint32_t raw[4 * HPW];
        if constexpr (HPW == 1)
          ptx::tmem_load_32x32b<4>(tmem + tq_lanes + kColDS + me.g * WS + 4 * hf, raw);
        else
          ptx::tmem_load_32x32b<8>(tmem + tq_lanes + kColDS + me.g * WS + 8 * hf, raw);
#pragma unroll
        for (int j = 0; j < HPW; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            sc[2 * j + e] = (__uint_as_float(raw[4 * j + e]) + __uint_as_float(raw[4 * j + 2 + e])) * alpha24;
      }
      const int pos0 = (g_begin + blk * NG) * GK;
      bool valid = me.g < nvalid;
      {
        unsigned hits = __ballot_sync(0xffffffffu, ret_pos >= pos0 && ret_pos < pos0 + kTok);
        const int my_pos = pos0 + me.g * GK + me.tok;
        while (hits) {
          const int src = __ffs(hits) - 1;
          hits &= hits - 1;
          if (__shfl_sync(0xffffffffu, ret_pos, src) == my_pos) valid = false;
        }
      }
      bool exceed = false;
#pragma unroll
      for (int i = 0; i < 2 * HPW; ++i) {
        const int hh = 2 * HPW * hf + i;
        if (!valid || hh >= NREP) sc[i] = -INFINITY;
        exceed |= sc[i] > m_reg[i] + kLazyRescale;
      }
      if (__any_sync(0xffffffffu, exceed)) {
#pragma unroll
        for (int i = 0; i < 2 * HPW; ++i) {
          float mx = sc[i];
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          if (lane == 0) sm_wmax[qd * 8 + 2 * HPW * hf + i] = mx;
        }
      } else if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 2 * HPW; ++i) sm_wmax[qd * 8 + 2 * HPW * hf + i] = -INFINITY;
      }
      if (ptx::bar_red_or(kComputeBar, kComputeThreads, exceed || bad)) {
        if (ptx::bar_red_or(kComputeBar, kComputeThreads, bad)) {
          failed = true;
          break;
        }
        // the reference maximum moves: rescale what was accumulated so far
        float a[2 * HPW];
#pragma unroll
        for (int i = 0; i < 2 * HPW; ++i) {
          float mn = m_reg[i];
#pragma unroll
          for (int ww = 0; ww < 4; ++ww) mn = fmaxf(mn, sm_wmax[ww * 8 + 2 * HPW * hf + i]);
          a[i] = (m_reg[i] == -INFINITY || mn == -INFINITY) ? 0.0f : ptx::ex2(m_reg[i] - mn);
          if (mn == m_reg[i]) a[i] = 1.0f;
          m_reg[i] = mn;
          lsum[i] *= a[i];
#pragma unroll
          for (int vg = 0; vg < G::NVG; ++vg) zs[vg][i] *= a[i];
        }
        if (blk > 0) {
#pragma unroll
          for (int vg = 0; vg < G::NVG; ++vg)
#pragma unroll
            for (int j = 0; j < HPW; ++j) {
              if (hf * HPW + j >= HP) continue;
              uint32_t acc[4];
              const uint32_t col = kColDP + vg * WS + 4 * (hf * HPW + j);
              ptx::tmem_load_32x32b<4>(tmem + tq_lanes + col, acc);
#pragma unroll
              for (int x = 0; x < 4; ++x) acc[x] = __float_as_uint(__uint_as_float(acc[x]) * a[2 * j + (x & 1)]);
              ptx::tmem_st_32x32b<4>(tmem + tq_lanes + col, acc);
            }
        }
      }
      {
        float pp[2 * HPW];
#pragma unroll
        for (int i = 0; i < 2 * HPW; ++i) {
          const float mu = m_reg[i] == -INFINITY ? 0.0f : m_reg[i];
          pp[i] = ptx::ex2(sc[i] - mu - my_pv);       // p * 2^-pv (0 when masked)
          lsum[i] += pp[i];
        }
        __half2 ph[HPW], pl[HPW];
#pragma unroll
        for (int j = 0; j < HPW; ++j) {
          ph[j] = __floats2half2_rn(pp[2 * j], pp[2 * j + 1]);
          const float2 f = __half22float2(ph[j]);
          pl[j] = __floats2half2_rn(pp[2 * j] - f.x, pp[2 * j + 1] - f.y);
        }
        uint32_t vm[G::NVG];
        lds_words<G::NVG>(S + G::S_VM + (me.g * GK + me.tok) * G::NVG * 4, vm);
#pragma unroll
        for (int vg = 0; vg < G::NVG; ++vg) {
          const __half2 sz = ptx::u32_as_h2(valid ? vm[vg] : 0u);
          const __half2 s2 = __low2half2(sz);
          const float zf = __high2float(sz);
#pragma unroll
          for (int i = 0; i < 2 * HPW; ++i) zs[vg][i] = fmaf(pp[i], zf, zs[vg][i]);
#pragma unroll
          for (int j = 0; j < HPW; ++j) {
            if (hf * HPW + j >= HP) continue;
            const __half2 hi = __hmul2(ph[j], s2);
            const __half2 lo = __hfma2(pl[j], s2, __hfma2(ph[j], s2, __hneg2(hi)));
            const int n = vg * WS + 4 * (hf * HPW + j);
            const int off = ((my_k >> 3) * (NP / 8) + (n >> 3)) * 128 + (my_k & 7) * 16 + (n & 7) * 2;
            *reinterpret_cast<uint2*>(sBP + off) = make_uint2(ptx::h2_as_u32(hi), ptx::h2_as_u32(lo));
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_pready);
    }

    // ---- the last p.V MMA, then the CTA totals and this split's partial ----
    if (!failed && n_blocks > 0 && !ptx::mbar_wait_bounded(bar_pdone, (n_blocks - 1) & 1, kWaitLimitNs))
      bad = true;
    ptx::tc_fence_after();
    failed = ptx::bar_red_or(kComputeBar, kComputeThreads, failed || bad);
    // sum p and sum p z of my heads: my share is in units of 2^-pv
    const float unscale = static_cast<float>(1 << me.pv);
    constexpr int NRED = G::NRED;
    float red[NRED];
#pragma unroll
    for (int i = 0; i < 2 * HPW; ++i) {
      red[i] = lsum[i] * unscale;
#pragma unroll
      for (int vg = 0; vg < G::NVG; ++vg) red[2 * HPW + vg * 2 * HPW + i] = zs[vg][i] * unscale;
    }
#pragma unroll
    for (int i = 0; i < NRED; ++i) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) red[i] += __shfl_xor_sync(0xffffffffu, red[i], o);
    }
    if (lane == 0)
#pragma unroll
      for (int i = 0; i < NRED; ++i) sm_red[warp * NRED + i] = red[i];
    ptx::bar_red_or(kComputeBar, kComputeThreads, false);
#pragma unroll
    for (int i = 0; i < NRED; ++i) {
      float t = 0.0f;
#pragma unroll
      for (int ww = 0; ww < 4; ++ww) t += sm_red[(4 * hf + ww) * NRED + i];
      red[i] = t;
    }
    // lane = channel 32qd + lane; my heads
    const int c = 32 * qd + lane, vg = (32 * qd) / GV;
#pragma unroll
    for (int j = 0; j < HPW; ++j) {
      const int pair = hf * HPW + j;
      if (pair >= HP) continue;
      uint32_t acc[4] = {0u, 0u, 0u, 0u};
      if (n_blocks > 0 && !failed) ptx::tmem_load_32x32b<4>(tmem + tq_lanes + kColDP + vg * WS + 4 * pair, acc);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hh = 2 * pair + e;
        if (hh >= NREP) continue;
        const float o = (__uint_as_float(acc[e]) + __uint_as_float(acc[2 + e])) * 16777216.0f +
                        red[2 * HPW + vg * 2 * HPW + 2 * j + e];
        const size_t pi = (static_cast<size_t>(b) * d.Hq + h * NREP + hh) * w.splits + split;
        part.o[pi * kDV + c] = failed ? 0.0f : o;
        if (c == 0) part.ml[pi] = failed ? make_float2(-INFINITY, 0.0f) : make_float2(m_reg[2 * j + e], red[2 * j + e]);
      }
    }
    if (failed && tid == 0) atomicOr(part.status, KVQ_STATUS_TIMEOUT);
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (control) {
    if (bad && lane == 0) atomicOr(part.status, KVQ_STATUS_TIMEOUT);
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int KB, int VB, int DK, int NREP, int GV, int GK>
cudaError_t launch(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                   const Partials& p, cudaStream_t s) {
  auto kern = decode_tc_kernel<KB, VB, DK, NREP, GV, GK>;
  // Every CTA asks for kSmemPerCta bytes (more than a third of the SM) so that no more
  // than two CTAs, 2 x kTmemCols columns, ever share an SM's tensor memory: an allocation
  // never has to wait for another CTA to free its columns.
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerCta);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(w.splits_q, d.Hkv, d.B);
  kern<<<grid, kThreads, kSmemPerCta, s>>>(d, c, w, q, p);
  return cudaGetLastError();
}

}  // namespace tc
}  // namespace kvq
