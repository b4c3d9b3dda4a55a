// Fused dequant + split-K flash-decoding kernel for the quantized groups of the
// cache, on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// One CTA = 4 warps = one split of one (b, kv head): a run of whole key groups.
// It walks its groups in blocks of 128 tokens (the MMA's M), and per block:
//
//   (a) keys.    Each warp unpacks the key codes of 32 tokens and stores them
//       with tcgen05.st into A_K (TMEM; lane = token, 128 x d_k fp16).  A b-bit
//       field masked in place inside a 16-bit lane is an fp16 subnormal of value
//       code * 2^(p-24), p its bit offset, so unpacking is one AND per two codes.
//   (b) query.   Per key group g and channel c the query is scaled by the key
//       scale ("HeadQ", §2.1: s_j = q.k_j / sqrt(d); "Thin Keys, Full Values",
//       §2: d = d_k) and by 2^-p of that channel's code field:
//       B_S[c][h] = q_h,c * 2^-p * s_g,c as an exact (hi, lo) fp16 pair, and
//       the zero-point term B_Z[c][h] = q_h,c * z_g,c likewise; both go to
//       shared memory as MN-major UMMA operands (N = head x {hi, lo} per group).
//   (c) one thread issues D_S = A_K x B_S + A_one x B_Z (A_one = 2^-24 in every
//       element, so the zero-point sum lands in the same scale as the codes),
//       while the others unpack the value codes into A_V (TMEM; lane = channel,
//       K = the block's tokens).  Values are stored channel-major inside each
//       key group, so a thread's codes for one channel are whole words.
//   (d) softmax. Thread t reads its token's scores from D_S (tcgen05.ld), keeps
//       a CTA-wide reference maximum per head that moves only when a score
//       exceeds it by more than kLazyRescale (log2 units), and writes the row
//       B_P[token][vg, h] = p_h * s_token,vg * 2^-p' as (hi, lo) fp16, p' being
//       the bit offset of that token's value field; sum_j p_j z_j,vg and sum_j p_j
//       are kept per thread.
//   (e) one thread issues D_PV += A_V x B_P and refills the block's ring stages.
//
// The score MMA of a block runs while the CTA unpacks its values, and its p.V
// MMA while the CTA unpacks the next block's keys.  The packed groups arrive by
// 1-D bulk copies (cp.async.bulk) into a ring of shared-memory stages, one key
// group per stage.  Token order inside a block is free ("LogQuant:
// Log-Distributed 2-Bit Quantization of KV Cache", §4), so tokens are assigned
// to TMEM lanes and K slots in whatever order makes the unpacking cheap; A_K
// lane l, B_P row k and A_V column k all name the same token through one map.
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

constexpr int kThreads = 128;                 // warp w owns TMEM lanes 32w .. 32w+31
constexpr int kTok = 128;                     // tokens per block
constexpr int kDV = 128;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kLazyRescale = 8.0f;
constexpr uint32_t kTmemCols = 256;           // two CTAs per SM share the 512 columns
constexpr int kColAK = 0, kColAV = 64, kColA1 = 128, kColDS = 160, kColDP = 192;
constexpr int kSmemPerCta = 112 * 1024;       // at most two CTAs per SM
constexpr int kMaxRing = 24;

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
  // one key group in a ring stage: key codes, key (s, z), value codes, value (s, z)
  static constexpr int K_OFF = 0;
  static constexpr int KROW = DK * KB / 8;
  static constexpr int KM_OFF = GK * KROW;
  static constexpr int V_OFF = KM_OFF + DK * 4;
  static constexpr int VM_OFF = V_OFF + GK * kDV * VB / 8;
  static constexpr int STAGE_BYTES = VM_OFF + GK * NVG * 4;
  // stages start 64 B apart modulo 128 so that two groups' rows fall in different banks
  static constexpr int STAGE_STRIDE = (STAGE_BYTES + 127) / 128 * 128 + 64;
  // shared memory: header, B_S, B_Z, B_P, ring
  static constexpr int SM_BAR_S = kMaxRing * 8;
  static constexpr int SM_BAR_P = SM_BAR_S + 8;
  static constexpr int SM_TMEM = SM_BAR_P + 8;
  static constexpr int SM_ISSUED = SM_TMEM + 8;                 // int [kMaxRing]
  static constexpr int SM_WMAX = SM_ISSUED + kMaxRing * 4;      // float [4][8]
  static constexpr int SM_RED = SM_WMAX + 4 * 8 * 4;            // float [4][NREP * (NVG + 1)]
  static constexpr int SM_BS = (SM_RED + 4 * NREP * (NVG + 1) * 4 + 127) / 128 * 128;
  static constexpr int SM_BZ = SM_BS + DK * NS * 2;
  static constexpr int SM_BP = SM_BZ + DK * NS * 2;
  static constexpr int SM_RING = (SM_BP + kTok * NP * 2 + 127) / 128 * 128;
  static constexpr int RING_FIT = (kSmemPerCta - SM_RING) / STAGE_STRIDE;
  static constexpr int RING = (RING_FIT > kMaxRing ? kMaxRing : RING_FIT) / NG * NG;
  static constexpr int SMEM = SM_RING + RING * STAGE_STRIDE;

  static_assert(NG >= 1 && kTok % GK == 0, "group_k must divide 128");
  static_assert(WPT >= 1, "key row too short for the fragment mapping");
  static_assert(DK % 16 == 0 && 128 % DK == 0, "d_k must divide 128");
  static_assert(RG * 2 >= RPWV, "value words too long for the group size");
  static_assert(NS <= 32 && NP <= 32, "TMEM column plan");
  static_assert(RING >= 2 * NG, "ring too small");
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

// Half of the registers of a word: registers [0, 8/B) of (w >> 8*hi).
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
// which keeps both the B_P row stores and the key-row loads free of bank conflicts.
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
  constexpr int NG = G::NG, RING = G::RING, WS = G::WS, NS = G::NS, NP = G::NP, HP = G::HP;
  extern __shared__ __align__(1024) unsigned char smem[];

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * d.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qr = lane >> 2, qi = lane & 3;

  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t bar_ring = sbase, bar_s = sbase + G::SM_BAR_S, bar_p = sbase + G::SM_BAR_P;
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

  if (warp == 0) {
    ptx::tmem_alloc(sbase + G::SM_TMEM, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < RING; ++s) {
      ptx::mbar_init(bar_ring + 8 * s, 1);
      sm_issued[s] = 0;
    }
    ptx::mbar_init(bar_s, 1);
    ptx::mbar_init(bar_p, 1);
    ptx::fence_barrier_init();
  }

  // one thread copies group u of this CTA into stage u % RING
  auto issue = [&](int u) {
    const int g = g_begin + u, st = u % RING;
    const uint32_t bar = bar_ring + 8 * st;
    const uint32_t dst = ring_s + st * G::STAGE_STRIDE;
    sm_issued[st] += 1;
    ptx::mbar_arrive_expect_tx(bar, G::STAGE_BYTES);
    const size_t grp = static_cast<size_t>(bh) * (d.lcap / GK) + g;
    const size_t tok = static_cast<size_t>(bh) * d.lcap + static_cast<size_t>(g) * GK;
    ptx::bulk_g2s(dst + G::K_OFF, cb.kcode + tok * G::KW, GK * G::KROW, bar);
    ptx::bulk_g2s(dst + G::KM_OFF, cb.ksz + grp * DK, DK * 4, bar);
    ptx::bulk_g2s(dst + G::V_OFF, cb.vcode + grp * (kDV * G::VRW), GK * kDV * VB / 8, bar);
    ptx::bulk_g2s(dst + G::VM_OFF, cb.vsz + tok * G::NVG, GK * G::NVG * 4, bar);
  };
  auto stage = [&](int u) -> const unsigned char* { return ring + (u % RING) * G::STAGE_STRIDE; };

  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + G::SM_TMEM);
  const uint32_t tlane = static_cast<uint32_t>(32 * warp) << 16;
  {
    // A_one: 2^-24 (the smallest fp16 subnormal) in both halves of 8 columns
    uint32_t one[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) one[i] = 0x00010001u;
    ptx::tmem_st_32x32b<8>(tmem + tlane + kColA1, one);
  }
  if (tid == 0)
    for (int u = 0; u < RING && u < n_units; ++u) issue(u);

  // ---- per-thread maps (fixed for the whole CTA) ----
  // key phase: rows of lanes 32w + 16hf + qr + 8e
  int kg[2][2], koff[2][2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const TokenSlot t = token_of_kslot<VB, GK>(kslot_of_lane(32 * warp + 16 * hf + qr + 8 * e));
      kg[hf][e] = t.g;
      koff[hf][e] = G::K_OFF + t.tok * G::KROW + qi * G::WPT * 4;
    }
  // softmax phase: my lane's token
  const int my_k = kslot_of_lane(tid);
  const TokenSlot me = token_of_kslot<VB, GK>(my_k);
  const float my_pv = static_cast<float>(me.pv);
  // query phase: K slot tid % DK of key groups tid / DK, tid / DK + 128 / DK, ...
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

  float m_reg[NREP], lsum[NREP], zs[G::NVG][NREP];
#pragma unroll
  for (int hh = 0; hh < NREP; ++hh) {
    m_reg[hh] = -INFINITY;
    lsum[hh] = 0.0f;
#pragma unroll
    for (int vg = 0; vg < G::NVG; ++vg) zs[vg][hh] = 0.0f;
  }
  int s_issued = 0, p_issued = 0;
  bool failed = false;   // uniform: set at a barrier from every thread's `bad`
  bool bad = false;      // this thread saw a bounded wait give up
  const uint32_t idesc_s = idesc_f16(NS), idesc_p = idesc_f16(NP);
  constexpr uint32_t LBO_S = (NS / 8) * 128, LBO_P = (NP / 8) * 128;

  for (int blk = 0; blk < n_blocks; ++blk) {
    const int u0 = blk * NG;
    const int nvalid = min(NG, n_units - u0);
    bool ok = true;
    for (int g = 0; g < nvalid; ++g) {
      const int u = u0 + g;
      ok = ok && ptx::mbar_wait_bounded(bar_ring + 8 * (u % RING), (u / RING) & 1, kWaitLimitNs);
    }
    bad |= !ok;

    // ---- (a) keys -> A_K ----
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t regs[4 * G::KSTEPS];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        uint32_t wds[G::WPT];
        lds_words<G::WPT>(stage(u0 + kg[hf][e]) + koff[hf][e], wds);
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
      ptx::tmem_st_16x256b<G::KSTEPS>(tmem + (static_cast<uint32_t>(32 * warp + 16 * hf) << 16) + kColAK,
                                      regs);
    }

    // ---- (b) query scaled per key group -> B_S, B_Z ----
#pragma unroll
    for (int gg0 = 0; gg0 < NG; gg0 += kThreads / DK) {
      const int gg = gg0 + tid / DK;
      if (gg < nvalid) {
        const __half2 sz = *reinterpret_cast<const __half2*>(stage(u0 + gg) + G::KM_OFF + bch.x * 4);
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
          const uint32_t x0 = vs[4 * c], x1 = vs[4 * c + 1];
          const uint32_t x2 = 4 * c + 2 < 2 * HP ? vs[4 * c + 2] : 0u;
          const uint32_t x3 = 4 * c + 3 < 2 * HP ? vs[4 * c + 3] : 0u;
          const uint32_t y0 = vz[4 * c], y1 = vz[4 * c + 1];
          const uint32_t y2 = 4 * c + 2 < 2 * HP ? vz[4 * c + 2] : 0u;
          const uint32_t y3 = 4 * c + 3 < 2 * HP ? vz[4 * c + 3] : 0u;
          *reinterpret_cast<uint4*>(sBS + off + c * 128) = make_uint4(x0, x1, x2, x3);
          *reinterpret_cast<uint4*>(sBZ + off + c * 128) = make_uint4(y0, y1, y2, y3);
        }
      }
    }
    ptx::tmem_wait_st();
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    if (__syncthreads_or(bad)) {
      failed = true;
      break;
    }
    if (tid == 0) {
      ptx::tc_fence_after();
      const uint32_t bs = ptx::smem_addr(sBS), bz = ptx::smem_addr(sBZ);
#pragma unroll
      for (int s = 0; s < G::KSTEPS; ++s)
        ptx::mma_f16_ts(tmem + kColDS, tmem + kColAK + 8 * s, smem_desc(bs + 2 * LBO_S * s, LBO_S, 128),
                        idesc_s, s > 0);
#pragma unroll
      for (int s = 0; s < G::KSTEPS; ++s)
        ptx::mma_f16_ts(tmem + kColDS, tmem + kColA1, smem_desc(bz + 2 * LBO_S * s, LBO_S, 128), idesc_s,
                        true);
      ptx::tc_commit(bar_s);
    }
    ++s_issued;

    // ---- (c) values -> A_V, once the previous block's p.V MMA has read it ----
    if (p_issued > 0 && !ptx::mbar_wait_bounded(bar_p, (p_issued - 1) & 1, kWaitLimitNs)) bad = true;
    ptx::tc_fence_after();
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t regs[32];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = 32 * warp + 16 * hf + qr + 8 * e;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          uint32_t r[G::RG];
          const unsigned char* row = stage(u0 + g) + G::V_OFF + c * (G::VRW * 4);
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
      ptx::tmem_st_16x256b<8>(tmem + (static_cast<uint32_t>(32 * warp + 16 * hf) << 16) + kColAV, regs);
    }

    // ---- (d) scores -> softmax -> B_P ----
    if (!ptx::mbar_wait_bounded(bar_s, (s_issued - 1) & 1, kWaitLimitNs)) bad = true;
    ptx::tc_fence_after();
    float sc[NREP];
    {
      uint32_t raw[WS];
      ptx::tmem_load_32x32b<WS>(tmem + tlane + kColDS + me.g * WS, raw);
#pragma unroll
      for (int hh = 0; hh < NREP; ++hh) {
        const int i = hh >> 1, e = hh & 1;
        sc[hh] = (__uint_as_float(raw[4 * i + e]) + __uint_as_float(raw[4 * i + 2 + e])) * alpha24;
      }
    }
    const int pos0 = (g_begin + u0) * GK;
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
    for (int hh = 0; hh < NREP; ++hh) {
      if (!valid) sc[hh] = -INFINITY;
      exceed |= sc[hh] > m_reg[hh] + kLazyRescale;
    }
    if (__any_sync(0xffffffffu, exceed)) {
#pragma unroll
      for (int hh = 0; hh < NREP; ++hh) {
        float mx = sc[hh];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) sm_wmax[warp * 8 + hh] = mx;
      }
    } else if (lane == 0) {
#pragma unroll
      for (int hh = 0; hh < NREP; ++hh) sm_wmax[warp * 8 + hh] = -INFINITY;
    }
    if (__syncthreads_or(exceed)) {
      // the reference maximum moves: rescale what was accumulated so far
      float a[NREP];
#pragma unroll
      for (int hh = 0; hh < NREP; ++hh) {
        float mn = m_reg[hh];
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) mn = fmaxf(mn, sm_wmax[ww * 8 + hh]);
        a[hh] = (m_reg[hh] == -INFINITY || mn == -INFINITY) ? 0.0f : ptx::ex2(m_reg[hh] - mn);
        if (mn == m_reg[hh]) a[hh] = 1.0f;
        m_reg[hh] = mn;
        lsum[hh] *= a[hh];
#pragma unroll
        for (int vg = 0; vg < G::NVG; ++vg) zs[vg][hh] *= a[hh];
      }
      if (p_issued > 0) {
        uint32_t acc[NP];
        ptx::tmem_load_32x32b<NP>(tmem + tlane + kColDP, acc);
#pragma unroll
        for (int n = 0; n < NP; ++n) {
          const int wi = n % WS, hh = 2 * (wi >> 2) + (wi & 1);
          const float f = hh < NREP ? a[hh] : 0.0f;
          acc[n] = __float_as_uint(__uint_as_float(acc[n]) * f);
        }
        ptx::tmem_st_32x32b<NP>(tmem + tlane + kColDP, acc);
      }
    }
    {
      float pp[NREP];
#pragma unroll
      for (int hh = 0; hh < NREP; ++hh) {
        const float mu = m_reg[hh] == -INFINITY ? 0.0f : m_reg[hh];
        pp[hh] = ptx::ex2(sc[hh] - mu - my_pv);       // p * 2^-pv (0 when masked)
        lsum[hh] += pp[hh];
      }
      __half2 ph[HP], pl[HP];
#pragma unroll
      for (int i = 0; i < HP; ++i) {
        const float p1 = 2 * i + 1 < NREP ? pp[2 * i + 1] : 0.0f;
        ph[i] = __floats2half2_rn(pp[2 * i], p1);
        const float2 hf = __half22float2(ph[i]);
        pl[i] = __floats2half2_rn(pp[2 * i] - hf.x, p1 - hf.y);
      }
      uint32_t vm[G::NVG];
      lds_words<G::NVG>(stage(u0 + me.g) + G::VM_OFF + me.tok * G::NVG * 4, vm);
#pragma unroll
      for (int vg = 0; vg < G::NVG; ++vg) {
        const uint32_t m = valid ? vm[vg] : 0u;
        const __half2 sz = ptx::u32_as_h2(m);
        const __half2 s2 = __low2half2(sz);
        const float zf = __high2float(sz);
        uint32_t x[2 * HP];
#pragma unroll
        for (int i = 0; i < HP; ++i) {
          const __half2 hi = __hmul2(ph[i], s2);
          const __half2 lo = __hfma2(pl[i], s2, __hfma2(ph[i], s2, __hneg2(hi)));
          x[2 * i] = ptx::h2_as_u32(hi);
          x[2 * i + 1] = ptx::h2_as_u32(lo);
        }
#pragma unroll
        for (int hh = 0; hh < NREP; ++hh) zs[vg][hh] = fmaf(pp[hh], zf, zs[vg][hh]);
        const int off = ((my_k >> 3) * (NP / 8) + vg * (WS / 8)) * 128 + (my_k & 7) * 16;
#pragma unroll
        for (int c = 0; c < WS / 8; ++c) {
          const uint32_t x2 = 4 * c + 2 < 2 * HP ? x[4 * c + 2] : 0u;
          const uint32_t x3 = 4 * c + 3 < 2 * HP ? x[4 * c + 3] : 0u;
          *reinterpret_cast<uint4*>(sBP + off + c * 128) = make_uint4(x[4 * c], x[4 * c + 1], x2, x3);
        }
      }
    }
    ptx::tmem_wait_st();
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    if (__syncthreads_or(bad)) {
      failed = true;
      break;
    }
    // ---- (e) p.V, then refill the block's stages ----
    if (tid == 0) {
      ptx::tc_fence_after();
      const uint32_t bp = ptx::smem_addr(sBP);
#pragma unroll
      for (int s = 0; s < kTok / 16; ++s)
        ptx::mma_f16_ts(tmem + kColDP, tmem + kColAV + 8 * s, smem_desc(bp + 2 * LBO_P * s, LBO_P, 128),
                        idesc_p, p_issued > 0 || s > 0);
      ptx::tc_commit(bar_p);
      ptx::fence_proxy_async_smem();
      for (int g = 0; g < NG; ++g)
        if (u0 + g + RING < n_units) issue(u0 + g + RING);
    }
    ++p_issued;
  }

  // ---- drain: the last p.V MMA (or, after a timeout, everything in flight) ----
  if (failed) {
    if (tid == 0) atomicOr(part.status, KVQ_STATUS_TIMEOUT);
    if (tid < RING && sm_issued[tid] > 0)
      ptx::mbar_wait_bounded(bar_ring + 8 * tid, (sm_issued[tid] - 1) & 1, kWaitLimitNs);
    if (s_issued > 0) ptx::mbar_wait_bounded(bar_s, (s_issued - 1) & 1, kWaitLimitNs);
  }
  const bool have_pv = p_issued > 0;
  if (have_pv && !ptx::mbar_wait_bounded(bar_p, (p_issued - 1) & 1, kWaitLimitNs)) {
    atomicOr(part.status, KVQ_STATUS_TIMEOUT);
    bad = true;
  }
  ptx::tc_fence_after();

  // ---- CTA totals of sum p and sum p z (each thread's share is in units of 2^-pv) ----
  const float unscale = static_cast<float>(1 << me.pv);
  constexpr int NRED = NREP * (G::NVG + 1);
  float red[NRED];
#pragma unroll
  for (int hh = 0; hh < NREP; ++hh) {
    red[hh] = lsum[hh] * unscale;
#pragma unroll
    for (int vg = 0; vg < G::NVG; ++vg) red[NREP + vg * NREP + hh] = zs[vg][hh] * unscale;
  }
#pragma unroll
  for (int i = 0; i < NRED; ++i) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) red[i] += __shfl_xor_sync(0xffffffffu, red[i], o);
  }
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < NRED; ++i) sm_red[warp * NRED + i] = red[i];
  failed = __syncthreads_or(failed || bad) != 0;
#pragma unroll
  for (int i = 0; i < NRED; ++i)
    red[i] = sm_red[i] + sm_red[NRED + i] + sm_red[2 * NRED + i] + sm_red[3 * NRED + i];

  // ---- the partial of this split: lane = channel tid ----
  {
    uint32_t acc[NP];
#pragma unroll
    for (int n = 0; n < NP; ++n) acc[n] = 0u;
    if (have_pv && !failed) ptx::tmem_load_32x32b<NP>(tmem + tlane + kColDP, acc);
    const int c = tid, vg = c / GV;
#pragma unroll
    for (int hh = 0; hh < NREP; ++hh) {
      const int i = hh >> 1, e = hh & 1;
      float o = 0.0f;
#pragma unroll
      for (int v = 0; v < G::NVG; ++v)
        if (v == vg)
          o = (__uint_as_float(acc[v * WS + 4 * i + e]) + __uint_as_float(acc[v * WS + 4 * i + 2 + e])) *
                  16777216.0f +
              red[NREP + v * NREP + hh];
      const size_t pi = (static_cast<size_t>(b) * d.Hq + h * NREP + hh) * w.splits + split;
      part.o[pi * kDV + c] = failed ? 0.0f : o;
      if (c == 0) part.ml[pi] = failed ? make_float2(-INFINITY, 0.0f) : make_float2(m_reg[hh], red[hh]);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int KB, int VB, int DK, int NREP, int GV, int GK>
cudaError_t launch(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                   const Partials& p, cudaStream_t s) {
  using G = Geom<KB, VB, DK, NREP, GV, GK>;
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
