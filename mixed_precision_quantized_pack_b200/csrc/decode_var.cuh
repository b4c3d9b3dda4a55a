// Tensor-core decode attention over caches with per-channel bit widths: the kernel
// ("Attention-Aware Transform Coding (AATC)", §Méthodologie, Allocation de Bits: each
// transformed channel gets its own number of bits, zero for the weakest).
//
// The split-K structure of the fixed-width kernel: one CTA per (split, kv head, sequence), four
// warps, a CTA-wide ring of bulk-copy stages, a partial (m, l, o) per query head and split that
// the combine kernel merges.  As in that kernel the MMA operands are built in registers from the
// packed words (no expanded copy of a tile is written anywhere); the map's layout comes from a
// plan made on the host, so any map within the shape limits below runs on this code:
//
// keys    Widths are non-increasing powers of two, so every field starts at a multiple of its
//         width and lies inside one byte.  Masking a word in place (w & m) gives the fields of
//         bytes 0 and 2 as fp16 subnormals code * 2^(p-24) (p = the field's bit in its byte),
//         and (w >> 8) & m those of bytes 1 and 3.  The plan pairs one register of each kind
//         from the same word (a couple: A registers a0 and a2 of one row in one k-step) and
//         gives couple 4s + qi to quad lane qi in k-step s, so a lane pays one word load and
//         three ALU operations per row and k-step.  B = (q_c 2^-p) s_c split into exact (hi, lo)
//         fp16 halves, formed once per key group from the group's (scale, zero) gathered into
//         couple order; sum_c q_c z_c by one more MMA per k-step.  score = (C_hi + C_lo) 2^24
//         alpha + alpha sum_c q_c z_c.
// values  A value group's G_v channels share one width b.  Quad row qr owns the run of G_v/8
//         consecutive channels of each group; a byte permute puts the runs of two tokens in
//         the two halves of one register (token 2qi low, 2qi + 1 high) and masks in place give
//         one register per channel.  Channels on M, tokens on K, B = p_t s_{t,g} split (hi, lo)
//         and transposed by movmatrix; o_c = C 2^(24-p) + sum_t p_t z_{t,g}.  A group's width
//         is a run-time value (one warp-uniform branch per group and key group); dropped groups
//         are skipped.
// fp16    Retained tokens and the window: rows loaded with ldmatrix as they are.
//
// A map known at build time (FixedMap) gets an instance in which the k-step count, the row
// strides and the value groups' widths and first bits are compile-time constants.
//
// Shape limits (other maps run on the generic kernel): d_k = d_v = 128, 1 or 4 query heads per
// kv head, value groups of 16, 32, 64 or 128 channels, and at most 32 couples in a key row
// (eight k-steps: every map whose key words each hold one width fits; a map whose words mix
// widths can need more).
#pragma once
#include <string.h>

#include "../../include/kvq.h"
#include "kvq_internal.cuh"
#include "ptx.cuh"

namespace kvq {
namespace var {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kDK = 128, kDV = 128;
constexpr int kKSteps = 8;                 // k-steps of 16 fields: a 128-channel row at most
constexpr int kCouples = 4 * kKSteps;
constexpr int kMaxRing = 8;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kLazyRescale = 8.0f;
// Three CTAs per SM (168 registers): the build-time map instances spill at four, and the run-time
// ones, which fit four, measured 3-6% faster at three.
constexpr int kCtasPerSm = 3;
constexpr int kSmemPerCta = 233472 / kCtasPerSm - 1024;
constexpr int KST = kDK * 2 + 16;          // padded fp16 row strides of an fp16 stage (bytes)
constexpr int VST = kDV * 2 + 16;
constexpr unsigned char kNone = 0xFF;

// The plan of a width map (a kernel parameter, made on the host by make_plan).
struct VarPlan {
  int nks;                                // k-steps of the score contraction
  uint32_t kwo[kCouples];                 // couple n: byte offset of its word in a key row
  uint32_t kma[kCouples], kmb[kCouples];  // masks of a0 = w & ma and a2 = (w >> 8) & mb
  unsigned char kch[kCouples][4];         // channels of (a0 lo, a0 hi, a2 lo, a2 hi); kNone: empty
  unsigned char kpos[kCouples][4];        // their field offsets p
  int vbits[8];                           // width of value group g (0: dropped)
  int vbit0[8];                           // first bit of value group g in a value row
};

// Shared memory of one CTA: mbarriers and stage bookkeeping, the couple descriptors, the query
// terms of each couple and head, per warp the current group's key (scale, zero) in couple
// order, then the ring of stages.
struct Smem {
  static constexpr int kBars = 0;
  static constexpr int kIssued = kBars + kMaxRing * 8;
  static constexpr int kTag = kIssued + kMaxRing * 4;
  static constexpr int kFail = kTag + kMaxRing * 4;
  static constexpr int kDesc = 256;                         // uint4 [couple]: word offset, ma, mb
  static constexpr int kQk = kDesc + kCouples * 16;         // uint4 [couple][4 heads]: qf0 qf1 qb0 qb1
  static constexpr int kKsz = kQk + kCouples * 4 * 16;      // uint4 [warp][couple]: (s, z) words
  static constexpr int kStages = kKsz + kWarps * kCouples * 16;
};

struct StageLayout {
  int k_off, kmeta_off, v_off, vmeta_off, bytes;
};

__host__ __device__ inline StageLayout var_stage_layout(const Dims& d) {
  StageLayout s;
  s.k_off = 0;
  s.kmeta_off = d.gk * d.kw * 4;
  s.v_off = s.kmeta_off + d.dk * 4;
  s.vmeta_off = s.v_off + d.gk * d.vw * 4;
  s.bytes = s.vmeta_off + d.gk * d.nvg * 4;
  return s;
}

__host__ __device__ inline int round128(int x) { return (x + 127) / 128 * 128; }

constexpr int kRawStage = (16 * (KST + VST) + 127) / 128 * 128;

// N consecutive words of shared memory at an address aligned to min(4N, 16) bytes.
template <int N>
__device__ __forceinline__ void load_row(const uint32_t* p, uint32_t* out) {
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
    out[0] = p[0];
  }
}

// The 16 / B codes of a 16-bit piece (field f at bit B f of each half) as registers: field f
// masked in place in x or in x >> 8, so at offset p = (B f) mod 8.
template <int B>
__device__ __forceinline__ void unpack_piece16(uint32_t x, uint32_t* r) {
  const uint32_t u = x >> 8;
#pragma unroll
  for (int f = 0; f < 16 / B; ++f) r[f] = (B * f < 8 ? x : u) & (((1u << B) - 1u) << ((B * f) & 7)) * 0x00010001u;
}

// p.V of one value group of width B: the lane's run (channels qr * G_v/8 ...) of tokens
// (ta, tb) and (ta + 8, tb + 8), swapped so that token 2qi lands in the low half, then G_v/16
// MMAs into the group's channel tiles c[0 .. G_v/16).
template <int B, int GV>
__device__ __forceinline__ void value_group(const uint32_t* svc, int vw, int ta, int tb, int qr, bool swap,
                                            uint32_t sel_lo, uint32_t sel_hi, int bit0, uint32_t bp0,
                                            uint32_t bp1, float (*c)[4]) {
  constexpr int CPG = GV / 8, MPG = CPG / 2, RUN = CPG * B;
  uint32_t ra[CPG], rb[CPG];
  const int ob = bit0 + qr * RUN;        // a multiple of RUN: the run never crosses a byte or word
  if constexpr (RUN < 16) {
    const int wv = ob >> 5;
    const uint32_t bs = static_cast<uint32_t>((ob >> 3) & 3);
    const uint32_t sel = swap ? ((4 + bs) | ((4 + bs) << 4) | (bs << 8) | (bs << 12))
                              : (bs | (bs << 4) | ((4 + bs) << 8) | ((4 + bs) << 12));
    const int sh = ob & 7;
    const uint32_t x0 = ptx::prmt(svc[ta * vw + wv], svc[tb * vw + wv], sel) >> sh;
    const uint32_t x1 = ptx::prmt(svc[(ta + 8) * vw + wv], svc[(tb + 8) * vw + wv], sel) >> sh;
#pragma unroll
    for (int e = 0; e < CPG; ++e) {
      ra[e] = x0 & (((1u << B) - 1u) << (B * e)) * 0x00010001u;
      rb[e] = x1 & (((1u << B) - 1u) << (B * e)) * 0x00010001u;
    }
  } else {
    constexpr int NP = RUN / 16, FP = 16 / B;     // 16-bit pieces of the run, fields per piece
#pragma unroll
    for (int pc = 0; pc < NP; ++pc) {
      const int bit = ob + 16 * pc;
      const int wv = bit >> 5;
      const uint32_t sel = (bit & 16) ? sel_hi : sel_lo;
      unpack_piece16<B>(ptx::prmt(svc[ta * vw + wv], svc[tb * vw + wv], sel), ra + pc * FP);
      unpack_piece16<B>(ptx::prmt(svc[(ta + 8) * vw + wv], svc[(tb + 8) * vw + wv], sel), rb + pc * FP);
    }
  }
#pragma unroll
  for (int ml = 0; ml < MPG; ++ml) ptx::mma_16816(c[ml], ra[ml], ra[ml + MPG], rb[ml], rb[ml + MPG], bp0, bp1);
}

// A width map known at build time: channel counts of widths 8, 4, 2 and 1 for keys (K*) and
// values (V*).  Its instance folds the k-step count, the row strides and every value group's width
// and first bit into the code (no branch on a group's width, immediate row offsets); the couple
// descriptors still come from the plan, which the host checks against these counts.
template <int K8, int K4, int K2, int K1, int V8, int V4, int V2, int V1>
struct FixedMap {
  static constexpr bool kFixed = true;
  static constexpr int kBitsK = 8 * K8 + 4 * K4 + 2 * K2 + K1;
  static constexpr int kBitsV = 8 * V8 + 4 * V4 + 2 * V2 + V1;
  static constexpr int KW = kBitsK > 32 ? (kBitsK + 31) / 32 : 1;
  static constexpr int VW = kBitsV > 32 ? (kBitsV + 31) / 32 : 1;
  static constexpr int kcnt(int i) { return i == 0 ? K8 : i == 1 ? K4 : i == 2 ? K2 : K1; }
  static constexpr int vcnt(int i) { return i == 0 ? V8 : i == 1 ? V4 : i == 2 ? V2 : V1; }
  // width of value channel c (0: dropped)
  static constexpr int vwidth(int c) {
    return c < V8 ? 8 : c < V8 + V4 ? 4 : c < V8 + V4 + V2 ? 2 : c < V8 + V4 + V2 + V1 ? 1 : 0;
  }
  // first bit of value group g of gv channels
  static constexpr int vbit0(int g, int gv) {
    int bit = 0;
    for (int i = 0; i < g; ++i) bit += gv * vwidth(i * gv);
    return bit;
  }
  // couples of a key row: per word, the larger field count of bytes (0, 2) and of bytes (1, 3)
  static constexpr int couples() {
    int cnt[32][4] = {};
    int q = 0;
    for (int i = 0; i < 4; ++i)
      for (int n = 0; n < kcnt(i); ++n) {
        cnt[(q >> 5) & 31][(q >> 3) & 3] += 1;
        q += 8 >> i;
      }
    int total = 0;
    for (int wd = 0; wd < 32; ++wd) {
      const int a = cnt[wd][0] > cnt[wd][2] ? cnt[wd][0] : cnt[wd][2];
      const int b = cnt[wd][1] > cnt[wd][3] ? cnt[wd][1] : cnt[wd][3];
      total += a > b ? a : b;
    }
    return total;
  }
  static constexpr int NKS = (couples() + 3) / 4;
};
struct RuntimeMap {
  static constexpr bool kFixed = false;
  static constexpr int KW = 0, VW = 0, NKS = 0;
  static constexpr int vwidth(int) { return 0; }
  static constexpr int vbit0(int, int) { return 0; }
};

// The maps with a build-time instance (1 or 4 query heads per kv head as listed, groups of 64
// tokens): keys 16 x 8, 64 x 4, 32 x 2 bits (16 dropped), values in groups of 32 channels at 4, 2,
// 2, 1 bits; keys 32 x 8, 96 x 2 bits, values in groups of 64 channels at 4 and 2 bits.
using MapK3V2 = FixedMap<16, 64, 32, 0, 0, 32, 64, 32>;
using MapK8K2 = FixedMap<32, 0, 96, 0, 0, 64, 64, 0>;

// p.V of one value group of width B over the MT tiles of a key group: per tile the (scale, zero)
// of the lane's two tokens, the B operand p_t s_{t,g} split (hi, lo) and transposed, and the
// group's MMAs; zsum accumulates sum_t p_t z_{t,g}.
template <int B, int GV, int MT, int NVG>
__device__ __forceinline__ void value_group_tiles(const uint32_t* svc, const uint32_t* svm, int vw, int gg, int qi,
                                                  int qr, bool swap, uint32_t sel_lo, uint32_t sel_hi, int bit0,
                                                  const float (&pw)[MT][2], float& zsum, float (*c)[4]) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int t0 = 16 * mt + qr;
    const float2 f0 = __half22float2(ptx::u32_as_h2(svm[t0 * NVG + gg]));
    const float2 f1 = __half22float2(ptx::u32_as_h2(svm[(t0 + 8) * NVG + gg]));
    zsum = fmaf(pw[mt][0], f0.y, fmaf(pw[mt][1], f1.y, zsum));
    const uint32_t bp0 = ptx::movmatrix_trans(ptx::split_hi_lo_trunc(pw[mt][0] * f0.x));
    const uint32_t bp1 = ptx::movmatrix_trans(ptx::split_hi_lo_trunc(pw[mt][1] * f1.x));
    const int ta = 16 * mt + 2 * qi + (swap ? 1 : 0);
    const int tb = 16 * mt + 2 * qi + (swap ? 0 : 1);
    value_group<B, GV>(svc, vw, ta, tb, qr, swap, sel_lo, sel_hi, bit0, bp0, bp1, c);
  }
}

template <int NREP, int GV, int GK, class MAP = RuntimeMap>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
decode_var_kernel(Dims d, CacheBufs cb, DecodeWork w, VarPlan plan, const __half* __restrict__ q,
                  Partials part) {
  constexpr int NVG = kDV / GV;          // value groups per row
  constexpr int CPG = GV / 8;            // channels of a lane's run in a group
  constexpr int MPG = CPG / 2;           // channel tiles (MMAs) per group
  extern __shared__ __align__(128) unsigned char smem[];
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * d.Hkv + h;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = lane & 3;          // C columns 2qi, 2qi+1 = head qi (hi, lo)
  const int qr = lane >> 2;         // A rows qr, qr + 8; B column qr
  const int bhead = qr >> 1;        // head of this thread's B column
  const bool blo = (qr & 1) != 0;   // B column holds the lo half
  const bool bvalid = bhead < NREP;
  const bool cvalid = qi < NREP;

  int* sm_issued = reinterpret_cast<int*>(smem + Smem::kIssued);
  volatile int* sm_tag = reinterpret_cast<volatile int*>(smem + Smem::kTag);
  int* sm_fail = reinterpret_cast<int*>(smem + Smem::kFail);
  const uint32_t bar0 = ptx::smem_addr(smem + Smem::kBars);
  const uint4* sm_desc = reinterpret_cast<const uint4*>(smem + Smem::kDesc);
  const uint4* sm_qk = reinterpret_cast<const uint4*>(smem + Smem::kQk);
  uint4* sm_ksz = reinterpret_cast<uint4*>(smem + Smem::kKsz) + warp * kCouples;
  unsigned char* stages = smem + Smem::kStages;
  const uint32_t stages_s = ptx::smem_addr(stages);

  const bool quant = split < w.splits_q;
  const StageLayout L = var_stage_layout(d);
  const int stage_bytes = quant ? round128(L.bytes) : kRawStage;
  int ring = (kSmemPerCta - Smem::kStages) / stage_bytes;
  ring = ring > kMaxRing ? kMaxRing : ring;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ring; ++s) {
      ptx::mbar_init(bar0 + 8 * s, 1);
      sm_issued[s] = 0;
      sm_tag[s] = -1;
    }
    *sm_fail = 0;
    ptx::fence_barrier_init();
  }
  const __half* qbase = q + (static_cast<size_t>(b) * d.Hq + h * NREP) * kDK;
  if (quant) {
    // the couple descriptors, and per couple and head the B terms (q_c 2^-p for the scores,
    // q_c for the zero-point MMA) of the couple's four channels; zeros for empty halves and
    // for heads past NREP
    for (int n = threadIdx.x; n < kCouples; n += kThreads)
      reinterpret_cast<uint4*>(smem + Smem::kDesc)[n] = make_uint4(plan.kwo[n], plan.kma[n], plan.kmb[n], 0u);
    for (int i = threadIdx.x; i < kCouples * 4; i += kThreads) {
      const int n = i >> 2, hh = i & 3;
      uint32_t f[2] = {0u, 0u}, g[2] = {0u, 0u};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        __half qf[2], qb[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int ch = plan.kch[n][2 * r + e];
          qb[e] = __float2half_rn(0.0f);
          qf[e] = qb[e];
          if (hh < NREP && ch != kNone) {
            qb[e] = qbase[hh * kDK + ch];
            qf[e] = __hmul(qb[e], __float2half_rn(1.0f / static_cast<float>(1 << plan.kpos[n][2 * r + e])));
          }
        }
        f[r] = ptx::h2_as_u32(__halves2half2(qf[0], qf[1]));
        g[r] = ptx::h2_as_u32(__halves2half2(qb[0], qb[1]));
      }
      reinterpret_cast<uint4*>(smem + Smem::kQk)[i] = make_uint4(f[0], f[1], g[0], g[1]);
    }
  }

  // ---------------- work list ----------------
  const SeqWork sw = seq_work(w, b, GK, d.log_retain);
  int unit_begin = 0, unit_end, list_begin = 0, list_end = 0;
  if (quant) {
    unit_begin = static_cast<int>(static_cast<long long>(split) * sw.n_groups / w.splits_q);
    unit_end = static_cast<int>(static_cast<long long>(split + 1) * sw.n_groups / w.splits_q);
  } else {
    const int f = split - w.splits_q;
    list_begin = static_cast<int>(static_cast<long long>(f) * sw.n_fp16 / w.splits_f);
    list_end = static_cast<int>(static_cast<long long>(f + 1) * sw.n_fp16 / w.splits_f);
    unit_end = (list_end - list_begin + 15) / 16;
  }
  const int n_units = unit_end - unit_begin;
  constexpr int gk = GK;

  // one lane copies unit k into stage k % ring: a key group (four runs), or up to 16 fp16
  // key and value rows (one lane per row and tensor)
  auto issue = [&](int k) {
    const int st = k % ring;
    const uint32_t bar = bar0 + 8 * st;
    const uint32_t dst = stages_s + st * stage_bytes;
    if (quant) {
      const int g = unit_begin + k;
      sm_issued[st] += 1;
      sm_tag[st] = k;
      // (test hook) one stage that never completes: its waits run into their bound
      const bool stall = w.stall && k == 0 && split == 0 && h == 0 && b == 0;
      ptx::mbar_arrive_expect_tx(bar, L.bytes + (stall ? 16u : 0u));
      size_t gi = KVQ_IN_BOUNDS(d, kSiteDecTable, g, d.max_groups) ? group_index(d, cb.table, b, h, g) : 0;
      // (bounds-check builds) a group outside the buffers is replaced by group 0, so that the
      // stage's copies still complete
      if (!KVQ_IN_BOUNDS(d, kSiteDecKCode, static_cast<long long>(gi), quant_groups(d))) gi = 0;
      const size_t tok = gi * gk;
      ptx::bulk_g2s(dst + L.k_off, cb.kcode + tok * d.kw, gk * d.kw * 4, bar);
      ptx::bulk_g2s(dst + L.kmeta_off, cb.ksz + gi * d.dk, d.dk * 4, bar);
      ptx::bulk_g2s(dst + L.v_off, cb.vcode + tok * d.vw, gk * d.vw * 4, bar);
      ptx::bulk_g2s(dst + L.vmeta_off, cb.vsz + tok * d.nvg, gk * d.nvg * 4, bar);
    } else {
      const int e0 = list_begin + 16 * k;
      const int nvalid = min(16, list_end - e0);
      if (lane == 0) {
        sm_issued[st] += 1;
        sm_tag[st] = k;
        const bool stall = w.stall && k == 0 && split == w.splits_q && h == 0 && b == 0;
        ptx::mbar_arrive_expect_tx(bar, nvalid * (kDK + kDV) * 2 + (stall ? 16 : 0));
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
          ptx::bulk_g2s(dst + row * KST, base_k + slot * kDK, kDK * 2, bar);
        else
          ptx::bulk_g2s(dst + 16 * KST + row * VST, base_v + slot * kDV, kDV * 2, bar);
      }
    }
  };

  // fp16 stages: stale shared memory must hold finite values (masked rows multiply p = 0)
  if (!quant) {
    for (int i = threadIdx.x; i < ring * stage_bytes / 16; i += kThreads)
      reinterpret_cast<uint4*>(stages)[i] = make_uint4(0, 0, 0, 0);
    ptx::fence_proxy_async_smem();
  }
  __syncthreads();
  if (quant) {
    if (threadIdx.x == 0)
      for (int k = 0; k < ring && k < n_units; ++k) issue(k);
  } else if (warp == 0) {
    for (int k = 0; k < ring && k < n_units; ++k) issue(k);
  }

  float m_run = -INFINITY, l_run = 0.0f;
  float zsum[NVG];                 // sum_t p_t z_{t,g}, lane-partial
#pragma unroll
  for (int g = 0; g < NVG; ++g) zsum[g] = 0.0f;
  float co[8][4];
#pragma unroll
  for (int mv = 0; mv < 8; ++mv)
#pragma unroll
    for (int e = 0; e < 4; ++e) co[mv][e] = 0.0f;
  bool failed = false;
  const float alpha = w.score_scale;                       // log2(e) / sqrt(d_k)
  const float alpha24 = w.score_scale * 16777216.0f;       // undoes the 2^-24 of subnormal codes

  if (quant) {
    // retained positions, one per lane (ascending), for masking the quantized tiles
    const int ret_pos = lane < sw.n_ret ? retained_position(sw.Q, lane) : -1;
    const int nks = MAP::kFixed ? MAP::NKS : plan.nks;
    constexpr int MT = GK / 16;         // 16-token tiles of a key group
    const int kw4 = MAP::kFixed ? MAP::KW * 4 : d.kw * 4;
    const int vw = MAP::kFixed ? MAP::VW : d.vw;
    // this lane's couple in the per-group gather of the key (scale, zero): four channel offsets
    uint32_t gofs[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int ch = plan.kch[lane][e];
      gofs[e] = ch == kNone ? 0u : static_cast<uint32_t>(ch) * 4u;
    }
    const bool swap = qi >= 2;          // bank-conflict-free value-row loads
    const uint32_t sel_lo = swap ? 0x1054u : 0x5410u;
    const uint32_t sel_hi = swap ? 0x3276u : 0x7632u;

    for (int k = warp; k < n_units; k += kWarps) {
      const int st = k % ring;
      const bool ok = ptx::wait_equal_bounded(sm_tag + st, k, kWaitLimitNs) &&
                      ptx::mbar_wait_bounded(bar0 + 8 * st, (k / ring) & 1, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        failed = true;
        break;
      }
      const unsigned char* S = stages + st * stage_bytes;

      // ---- group prologue: the key (scale, zero) in couple order, B of each k-step, bias ----
      {
        const unsigned char* km = S + L.kmeta_off;
        uint4 g4;
        g4.x = *reinterpret_cast<const uint32_t*>(km + gofs[0]);
        g4.y = *reinterpret_cast<const uint32_t*>(km + gofs[1]);
        g4.z = *reinterpret_cast<const uint32_t*>(km + gofs[2]);
        g4.w = *reinterpret_cast<const uint32_t*>(km + gofs[3]);
        sm_ksz[lane] = g4;
      }
      __syncwarp();
      uint32_t bq[kKSteps][2];
      float cb0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cb1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int s = 0; s < kKSteps; ++s) bq[s][0] = bq[s][1] = 0u;
#pragma unroll
      for (int s = 0; s < kKSteps; ++s) {
        if (s >= nks) break;
        {
          const uint4 sz = sm_ksz[4 * s + qi];
          const uint4 qq = sm_qk[(4 * s + qi) * 4 + bhead];   // zeros for heads past NREP
          const __half2 s0 = ptx::u32_as_h2(ptx::prmt(sz.x, sz.y, 0x5410u));
          const __half2 s1 = ptx::u32_as_h2(ptx::prmt(sz.z, sz.w, 0x5410u));
          const uint32_t z0 = ptx::prmt(sz.x, sz.y, 0x7632u);
          const uint32_t z1 = ptx::prmt(sz.z, sz.w, 0x7632u);
          const __half2 f0 = ptx::u32_as_h2(qq.x), f1 = ptx::u32_as_h2(qq.y);
          const __half2 hi0 = __hmul2(f0, s0), hi1 = __hmul2(f1, s1);
          bq[s][0] = blo ? ptx::h2_as_u32(__hfma2(f0, s0, __hneg2(hi0))) : ptx::h2_as_u32(hi0);
          bq[s][1] = blo ? ptx::h2_as_u32(__hfma2(f1, s1, __hneg2(hi1))) : ptx::h2_as_u32(hi1);
          if (s & 1) ptx::mma_16816(cb1, z0, z0, z1, z1, qq.z, qq.w);
          else ptx::mma_16816(cb0, z0, z0, z1, z1, qq.z, qq.w);
        }
      }
      const float beta = (cb0[0] + cb1[0]) * alpha;

      // ---- scores of the whole group ----
      // per k-step: the lane's word in row qr of the group's first tile, and the two masks
      const unsigned char* kp[kKSteps];
      uint32_t kma[kKSteps], kmb[kKSteps];
#pragma unroll
      for (int s = 0; s < kKSteps; ++s) {
        const uint4 dsc = sm_desc[4 * s + qi];
        kp[s] = S + L.k_off + qr * kw4 + dsc.x;
        kma[s] = dsc.y;
        kmb[s] = dsc.z;
      }
      float sc[MT][2];
      if constexpr (MAP::kFixed) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int s = 0; s < kKSteps; ++s) {
            if (s >= nks) break;
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(kp[s] + 16 * mt * kw4);
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(kp[s] + (16 * mt + 8) * kw4);
            ptx::mma_16816(cs, w0 & kma[s], w1 & kma[s], (w0 >> 8) & kmb[s], (w1 >> 8) & kmb[s], bq[s][0],
                           bq[s][1]);
          }
          sc[mt][0] = fmaf(cs[0] + cs[1], alpha24, beta);
          sc[mt][1] = fmaf(cs[2] + cs[3], alpha24, beta);
        }
      } else {
        // a run-time k-step count: the k-steps outside, the tiles inside (one branch per k-step
        // and key group)
        float cs[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) cs[mt][0] = cs[mt][1] = cs[mt][2] = cs[mt][3] = 0.0f;
#pragma unroll
        for (int s = 0; s < kKSteps; ++s) {
          if (s >= nks) break;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(kp[s] + 16 * mt * kw4);
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(kp[s] + (16 * mt + 8) * kw4);
            ptx::mma_16816(cs[mt], w0 & kma[s], w1 & kma[s], (w0 >> 8) & kmb[s], (w1 >> 8) & kmb[s], bq[s][0],
                           bq[s][1]);
          }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          sc[mt][0] = fmaf(cs[mt][0] + cs[mt][1], alpha24, beta);
          sc[mt][1] = fmaf(cs[mt][2] + cs[mt][3], alpha24, beta);
        }
      }
      // retained tokens of this group are read from the fp16 list: mask them here
      const int g0 = (unit_begin + k) * GK;
      unsigned hits = __ballot_sync(0xffffffffu, ret_pos >= g0 && ret_pos < g0 + GK);
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
      // the reference maximum moves only when a score exceeds it by more than kLazyRescale
      const float m_new = fmaxf(m_run, gmax);
      if (__any_sync(0xffffffffu, m_new > m_run + kLazyRescale)) {
        const float a = (m_new == -INFINITY) ? 1.0f : ptx::ex2(m_run - m_new);
        l_run *= a;
#pragma unroll
        for (int g = 0; g < NVG; ++g) zsum[g] *= a;
#pragma unroll
        for (int mv = 0; mv < 8; ++mv)
#pragma unroll
          for (int e = 0; e < 4; ++e) co[mv][e] *= a;
        m_run = m_new;
      }
      const float m_use = m_run == -INFINITY ? 0.0f : m_run;   // all masked: every p is 0

      // ---- p.V over the group ----
      const uint32_t* svc = reinterpret_cast<const uint32_t*>(S + L.v_off);
      const uint32_t* svm = reinterpret_cast<const uint32_t*>(S + L.vmeta_off);
      if constexpr (!MAP::kFixed) {
        // a run-time map: one branch on each group's width per key group (not per tile), the
        // group's tiles inside
        float pw[MT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          pw[mt][0] = ptx::ex2(sc[mt][0] - m_use);
          pw[mt][1] = ptx::ex2(sc[mt][1] - m_use);
          l_run += pw[mt][0] + pw[mt][1];
        }
#pragma unroll
        for (int gg = 0; gg < NVG; ++gg) {
          const int bit0 = plan.vbit0[gg];
          float(*cg)[4] = co + gg * MPG;
          switch (plan.vbits[gg]) {
            case 8: value_group_tiles<8, GV, MT, NVG>(svc, svm, vw, gg, qi, qr, swap, sel_lo, sel_hi, bit0, pw, zsum[gg], cg); break;
            case 4: value_group_tiles<4, GV, MT, NVG>(svc, svm, vw, gg, qi, qr, swap, sel_lo, sel_hi, bit0, pw, zsum[gg], cg); break;
            case 2: value_group_tiles<2, GV, MT, NVG>(svc, svm, vw, gg, qi, qr, swap, sel_lo, sel_hi, bit0, pw, zsum[gg], cg); break;
            case 1: value_group_tiles<1, GV, MT, NVG>(svc, svm, vw, gg, qi, qr, swap, sel_lo, sel_hi, bit0, pw, zsum[gg], cg); break;
            default: break;                  // a dropped group: no codes, (scale, zero) = 0
          }
        }
      } else {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        {
          const int t0 = 16 * mt + qr;
          const float p0 = ptx::ex2(sc[mt][0] - m_use);
          const float p1 = ptx::ex2(sc[mt][1] - m_use);
          l_run += p0 + p1;
          // value (scale, zero) of the two tokens this thread weights, every group
          uint32_t vm0[NVG], vm1[NVG];
          load_row<NVG>(svm + t0 * NVG, vm0);
          load_row<NVG>(svm + (t0 + 8) * NVG, vm1);
          // tokens 2qi, 2qi+1, 2qi+8, 2qi+9 of the tile, the pair swapped for qi >= 2
          const int ta = 16 * mt + 2 * qi + (swap ? 1 : 0);
          const int tb = 16 * mt + 2 * qi + (swap ? 0 : 1);
#pragma unroll
          for (int gg = 0; gg < NVG; ++gg) {
            const int vb = MAP::kFixed ? MAP::vwidth(gg * GV) : plan.vbits[gg];
            if (vb == 0) continue;                 // a dropped group: no codes, (scale, zero) = 0
            const float2 f0 = __half22float2(ptx::u32_as_h2(vm0[gg]));
            const float2 f1 = __half22float2(ptx::u32_as_h2(vm1[gg]));
            zsum[gg] = fmaf(p0, f0.y, fmaf(p1, f1.y, zsum[gg]));
            const uint32_t bp0 = ptx::movmatrix_trans(ptx::split_hi_lo_trunc(p0 * f0.x));
            const uint32_t bp1 = ptx::movmatrix_trans(ptx::split_hi_lo_trunc(p1 * f1.x));
            const int bit0 = MAP::kFixed ? MAP::vbit0(gg, GV) : plan.vbit0[gg];
            float(*cg)[4] = co + gg * MPG;
            switch (vb) {
              case 8: value_group<8, GV>(svc, vw, ta, tb, qr, swap, sel_lo, sel_hi, bit0, bp0, bp1, cg); break;
              case 4: value_group<4, GV>(svc, vw, ta, tb, qr, swap, sel_lo, sel_hi, bit0, bp0, bp1, cg); break;
              case 2: value_group<2, GV>(svc, vw, ta, tb, qr, swap, sel_lo, sel_hi, bit0, bp0, bp1, cg); break;
              default: value_group<1, GV>(svc, vw, ta, tb, qr, swap, sel_lo, sel_hi, bit0, bp0, bp1, cg); break;
            }
          }
        }
      }
      }

      // ---- release the stage: refill it with unit k + ring ----
      __syncwarp();
      if (lane == 0 && k + ring < n_units) {
        ptx::fence_proxy_async_smem();
        issue(k + ring);
      }
    }
  } else {
    // ---------------- fp16 rows: retained tokens, then the window ----------------
    const __half* qrow = qbase + (bvalid ? bhead : 0) * kDK;
    uint32_t qn[8][2];
#pragma unroll
    for (int s = 0; s < 8; ++s)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = 16 * s + 2 * qi + 8 * j;
        qn[s][j] = (bvalid && !blo) ? ptx::h2_as_u32(__halves2half2(qrow[c], qrow[c + 1])) : 0u;
      }
    const int mi = lane >> 3;                         // which 8x8 matrix this lane addresses
    const int arow = (mi & 1) * 8 + (lane & 7);
    const int vrow = (mi >> 1) * 8 + (lane & 7);
    for (int k = warp; k < n_units; k += kWarps) {
      const int st = k % ring;
      const bool ok = ptx::wait_equal_bounded(sm_tag + st, k, kWaitLimitNs) &&
                      ptx::mbar_wait_bounded(bar0 + 8 * st, (k / ring) & 1, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        failed = true;
        break;
      }
      const uint32_t S = stages_s + st * stage_bytes;
      const int nvalid = min(16, list_end - (list_begin + 16 * k));
      // scores: A = 16 key rows via ldmatrix, B = q (hi columns only)
      float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t a0, a1, a2, a3;
        ptx::ldmatrix_x4(S + arow * KST + (16 * s + (mi >> 1) * 8) * 2, a0, a1, a2, a3);
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
      const uint32_t bp0 = ptx::movmatrix_trans(ptx::split_hi_lo_trunc(p0));
      const uint32_t bp1 = ptx::movmatrix_trans(ptx::split_hi_lo_trunc(p1));
      // p.V: A = V^T tiles via ldmatrix.trans (rows = tokens in shared memory)
#pragma unroll
      for (int mv = 0; mv < 8; ++mv) {
        uint32_t a0, a1, a2, a3;
        ptx::ldmatrix_x4_trans(S + 16 * KST + vrow * VST + (16 * mv + (mi & 1) * 8) * 2, a0, a1, a2, a3);
        ptx::mma_16816(co[mv], a0, a1, a2, a3, bp0, bp1);
      }
      __syncwarp();
      if (k + ring < n_units) {
        if (lane == 0) ptx::fence_proxy_async_smem();
        issue(k + ring);
      }
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
    if (threadIdx.x < ring && sm_issued[threadIdx.x] > 0)
      ptx::mbar_wait_bounded(bar0 + 8 * threadIdx.x, (sm_issued[threadIdx.x] - 1) & 1, kWaitLimitNs);
    failed = true;     // the CTA's partial is dropped as a whole
  }

  // ---------------- warp totals, then the CTA merge ----------------
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 4);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
#pragma unroll
  for (int g = 0; g < NVG; ++g) {
    zsum[g] += __shfl_xor_sync(0xffffffffu, zsum[g], 4);
    zsum[g] += __shfl_xor_sync(0xffffffffu, zsum[g], 8);
    zsum[g] += __shfl_xor_sync(0xffffffffu, zsum[g], 16);
  }
  if (failed) {
    m_run = -INFINITY;
    l_run = 0.0f;
  }
  __syncthreads();   // every warp is done with the stages: reuse them for the merge
  float* sm_o = reinterpret_cast<float*>(stages);                    // [kWarps][NREP][kDV]
  float* sm_ml = sm_o + kWarps * NREP * kDV;                         // [kWarps][NREP][2]
  if (cvalid) {
    float* dst = sm_o + (warp * NREP + qi) * kDV;
#pragma unroll
    for (int mv = 0; mv < 8; ++mv) {
      float o0 = co[mv][0] + co[mv][1];
      float o1 = co[mv][2] + co[mv][3];
      int c0, c1;
      if (quant) {
        // channel tile mv = group gg, tile ml: rows qr, qr + 8 hold fields ml, ml + MPG of the
        // lane's run, at offsets (b * field) mod 8 in their bytes
        const int gg = mv / MPG, ml = mv % MPG;
        const int vb = MAP::kFixed ? MAP::vwidth(gg * GV) : plan.vbits[gg];
        c0 = gg * GV + qr * CPG + ml;
        c1 = c0 + MPG;
        o0 = fmaf(o0, __int_as_float((127 + 24 - ((vb * ml) & 7)) << 23), zsum[gg]);
        o1 = fmaf(o1, __int_as_float((127 + 24 - ((vb * (ml + MPG)) & 7)) << 23), zsum[gg]);
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


template <int NREP, int GV, int GK, class M = RuntimeMap>
cudaError_t launch_var(const Dims& d, const CacheBufs& c, const DecodeWork& w, const VarPlan& vp,
                       const __half* q, const Partials& p, cudaStream_t s) {
  auto kern = decode_var_kernel<NREP, GV, GK, M>;
  constexpr int smem = kSmemPerCta;
  static bool configured = false;
  if (!configured) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(w.splits, d.Hkv, d.B);
  kern<<<grid, kThreads, smem, s>>>(d, c, w, vp, q, p);
  return cudaGetLastError();
}

}  // namespace var
}  // namespace kvq
