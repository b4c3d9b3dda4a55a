// Tensor-core decode attention over caches with per-channel bit widths
// ("Attention-Aware Transform Coding (AATC)", §Méthodologie, Allocation de Bits: each
// transformed channel gets its own number of bits, zero for the weakest).
//
// Same flash-decoding split-K structure as the fixed-width kernel (one CTA per (split, kv
// head, sequence), four warps, a CTA-wide ring of bulk-copy stages, a partial (m, l, o) per
// query head and split), but the codes of a 16-token tile are first expanded in shared
// memory: every packed word of width b yields 16/b registers, each the pair of fields at
// bits (8j + p, 8j + p + 16) masked in place, i.e. two codes as fp16 subnormals with value
// code * 2^(p-24).  Register m of a row is stored at fp16 slots (2m, 2m+1), so a tile is a
// [16 tokens][slots] fp16 matrix that ldmatrix feeds to m16n8k16 MMAs:
//   scores: A = key slots, B = (q_c * s_c * 2^(8-p)) split into (hi, lo) fp16 halves
//           (columns 2h, 2h+1 of head h), score = (C_hi + C_lo) * 2^16 + sum_c z_c q_c;
//   p.V:    A = value slots (transposed), B = (p_t * s_{t,g}) split (hi, lo), per value
//           group g; o_c = C * 2^(24-p) + sum_t p_t z_{t,g}.
// Dropped channels (width 0) have no slot and read 0.  fp16 rows (retained tokens and the
// window) use the same tile core with the rows copied in as they are (slot = channel).
//
// Shape limits of this kernel (others run on the generic kernel): d_k = d_v = 128, 1 or 4
// query heads per kv head, value groups of >= 16 channels (>= 32 for 1-bit groups), and the
// channels of each width filling whole 32-bit words.  The map is read at run time from the
// slot tables; a map listed at build time (MapSpec) gets an instance whose expansion loops
// are unrolled and whose value-group tables are constants.
#include <string.h>

#include "../../include/kvq.h"
#include "kvq_internal.cuh"
#include "ptx.cuh"

namespace kvq {
namespace var {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kDK = 128, kDV = 128;
constexpr int kMaxRing = 8;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kLazyRescale = 8.0f;
constexpr int kCtasPerSm = 3;
constexpr int kSmemPerCta = 233472 / kCtasPerSm - 1024;
constexpr int KST = kDK * 2 + 16;         // padded tile row strides (bytes)
constexpr int VST = kDV * 2 + 16;
constexpr int kTileBytes = 16 * (KST > VST ? KST : VST);

// The slot tables of a width map (a kernel parameter; built on the host by make_map).
struct VarMap {
  int kslots, vslots;               // slots in use (coded channels)
  unsigned char kch[256], kp[256];        // per key slot: channel, field position p
  unsigned char vch[128], vp[128];        // per value slot: channel, field position p
  signed char vgroup[8];                  // value group of slot tile mv (-1: unused)
  signed char vhead[8];                   // first slot tile of the group of tile mv
  int kwb[5], vwb[5];                     // words of width 8 >> i: [wb[i], wb[i + 1])
  int kmb[4], vmb[4];                     // their first register (slot pair)
  int vtiles;                             // slot tiles of 16 in use
};

// Shared-memory layout of one CTA.
struct Smem {
  static constexpr int kBars = 0;                       // kMaxRing mbarriers
  static constexpr int kIssued = kBars + kMaxRing * 8;
  static constexpr int kTag = kIssued + kMaxRing * 4;
  static constexpr int kFail = kTag + kMaxRing * 4;
  static constexpr int kKCh = 256;                      // VarMap slot tables, copied in
  static constexpr int kKP = kKCh + 256;
  static constexpr int kVCh = kKP + 256;
  static constexpr int kVP = kVCh + 128;
  static constexpr int kQ = kVP + 128;                  // q * score_scale, fp32 [4][128], channel order
  static constexpr int kQS = kQ + 4 * kDK * 4;          // the same in slot order, times 2^(8-p)
  static constexpr int kTiles = kQS + 4 * kDK * 4;      // per warp: one expanded tile
  static constexpr int kStages = kTiles + kWarps * kTileBytes;
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

// The 16/B registers of one packed word of width B: register (j, p) = (x >> 8j) & (field
// mask at bit p of both halves), j-major, p = 0, B, ..., 8 - B.
template <int B>
__device__ __forceinline__ void expand_word(uint32_t x, uint32_t (&r)[16 / B]) {
  const uint32_t u = x >> 8;
#pragma unroll
  for (int p = 0; p < 8; p += B) {
    r[p / B] = x & ((((1u << B) - 1u) << p) * 0x00010001u);
    r[8 / B + p / B] = u & ((((1u << B) - 1u) << p) * 0x00010001u);
  }
}

// Expands the words [w0, w1) of width B of one packed row into the tile row: word w0 + i
// goes to registers m0 + i * 16/B (64-bit stores).  The two half-warps take alternate words.
template <int B>
__device__ __forceinline__ void expand_class(const uint32_t* rowp, uint32_t* trow, int w0, int w1,
                                             int m0, int ehalf) {
  constexpr int R = 16 / B;
#pragma unroll 2
  for (int wd = w0 + ehalf; wd < w1; wd += 2) {
    uint32_t r[R];
    expand_word<B>(rowp[wd], r);
    uint2* dst = reinterpret_cast<uint2*>(trow + m0 + (wd - w0) * R);
#pragma unroll
    for (int i = 0; i < R; i += 2) dst[i / 2] = make_uint2(r[i], r[i + 1]);
  }
}

// The class boundaries come as values (indexing the kernel's parameter arrays through a
// reference would copy them to local memory).
__device__ __forceinline__ void expand_row(const uint32_t* rowp, uint32_t* trow, int w1, int w2,
                                           int w3, int w4, int m1, int m2, int m3, int ehalf) {
  expand_class<8>(rowp, trow, 0, w1, 0, ehalf);
  expand_class<4>(rowp, trow, w1, w2, m1, ehalf);
  expand_class<2>(rowp, trow, w2, w3, m2, ehalf);
  expand_class<1>(rowp, trow, w3, w4, m3, ehalf);
}

// A width map fixed at build time: channel counts of widths 8, 4, 2, 1 for keys (K*) and
// values (V*), and the value group size.  K8 < 0 means "taken from the VarMap at run time".
template <int K8_, int K4_, int K2_, int K1_, int V8_, int V4_, int V2_, int V1_, int GV_>
struct MapSpec {
  static constexpr bool kFixed = K8_ >= 0;
  static constexpr int K8 = K8_, K4 = K4_, K2 = K2_, K1 = K1_;
  static constexpr int V8 = V8_, V4 = V4_, V2 = V2_, V1 = V1_, GV = GV_;
};
using RuntimeMap = MapSpec<-1, 0, 0, 0, 0, 0, 0, 0, 0>;

// Words [W0, W1) of width B at register M0, with every bound a compile-time constant: the
// half-warp ehalf takes words W0 + ehalf, W0 + ehalf + 2, ...
template <int B, int W0, int W1, int M0>
__device__ __forceinline__ void expand_class_fixed(const uint32_t* rowp, uint32_t* trow, int ehalf) {
  constexpr int R = 16 / B, N = W1 - W0;
#pragma unroll
  for (int i = 0; i < (N + 1) / 2; ++i) {
    if (N % 2 == 0 || 2 * i + ehalf < N) {
      uint32_t r[R];
      expand_word<B>(rowp[W0 + 2 * i + ehalf], r);
      uint2* dst = reinterpret_cast<uint2*>(trow + M0 + (2 * i + ehalf) * R);
#pragma unroll
      for (int k = 0; k < R; k += 2) dst[k / 2] = make_uint2(r[k], r[k + 1]);
    }
  }
}

template <int C8, int C4, int C2, int C1>
__device__ __forceinline__ void expand_row_fixed(const uint32_t* rowp, uint32_t* trow, int ehalf) {
  constexpr int N8 = C8 / 4, N4 = C4 / 8, N2 = C2 / 16, N1 = C1 / 32;      // words per class
  expand_class_fixed<8, 0, N8, 0>(rowp, trow, ehalf);
  expand_class_fixed<4, N8, N8 + N4, 2 * N8>(rowp, trow, ehalf);
  expand_class_fixed<2, N8 + N4, N8 + N4 + N2, 2 * N8 + 4 * N4>(rowp, trow, ehalf);
  expand_class_fixed<1, N8 + N4 + N2, N8 + N4 + N2 + N1, 2 * N8 + 4 * N4 + 8 * N2>(rowp, trow, ehalf);
}

// Channel of slot s of a fixed map (the order expand_word produces; -1 past the used slots).
__host__ __device__ constexpr int fixed_slot_channel(int s, int c8, int c4, int c2, int c1) {
  const int cnt[4] = {c8, c4, c2, c1};
  int m = s / 2, hi = s % 2, c = 0, pairs = 0;
  for (int i = 0; i < 4; ++i) {
    const int b = 8 >> i, words = cnt[i] * b / 32, regs = 16 / b;
    if (m < pairs + words * regs) {
      const int k = (m - pairs) / regs, r = (m - pairs) % regs;
      const int j = r / (8 / b), p = (r % (8 / b)) * b;
      return c + k * (32 / b) + (8 * j + p + 16 * hi) / b;
    }
    pairs += words * regs;
    c += cnt[i];
  }
  return -1;
}

// Value group of slot tile mv of a fixed map, and the first tile of that group (-1: unused).
template <class M>
__host__ __device__ constexpr int fixed_tile_group(int mv) {
  const int ch = fixed_slot_channel(16 * mv, M::V8, M::V4, M::V2, M::V1);
  return ch < 0 ? -1 : ch / M::GV;
}
template <class M>
__host__ __device__ constexpr int fixed_tile_head(int mv) {
  return fixed_tile_group<M>(mv) < 0 ? -1
         : (mv > 0 && fixed_tile_group<M>(mv - 1) == fixed_tile_group<M>(mv)) ? fixed_tile_head<M>(mv - 1)
                                                                              : mv;
}

// Value group and group-head tile of every slot tile of a fixed map, as one compile-time table.
struct TileTable {
  int group[8], head[8];
};
template <class M>
__host__ __device__ constexpr TileTable fixed_tile_table() {
  TileTable t{};
  for (int mv = 0; mv < 8; ++mv) {
    t.group[mv] = fixed_tile_group<M>(mv);
    t.head[mv] = t.group[mv] < 0 ? -1 : (mv > 0 && t.group[mv - 1] == t.group[mv]) ? t.head[mv - 1] : mv;
  }
  return t;
}

template <int NREP, class M = RuntimeMap>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
decode_var_kernel(Dims d, CacheBufs cb, DecodeWork w, VarMap vm, const __half* __restrict__ q,
                  Partials part) {
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
  unsigned char* kch = smem + Smem::kKCh;
  unsigned char* kp = smem + Smem::kKP;
  unsigned char* vch = smem + Smem::kVCh;
  unsigned char* vp = smem + Smem::kVP;
  float* sm_q = reinterpret_cast<float*>(smem + Smem::kQ);
  float* sm_qs = reinterpret_cast<float*>(smem + Smem::kQS);
  unsigned char* tile = smem + Smem::kTiles + warp * kTileBytes;
  const uint32_t tile_s = ptx::smem_addr(tile);
  unsigned char* stages = smem + Smem::kStages;
  const uint32_t stages_s = ptx::smem_addr(stages);

  const bool quant = split < w.splits_q;
  const StageLayout L = var_stage_layout(d);
  const int stage_bytes = quant ? round128(L.bytes) : round128(16 * (KST + VST));
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
  // the width map's tables; the query rows (times the score scale) in channel order
  for (int i = threadIdx.x; i < 256; i += kThreads) {
    kch[i] = vm.kch[i];
    kp[i] = vm.kp[i];
  }
  for (int i = threadIdx.x; i < 128; i += kThreads) {
    vch[i] = vm.vch[i];
    vp[i] = vm.vp[i];
  }
  const __half* qbase = q + (static_cast<size_t>(b) * d.Hq + h * NREP) * kDK;
  for (int i = threadIdx.x; i < 4 * kDK; i += kThreads)
    sm_q[i] = i < NREP * kDK ? __half2float(qbase[i]) * w.score_scale : 0.0f;
  // the expanded tiles start as zeros: slots no code is written to must hold finite values
  for (int i = threadIdx.x; i < kWarps * kTileBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + Smem::kTiles)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  // slot order (quantized CTAs: times 2^(8-p) for the subnormal codes and the 2^-16 range
  // factor; fp16 CTAs: slot = channel)
  for (int i = threadIdx.x; i < 4 * kDK; i += kThreads) {
    const int hh = i / kDK, sl = i % kDK;
    float x = 0.0f;
    if (quant) {
      if (sl < vm.kslots) x = sm_q[hh * kDK + kch[sl]] * __int_as_float((127 + 8 - kp[sl]) << 23);
    } else {
      x = sm_q[i];
    }
    sm_qs[i] = x;
  }

  // ---------------- work list ----------------
  const SeqWork sw = seq_work(w, b, d.gk, d.log_retain);
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
  const int gk = d.gk;

  // one lane copies unit k into stage k % ring: a key group (four runs), or up to 16 fp16
  // key and value rows
  auto issue = [&](int k) {
    const int st = k % ring;
    const uint32_t bar = bar0 + 8 * st;
    const uint32_t dst = stages_s + st * stage_bytes;
    if (quant) {
      const int g = unit_begin + k;
      sm_issued[st] += 1;
      sm_tag[st] = k;
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

  // retained positions, one per lane (ascending), for masking the quantized tiles
  const int ret_pos = quant && lane < sw.n_ret ? retained_position(sw.Q, lane) : -1;

  // B operands of the scores for fp16 units (q itself), fixed for the CTA
  uint32_t bq[8][2];
  auto build_bq = [&](const __half2* kmeta) {
#pragma unroll
    for (int s = 0; s < 8; ++s)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int sl = 16 * s + 2 * qi + 8 * j;
        float x0 = 0.0f, x1 = 0.0f;
        if (bvalid) {
          const float2 qq = *reinterpret_cast<const float2*>(sm_qs + bhead * kDK + sl);
          x0 = qq.x;
          x1 = qq.y;
          if (kmeta) {
            x0 *= __low2float(kmeta[kch[sl]]);
            x1 *= __low2float(kmeta[kch[sl + 1]]);
          }
        }
        const uint32_t s0 = ptx::split_hi_lo_trunc(x0), s1 = ptx::split_hi_lo_trunc(x1);
        // (hi, lo) of each: keep this column's half of both
        bq[s][j] = blo ? ptx::prmt(s0, s1, 0x7632u) : ptx::prmt(s0, s1, 0x5410u);
      }
  };
  if (!quant) build_bq(nullptr);

  float m_run = -INFINITY, l_run = 0.0f;
  float zsum[8];                 // sum_t p_t z_{t,g}, lane-partial, under the group's first tile
#pragma unroll
  for (int g = 0; g < 8; ++g) zsum[g] = 0.0f;
  float co[8][4];
#pragma unroll
  for (int mv = 0; mv < 8; ++mv)
#pragma unroll
    for (int e = 0; e < 4; ++e) co[mv][e] = 0.0f;
  bool failed = false;
  const int mi = lane >> 3;                 // which 8x8 matrix this lane addresses in ldmatrix
  const int arow = (mi & 1) * 8 + (lane & 7);
  const int vrow = (mi >> 1) * 8 + (lane & 7);
  const int erow = lane & 15, ehalf = lane >> 4;      // expansion: row, word parity

  for (int k = warp; k < n_units; k += kWarps) {
    const int st = k % ring;
    const bool ok = ptx::wait_equal_bounded(sm_tag + st, k, kWaitLimitNs) &&
                    ptx::mbar_wait_bounded(bar0 + 8 * st, (k / ring) & 1, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) {
      failed = true;
      break;
    }
    unsigned char* S = stages + st * stage_bytes;
    const uint32_t S_s = stages_s + st * stage_bytes;
    float kbias = 0.0f;                 // sum_c z_c q_c of head qi (quantized units)
    uint32_t rm0 = 0u, rm1 = 0u, rm2 = 0u, rm3 = 0u;   // retained rows of the group (up to 128)
    int n_tiles, nvalid_last = 16;
    if (quant) {
      const __half2* kmeta = reinterpret_cast<const __half2*>(S + L.kmeta_off);
      build_bq(kmeta);
      // key zero-point bias of each head: lanes over channels, then a warp sum
      float zb[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int i = 0; i < kDK / 32; ++i) {
        const int c = lane + 32 * i;
        const float z = __high2float(kmeta[c]);
#pragma unroll
        for (int hh = 0; hh < NREP; ++hh) zb[hh] = fmaf(z, sm_q[hh * kDK + c], zb[hh]);
      }
#pragma unroll
      for (int hh = 0; hh < NREP; ++hh)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) zb[hh] += __shfl_xor_sync(0xffffffffu, zb[hh], off);
      kbias = qi == 0 ? zb[0] : qi == 1 ? zb[1] : qi == 2 ? zb[2] : zb[3];
      const int g0 = (unit_begin + k) * gk;
      unsigned hits = __ballot_sync(0xffffffffu, ret_pos >= g0 && ret_pos < g0 + gk);
      while (hits) {
        const int src = __ffs(hits) - 1;
        hits &= hits - 1;
        const int off = __shfl_sync(0xffffffffu, ret_pos, src) - g0;
        const uint32_t bit = 1u << (off & 31);
        const int wsel = off >> 5;
        rm0 |= wsel == 0 ? bit : 0u;
        rm1 |= wsel == 1 ? bit : 0u;
        rm2 |= wsel == 2 ? bit : 0u;
        rm3 |= wsel == 3 ? bit : 0u;
      }
      n_tiles = gk / 16;
    } else {
      n_tiles = 1;
      nvalid_last = min(16, list_end - (list_begin + 16 * k));
    }

    for (int t = 0; t < n_tiles; ++t) {
      uint32_t KT, VT;     // shared addresses of the key and value tiles
      if (quant) {
        // expand the 16 key rows of the tile: lane = (row, word parity)
        const uint32_t* rowp = reinterpret_cast<const uint32_t*>(S + L.k_off) + (16 * t + erow) * d.kw;
        if constexpr (M::kFixed)
          expand_row_fixed<M::K8, M::K4, M::K2, M::K1>(rowp, reinterpret_cast<uint32_t*>(tile + erow * KST), ehalf);
        else
          expand_row(rowp, reinterpret_cast<uint32_t*>(tile + erow * KST), vm.kwb[1], vm.kwb[2], vm.kwb[3],
                     vm.kwb[4], vm.kmb[1], vm.kmb[2], vm.kmb[3], ehalf);
        __syncwarp();
        KT = tile_s;
      } else {
        KT = S_s;
      }
      // scores: C rows = tokens (qr, qr + 8), columns (2qi, 2qi + 1) = head qi (hi, lo)
      float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t a0, a1, a2, a3;
        ptx::ldmatrix_x4(KT + arow * KST + (16 * s + (mi >> 1) * 8) * 2, a0, a1, a2, a3);
        ptx::mma_16816(cs, a0, a1, a2, a3, bq[s][0], bq[s][1]);
      }
      float s0, s1;
      if (quant) {
        s0 = fmaf(cs[0] + cs[1], 65536.0f, kbias);
        s1 = fmaf(cs[2] + cs[3], 65536.0f, kbias);
        // rows 16t + qr and 16t + qr + 8 lie in word t / 2 of the mask, half t % 2
        const uint32_t mw = (t >> 1) == 0 ? rm0 : (t >> 1) == 1 ? rm1 : (t >> 1) == 2 ? rm2 : rm3;
        const int r0 = 16 * (t & 1) + qr;
        if ((mw >> r0) & 1u) s0 = -INFINITY;
        if ((mw >> (r0 + 8)) & 1u) s1 = -INFINITY;
      } else {
        s0 = cs[0] + cs[1];
        s1 = cs[2] + cs[3];
        if (qr >= nvalid_last) s0 = -INFINITY;
        if (qr + 8 >= nvalid_last) s1 = -INFINITY;
      }
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
#pragma unroll
        for (int g = 0; g < 8; ++g) zsum[g] *= a;
        m_run = m_new;
      }
      const float m_use = m_run == -INFINITY ? 0.0f : m_run;
      const float p0 = ptx::ex2(s0 - m_use);
      const float p1 = ptx::ex2(s1 - m_use);
      l_run += p0 + p1;

      if (quant) {
        // expand the 16 value rows into the same tile (the key slots are consumed)
        __syncwarp();
        const uint32_t* rowp = reinterpret_cast<const uint32_t*>(S + L.v_off) + (16 * t + erow) * d.vw;
        if constexpr (M::kFixed)
          expand_row_fixed<M::V8, M::V4, M::V2, M::V1>(rowp, reinterpret_cast<uint32_t*>(tile + erow * VST), ehalf);
        else
          expand_row(rowp, reinterpret_cast<uint32_t*>(tile + erow * VST), vm.vwb[1], vm.vwb[2], vm.vwb[3],
                     vm.vwb[4], vm.vmb[1], vm.vmb[2], vm.vmb[3], ehalf);
        __syncwarp();
        VT = tile_s;
      } else {
        VT = S_s + 16 * KST;
      }
      // p.V: A = V^T tiles of 16 slots via ldmatrix.trans, B = p (times the value group's
      // scale of each token), one (hi, lo) pair per token transposed by movmatrix
      const __half2* vmeta = quant ? reinterpret_cast<const __half2*>(S + L.vmeta_off) : nullptr;
      uint32_t bp0 = 0u, bp1 = 0u;
#pragma unroll
      for (int mv = 0; mv < 8; ++mv) {
        int head, g;
        if constexpr (M::kFixed) {
          constexpr TileTable tt = fixed_tile_table<M>();
          head = tt.head[mv];
          g = tt.group[mv];
        } else {
          head = vm.vhead[mv];
          g = vm.vgroup[mv];
        }
        if (quant && g < 0) break;
        float zz = 0.0f;
        if (quant ? head == mv : mv == 0) {      // the first tile of a value group
          float x0 = p0, x1 = p1;
          if (quant) {
            const float2 sz0 = __half22float2(vmeta[(16 * t + qr) * d.nvg + g]);
            const float2 sz1 = __half22float2(vmeta[(16 * t + qr + 8) * d.nvg + g]);
            x0 *= sz0.x;
            x1 *= sz1.x;
            zz = fmaf(p0, sz0.y, p1 * sz1.y);
          }
          bp0 = ptx::movmatrix_trans(ptx::split_hi_lo_trunc(x0));
          bp1 = ptx::movmatrix_trans(ptx::split_hi_lo_trunc(x1));
        }
        zsum[mv] += zz;          // a group's sum is kept under its first tile
        uint32_t a0, a1, a2, a3;
        ptx::ldmatrix_x4_trans(VT + vrow * VST + (16 * mv + (mi & 1) * 8) * 2, a0, a1, a2, a3);
        ptx::mma_16816(co[mv], a0, a1, a2, a3, bp0, bp1);
      }
      __syncwarp();        // the tile is read before the next expansion overwrites it
    }

    if (k + ring < n_units) {
      if (quant) {
        if (lane == 0) {
          ptx::fence_proxy_async_smem();
          issue(k + ring);
        }
      } else {
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
  for (int g = 0; g < 8; ++g) {
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
  for (int i = threadIdx.x; i < kWarps * NREP * kDV; i += kThreads) sm_o[i] = 0.0f;   // dropped channels
  __syncthreads();
  if (cvalid) {
    float* dst = sm_o + (warp * NREP + qi) * kDV;
#pragma unroll
    for (int mv = 0; mv < 8; ++mv) {
      float o0 = co[mv][0] + co[mv][1];
      float o1 = co[mv][2] + co[mv][3];
      const int sl0 = 16 * mv + qr, sl1 = sl0 + 8;
      int c0 = sl0, c1 = sl1;
      bool w0 = true, w1 = true;
      if (quant) {
        w0 = mv < vm.vtiles && sl0 < vm.vslots;
        w1 = mv < vm.vtiles && sl1 < vm.vslots;
        // a group's tiles are consecutive: carry the first tile's sum forward
        if (vm.vhead[mv] != mv && mv > 0) zsum[mv] = zsum[mv > 0 ? mv - 1 : 0];
        const float zg = zsum[mv];
        if (w0) {
          c0 = vch[sl0];
          o0 = fmaf(o0, __int_as_float((127 + 24 - vp[sl0]) << 23), zg);
        }
        if (w1) {
          c1 = vch[sl1];
          o1 = fmaf(o1, __int_as_float((127 + 24 - vp[sl1]) << 23), zg);
        }
      }
      if (failed) o0 = o1 = 0.0f;
      if (w0) dst[c0] = o0;
      if (w1) dst[c1] = o1;
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

// Slots of one width map: words in row order, each word's registers (j, p) in the order
// expand_word stores them; channels of register (j, p) of a word starting at channel c0 of
// width b: c0 + (8j + p) / b (low half) and c0 + (8j + p + 16) / b (high half).
bool build_slots(const int* cnt, unsigned char* ch, unsigned char* fp, int* nslots, int* wb, int* mb) {
  int c = 0, wd = 0, m = 0;
  for (int i = 0; i < 4; ++i) {
    const int bw = 8 >> i;
    if ((cnt[i] * bw) % 32 != 0) return false;          // a word would mix widths
    const int words = cnt[i] * bw / 32;
    wb[i] = wd;
    mb[i] = m;
    for (int k = 0; k < words; ++k) {
      if (wd >= 64) return false;
      const int c0 = c + k * (32 / bw);
      for (int j = 0; j < 2; ++j)
        for (int p = 0; p < 8; p += bw) {
          ch[2 * m] = static_cast<unsigned char>(c0 + (8 * j + p) / bw);
          ch[2 * m + 1] = static_cast<unsigned char>(c0 + (8 * j + p + 16) / bw);
          fp[2 * m] = fp[2 * m + 1] = static_cast<unsigned char>(p);
          ++m;
        }
      ++wd;
    }
    c += cnt[i];
  }
  wb[4] = wd;
  *nslots = 2 * m;
  return true;
}

bool make_map(const Dims& d, VarMap* vm) {
  memset(vm, 0, sizeof(*vm));
  if (!build_slots(d.kcnt, vm->kch, vm->kp, &vm->kslots, vm->kwb, vm->kmb)) return false;
  if (!build_slots(d.vcnt, vm->vch, vm->vp, &vm->vslots, vm->vwb, vm->vmb)) return false;
  if (vm->kslots > kDK || vm->vslots > kDV) return false;
  // every tile of 16 value slots must lie in one value group
  vm->vtiles = (vm->vslots + 15) / 16;
  for (int mv = 0; mv < 8; ++mv) {
    vm->vgroup[mv] = -1;
    vm->vhead[mv] = -1;
    for (int sl = 16 * mv; sl < 16 * mv + 16 && sl < vm->vslots; ++sl) {
      const int g = vm->vch[sl] / d.gv;
      if (vm->vgroup[mv] < 0) vm->vgroup[mv] = static_cast<signed char>(g);
      else if (vm->vgroup[mv] != g) return false;
    }
    if (mv < vm->vtiles)
      vm->vhead[mv] = (mv > 0 && vm->vgroup[mv - 1] == vm->vgroup[mv]) ? vm->vhead[mv - 1]
                                                                         : static_cast<signed char>(mv);
  }
  // a group's tiles are consecutive (slots follow the channel order)
  for (int mv = 1; mv < vm->vtiles; ++mv)
    if (vm->vgroup[mv] < vm->vgroup[mv - 1]) return false;
  return true;
}

}  // namespace

bool supported(const Dims& d) {
  if (!d.var || d.dk != kDK || d.dv != kDV || (d.n_rep != 1 && d.n_rep != 4) || d.gv < 16 || d.nvg > 8)
    return false;
  VarMap vm;
  if (!make_map(d, &vm)) return false;
  const int stage = round128(var_stage_layout(d).bytes);
  return (kSmemPerCta - Smem::kStages) / stage >= 1 && kWarps * 4 * kDV * 4 + 256 <= kSmemPerCta - Smem::kStages;
}

namespace {

// Maps with a build-time instance: keys 16 x 8, 64 x 4, 32 x 2 bits (+ 16 dropped), values in
// groups of 32 channels at 4, 2, 2, 1 bits.
using MapK3V2 = MapSpec<16, 64, 32, 0, 0, 32, 64, 32, 32>;

// The instance's compile-time tables must be those of the run-time map.
template <class M>
bool fixed_map_matches(const Dims& d, const VarMap& vm) {
  const int k[4] = {M::K8, M::K4, M::K2, M::K1}, v[4] = {M::V8, M::V4, M::V2, M::V1};
  for (int i = 0; i < 4; ++i)
    if (d.kcnt[i] != k[i] || d.vcnt[i] != v[i]) return false;
  if (d.gv != M::GV) return false;
  for (int sl = 0; sl < vm.kslots; ++sl)
    if (fixed_slot_channel(sl, M::K8, M::K4, M::K2, M::K1) != vm.kch[sl]) return false;
  for (int sl = 0; sl < vm.vslots; ++sl)
    if (fixed_slot_channel(sl, M::V8, M::V4, M::V2, M::V1) != vm.vch[sl]) return false;
  for (int mv = 0; mv < 8; ++mv)
    if (fixed_tile_group<M>(mv) != vm.vgroup[mv] || fixed_tile_head<M>(mv) != vm.vhead[mv]) return false;
  return true;
}

}  // namespace

cudaError_t launch(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                   const Partials& p, cudaStream_t s) {
  VarMap vm;
  if (!supported(d) || !make_map(d, &vm)) return cudaErrorNotSupported;
  void (*kern)(Dims, CacheBufs, DecodeWork, VarMap, const __half*, Partials);
  int which;
  if (fixed_map_matches<MapK3V2>(d, vm)) {
    kern = d.n_rep == 4 ? decode_var_kernel<4, MapK3V2> : decode_var_kernel<1, MapK3V2>;
    which = d.n_rep == 4 ? 2 : 3;
  } else {
    kern = d.n_rep == 4 ? decode_var_kernel<4> : decode_var_kernel<1>;
    which = d.n_rep == 4 ? 0 : 1;
  }
  static bool configured[4] = {false, false, false, false};
  if (!configured[which]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerCta);
    if (e != cudaSuccess) return e;
    configured[which] = true;
  }
  dim3 grid(w.splits, d.Hkv, d.B);
  kern<<<grid, kThreads, kSmemPerCta, s>>>(d, c, w, vm, q, p);
  return cudaGetLastError();
}

}  // namespace var

bool decode_var_supported(const Dims& d) { return var::supported(d); }

cudaError_t launch_decode_var(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                              const Partials& p, cudaStream_t s) {
  return var::launch(d, c, w, q, p, s);
}

}  // namespace kvq
