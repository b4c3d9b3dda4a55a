// Write path of the cache: groupwise min-max quantize-and-pack, window and
// retained-token copies.
//
// Quantizer (asymmetric uniform min-max with an fp16 scale and zero per group;
// the form is this library's reading of the groupwise quantizers named in
// "Quantize What Counts: More for Keys, Less for Values", §Méthodologie, and
// "LogQuant: Log-Distributed 2-Bit Quantization of KV Cache", §5):
//   s = fp16(fl32(max - min) / (2^b - 1))  (+0 when zero),  z = fp16(min + 0)
//   code = s == 0 ? 0 : clamp(rint(fl32(fl32(x - z) / s)), 0, 2^b - 1)
// Every step is an explicit IEEE round-to-nearest intrinsic so that no FMA
// contraction or fast-math rewrite can change a code.  Keys: one group per
// channel over group_k consecutive tokens (LogQuant §5, per-channel keys); a group's
// (scale, zero) block is stored in the order the decode kernel pairs channels.
// Values: one group per token over group_v consecutive channels.
#include <type_traits>

#include "kvq_internal.cuh"
#include "ptx.cuh"

namespace kvq {
namespace {

// Shared-memory tables of the key quantizer: (zero, 1/scale, scale) per (group of a CTA,
// channel) and the groups' (scale, zero) blocks; a CTA holds at most 2048 / gk * R channels'
// parameters (512 for gk = 16 with 4 rows per thread).
constexpr int kKeyPrm = 512;
constexpr int kKeyBlk = 2 * kKeyPrm;

struct GroupParams {
  float scale;   // fp32 value of the fp16 scale
  float zero;    // fp32 value of the fp16 zero
  __half2 sz;    // (scale, zero) as stored
};

__device__ __forceinline__ GroupParams group_params_b(float mn, float mx, int bits) {
  const float levels = static_cast<float>((1 << bits) - 1);
  const float s32 = __fdiv_rn(__fsub_rn(mx, mn), levels);
  __half s16 = __float2half_rn(s32);
  if (__half2float(s16) == 0.0f) s16 = __ushort_as_half(0);          // canonical +0
  const __half z16 = __float2half_rn(__fadd_rn(mn, 0.0f));            // exact, -0 -> +0
  GroupParams g;
  g.scale = __half2float(s16);
  g.zero = __half2float(z16);
  g.sz = __halves2half2(s16, z16);
  return g;
}

__device__ __forceinline__ uint32_t quant_code_b(float x, const GroupParams& g, int bits) {
  if (g.scale == 0.0f) return 0u;
  const float levels = static_cast<float>((1 << bits) - 1);
  float c = rintf(__fdiv_rn(__fsub_rn(x, g.zero), g.scale));          // half-to-even
  c = fminf(fmaxf(c, 0.0f), levels);
  return static_cast<uint32_t>(c);
}

template <int BITS>
__device__ __forceinline__ GroupParams group_params(float mn, float mx) { return group_params_b(mn, mx, BITS); }

template <int BITS>
__device__ __forceinline__ uint32_t quant_code(float x, const GroupParams& g) { return quant_code_b(x, g, BITS); }

// The code of one element from the group's zero z and the reciprocal r = fl32(1/s) of its
// scale, equal to the quantizer's clamp(rint(fl32(fl32(x - z) / s)), 0, 2^b - 1) wherever
// `near` stays false:
//   with d = fl32(x - z) >= 0, the exact quotient Q = d/s is below 512 (s is the fp16 rounding
//   of (max - min)/(2^b - 1) with b <= 8, or a subnormal at most 1.5x smaller; s = 0 gives
//   r = 0 and code 0).  P = d * r = Q (1 + e), |e| <= 2^-24, so |P - Q| < 2^-15, and the IEEE
//   quotient F = fl32(Q) is within half an ulp, 2^-16, of Q.  y = fma(d, r, 1.5 * 2^23) rounds
//   the exact P to the nearest integer c (ties to even: spacing 1 at that magnitude, and the
//   constant is even), c = y - 1.5 * 2^23 exactly, and t = fma(d, r, -c) is P - c up to 2^-25.
//   If |t| <= 1/2 - 2^-13 then |F - c| < 1/2 - 2^-14, so rint(F) = c; otherwise `near` is set
//   and the caller takes the IEEE division.  No float-to-integer conversion is needed: the
//   integer c is the low bits of y.
constexpr float kNearHalf = 0.5f - 1.0f / 8192.0f;
constexpr float kRoundMagic = 12582912.0f;         // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

__device__ __forceinline__ uint32_t code_fast_l(float x, float z, float r, uint32_t levels, bool& near) {
  const float d = __fsub_rn(x, z);
  const float y = __fmaf_rn(d, r, kRoundMagic);
  const float c = __fsub_rn(y, kRoundMagic);
  near |= fabsf(__fmaf_rn(d, r, -c)) > kNearHalf;
  return min(__float_as_uint(y) - kRoundMagicBits, levels);
}

// The quantizer's code with the IEEE division (the rare elements code_fast leaves undecided).
__device__ __forceinline__ uint32_t code_exact_l(float x, float z, float s, uint32_t levels) {
  if (s == 0.0f) return 0u;
  float c = rintf(__fdiv_rn(__fsub_rn(x, z), s));
  c = fminf(fmaxf(c, 0.0f), static_cast<float>(levels));
  return static_cast<uint32_t>(c);
}

template <int BITS>
__device__ __forceinline__ uint32_t code_fast(float x, float z, float r, bool& near) {
  return code_fast_l(x, z, r, (1u << BITS) - 1u, near);
}

template <int BITS>
__device__ __forceinline__ uint32_t code_exact(float x, float z, float s) {
  return code_exact_l(x, z, s, (1u << BITS) - 1u);
}

// The packed codes of one 16-byte chunk: 8 * BITS bits (a 32-bit word below 8 bits).
template <int BITS>
using ChunkBits = typename std::conditional<(BITS == 8), uint64_t, uint32_t>::type;

// Codes of 8 consecutive channels (one 16-byte chunk of fp16) packed LSB-first: 8 * BITS bits.
// Channel j's group has zero z[j], reciprocal scale r[j] and scale sc[j] (keys: one group per
// channel), or every channel the same (values: STRIDE 0 reads element 0 for all j).
template <int BITS, int STRIDE>
__device__ __forceinline__ ChunkBits<BITS> pack_chunk(const uint4& raw, const float* z, const float* r,
                                                      const float* sc) {
  using W = ChunkBits<BITS>;
  const __half2* hx = reinterpret_cast<const __half2*>(&raw);
  float x[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(hx[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
  bool near = false;
  W bits = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    bits |= static_cast<W>(code_fast<BITS>(x[j], z[j * STRIDE], r[j * STRIDE], near)) << (j * BITS);
  if (near) {             // rare: a quotient within 2^-13 of a half-integer
    bits = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      bits |= static_cast<W>(code_exact<BITS>(x[j], z[j * STRIDE], sc[j * STRIDE])) << (j * BITS);
  }
  return bits;
}

// Stores a chunk's packed codes at chunk index `idx` of a row array of (8 * BITS)-bit units.
template <int BITS>
__device__ __forceinline__ void store_chunk(uint32_t* base, size_t idx, ChunkBits<BITS> bits) {
  if constexpr (BITS == 2)
    reinterpret_cast<uint16_t*>(base)[idx] = static_cast<uint16_t>(bits);
  else if constexpr (BITS == 4)
    base[idx] = static_cast<uint32_t>(bits);
  else
    reinterpret_cast<uint2*>(base)[idx] = make_uint2(static_cast<uint32_t>(bits), static_cast<uint32_t>(bits >> 32));
}

__host__ __device__ constexpr int ilog2c(int x) { return x <= 1 ? 0 : 1 + ilog2c(x / 2); }

// The part of the key quantizer after a tile's chunks are in registers: thread (group gi of the
// CTA, slab rs, chunk cc) holds rows rs, rs + gk/R, ... of chunk cc of group g_begin + g_first + gi
// (of the launch's n_groups) of row bh = b * Hkv + h (sequence b, kv head h).  Per-channel min and max in fp16 (exact),
// reduced over the slabs in shared memory; (scale, zero) per channel, written as the groups'
// blocks; then the codes from the registers.  Every size here is a power of two, so the index
// arithmetic is shifts and masks.  Called by every thread of the CTA (barriers).
template <int BITS, int R>
__device__ __forceinline__ void key_tile(const uint4 (&x)[R], int bh, int g_begin, int g_first,
                                         int n_groups, uint32_t* __restrict__ kcode, __half2* __restrict__ ksz,
                                         const int* __restrict__ table, const Dims& d,
                                         __half2 (*red)[256][4], float (*prm)[kKeyPrm], __half* blk) {
  const int dk = d.dk;
  const int ldk = __ffs(dk) - 1, lcpr = ldk - 3, lslabs = __ffs(d.gk) - 1 - ilog2c(R);
  const int ltpg = lcpr + lslabs, slabs = 1 << lslabs, gpc = 256 >> ltpg;
  const int tid = threadIdx.x;
  const int gi = tid >> ltpg, lt = tid & ((1 << ltpg) - 1), cc = lt & ((1 << lcpr) - 1), rs = lt >> lcpr;
  const bool active = g_first + gi < n_groups;
  const int g = g_begin + g_first + gi;
  {
    const __half2* h0 = reinterpret_cast<const __half2*>(&x[0]);
    __half2 mn[4], mx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) mn[k] = mx[k] = h0[k];
#pragma unroll
    for (int i = 1; i < R; ++i) {
      const __half2* hi = reinterpret_cast<const __half2*>(&x[i]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mn[k] = __hmin2(mn[k], hi[k]);
        mx[k] = __hmax2(mx[k], hi[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      red[0][tid][k] = mn[k];
      red[1][tid][k] = mx[k];
    }
  }
  __syncthreads();
  // per (group of the CTA, channel pair): reduce over the slabs, then (scale, zero)
  constexpr int per_w = 32 / BITS, half_w = 16 / BITS;
  const int lwords = ldk - ilog2c(per_w);                  // words per key row, log2
  const int lquarter = lwords >= 2 ? lwords - 2 : -1;      // quarter-interleaved when 4 | words
  for (int p = tid; p < (gpc << (ldk - 1)); p += 256) {
    const int g2 = p >> (ldk - 1), pp = p & ((dk >> 1) - 1), c2 = pp >> 2, k = pp & 3;
    const int t0 = (g2 << ltpg) + c2;
    __half2 mn = red[0][t0][k], mx = red[1][t0][k];
    for (int sl = 1; sl < slabs; ++sl) {
      mn = __hmin2(mn, red[0][t0 + (sl << lcpr)][k]);
      mx = __hmax2(mx, red[1][t0 + (sl << lcpr)][k]);
    }
    const float2 fmn = __half22float2(mn), fmx = __half22float2(mx);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int c = 8 * c2 + 2 * k + e;
      const GroupParams gp = group_params<BITS>(e ? fmn.y : fmn.x, e ? fmx.y : fmx.x);
      prm[0][(g2 << ldk) + c] = gp.zero;
      prm[1][(g2 << ldk) + c] = gp.scale == 0.0f ? 0.0f : __frcp_rn(gp.scale);
      prm[2][(g2 << ldk) + c] = gp.scale;
      // the group's block of 2*dk fp16: per packed word w, the scales of channels
      // (w*per + i, w*per + i + per/2) for i < per/2, then their zeros in the same order;
      // the words' blocks quarter-interleaved when 4 divides the words per row
      const int wd = c / per_w, r = c % per_w;
      const int pos = lquarter >= 0 ? ((wd & ((1 << lquarter) - 1)) << 2) + (wd >> lquarter) : wd;
      const int slot = pos * 2 * per_w + (r % half_w) * 2 + r / half_w;
      blk[(g2 << (ldk + 1)) + slot] = __low2half(gp.sz);
      blk[(g2 << (ldk + 1)) + slot + per_w] = __high2half(gp.sz);
    }
  }
  __syncthreads();
  for (int i = tid; i < (gpc << (ldk - 2)); i += 256) {     // 16 B of a block per thread
    const int g2 = i >> (ldk - 2), j = i & ((dk >> 2) - 1);
    if (g_first + g2 >= n_groups) continue;
    const size_t gidx = group_index_bh(d, table, bh, g_begin + g_first + g2);
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteQKeyMeta, static_cast<long long>(gidx * 2 * dk) + 8 * j, 8,
                             quant_groups(d) * 2 * dk))
      continue;
    reinterpret_cast<uint4*>(reinterpret_cast<__half*>(ksz) + gidx * 2 * dk)[j] =
        reinterpret_cast<const uint4*>(blk + (g2 << (ldk + 1)))[j];
  }
  if (!active) return;   // (the caller's loop has no barrier after this call)
  float z[8], r[8], sc[8];
#pragma unroll
  for (int j = 0; j < 8; j += 4) {
    *reinterpret_cast<float4*>(z + j) = *reinterpret_cast<const float4*>(&prm[0][(gi << ldk) + 8 * cc + j]);
    *reinterpret_cast<float4*>(r + j) = *reinterpret_cast<const float4*>(&prm[1][(gi << ldk) + 8 * cc + j]);
    *reinterpret_cast<float4*>(sc + j) = *reinterpret_cast<const float4*>(&prm[2][(gi << ldk) + 8 * cc + j]);
  }
  const size_t row0 = group_row_bh(d, table, bh, g);
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const ChunkBits<BITS> bits = pack_chunk<BITS, 1>(x[i], z, r, sc);
    const size_t row = row0 + rs + slabs * i;
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteQKeyCode, static_cast<long long>(row * (dk * BITS / 8)) + cc * BITS, BITS,
                             quant_rows(d) * d.kw * 4))
      continue;
    store_chunk<BITS>(kcode, (row << lcpr) + cc, bits);
  }
}

template <int BITS, int R, bool ROT>
__global__ void __launch_bounds__(256) quantize_keys_kernel(
    const __half* __restrict__ src, int src_rows, int g_begin, int n_groups,
    uint32_t* __restrict__ kcode, __half2* __restrict__ ksz, const int* __restrict__ table, Dims d) {
  extern __shared__ __align__(16) unsigned char sm_dyn[];          // ROT: [gpc * gk][dk] fp16
  __shared__ __align__(16) __half2 red[2][256][4];                  // per thread: min, max
  __shared__ __align__(16) float prm[3][kKeyPrm];                   // zero, 1/scale, scale
  __shared__ __align__(16) __half blk[kKeyBlk];                     // (scale, zero) blocks
  const int dk = d.dk, gk = d.gk;
  const int cpr = dk / 8, slabs = gk / R, tpg = cpr * slabs, gpc = 256 / tpg;
  const int tid = threadIdx.x;
  const int gi = tid / tpg, lt = tid % tpg, cc = lt % cpr, rs = lt % tpg / cpr;
  const int bh = blockIdx.y;
  const int g_first = blockIdx.x * gpc;           // first group of the CTA, among the launch's
  const bool active = g_first + gi < n_groups;
  const int g = g_begin + g_first + gi;
  const size_t base = static_cast<size_t>(bh) * src_rows;
  [[maybe_unused]] const long long src_ext = static_cast<long long>(d.B) * d.Hkv * src_rows * dk;

  uint4 x[R];
  if constexpr (ROT) {
    __half* rot = reinterpret_cast<__half*>(sm_dyn);
    const int lane = tid & 31, warp = tid >> 5;
    for (int rr = warp; rr < gpc * gk; rr += 8) {
      const int yy = rr / gk, t = rr % gk;
      if (g_first + yy >= n_groups) continue;                     // uniform per warp
      const int row = ((g_begin + g_first + yy) * gk + t) % src_rows;
      float v[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const long long si = static_cast<long long>((base + row) * dk) + lane + 32 * m;
        v[m] = m < dk / 32 && KVQ_IN_BOUNDS(d, kSiteQKeySrc, si, src_ext) ? __half2float(src[si]) : 0.0f;
      }
      rotate_row_warp<8>(v, dk / 32, d.rot_signs, d.rot_inv_ck, lane);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (m < dk / 32) rot[static_cast<size_t>(rr) * dk + lane + 32 * m] = __float2half_rn(v[m]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < R; ++i)
      x[i] = reinterpret_cast<const uint4*>(rot)[(gi * gk + rs + slabs * i) * cpr + cc];
  } else {
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int tk = g * gk + rs + slabs * i;
      const int row = tk < src_rows ? tk : tk % src_rows;            // the window is a ring
      const long long si = static_cast<long long>((base + row) * dk) + 8 * cc;
      x[i] = active && KVQ_RANGE_IN_BOUNDS(d, kSiteQKeySrc, si, 8, src_ext)
                 ? __ldg(reinterpret_cast<const uint4*>(src + (base + row) * dk) + cc)
                 : make_uint4(0, 0, 0, 0);
    }
  }
  key_tile<BITS, R>(x, bh, g_begin, g_first, n_groups, kcode, ksz, table, d, red, prm, blk);
}

// Side code of key groups ("HeadQ: Distortion visible par le modele et correction dans
// l'espace des scores pour la quantification du cache KV", §3, Aperçu de l'algorithme,
// step 2): for every token of the group the base residual e = k - (code*s + z) of each
// channel, its projection y = U_h^T e on the kv head's basis (fp32, channels summed in
// ascending order, one rounded product and one rounded sum per channel), then the
// min-max quantizer above per coordinate over the group's tokens.  The base codes and
// (scale, zero) are read back from kcode / ksz, so both describe the same key.
// One CTA per (group, b * kv head).  Shared memory: e [gk][dk + 1] (padded so that the
// threads of a warp, which read one channel of several tokens, hit distinct banks),
// U_h [dk][sr] and y [gk][sr].
template <int SQ, bool ROT>
__global__ void quantize_side_kernel(const __half* __restrict__ src, int src_rows, int dk, int kb,
                                     int gk, int g_begin, int lcap, int hkv, int sr, int zb,
                                     const uint32_t* __restrict__ kcode,
                                     const __half2* __restrict__ ksz,
                                     const float* __restrict__ side_u,
                                     uint8_t* __restrict__ zcode, __half2* __restrict__ zsz,
                                     const int* __restrict__ table, Dims d) {
  extern __shared__ float sm_side[];
  __shared__ float2 params[8];
  const int es = dk + 1;
  float* e = sm_side;
  float* u = e + gk * es;
  float* y = u + dk * sr;
  const int g = g_begin + blockIdx.x;
  const int bh = blockIdx.y;
  const int h = bh % hkv;
  const size_t base = static_cast<size_t>(bh) * src_rows;
  const int per = 32 / kb, half = per / 2, words = dk / per;
  const int quarter = words % 4 == 0 ? words / 4 : 0;
  const size_t row0 = group_row(d, table, bh / hkv, h, g);
  const size_t gidx = group_index(d, table, bh / hkv, h, g);
  const __half* blk = reinterpret_cast<const __half*>(ksz) + gidx * 2 * dk;
  // the cached key of token t, channel c: the source key, or its rotation (ROT: rotated
  // by warps into e, then read back from there)
  if constexpr (ROT) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x / 32;
    for (int t = warp; t < gk; t += nwarps) {
      const int row = (g * gk + t) % src_rows;
      float x[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const long long si = static_cast<long long>((base + row) * dk) + lane + 32 * m;
        x[m] = m < dk / 32 && KVQ_IN_BOUNDS(d, kSiteSideSrc, si, static_cast<long long>(d.B) * hkv * src_rows * dk)
                   ? __half2float(src[si]) : 0.0f;
      }
      rotate_row_warp<8>(x, dk / 32, d.rot_signs, d.rot_inv_ck, lane);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (m < dk / 32) e[t * es + lane + 32 * m] = __half2float(__float2half_rn(x[m]));
    }
    __syncthreads();
  }
  // the residual e of every token, one channel per thread (dk, the words per row and the
  // (scale, zero) block's quarters are powers of two): the channel's (scale, zero), word and
  // field are fixed for the thread, its tokens step by blockDim / dk
  {
    const int ldk = __ffs(dk) - 1, lper = __ffs(per) - 1;
    const int c = threadIdx.x & (dk - 1);
    const int tstep = blockDim.x >> ldk;
    const int wd = c >> lper, r = c & (per - 1);
    const int pos = quarter ? (wd & (quarter - 1)) * 4 + (wd >> (__ffs(quarter) - 1)) : wd;
    const int slot = pos * 2 * per + (r & (half - 1)) * 2 + (r >> (__ffs(half) - 1));
    const bool meta_ok = KVQ_RANGE_IN_BOUNDS(d, kSiteSideMeta, static_cast<long long>(gidx * 2 * dk) + slot, per + 1,
                                             quant_groups(d) * 2 * dk);
    const float sc = meta_ok ? __half2float(blk[slot]) : 0.0f;
    const float zc = meta_ok ? __half2float(blk[slot + per]) : 0.0f;
    const int shift = r * kb;
    const uint32_t mask = (1u << kb) - 1u;
    auto residual = [&](int t, float x) {
      const long long ki = static_cast<long long>((row0 + t) * words) + wd;
      const uint32_t w = KVQ_IN_BOUNDS(d, kSiteSideCode, ki, quant_rows(d) * words) ? kcode[ki] : 0u;
      const uint32_t code = (w >> shift) & mask;
      const float kh = __fadd_rn(__fmul_rn(static_cast<float>(code), sc), zc);
      e[t * es + c] = __fsub_rn(x, kh);
    };
    int t = threadIdx.x >> ldk;
    if (ROT || static_cast<long long>(g + 1) * gk <= src_rows) {
      // the group's rows are contiguous in the source (a prefill): independent iterations, so
      // that the loads of several tokens are in flight together
#pragma unroll 8
      for (int tt = t; tt < gk; tt += tstep) {
        float x;
        if constexpr (ROT) {
          x = e[tt * es + c];
        } else {
          const long long si = static_cast<long long>((base + static_cast<long long>(g) * gk + tt) * dk) + c;
          x = KVQ_IN_BOUNDS(d, kSiteSideSrc, si, static_cast<long long>(d.B) * hkv * src_rows * dk)
                  ? __half2float(src[si]) : 0.0f;
        }
        residual(tt, x);
      }
      t = gk;
    }
    int row = static_cast<int>((static_cast<long long>(g) * gk + t) % src_rows);   // source row of token t
    for (; t < gk; t += tstep) {
      float x;
      if constexpr (ROT) {
        x = e[t * es + c];
      } else {
        const long long si = static_cast<long long>((base + row) * dk) + c;
        x = KVQ_IN_BOUNDS(d, kSiteSideSrc, si, static_cast<long long>(d.B) * hkv * src_rows * dk)
                ? __half2float(src[si]) : 0.0f;
      }
      residual(t, x);
      row += tstep;
      while (row >= src_rows) row -= src_rows;
    }
  }
  for (int idx = threadIdx.x; idx < dk * sr; idx += blockDim.x)
    u[idx] = KVQ_IN_BOUNDS(d, kSiteSideU, static_cast<long long>(h) * dk * sr + idx, static_cast<long long>(hkv) * dk * sr)
                 ? side_u[static_cast<size_t>(h) * dk * sr + idx] : 0.0f;
  __syncthreads();
  const int lsr = __ffs(sr) - 1;
  for (int idx = threadIdx.x; idx < gk * sr; idx += blockDim.x) {
    const int t = idx >> lsr, i = idx & (sr - 1);
    float acc = 0.0f;
#pragma unroll 8
    for (int c = 0; c < dk; ++c) acc = __fadd_rn(acc, __fmul_rn(e[t * es + c], u[c * sr + i]));
    y[idx] = acc;
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = warp; i < sr; i += blockDim.x / 32) {
    float mn = INFINITY, mx = -INFINITY;
    for (int t = lane; t < gk; t += 32) {
      mn = fminf(mn, y[t * sr + i]);
      mx = fmaxf(mx, y[t * sr + i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    if (lane == 0) {
      const GroupParams gp = group_params<SQ>(mn, mx);
      if (KVQ_IN_BOUNDS(d, kSiteSideZMeta, static_cast<long long>(gidx * sr) + i, quant_groups(d) * sr))
        zsz[gidx * sr + i] = gp.sz;
      params[i] = make_float2(gp.scale, gp.zero);
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < gk; t += blockDim.x) {
    uint32_t row = 0;
    for (int i = 0; i < sr; ++i) {
      GroupParams gp;
      gp.scale = params[i].x;
      gp.zero = params[i].y;
      row |= quant_code<SQ>(y[t * sr + i], gp) << (i * SQ);
    }
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteSideZCode, static_cast<long long>((row0 + t) * zb), zb, quant_rows(d) * zb))
      continue;
    uint8_t* dst = zcode + (row0 + t) * zb;
    if (zb == 4)
      *reinterpret_cast<uint32_t*>(dst) = row;
    else
      *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(row);
  }
}

__device__ __forceinline__ uint32_t ptx_h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 ptx_u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Extremes of a value group over its gl lanes (each holding 8 channels of the row), as the half2
// (min, -max): one min-reduction over both (fp16 min and max are exact).
__device__ __forceinline__ __half2 group_extremes(const uint4& raw, int gl) {
  const __half2* hx = reinterpret_cast<const __half2*>(&raw);
  const __half2 mn2 = __hmin2(__hmin2(hx[0], hx[1]), __hmin2(hx[2], hx[3]));
  const __half2 mx2 = __hmax2(__hmax2(hx[0], hx[1]), __hmax2(hx[2], hx[3]));
  __half2 e = __halves2half2(__hmin(__low2half(mn2), __high2half(mn2)),
                             __hneg(__hmax(__low2half(mx2), __high2half(mx2))));
  for (int off = 1; off < gl; off <<= 1)
    e = __hmin2(e, ptx_u32_as_h2(__shfl_xor_sync(0xffffffffu, ptx_h2_as_u32(e), off)));
  return e;
}

// Value quantize-pack, per token row over groups of gv channels.  CTA (x, y) covers tokens of
// (b, kv head) row y; a token row is dv/8 16-byte chunks of 8 channels, one chunk per lane, so a
// warp covers 32 / (dv/8) rows per load and each lane R rows (rows rsub, rsub + 32/(dv/8), ...
// of the warp's block).  A value group is gv/8 consecutive lanes (gv is a multiple of 8): min
// and max in fp16 per lane, then by shuffles across the group's lanes; every lane of a group
// derives the same (scale, zero).  Lane 0 of a group writes its (scale, zero); each lane writes
// The part of the value quantizer after a warp's rows are in registers: lane (rsub, cc) holds
// chunk cc of tokens t_begin + ti[i] (valid when ti[i] < n_tokens) of row bh = b * Hkv + h.
// Group extremes by shuffles; (scale, zero) and 1/scale per row and group; codes and (scale,
// zero) stored.  Sizes are powers of two (shifts and masks).  Called by every lane of the warp.
template <int BITS, int R>
__device__ __forceinline__ void value_rows(const uint4 (&x)[R], const int (&ti)[R], int bh, int t_begin,
                                           int n_tokens, uint32_t* __restrict__ vcode,
                                           __half2* __restrict__ vsz, const int* __restrict__ table,
                                           const Dims& d) {
  const int lcpr = __ffs(d.dv) - 4, lgl = __ffs(d.gv) - 4, lnvg = lcpr - lgl;
  const int gl = 1 << lgl;
  const int lane = threadIdx.x & 31;
  const int cc = lane & ((1 << lcpr) - 1);
  const int lgk = __ffs(d.gk) - 1;
  // each row's group extremes as one half2 (min, -max), reduced over the group's lanes
  // (aligned and consecutive)
  __half2 ext[R];
#pragma unroll
  for (int i = 0; i < R; ++i) ext[i] = group_extremes(x[i], gl);
  // (scale, zero) and 1/scale of the R rows: with groups of at least R lanes, lane j of a group
  // derives row j's in one pass and the rows are broadcast; otherwise every lane derives its own
  const int gsub = cc & (gl - 1), gbase = lane - gsub, vg = cc >> lgl;
  __half2 rsz[R];
  float rrc[R];
  if (gl >= R) {
    __half2 e = ext[0];
#pragma unroll
    for (int i = 1; i < R; ++i)
      if (gsub == i) e = ext[i];
    const GroupParams gp = group_params<BITS>(__low2float(e), -__high2float(e));
    const uint32_t sz = ptx_h2_as_u32(gp.sz);
    const float rc = gp.scale == 0.0f ? 0.0f : __frcp_rn(gp.scale);
#pragma unroll
    for (int i = 0; i < R; ++i) {
      rsz[i] = ptx_u32_as_h2(__shfl_sync(0xffffffffu, sz, gbase + i));
      rrc[i] = __shfl_sync(0xffffffffu, rc, gbase + i);
    }
  } else {
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const GroupParams gp = group_params<BITS>(__low2float(ext[i]), -__high2float(ext[i]));
      rsz[i] = gp.sz;
      rrc[i] = gp.scale == 0.0f ? 0.0f : __frcp_rn(gp.scale);
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (ti[i] >= n_tokens) continue;
    const float2 szf = __half22float2(rsz[i]);             // (scale, zero), exact
    const int t = t_begin + ti[i];
    const size_t vrow = group_row_bh(d, table, bh, t >> lgk) + (t & (d.gk - 1));
    if (gsub == 0 && KVQ_IN_BOUNDS(d, kSiteQValMeta, static_cast<long long>(vrow << lnvg) + vg,
                                   quant_rows(d) * d.nvg))
      vsz[(vrow << lnvg) + vg] = rsz[i];
    const ChunkBits<BITS> bits = pack_chunk<BITS, 0>(x[i], &szf.y, &rrc[i], &szf.x);
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteQValCode, static_cast<long long>(vrow * (d.dv * BITS / 8)) + cc * BITS, BITS,
                             quant_rows(d) * d.vw * 4))
      continue;
    store_chunk<BITS>(vcode, (vrow << lcpr) + cc, bits);
  }
}

template <int BITS, int R>
__global__ void __launch_bounds__(256) quantize_values_kernel(
    const __half* __restrict__ src, int src_rows, int t_begin, int n_tokens,
    uint32_t* __restrict__ vcode, __half2* __restrict__ vsz, const int* __restrict__ table, Dims d) {
  const int dv = d.dv, cpr = dv / 8, rpw = 32 / cpr;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cc = lane % cpr, rsub = lane / cpr;
  const int bh = blockIdx.y;
  const int t_first = (blockIdx.x * 8 + warp) * rpw * R;             // this warp's block of tokens
  if (t_first >= n_tokens) return;                                    // uniform per warp
  const size_t src_base = static_cast<size_t>(bh) * src_rows;
  {
    uint4 x[R];
    int ti[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      ti[i] = t_first + rsub + rpw * i;
      const int t = t_begin + ti[i];
      const int row = t < src_rows ? t : t % src_rows;                // the window is a ring
      const long long si = static_cast<long long>((src_base + row) * dv) + 8 * cc;
      if (ti[i] < n_tokens && KVQ_RANGE_IN_BOUNDS(d, kSiteQValSrc, si, 8, static_cast<long long>(d.B) * d.Hkv * src_rows * dv)) {
        x[i] = __ldg(reinterpret_cast<const uint4*>(src + (src_base + row) * dv) + cc);
      } else {
        x[i] = make_uint4(0, 0, 0, 0);
      }
    }
    value_rows<BITS, R>(x, ti, bh, t_begin, n_tokens, vcode, vsz, table, d);
  }
}

// ---- prefill quantizers over a contiguous source, persistent and staged ----
// CTA c takes tiles c, c + gridDim.x, ... of the launch (a key tile: the gpc consecutive groups
// of one (b, kv head) that a CTA holds; a value tile: 1024 / (dv/8) consecutive token rows of one
// (b, kv head), 16 KB), each brought into shared memory by one 1-D bulk copy (cp.async.bulk) two
// tiles ahead (double buffer, one mbarrier per stage), so HBM reads overlap the quantizer's
// arithmetic.  The rows of a tile must be contiguous in the source (a prefill input: row t of
// (b, h) at (b * Hkv + h) * src_rows + t); waits are bounded and a CTA whose wait gives up stops.
constexpr uint64_t kStageWaitNs = 1000000000ull;

struct StageRing {
  uint64_t bars[2];
  int issued[2];
  int adv_bh, adv_tr;   // gridDim.x tiles as (rows, tiles of a row): the step of a CTA's tile walk
};

// Waits (bounded) for the copies still in flight into the two stages before a CTA exits.
__device__ __forceinline__ void drain_stages(StageRing* ring) {
  if (threadIdx.x == 0)
    for (int s = 0; s < 2; ++s)
      if (ring->issued[s] > 0)
        ptx::mbar_wait_bounded(ptx::smem_addr(&ring->bars[s]), (ring->issued[s] - 1) & 1, kStageWaitNs);
  __syncthreads();
}

// Rotates n rows of 32 * M fp16 channels in shared memory in place (a warp per row, two rows at
// a time so that the butterfly chains of the two interleave), as rotate_row_warp then one
// rounding to fp16.
template <int M>
__device__ __forceinline__ void rotate_stage_rows(__half* rows, int n, const Dims& d) {
  constexpr int dk = 32 * M;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r0 = 2 * warp; r0 < n; r0 += 16) {
    const bool two = r0 + 1 < n;
    float a[M], b[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      a[m] = __half2float(rows[r0 * dk + lane + 32 * m]);
      b[m] = two ? __half2float(rows[(r0 + 1) * dk + lane + 32 * m]) : 0.0f;
    }
    rotate_row_warp<M>(a, M, d.rot_signs, d.rot_inv_ck, lane);
    rotate_row_warp<M>(b, M, d.rot_signs, d.rot_inv_ck, lane);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      rows[r0 * dk + lane + 32 * m] = __float2half_rn(a[m]);
      if (two) rows[(r0 + 1) * dk + lane + 32 * m] = __float2half_rn(b[m]);
    }
  }
}

template <int BITS, int R, bool ROT>
__global__ void __launch_bounds__(256, 16 / R) quantize_keys_staged_kernel(
    const __half* __restrict__ src, int src_rows, int g_begin, int n_groups,
    uint32_t* __restrict__ kcode, __half2* __restrict__ ksz, const int* __restrict__ table, Dims d) {
  extern __shared__ __align__(128) unsigned char sm_stage[];        // 2 x [gpc * gk][dk] fp16
  __shared__ __align__(16) __half2 red[2][256][4];
  __shared__ __align__(16) float prm[3][kKeyPrm];
  __shared__ __align__(16) __half blk[kKeyBlk];
  __shared__ __align__(8) StageRing ring;
  const int dk = d.dk, gk = d.gk;
  const int cpr = dk / 8, slabs = gk / R, tpg = cpr * slabs, gpc = 256 / tpg;
  const int tid = threadIdx.x;
  const int gi = tid / tpg, lt = tid % tpg, cc = lt % cpr, rs = lt / cpr;
  const int tiles_per_row = (n_groups + gpc - 1) / gpc;
  const long long n_tiles = static_cast<long long>(d.B) * d.Hkv * tiles_per_row;
  const int stage_bytes = gpc * gk * dk * 2;
  const uint32_t st0 = ptx::smem_addr(sm_stage);
  [[maybe_unused]] const long long src_ext = static_cast<long long>(d.B) * d.Hkv * src_rows * dk;
  // thread 0 copies tile `tile` (its groups' gk rows each) into stage st
  auto issue = [&](long long tile, int st) {
    const int bh = static_cast<int>(tile / tiles_per_row), g_first = static_cast<int>(tile % tiles_per_row) * gpc;
    const int ng = min(gpc, n_groups - g_first);
    long long first = (static_cast<long long>(bh) * src_rows + static_cast<long long>(g_begin + g_first) * gk) * dk;
    const uint32_t bytes = static_cast<uint32_t>(ng) * gk * dk * 2;
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteQKeySrc, first, static_cast<long long>(ng) * gk * dk, src_ext)) first = 0;
    ring.issued[st] += 1;
    ptx::mbar_arrive_expect_tx(ptx::smem_addr(&ring.bars[st]), bytes);
    ptx::bulk_g2s(st0 + st * stage_bytes, src + first, bytes, ptx::smem_addr(&ring.bars[st]));
  };
  if (tid == 0) {
    for (int st = 0; st < 2; ++st) {
      ptx::mbar_init(ptx::smem_addr(&ring.bars[st]), 1);
      ring.issued[st] = 0;
    }
    ring.adv_bh = static_cast<int>(gridDim.x / tiles_per_row);
    ring.adv_tr = static_cast<int>(gridDim.x % tiles_per_row);
    ptx::fence_barrier_init();
    for (int k = 0; k < 2; ++k)
      if (blockIdx.x + static_cast<long long>(k) * gridDim.x < n_tiles) issue(blockIdx.x + static_cast<long long>(k) * gridDim.x, k);
  }
  __syncthreads();
  // (row bh, tile of the row) of the current tile, advanced by gridDim.x tiles per iteration
  // without a division (the step is read from shared memory: it holds no registers)
  int bh = static_cast<int>(blockIdx.x / tiles_per_row), tr = static_cast<int>(blockIdx.x % tiles_per_row);
  for (int it = 0; bh < d.B * d.Hkv; ++it) {                         // tile bh * tiles_per_row + tr
    const int st = it & 1;
    const bool ok = ptx::mbar_wait_bounded(ptx::smem_addr(&ring.bars[st]), (it >> 1) & 1, kStageWaitNs);
    if (!__syncthreads_and(ok)) break;                                 // a wait gave up: stop
    if constexpr (ROT) {
      // key-only rotation: each warp rotates rows of the stage in place (fp32 butterflies, one
      // rounding to fp16), before any thread reads its chunks
      __half* rows = reinterpret_cast<__half*>(sm_stage + st * stage_bytes);
      switch (dk) {
        case 32: rotate_stage_rows<1>(rows, gpc * gk, d); break;
        case 64: rotate_stage_rows<2>(rows, gpc * gk, d); break;
        case 128: rotate_stage_rows<4>(rows, gpc * gk, d); break;
        default: rotate_stage_rows<8>(rows, gpc * gk, d); break;
      }
      __syncthreads();
    }
    const uint4* stage = reinterpret_cast<const uint4*>(sm_stage + st * stage_bytes);
    uint4 x[R];
#pragma unroll
    for (int i = 0; i < R; ++i) x[i] = stage[(gi * gk + rs + slabs * i) * cpr + cc];
    __syncthreads();                                                   // the stage may be refilled
    const long long next = static_cast<long long>(bh) * tiles_per_row + tr + 2LL * gridDim.x;
    if (tid == 0 && next < n_tiles) {
      ptx::fence_proxy_async_smem();
      issue(next, st);
    }
    key_tile<BITS, R>(x, bh, g_begin, tr * gpc, n_groups, kcode, ksz, table, d, red, prm, blk);
    __syncthreads();                                                   // red, prm, blk are reused
    bh += ring.adv_bh;
    tr += ring.adv_tr;
    if (tr >= tiles_per_row) {
      tr -= tiles_per_row;
      ++bh;
    }
  }
  drain_stages(&ring);
}

template <int BITS, int R>
__global__ void __launch_bounds__(256, 4) quantize_values_staged_kernel(
    const __half* __restrict__ src, int src_rows, int t_begin, int n_tokens,
    uint32_t* __restrict__ vcode, __half2* __restrict__ vsz, const int* __restrict__ table, Dims d) {
  extern __shared__ __align__(128) unsigned char sm_stage[];        // 2 x [tile rows][dv] fp16
  __shared__ __align__(8) StageRing ring;
  const int dv = d.dv, cpr = dv / 8, rpw = 32 / cpr;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cc = lane % cpr, rsub = lane / cpr;
  const int tile_rows = 8 * rpw * R;                                  // 16 KB of fp16 rows
  const int tiles_per_row = (n_tokens + tile_rows - 1) / tile_rows;
  const long long n_tiles = static_cast<long long>(d.B) * d.Hkv * tiles_per_row;
  const int stage_bytes = tile_rows * dv * 2;
  const uint32_t st0 = ptx::smem_addr(sm_stage);
  [[maybe_unused]] const long long src_ext = static_cast<long long>(d.B) * d.Hkv * src_rows * dv;
  auto issue = [&](long long tile, int st) {
    const int bh = static_cast<int>(tile / tiles_per_row), t0 = static_cast<int>(tile % tiles_per_row) * tile_rows;
    const int nr = min(tile_rows, n_tokens - t0);
    long long first = (static_cast<long long>(bh) * src_rows + t_begin + t0) * dv;
    const uint32_t bytes = static_cast<uint32_t>(nr) * dv * 2;
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteQValSrc, first, static_cast<long long>(nr) * dv, src_ext)) first = 0;
    ring.issued[st] += 1;
    ptx::mbar_arrive_expect_tx(ptx::smem_addr(&ring.bars[st]), bytes);
    ptx::bulk_g2s(st0 + st * stage_bytes, src + first, bytes, ptx::smem_addr(&ring.bars[st]));
  };
  if (threadIdx.x == 0) {
    for (int st = 0; st < 2; ++st) {
      ptx::mbar_init(ptx::smem_addr(&ring.bars[st]), 1);
      ring.issued[st] = 0;
    }
    ring.adv_bh = static_cast<int>(gridDim.x / tiles_per_row);
    ring.adv_tr = static_cast<int>(gridDim.x % tiles_per_row);
    ptx::fence_barrier_init();
    for (int k = 0; k < 2; ++k)
      if (blockIdx.x + static_cast<long long>(k) * gridDim.x < n_tiles) issue(blockIdx.x + static_cast<long long>(k) * gridDim.x, k);
  }
  __syncthreads();
  // (row bh, tile of the row) of the current tile, advanced by gridDim.x tiles per iteration
  // without a division (the step is read from shared memory: it holds no registers)
  int bh = static_cast<int>(blockIdx.x / tiles_per_row), tr = static_cast<int>(blockIdx.x % tiles_per_row);
  for (int it = 0; bh < d.B * d.Hkv; ++it) {                         // tile bh * tiles_per_row + tr
    const int st = it & 1;
    const bool ok = ptx::mbar_wait_bounded(ptx::smem_addr(&ring.bars[st]), (it >> 1) & 1, kStageWaitNs);
    if (!__syncthreads_and(ok)) break;                                 // a wait gave up: stop
    const int t0 = tr * tile_rows;
    const uint4* stage = reinterpret_cast<const uint4*>(sm_stage + st * stage_bytes);
    uint4 x[R];
    int ti[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int r = warp * rpw * R + rsub + rpw * i;                  // row within the tile
      ti[i] = t0 + r;
      x[i] = ti[i] < n_tokens ? stage[r * cpr + cc] : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();                                                   // the stage may be refilled
    const long long next = static_cast<long long>(bh) * tiles_per_row + tr + 2LL * gridDim.x;
    if (threadIdx.x == 0 && next < n_tiles) {
      ptx::fence_proxy_async_smem();
      issue(next, st);
    }
    value_rows<BITS, R>(x, ti, bh, t_begin, n_tokens, vcode, vsz, table, d);
    bh += ring.adv_bh;
    tr += ring.adv_tr;
    if (tr >= tiles_per_row) {
      tr -= tiles_per_row;
      ++bh;
    }
  }
  drain_stages(&ring);
}

// ---- per-channel widths ("Attention-Aware Transform Coding (AATC)", §Méthodologie,
// Allocation de Bits): channel c has its own width (8, 4, 2, 1 or 0 = dropped), widths
// non-increasing over the channels; the same quantizer with that many bits; a row packs
// the codes channel after channel, channel c at the sum of the widths before it.

// Codes of a 16-byte chunk of 8 channels with per-channel widths w[j] (0 = dropped, no bits),
// packed at bit offsets o[j] - o[0] (the offsets in the row are non-decreasing and a channel's
// offset is a multiple of its width); 8 * w[0] bits at most.
__device__ __forceinline__ uint64_t pack_chunk_var(const uint4& raw, const float* z, const float* r,
                                                   const float* sc, const int* w, const int* o) {
  const __half2* hx = reinterpret_cast<const __half2*>(&raw);
  float x[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(hx[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
  bool near = false;
  uint64_t bits = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (w[j]) bits |= static_cast<uint64_t>(code_fast_l(x[j], z[j], r[j], (1u << w[j]) - 1u, near)) << (o[j] - o[0]);
  if (near) {
    bits = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (w[j]) bits |= static_cast<uint64_t>(code_exact_l(x[j], z[j], sc[j], (1u << w[j]) - 1u)) << (o[j] - o[0]);
  }
  return bits;
}

// ORs a chunk's bits, which start at bit `off` of a row of 32-bit words, into that row.  A chunk
// whose first channel has 8 bits starts on a 64-bit boundary (every channel before it has 8
// bits); otherwise it spans at most 32 bits; so the bits fit in 64 bits after the shift.
__device__ __forceinline__ void or_into_row(uint32_t* row, int off, uint64_t bits) {
  const uint64_t v = bits << (off % 32);
  if (static_cast<uint32_t>(v)) atomicOr(&row[off / 32], static_cast<uint32_t>(v));
  if (v >> 32) atomicOr(&row[off / 32 + 1], static_cast<uint32_t>(v >> 32));
}

// Key quantize-pack with per-channel widths: the fixed-width kernel's tiling (16-byte chunks of
// 8 channels, R rows per thread, each key read once, min/max reduced in shared memory), channel
// c quantized with its own width; the codes are ORed into the CTA's rows in shared memory
// ([gpc * gk][kw] words), which are then written out whole.  (scale, zero) are stored plainly,
// [dk][2] per group; a dropped channel stores (0, 0).
// The part of the width-map key quantizer after a tile's chunks are in registers (the layout of
// key_tile; sm_rows: [gpc * gk][kw] words of the CTA's rows, zeroed here).  Called by every thread
// of the CTA (barriers).
template <int R>
__device__ __forceinline__ void key_tile_var(const uint4 (&x)[R], int b, int h, int g_begin, int g_first,
                                             int n_groups, uint32_t* __restrict__ kcode, __half2* __restrict__ ksz,
                                             const int* __restrict__ table, const Dims& d,
                                             __half2 (*red)[256][4], float (*prm)[kKeyPrm], __half2* blk,
                                             uint32_t* sm_rows, const int (&w)[8], const int (&o)[8]) {
  const int dk = d.dk, gk = d.gk, kw = d.kw;
  const int ldk = __ffs(dk) - 1, lcpr = ldk - 3, lslabs = __ffs(gk) - 1 - ilog2c(R);
  const int ltpg = lcpr + lslabs, slabs = 1 << lslabs, tpg = 1 << ltpg, gpc = 256 >> ltpg;
  const int cpr = 1 << lcpr;
  const int tid = threadIdx.x;
  const int gi = tid >> ltpg, lt = tid & (tpg - 1), cc = lt & (cpr - 1), rs = lt >> lcpr;
  const bool active = g_first + gi < n_groups;
  for (int i = tid; i < gpc * gk * kw; i += 256) sm_rows[i] = 0u;
  {
    const __half2* h0 = reinterpret_cast<const __half2*>(&x[0]);
    __half2 mn[4], mx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) mn[k] = mx[k] = h0[k];
#pragma unroll
    for (int i = 1; i < R; ++i) {
      const __half2* hi = reinterpret_cast<const __half2*>(&x[i]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mn[k] = __hmin2(mn[k], hi[k]);
        mx[k] = __hmax2(mx[k], hi[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      red[0][tid][k] = mn[k];
      red[1][tid][k] = mx[k];
    }
  }
  __syncthreads();
  for (int p = tid; p < (gpc << (ldk - 1)); p += 256) {
    const int g2 = p >> (ldk - 1), pp = p & ((dk >> 1) - 1), c2 = pp >> 2, k = pp & 3;
    const int t0 = (g2 << ltpg) + c2;
    __half2 mn = red[0][t0][k], mx = red[1][t0][k];
    for (int sl = 1; sl < slabs; ++sl) {
      mn = __hmin2(mn, red[0][t0 + (sl << lcpr)][k]);
      mx = __hmax2(mx, red[1][t0 + (sl << lcpr)][k]);
    }
    const float2 fmn = __half22float2(mn), fmx = __half22float2(mx);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int c = 8 * c2 + 2 * k + e;
      int width, offset;
      channel_width(d.kcnt, c, &width, &offset);
      GroupParams gp;
      gp.scale = gp.zero = 0.0f;
      gp.sz = __floats2half2_rn(0.0f, 0.0f);
      if (width) gp = group_params_b(e ? fmn.y : fmn.x, e ? fmx.y : fmx.x, width);
      prm[0][(g2 << ldk) + c] = gp.zero;
      prm[1][(g2 << ldk) + c] = gp.scale == 0.0f ? 0.0f : __frcp_rn(gp.scale);
      prm[2][(g2 << ldk) + c] = gp.scale;
      blk[(g2 << ldk) + c] = gp.sz;
    }
  }
  __syncthreads();
  for (int i = tid; i < (gpc << (ldk - 2)); i += 256) {           // 16 B of (scale, zero) per thread
    const int g2 = i >> (ldk - 2), j = i & ((dk >> 2) - 1);
    if (g_first + g2 >= n_groups) continue;
    const size_t gidx = group_index(d, table, b, h, g_begin + g_first + g2);
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteQKeyMeta, static_cast<long long>(gidx * dk) + 4 * j, 4, quant_groups(d) * dk))
      continue;
    reinterpret_cast<uint4*>(ksz + gidx * dk)[j] = reinterpret_cast<const uint4*>(blk + g2 * dk)[j];
  }
  if (active) {
    float z[8], r[8], sc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      z[j] = prm[0][(gi << ldk) + 8 * cc + j];
      r[j] = prm[1][(gi << ldk) + 8 * cc + j];
      sc[j] = prm[2][(gi << ldk) + 8 * cc + j];
    }
    if (w[0]) {
#pragma unroll
      for (int i = 0; i < R; ++i)
        or_into_row(sm_rows + (gi * gk + rs + slabs * i) * kw, o[0], pack_chunk_var(x[i], z, r, sc, w, o));
    }
  }
  __syncthreads();
  // the packed rows out: a group's gk rows are contiguous in the cache
  for (int g2 = 0; g2 < gpc && g_first + g2 < n_groups; ++g2) {
    const long long k0 = static_cast<long long>(group_row(d, table, b, h, g_begin + g_first + g2) * kw);
    const uint32_t* src_rows_sm = sm_rows + g2 * gk * kw;
    for (int j = tid; j < gk * kw; j += 256)
      if (KVQ_IN_BOUNDS(d, kSiteQKeyCode, k0 + j, quant_rows(d) * kw)) kcode[k0 + j] = src_rows_sm[j];
  }
}

// The widths and row bit offsets of the 8 channels of chunk cc (0 and the row's end for dropped
// channels).
__device__ __forceinline__ void chunk_widths(const Dims& d, int cc, int (&w)[8], int (&o)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) channel_width(d.kcnt, 8 * cc + j, &w[j], &o[j]);
}

template <int R>
__global__ void __launch_bounds__(256) quantize_keys_var_kernel(
    const __half* __restrict__ src, int src_rows, int g_begin, int n_groups,
    uint32_t* __restrict__ kcode, __half2* __restrict__ ksz, const int* __restrict__ table, Dims d) {
  extern __shared__ __align__(16) uint32_t sm_rows[];               // [gpc * gk][kw]
  __shared__ __align__(16) __half2 red[2][256][4];
  __shared__ __align__(16) float prm[3][kKeyPrm];
  __shared__ __align__(16) __half2 blk[kKeyPrm];
  const int dk = d.dk, gk = d.gk;
  const int cpr = dk / 8, slabs = gk / R, tpg = cpr * slabs, gpc = 256 / tpg;
  const int tid = threadIdx.x;
  const int gi = tid / tpg, lt = tid % tpg, cc = lt % cpr, rs = lt / cpr;
  const int bh = blockIdx.y;
  const int g_first = blockIdx.x * gpc;
  const bool active = g_first + gi < n_groups;
  const int g = g_begin + g_first + gi;
  const size_t base = static_cast<size_t>(bh) * src_rows;
  uint4 x[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int tk = g * gk + rs + slabs * i;
    const int row = tk < src_rows ? tk : tk % src_rows;              // the window is a ring
    const long long si = static_cast<long long>((base + row) * dk) + 8 * cc;
    x[i] = active && KVQ_RANGE_IN_BOUNDS(d, kSiteQKeySrc, si, 8, static_cast<long long>(d.B) * d.Hkv * src_rows * dk)
               ? __ldg(reinterpret_cast<const uint4*>(src + (base + row) * dk) + cc)
               : make_uint4(0, 0, 0, 0);
  }
  int w[8], o[8];
  chunk_widths(d, cc, w, o);
  key_tile_var<R>(x, bh / d.Hkv, bh % d.Hkv, g_begin, g_first, n_groups, kcode, ksz, table, d, red, prm, blk, sm_rows,
                  w, o);
}

// The width-map key quantizer for a contiguous source (prefill): the persistent staged form of
// quantize_keys_var_kernel (two stages of raw rows by bulk copies, as quantize_keys_staged_kernel),
// the CTA's packed rows after the stages in dynamic shared memory.
template <int R>
__global__ void __launch_bounds__(256, R == 4 ? 3 : 2) quantize_keys_var_staged_kernel(
    const __half* __restrict__ src, int src_rows, int g_begin, int n_groups,
    uint32_t* __restrict__ kcode, __half2* __restrict__ ksz, const int* __restrict__ table, Dims d) {
  extern __shared__ __align__(128) unsigned char sm_stage[];        // 2 x [gpc * gk][dk] fp16, rows
  __shared__ __align__(16) __half2 red[2][256][4];
  __shared__ __align__(16) float prm[3][kKeyPrm];
  __shared__ __align__(16) __half2 blk[kKeyPrm];
  __shared__ __align__(8) StageRing ring;
  const int dk = d.dk, gk = d.gk;
  const int cpr = dk / 8, slabs = gk / R, tpg = cpr * slabs, gpc = 256 / tpg;
  const int tid = threadIdx.x;
  const int gi = tid / tpg, lt = tid % tpg, cc = lt % cpr, rs = lt / cpr;
  const int tiles_per_row = (n_groups + gpc - 1) / gpc;
  const long long n_tiles = static_cast<long long>(d.B) * d.Hkv * tiles_per_row;
  const int stage_bytes = gpc * gk * dk * 2;
  uint32_t* sm_rows = reinterpret_cast<uint32_t*>(sm_stage + 2 * stage_bytes);
  const uint32_t st0 = ptx::smem_addr(sm_stage);
  int w[8], o[8];
  chunk_widths(d, cc, w, o);
  [[maybe_unused]] const long long src_ext = static_cast<long long>(d.B) * d.Hkv * src_rows * dk;
  auto issue = [&](long long tile, int st) {
    const int bh = static_cast<int>(tile / tiles_per_row), g_first = static_cast<int>(tile % tiles_per_row) * gpc;
    const int ng = min(gpc, n_groups - g_first);
    long long first = (static_cast<long long>(bh) * src_rows + static_cast<long long>(g_begin + g_first) * gk) * dk;
    const uint32_t bytes = static_cast<uint32_t>(ng) * gk * dk * 2;
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteQKeySrc, first, static_cast<long long>(ng) * gk * dk, src_ext)) first = 0;
    ring.issued[st] += 1;
    ptx::mbar_arrive_expect_tx(ptx::smem_addr(&ring.bars[st]), bytes);
    ptx::bulk_g2s(st0 + st * stage_bytes, src + first, bytes, ptx::smem_addr(&ring.bars[st]));
  };
  if (tid == 0) {
    for (int st = 0; st < 2; ++st) {
      ptx::mbar_init(ptx::smem_addr(&ring.bars[st]), 1);
      ring.issued[st] = 0;
    }
    ptx::fence_barrier_init();
    for (int k = 0; k < 2; ++k)
      if (blockIdx.x + static_cast<long long>(k) * gridDim.x < n_tiles) issue(blockIdx.x + static_cast<long long>(k) * gridDim.x, k);
  }
  __syncthreads();
  for (int it = 0;; ++it) {
    const long long tile = blockIdx.x + static_cast<long long>(it) * gridDim.x;
    if (tile >= n_tiles) break;
    const int st = it & 1;
    const bool ok = ptx::mbar_wait_bounded(ptx::smem_addr(&ring.bars[st]), (it >> 1) & 1, kStageWaitNs);
    if (!__syncthreads_and(ok)) break;                                 // a wait gave up: stop
    const uint4* stage = reinterpret_cast<const uint4*>(sm_stage + st * stage_bytes);
    uint4 x[R];
#pragma unroll
    for (int i = 0; i < R; ++i) x[i] = stage[(gi * gk + rs + slabs * i) * cpr + cc];
    __syncthreads();                                                   // the stage may be refilled
    if (tid == 0 && tile + 2LL * gridDim.x < n_tiles) {
      ptx::fence_proxy_async_smem();
      issue(tile + 2LL * gridDim.x, st);
    }
    const int t32 = static_cast<int>(tile), bh = t32 / tiles_per_row, g_first = (t32 - bh * tiles_per_row) * gpc;
    key_tile_var<R>(x, bh / d.Hkv, bh % d.Hkv, g_begin, g_first, n_groups, kcode, ksz, table, d, red, prm, blk,
                    sm_rows, w, o);
    __syncthreads();                                                   // red, prm, blk, rows are reused
  }
  drain_stages(&ring);
}

// Value quantize-pack with per-group widths: the fixed-width value kernel's tiling (a lane per
// 16-byte chunk of a row, R rows per lane, group extremes by shuffles); a chunk lies in one
// value group, so its 8 channels share the group's width.  Each warp ORs its block's codes into
// rows in shared memory, then writes the rows out whole.
// One warp's block of value rows with per-group widths: lane (rsub, cc) holds chunk cc of rows
// t_first + rsub + rpw * i (i < R) in x; (scale, zero) per group and row, codes ORed into the
// warp's rows in shared memory (rows_sm: block_rows x vw words), which are then stored whole.
template <int R>
__device__ __forceinline__ void value_block_var(const uint4 (&x)[R], int bh, int t_begin, int t_first, int n_tokens,
                                                uint32_t* __restrict__ vcode, __half2* __restrict__ vsz,
                                                const int* __restrict__ table, const Dims& d, uint32_t* rows_sm) {
  const int dv = d.dv, cpr = dv / 8, rpw = 32 / cpr, gl = d.gv / 8, vw = d.vw;
  const int lane = threadIdx.x & 31;
  const int cc = lane % cpr, rsub = lane / cpr;
  int width, offset;
  channel_width(d.vcnt, 8 * cc, &width, &offset);
  const uint32_t levels = (1u << width) - 1u;
  const int lg = __ffs(d.gk) - 1;
  const int block_rows = rpw * R;
  for (int k = lane; k < block_rows * vw; k += 32) rows_sm[k] = 0u;
  __syncwarp();
  int ti[R];
#pragma unroll
  for (int i = 0; i < R; ++i) ti[i] = t_first + rsub + rpw * i;
  // (scale, zero) of the R rows: with groups of at least R lanes, lane j of a group derives row
  // j's and the rows are broadcast; otherwise every lane derives its own
  __half2 ext[R];
#pragma unroll
  for (int i = 0; i < R; ++i) ext[i] = group_extremes(x[i], gl);
  const int gsub = cc % gl, gbase = lane - gsub;
  GroupParams rgp[R];
  if (gl >= R) {
    __half2 e = ext[0];
#pragma unroll
    for (int i = 1; i < R; ++i)
      if (gsub == i) e = ext[i];
    GroupParams gp;
    gp.scale = gp.zero = 0.0f;
    gp.sz = __floats2half2_rn(0.0f, 0.0f);
    if (width) gp = group_params_b(__low2float(e), -__high2float(e), width);
    const uint32_t sz = ptx_h2_as_u32(gp.sz);
#pragma unroll
    for (int i = 0; i < R; ++i) {
      rgp[i].sz = ptx_u32_as_h2(__shfl_sync(0xffffffffu, sz, gbase + i));
      rgp[i].scale = __low2float(rgp[i].sz);
      rgp[i].zero = __high2float(rgp[i].sz);
    }
  } else {
#pragma unroll
    for (int i = 0; i < R; ++i) {
      rgp[i].scale = rgp[i].zero = 0.0f;
      rgp[i].sz = __floats2half2_rn(0.0f, 0.0f);
      if (width) rgp[i] = group_params_b(__low2float(ext[i]), -__high2float(ext[i]), width);
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (ti[i] >= n_tokens) continue;
    const GroupParams gp = rgp[i];
    const int t = t_begin + ti[i];
    const size_t vrow = group_row(d, table, bh / d.Hkv, bh % d.Hkv, t >> lg) + (t & (d.gk - 1));
    if (cc % gl == 0 && KVQ_IN_BOUNDS(d, kSiteQValMeta, static_cast<long long>(vrow * d.nvg) + cc / gl,
                                      quant_rows(d) * d.nvg))
      vsz[vrow * d.nvg + cc / gl] = gp.sz;
    if (!width) continue;
    const float rcp = gp.scale == 0.0f ? 0.0f : __frcp_rn(gp.scale);
    const __half2* h2 = reinterpret_cast<const __half2*>(&x[i]);
    bool near = false;
    uint64_t bits = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h2[e]);
      bits |= static_cast<uint64_t>(code_fast_l(f.x, gp.zero, rcp, levels, near)) << (2 * e * width);
      bits |= static_cast<uint64_t>(code_fast_l(f.y, gp.zero, rcp, levels, near)) << ((2 * e + 1) * width);
    }
    if (near) {
      bits = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h2[e]);
        bits |= static_cast<uint64_t>(code_exact_l(f.x, gp.zero, gp.scale, levels)) << (2 * e * width);
        bits |= static_cast<uint64_t>(code_exact_l(f.y, gp.zero, gp.scale, levels)) << ((2 * e + 1) * width);
      }
    }
    or_into_row(rows_sm + (rsub + rpw * i) * vw, offset, bits);
  }
  __syncwarp();
  // the warp's rows out, row by row (a row's words are consecutive in the cache)
  for (int rr = 0; rr < block_rows && t_first + rr < n_tokens; ++rr) {
    const int t = t_begin + t_first + rr;
    const size_t vrow = group_row(d, table, bh / d.Hkv, bh % d.Hkv, t >> lg) + (t & (d.gk - 1));
    for (int j = lane; j < vw; j += 32) {
      const long long vi = static_cast<long long>(vrow * vw) + j;
      if (KVQ_IN_BOUNDS(d, kSiteQValCode, vi, quant_rows(d) * vw)) vcode[vi] = rows_sm[rr * vw + j];
    }
  }
  __syncwarp();
}

template <int R>
__global__ void __launch_bounds__(256) quantize_values_var_kernel(
    const __half* __restrict__ src, int src_rows, int t_begin, int n_tokens,
    uint32_t* __restrict__ vcode, __half2* __restrict__ vsz, const int* __restrict__ table, Dims d) {
  __shared__ uint32_t sm_rows[8][64 * R];           // per warp: 256 R / dv rows of <= dv / 4 words
  const int dv = d.dv, cpr = dv / 8, rpw = 32 / cpr;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cc = lane % cpr, rsub = lane / cpr;
  const int bh = blockIdx.y;
  const int block_rows = rpw * R;
  const int t_first = (blockIdx.x * 8 + warp) * block_rows;          // this warp's block of tokens
  if (t_first >= n_tokens) return;                                    // uniform per warp
  const size_t src_base = static_cast<size_t>(bh) * src_rows;
  uint4 x[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int ti = t_first + rsub + rpw * i;
    const int t = t_begin + ti;
    const int row = t < src_rows ? t : t % src_rows;                  // the window is a ring
    const long long si = static_cast<long long>((src_base + row) * dv) + 8 * cc;
    x[i] = ti < n_tokens && KVQ_RANGE_IN_BOUNDS(d, kSiteQValSrc, si, 8, static_cast<long long>(d.B) * d.Hkv * src_rows * dv)
               ? __ldg(reinterpret_cast<const uint4*>(src + (src_base + row) * dv) + cc)
               : make_uint4(0, 0, 0, 0);
  }
  value_block_var<R>(x, bh, t_begin, t_first, n_tokens, vcode, vsz, table, d, sm_rows[warp]);
}

// dst[bh][(dst_base + i) % dst_rows] = src[bh][(src_base + i) % src_rows], i < n, 16 B at a time.
__global__ void copy_rows_kernel(const __half* __restrict__ src, int src_rows, int src_base,
                                 __half* __restrict__ dst, int dst_rows, int dst_base, int n,
                                 int width, int nbh, Dims d) {
  const int vec = width / 8;
  const long long total = static_cast<long long>(nbh) * n * vec;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(idx % vec);
    const long long r = idx / vec;
    const int i = static_cast<int>(r % n);
    const int bh = static_cast<int>(r / n);
    const int sr = (src_base + i) % src_rows;
    const int dr = (dst_base + i) % dst_rows;
    const long long si = static_cast<long long>((static_cast<size_t>(bh) * src_rows + sr) * width) + 8 * e;
    const long long di = static_cast<long long>((static_cast<size_t>(bh) * dst_rows + dr) * width) + 8 * e;
    if (!KVQ_RANGE_IN_BOUNDS(d, kSiteCopySrc, si, 8, static_cast<long long>(nbh) * src_rows * width) ||
        !KVQ_RANGE_IN_BOUNDS(d, kSiteCopyDst, di, 8, static_cast<long long>(nbh) * dst_rows * width))
      continue;
    const uint4* s = reinterpret_cast<const uint4*>(src + (static_cast<size_t>(bh) * src_rows + sr) * width);
    uint4* t = reinterpret_cast<uint4*>(dst + (static_cast<size_t>(bh) * dst_rows + dr) * width);
    t[e] = s[e];
  }
}

// Append: the new token's key and value rows of every (b, kv head) into the window slot of
// sequence b (none when it is -1), 16 B per thread; k null: values only.
__global__ void append_token_kernel(const __half* __restrict__ k, const __half* __restrict__ v,
                                    __half* __restrict__ win_k, __half* __restrict__ win_v,
                                    SlotMap slots, int hkv, int cap, int dk, int dv, int nbh, Dims d) {
  const int vk = dk / 8, vv = dv / 8;
  const int total = nbh * (vk + vv);
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += gridDim.x * blockDim.x) {
    const int bh = idx / (vk + vv), e = idx % (vk + vv);
    const int slot = slots.slot[bh / hkv];
    if (slot < 0) continue;
    if (!KVQ_IN_BOUNDS(d, kSiteAppendWin, slot, cap)) continue;
    if (e < vk) {
      if (k)
        reinterpret_cast<uint4*>(win_k + (static_cast<size_t>(bh) * cap + slot) * dk)[e] =
            reinterpret_cast<const uint4*>(k + static_cast<size_t>(bh) * dk)[e];
    } else {
      reinterpret_cast<uint4*>(win_v + (static_cast<size_t>(bh) * cap + slot) * dv)[e - vk] =
          reinterpret_cast<const uint4*>(v + static_cast<size_t>(bh) * dv)[e - vk];
    }
  }
}

// Rotated key rows, one warp per (b * kv head, row i < n): source row (src_base + i) %
// src_rows, or list->pos[i], into destination row (dst_base + i) % dst_rows, or, with
// use_slots, into row slots.slot[b] (skipped when -1).
__global__ void rotate_key_rows_kernel(const __half* __restrict__ src, int src_rows, int src_base,
                                       __half* __restrict__ dst, int dst_rows, int dst_base, int n,
                                       int nbh, RetList list, int use_list, SlotMap slots,
                                       int use_slots, Dims d) {
  const int lane = threadIdx.x & 31;
  const long long total = static_cast<long long>(nbh) * n;
  const int dk = d.dk;
  for (long long r = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) / 32; r < total;
       r += static_cast<long long>(gridDim.x) * blockDim.x / 32) {
    const int i = static_cast<int>(r % n);
    const int bh = static_cast<int>(r / n);
    const int sr = use_list ? list.pos[i] : (src_base + i) % src_rows;
    const int dr = use_slots ? slots.slot[bh / d.Hkv] : (dst_base + i) % dst_rows;
    if (dr < 0) continue;                                   // uniform per warp
    if (!KVQ_IN_BOUNDS(d, kSiteRotSrc, sr, src_rows) || !KVQ_IN_BOUNDS(d, kSiteRotDst, dr, dst_rows)) continue;
    const __half* s = src + (static_cast<size_t>(bh) * src_rows + sr) * dk;
    __half* t = dst + (static_cast<size_t>(bh) * dst_rows + dr) * dk;
    float x[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) x[m] = m < dk / 32 ? __half2float(s[lane + 32 * m]) : 0.0f;
    rotate_row_warp<8>(x, dk / 32, d.rot_signs, d.rot_inv_ck, lane);
#pragma unroll
    for (int m = 0; m < 8; ++m)
      if (m < dk / 32) t[lane + 32 * m] = __float2half_rn(x[m]);
  }
}

// Prefill: ret[bh][j] = K[bh][pos[j]] for the retained positions (keys and values).
__global__ void copy_retained_kernel(const __half* __restrict__ k, const __half* __restrict__ v,
                                     int L, int dk, int dv, RetList ret,
                                     __half* __restrict__ ret_k, __half* __restrict__ ret_v, Dims d) {
  const int bh = blockIdx.x;
  for (int j = 0; j < ret.n; ++j) {
    if (!KVQ_IN_BOUNDS(d, kSiteRetSrc, ret.pos[j], L) || !KVQ_IN_BOUNDS(d, kSiteRetDst, j, kMaxRetained)) continue;
    const size_t src = static_cast<size_t>(bh) * L + ret.pos[j];
    const size_t dst = static_cast<size_t>(bh) * kMaxRetained + j;
    if (k)
      for (int c = threadIdx.x; c < dk / 8; c += blockDim.x)
        reinterpret_cast<uint4*>(ret_k + dst * dk)[c] = reinterpret_cast<const uint4*>(k + src * dk)[c];
    for (int c = threadIdx.x; c < dv / 8; c += blockDim.x)
      reinterpret_cast<uint4*>(ret_v + dst * dv)[c] = reinterpret_cast<const uint4*>(v + src * dv)[c];
  }
}

// Append: rebuild the retained list in place, entry i from an old slot >= i or from
// a window slot.  Entries are handled in ascending order, so an old slot is read
// before any later entry overwrites it.
__global__ void update_retained_kernel(RetUpdate up, int cap, int dk, int dv,
                                       const __half* __restrict__ win_k,
                                       const __half* __restrict__ win_v, __half* ret_k,
                                       __half* ret_v, Dims d) {
  const int bh = blockIdx.x;
  for (int i = 0; i < up.n; ++i) {
    // uniform per CTA: the loop's barriers stay matched
    if (!KVQ_IN_BOUNDS(d, kSiteRetUpd, up.index[i], up.from_window[i] ? cap : kMaxRetained) ||
        !KVQ_IN_BOUNDS(d, kSiteRetDst, i, kMaxRetained))
      continue;
    const size_t dst = static_cast<size_t>(bh) * kMaxRetained + i;
    const __half* sk;
    const __half* sv;
    if (up.from_window[i]) {
      const size_t s = static_cast<size_t>(bh) * cap + up.index[i];
      sk = win_k + s * dk;
      sv = win_v + s * dv;
    } else {
      const size_t s = static_cast<size_t>(bh) * kMaxRetained + up.index[i];
      sk = ret_k + s * dk;
      sv = ret_v + s * dv;
    }
    uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
    const bool ka = threadIdx.x < dk / 8, va = threadIdx.x < dv / 8;
    if (ka) a = reinterpret_cast<const uint4*>(sk)[threadIdx.x];
    if (va) b = reinterpret_cast<const uint4*>(sv)[threadIdx.x];
    __syncthreads();
    if (ka) reinterpret_cast<uint4*>(ret_k + dst * dk)[threadIdx.x] = a;
    if (va) reinterpret_cast<uint4*>(ret_v + dst * dv)[threadIdx.x] = b;
    __syncthreads();
  }
}

// Block-table entries of a paged cache: table[idx[i]] = page[i].
__global__ void table_writes_kernel(int* __restrict__ table, TableWrites tw, Dims d) {
  for (int i = threadIdx.x; i < tw.n; i += blockDim.x)
    if (KVQ_IN_BOUNDS(d, kSiteTableIdx, tw.idx[i], static_cast<long long>(d.B) * d.max_groups) &&
        KVQ_IN_BOUNDS(d, kSiteTablePage, tw.page[i], d.n_pages))
      table[tw.idx[i]] = tw.page[i];
}

inline int grid_for(long long items, int block) {
  long long g = (items + block - 1) / block;
  if (g > 148LL * 32) g = 148LL * 32;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

template <int BITS, bool ROT>
cudaError_t launch_quantize_keys_t(const Dims& d, const __half* src, int src_rows, int g_begin,
                                   int n_groups, uint32_t* kcode, __half2* ksz, const int* table,
                                   cudaStream_t s) {
  // rows per thread: at least 4, and enough that one group needs at most 256 threads
  const int cpr = d.dk / 8;
  int rows = 4;
  while (cpr * d.gk / rows > 256) rows *= 2;
  const int tpg = cpr * d.gk / rows, gpc = 256 / tpg;
  dim3 grid((n_groups + gpc - 1) / gpc, d.B * d.Hkv);
  const size_t smem = ROT ? static_cast<size_t>(gpc) * d.gk * d.dk * 2 : 0;
  auto kern = rows == 4 ? quantize_keys_kernel<BITS, 4, ROT>
            : rows == 8 ? quantize_keys_kernel<BITS, 8, ROT> : quantize_keys_kernel<BITS, 16, ROT>;
  if (rows > 16 || gpc * d.dk > kKeyPrm || gpc * 2 * d.dk > kKeyBlk) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  if (static_cast<long long>(g_begin + n_groups) * d.gk <= src_rows) {
    // a contiguous source (prefill): the persistent staged kernel (rotating the staged rows in
    // place when the keys are rotated)
    // with G_k >= 64 at least eight rows per thread (two CTAs per SM): the per-tile work is
    // spread over more chunks (measured 2.91 against 2.96 ms on the 32k rotated-key prefill)
    const int rs8 = d.gk >= 64 && rows < 8 ? 8 : rows;
    const int gpc8 = 256 / (cpr * d.gk / rs8);
    if (gpc8 * d.dk > kKeyPrm || gpc8 * 2 * d.dk > kKeyBlk) return cudaErrorInvalidValue;
    auto staged = rs8 == 4 ? quantize_keys_staged_kernel<BITS, 4, ROT>
                : rs8 == 8 ? quantize_keys_staged_kernel<BITS, 8, ROT> : quantize_keys_staged_kernel<BITS, 16, ROT>;
    const int sbytes = 2 * gpc8 * d.gk * d.dk * 2;
    // static + dynamic shared memory above 48 KB needs the opt-in (set on every launch: it is a
    // property of the current device's context)
    const cudaError_t e = cudaFuncSetAttribute(staged, cudaFuncAttributeMaxDynamicSharedMemorySize, sbytes);
    if (e != cudaSuccess) return e;
    const long long tiles = static_cast<long long>(d.B) * d.Hkv * ((n_groups + gpc8 - 1) / gpc8);
    const long long slots = static_cast<long long>(d.sm_count > 0 ? d.sm_count : 148) * (16 / rs8);
    staged<<<static_cast<int>(tiles < slots ? tiles : slots), 256, sbytes, s>>>(src, src_rows, g_begin, n_groups,
                                                                               kcode, ksz, table, d);
    return cudaGetLastError();
  }
  kern<<<grid, 256, smem, s>>>(src, src_rows, g_begin, n_groups, kcode, ksz, table, d);
  return cudaGetLastError();
}

template <bool ROT>
cudaError_t launch_quantize_keys_r(const Dims& d, const __half* src, int src_rows, int g_begin,
                                   int n_groups, uint32_t* kcode, __half2* ksz, const int* table,
                                   cudaStream_t s) {
  switch (d.kb) {
    case 2: return launch_quantize_keys_t<2, ROT>(d, src, src_rows, g_begin, n_groups, kcode, ksz, table, s);
    case 4: return launch_quantize_keys_t<4, ROT>(d, src, src_rows, g_begin, n_groups, kcode, ksz, table, s);
    case 8: return launch_quantize_keys_t<8, ROT>(d, src, src_rows, g_begin, n_groups, kcode, ksz, table, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize_keys(const Dims& d, const __half* src, int src_rows, int g_begin,
                                 int n_groups, uint32_t* kcode, __half2* ksz, const int* table,
                                 bool rotate, cudaStream_t s) {
  if (n_groups <= 0) return cudaSuccess;
  if (d.var) {
    if (rotate) return cudaErrorInvalidValue;
    const int cpr = d.dk / 8;
    int rows = 4;
    while (cpr * d.gk / rows > 256) rows *= 2;
    const int tpg = cpr * d.gk / rows, gpc = 256 / tpg;
    const int smem = gpc * d.gk * d.kw * 4;
    auto kern = rows == 4 ? quantize_keys_var_kernel<4>
              : rows == 8 ? quantize_keys_var_kernel<8> : quantize_keys_var_kernel<16>;
    if (rows > 16 || gpc * d.dk > kKeyPrm) return cudaErrorInvalidValue;
    if (static_cast<long long>(g_begin + n_groups) * d.gk <= src_rows) {
      // a contiguous source (prefill): the persistent staged kernel, three CTAs per SM (two when
      // a thread holds more than four rows)
      auto staged = rows == 4 ? quantize_keys_var_staged_kernel<4>
                  : rows == 8 ? quantize_keys_var_staged_kernel<8> : quantize_keys_var_staged_kernel<16>;
      const int sbytes = 2 * gpc * d.gk * d.dk * 2 + smem;
      const cudaError_t e = cudaFuncSetAttribute(staged, cudaFuncAttributeMaxDynamicSharedMemorySize, sbytes);
      if (e != cudaSuccess) return e;
      const long long tiles = static_cast<long long>(d.B) * d.Hkv * ((n_groups + gpc - 1) / gpc);
      const long long slots = static_cast<long long>(d.sm_count > 0 ? d.sm_count : 148) * (rows == 4 ? 3 : 2);
      staged<<<static_cast<int>(tiles < slots ? tiles : slots), 256, sbytes, s>>>(src, src_rows, g_begin, n_groups,
                                                                                 kcode, ksz, table, d);
      return cudaGetLastError();
    }
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
    }
    kern<<<dim3((n_groups + gpc - 1) / gpc, d.B * d.Hkv), 256, smem, s>>>(src, src_rows, g_begin, n_groups,
                                                                         kcode, ksz, table, d);
    return cudaGetLastError();
  }
  return rotate ? launch_quantize_keys_r<true>(d, src, src_rows, g_begin, n_groups, kcode, ksz, table, s)
                : launch_quantize_keys_r<false>(d, src, src_rows, g_begin, n_groups, kcode, ksz, table, s);
}

cudaError_t launch_table_writes(const Dims& d, int* table, const TableWrites& tw, cudaStream_t s) {
  if (tw.n <= 0) return cudaSuccess;
  table_writes_kernel<<<1, 256, 0, s>>>(table, tw, d);
  return cudaGetLastError();
}

cudaError_t launch_rotate_key_rows(const Dims& d, const __half* src, int src_rows, int src_base,
                                   __half* dst, int dst_rows, int dst_base, int n,
                                   const RetList* list, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int nbh = d.B * d.Hkv;
  const long long warps = static_cast<long long>(nbh) * n;
  RetList empty;
  empty.n = 0;
  SlotMap none;
  none.slot[0] = -1;
  rotate_key_rows_kernel<<<grid_for(warps * 32, 256), 256, 0, s>>>(
      src, src_rows, src_base, dst, dst_rows, dst_base, n, nbh, list ? *list : empty, list ? 1 : 0,
      none, 0, d);
  return cudaGetLastError();
}

cudaError_t launch_quantize_side(const Dims& d, const __half* src, int src_rows, int g_begin,
                                 int n_groups, const uint32_t* kcode, const __half2* ksz,
                                 const float* side_u, uint8_t* zcode, __half2* zsz, const int* table,
                                 bool rotate, cudaStream_t s) {
  if (n_groups <= 0 || d.sr == 0) return cudaSuccess;
  const size_t smem = (static_cast<size_t>(d.gk) * (d.dk + 1) + d.dk * d.sr + d.gk * d.sr) * 4;
  dim3 grid(n_groups, d.B * d.Hkv);
  auto kern = d.sq == 4 ? (rotate ? quantize_side_kernel<4, true> : quantize_side_kernel<4, false>)
                        : (rotate ? quantize_side_kernel<8, true> : quantize_side_kernel<8, false>);
  if (d.sq != 4 && d.sq != 8) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, 256, smem, s>>>(src, src_rows, d.dk, d.kb, d.gk, g_begin, d.lcap, d.Hkv, d.sr, d.zb,
                               kcode, ksz, side_u, zcode, zsz, table, d);
  return cudaGetLastError();
}

cudaError_t launch_quantize_values(const Dims& d, const __half* src, int src_rows, int t_begin,
                                   int n_tokens, uint32_t* vcode, __half2* vsz, const int* table,
                                   cudaStream_t s) {
  if (n_tokens <= 0) return cudaSuccess;
  const int nbh = d.B * d.Hkv;
  // CTA (x, y): tokens [x * per_cta, (x + 1) * per_cta) of (b, kv head) row y; 8 warps, each
  // a block of 32 / (dv / 8) * kRows tokens
  constexpr int kRows = 4;
  const int per_cta = 8 * (32 / (d.dv / 8)) * kRows;
  const dim3 grid((n_tokens + per_cta - 1) / per_cta, nbh);
  if (d.var) {
    // (a staged form of this kernel measured slower: 2.58 against 2.07 ms on the 32k width map)
    quantize_values_var_kernel<kRows><<<grid, 256, 0, s>>>(src, src_rows, t_begin, n_tokens, vcode, vsz, table, d);
    return cudaGetLastError();
  }
  if (t_begin + n_tokens <= src_rows) {
    // a contiguous source (prefill): the persistent staged kernel (two 16 KB stages)
    const long long tiles = static_cast<long long>(nbh) * ((n_tokens + per_cta - 1) / per_cta);
    const long long slots = static_cast<long long>(d.sm_count > 0 ? d.sm_count : 148) * 4;
    const dim3 pgrid(static_cast<unsigned>(tiles < slots ? tiles : slots));
    const int sbytes = 2 * per_cta * d.dv * 2;         // 32 KB: below the 48 KB default
    switch (d.vb) {
      case 2: quantize_values_staged_kernel<2, kRows><<<pgrid, 256, sbytes, s>>>(src, src_rows, t_begin, n_tokens, vcode, vsz, table, d); break;
      case 4: quantize_values_staged_kernel<4, kRows><<<pgrid, 256, sbytes, s>>>(src, src_rows, t_begin, n_tokens, vcode, vsz, table, d); break;
      case 8: quantize_values_staged_kernel<8, kRows><<<pgrid, 256, sbytes, s>>>(src, src_rows, t_begin, n_tokens, vcode, vsz, table, d); break;
      default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
  }
  switch (d.vb) {
    case 2: quantize_values_kernel<2, kRows><<<grid, 256, 0, s>>>(src, src_rows, t_begin, n_tokens, vcode, vsz, table, d); break;
    case 4: quantize_values_kernel<4, kRows><<<grid, 256, 0, s>>>(src, src_rows, t_begin, n_tokens, vcode, vsz, table, d); break;
    case 8: quantize_values_kernel<8, kRows><<<grid, 256, 0, s>>>(src, src_rows, t_begin, n_tokens, vcode, vsz, table, d); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_copy_rows(const Dims& d, const __half* src, int src_rows, int src_base, __half* dst,
                             int dst_rows, int dst_base, int n, int width, int nbh, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const long long items = static_cast<long long>(nbh) * n * (width / 8);
  const int block = 256;
  copy_rows_kernel<<<grid_for(items, block), block, 0, s>>>(src, src_rows, src_base, dst, dst_rows,
                                                            dst_base, n, width, nbh, d);
  return cudaGetLastError();
}

cudaError_t launch_append_token(const Dims& d, const __half* k, const __half* v, __half* win_k,
                                __half* win_v, const SlotMap& slots, cudaStream_t s) {
  const int nbh = d.B * d.Hkv;
  const int total = nbh * (d.dk + d.dv) / 8;
  const int block = 256;
  append_token_kernel<<<(total + block - 1) / block, block, 0, s>>>(
      d.rot ? nullptr : k, v, win_k, win_v, slots, d.Hkv, d.cap, d.dk, d.dv, nbh, d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !d.rot) return e;
  // rotated keys: one warp per (b, kv head) row
  RetList empty;
  empty.n = 0;
  rotate_key_rows_kernel<<<grid_for(static_cast<long long>(nbh) * 32, 256), 256, 0, s>>>(
      k, 1, 0, win_k, d.cap, 0, 1, nbh, empty, 0, slots, 1, d);
  return cudaGetLastError();
}

cudaError_t launch_copy_retained(const Dims& d, const __half* k, const __half* v, int L,
                                 const RetList& ret, __half* ret_k, __half* ret_v, cudaStream_t s) {
  if (ret.n <= 0) return cudaSuccess;
  copy_retained_kernel<<<d.B * d.Hkv, 64, 0, s>>>(k, v, L, d.dk, d.dv, ret, ret_k, ret_v, d);
  return cudaGetLastError();
}

cudaError_t launch_update_retained(const Dims& d, const RetUpdate& up, __half* win_k,
                                   __half* win_v, __half* ret_k, __half* ret_v, cudaStream_t s) {
  if (up.n <= 0) return cudaSuccess;
  const int threads = ((d.dk > d.dv ? d.dk : d.dv) / 8 + 31) / 32 * 32;
  update_retained_kernel<<<d.B * d.Hkv, threads, 0, s>>>(up, d.cap, d.dk, d.dv, win_k, win_v,
                                                          ret_k, ret_v, d);
  return cudaGetLastError();
}

}  // namespace kvq
