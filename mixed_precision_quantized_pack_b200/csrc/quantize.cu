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
#include "kvq_internal.cuh"

namespace kvq {
namespace {

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

// One thread per (key group, channel); blockDim = (dk, groups per block).  The
// 32/BITS lanes holding the channels of one packed word OR their codes together.
// ROT: the source keys are unrotated; the block's warps first rotate the rows of its
// groups into shared memory ([groups per block][gk][dk] fp16) and the quantizer reads
// those.
template <int BITS, bool ROT>
__global__ void quantize_keys_kernel(const __half* __restrict__ src, int src_rows, int dk,
                                     int gk, int g_begin, int n_groups, int lcap,
                                     uint32_t* __restrict__ kcode, __half2* __restrict__ ksz,
                                     const int* __restrict__ table, Dims d) {
  extern __shared__ __half sm_rot[];
  const int c = threadIdx.x;
  const int gi = blockIdx.x * blockDim.y + threadIdx.y;
  const int bh = blockIdx.y;
  const size_t base = static_cast<size_t>(bh) * src_rows;
  if constexpr (ROT) {
    const int tid = threadIdx.y * blockDim.x + threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x * blockDim.y / 32;
    for (int rr = warp; rr < blockDim.y * gk; rr += nwarps) {
      const int yy = rr / gk, t = rr % gk;
      const int gg = blockIdx.x * blockDim.y + yy;
      if (gg >= n_groups) continue;                  // uniform per warp
      const int row = ((g_begin + gg) * gk + t) % src_rows;
      float x[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) x[m] = m < dk / 32 ? __half2float(src[(base + row) * dk + lane + 32 * m]) : 0.0f;
      rotate_row_warp<8>(x, dk / 32, d.rot_signs, d.rot_inv_ck, lane);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (m < dk / 32) sm_rot[(static_cast<size_t>(yy) * gk + t) * dk + lane + 32 * m] = __float2half_rn(x[m]);
    }
    __syncthreads();
  }
  if (gi >= n_groups) return;                       // uniform per warp: dk % 32 == 0
  const int g = g_begin + gi;
  // key t of the group, channel c
  auto key = [&](int t) -> float {
    if constexpr (ROT) return __half2float(sm_rot[(static_cast<size_t>(threadIdx.y) * gk + t) * dk + c]);
    const int row = (g * gk + t) % src_rows;
    return __half2float(src[(base + row) * dk + c]);
  };
  float mn = INFINITY, mx = -INFINITY;
  for (int t = 0; t < gk; ++t) {
    const float x = key(t);
    mn = fminf(mn, x);
    mx = fmaxf(mx, x);
  }
  const GroupParams gp = group_params<BITS>(mn, mx);
  {
    // the group's block of 2*dk fp16: per packed word w, the scales of channels
    // (w*per + i, w*per + i + per/2) for i < per/2, then their zeros in the same order;
    // the words' blocks quarter-interleaved when 4 divides the words per row
    constexpr int per_w = 32 / BITS, half_w = 16 / BITS;
    const int words = dk / per_w, quarter = words % 4 == 0 ? words / 4 : 0;
    const int wd = c / per_w, r = c % per_w;
    const int pos = quarter ? (wd % quarter) * 4 + wd / quarter : wd;
    const int slot = pos * 2 * per_w + (r % half_w) * 2 + r / half_w;
    __half* blk = reinterpret_cast<__half*>(ksz) + group_index(d, table, bh / d.Hkv, bh % d.Hkv, g) * 2 * dk;
    blk[slot] = __low2half(gp.sz);
    blk[slot + per_w] = __high2half(gp.sz);
  }
  constexpr int per = 32 / BITS;                    // channels per word
  const int words = dk / per;
  const size_t row0 = group_row(d, table, bh / d.Hkv, bh % d.Hkv, g);
  for (int t = 0; t < gk; ++t) {
    const float x = key(t);
    uint32_t part = quant_code<BITS>(x, gp) << ((c % per) * BITS);
#pragma unroll
    for (int off = 1; off < per; off <<= 1) part |= __shfl_xor_sync(0xffffffffu, part, off);
    if (c % per == 0)
      kcode[(row0 + t) * words + c / per] = part;
  }
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
      for (int m = 0; m < 8; ++m) x[m] = m < dk / 32 ? __half2float(src[(base + row) * dk + lane + 32 * m]) : 0.0f;
      rotate_row_warp<8>(x, dk / 32, d.rot_signs, d.rot_inv_ck, lane);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (m < dk / 32) e[t * es + lane + 32 * m] = __half2float(__float2half_rn(x[m]));
    }
    __syncthreads();
  }
  for (int idx = threadIdx.x; idx < gk * dk; idx += blockDim.x) {
    const int t = idx / dk, c = idx % dk;
    float x;
    if constexpr (ROT) {
      x = e[t * es + c];
    } else {
      const int row = (g * gk + t) % src_rows;
      x = __half2float(src[(base + row) * dk + c]);
    }
    const uint32_t w = kcode[(row0 + t) * words + c / per];
    const uint32_t code = (w >> ((c % per) * kb)) & ((1u << kb) - 1u);
    // the channel's (scale, zero) slots in the group's paired, quarter-interleaved block
    const int wd = c / per, r = c % per;
    const int pos = quarter ? (wd % quarter) * 4 + wd / quarter : wd;
    const int slot = pos * 2 * per + (r % half) * 2 + r / half;
    const float kh = __fadd_rn(__fmul_rn(static_cast<float>(code), __half2float(blk[slot])),
                               __half2float(blk[slot + per]));
    e[t * es + c] = __fsub_rn(x, kh);
  }
  for (int idx = threadIdx.x; idx < dk * sr; idx += blockDim.x)
    u[idx] = side_u[static_cast<size_t>(h) * dk * sr + idx];
  __syncthreads();
  for (int idx = threadIdx.x; idx < gk * sr; idx += blockDim.x) {
    const int t = idx / sr, i = idx % sr;
    float acc = 0.0f;
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
    uint8_t* dst = zcode + (row0 + t) * zb;
    if (zb == 4)
      *reinterpret_cast<uint32_t*>(dst) = row;
    else
      *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(row);
  }
}

// One thread per (kv row, token, value group).  gv is a multiple of 8 and of 32/BITS.
template <int BITS>
__global__ void quantize_values_kernel(const __half* __restrict__ src, int src_rows, int dv,
                                       int gv, int t_begin, int n_tokens, int nbh, int lcap,
                                       uint32_t* __restrict__ vcode, __half2* __restrict__ vsz,
                                       const int* __restrict__ table, Dims d) {
  const int nvg = dv / gv;
  const long long total = static_cast<long long>(nbh) * n_tokens * nvg;
  constexpr int per = 32 / BITS;
  const int vw = dv / per;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int gidx = static_cast<int>(idx % nvg);
    const long long r = idx / nvg;
    const int t = t_begin + static_cast<int>(r % n_tokens);
    const int bh = static_cast<int>(r / n_tokens);
    const int row = t % src_rows;
    const __half* x = src + (static_cast<size_t>(bh) * src_rows + row) * dv + gidx * gv;
    float mn = INFINITY, mx = -INFINITY;
    for (int j = 0; j < gv; j += 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(x + j);
      const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        mn = fminf(mn, fminf(f.x, f.y));
        mx = fmaxf(mx, fmaxf(f.x, f.y));
      }
    }
    const GroupParams gp = group_params<BITS>(mn, mx);
    const size_t vrow = group_row(d, table, bh / d.Hkv, bh % d.Hkv, t / d.gk) + t % d.gk;
    vsz[vrow * nvg + gidx] = gp.sz;
    uint32_t* out = vcode + vrow * vw + gidx * (gv / per);
    for (int w = 0; w < gv / per; ++w) {
      uint32_t word = 0;
      for (int k = 0; k < per; ++k) {
        const float xv = __half2float(x[w * per + k]);
        word |= quant_code<BITS>(xv, gp) << (k * BITS);
      }
      out[w] = word;
    }
  }
}

// ---- per-channel widths ("Attention-Aware Transform Coding (AATC)", §Méthodologie,
// Allocation de Bits): channel c has its own width (8, 4, 2, 1 or 0 = dropped), widths
// non-increasing over the channels; the same quantizer with that many bits; a row packs
// the codes channel after channel, channel c at the sum of the widths before it.

// One CTA of dk threads per (key group, b * kv head): thread c quantizes channel c over the
// group's gk tokens; the codes are ORed into the group's rows in shared memory
// ([gk][kw] u32, at most 128 x 64 words), which are then written out whole.  The group's
// (scale, zero) are stored plainly, [dk][2]; a dropped channel stores (0, 0).
__global__ void quantize_keys_var_kernel(const __half* __restrict__ src, int src_rows, int g_begin,
                                         uint32_t* __restrict__ kcode, __half2* __restrict__ ksz,
                                         const int* __restrict__ table, Dims d) {
  extern __shared__ uint32_t sm_rows[];
  const int c = threadIdx.x, nt = blockDim.x;
  const int g = g_begin + blockIdx.x, bh = blockIdx.y;
  const int gk = d.gk, kw = d.kw;
  for (int i = c; i < gk * kw; i += nt) sm_rows[i] = 0u;
  __syncthreads();
  int width, offset;
  channel_width(d.kcnt, c, &width, &offset);
  const size_t base = static_cast<size_t>(bh) * src_rows;
  auto key = [&](int t) { return __half2float(src[(base + (g * gk + t) % src_rows) * d.dk + c]); };
  const size_t gidx = group_index(d, table, bh / d.Hkv, bh % d.Hkv, g);
  __half2 sz = __floats2half2_rn(0.0f, 0.0f);
  if (width) {
    float mn = INFINITY, mx = -INFINITY;
    for (int t = 0; t < gk; ++t) {
      const float x = key(t);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    const GroupParams gp = group_params_b(mn, mx, width);
    sz = gp.sz;
    for (int t = 0; t < gk; ++t)
      atomicOr(&sm_rows[t * kw + offset / 32], quant_code_b(key(t), gp, width) << (offset % 32));
  }
  ksz[gidx * d.dk + c] = sz;
  __syncthreads();
  const size_t row0 = group_row(d, table, bh / d.Hkv, bh % d.Hkv, g);
  for (int i = c; i < gk * kw; i += nt) kcode[row0 * kw + i] = sm_rows[i];
}

// One CTA of dv threads per 16 consecutive (b * kv head, token) rows: thread c holds channel
// c; a value group's min and max are reduced over its gv channels (shuffles within a warp,
// then shared memory across warps when gv > 32), and the codes are ORed into the row in
// shared memory ([kw] u32) before it is written out.
__global__ void quantize_values_var_kernel(const __half* __restrict__ src, int src_rows, int t_begin,
                                           int n_tokens, uint32_t* __restrict__ vcode,
                                           __half2* __restrict__ vsz, const int* __restrict__ table,
                                           Dims d) {
  __shared__ uint32_t sm_row[64];
  __shared__ float sm_mn[8], sm_mx[8];
  const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
  const int gv = d.gv, vw = d.vw;
  int width, offset;
  channel_width(d.vcnt, c, &width, &offset);
  const long long rows = static_cast<long long>(d.B) * d.Hkv * n_tokens;
  for (long long r = static_cast<long long>(blockIdx.x) * 16; r < rows; r += static_cast<long long>(gridDim.x) * 16) {
    for (int rr = 0; rr < 16 && r + rr < rows; ++rr) {
      const long long rowi = r + rr;
      const int t = t_begin + static_cast<int>(rowi % n_tokens);
      const int bh = static_cast<int>(rowi / n_tokens);
      for (int i = c; i < vw; i += blockDim.x) sm_row[i] = 0u;
      const float x = __half2float(src[(static_cast<size_t>(bh) * src_rows + t % src_rows) * d.dv + c]);
      float mn = x, mx = x;
      const int span = gv < 32 ? gv : 32;
      for (int off = 1; off < span; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      }
      if (gv > 32) {
        if (lane == 0) {
          sm_mn[warp] = mn;
          sm_mx[warp] = mx;
        }
        __syncthreads();
        const int w0 = (c / gv) * (gv / 32);
        mn = sm_mn[w0];
        mx = sm_mx[w0];
        for (int k = 1; k < gv / 32; ++k) {
          mn = fminf(mn, sm_mn[w0 + k]);
          mx = fmaxf(mx, sm_mx[w0 + k]);
        }
      }
      __syncthreads();        // the row is cleared; the warps' extremes are read
      const size_t vrow = group_row(d, table, bh / d.Hkv, bh % d.Hkv, t / d.gk) + t % d.gk;
      __half2 sz = __floats2half2_rn(0.0f, 0.0f);
      if (width) {
        const GroupParams gp = group_params_b(mn, mx, width);
        sz = gp.sz;
        atomicOr(&sm_row[offset / 32], quant_code_b(x, gp, width) << (offset % 32));
      }
      if (c % gv == 0) vsz[vrow * d.nvg + c / gv] = sz;
      __syncthreads();
      for (int i = c; i < vw; i += blockDim.x) vcode[vrow * vw + i] = sm_row[i];
      __syncthreads();        // before the next row clears sm_row and sm_mn / sm_mx
    }
  }
}

// dst[bh][(dst_base + i) % dst_rows] = src[bh][(src_base + i) % src_rows], i < n, 16 B at a time.
__global__ void copy_rows_kernel(const __half* __restrict__ src, int src_rows, int src_base,
                                 __half* __restrict__ dst, int dst_rows, int dst_base, int n,
                                 int d, int nbh) {
  const int vec = d / 8;
  const long long total = static_cast<long long>(nbh) * n * vec;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(idx % vec);
    const long long r = idx / vec;
    const int i = static_cast<int>(r % n);
    const int bh = static_cast<int>(r / n);
    const int sr = (src_base + i) % src_rows;
    const int dr = (dst_base + i) % dst_rows;
    const uint4* s = reinterpret_cast<const uint4*>(src + (static_cast<size_t>(bh) * src_rows + sr) * d);
    uint4* t = reinterpret_cast<uint4*>(dst + (static_cast<size_t>(bh) * dst_rows + dr) * d);
    t[e] = s[e];
  }
}

// Append: the new token's key and value rows of every (b, kv head) into the window slot of
// sequence b (none when it is -1), 16 B per thread; k null: values only.
__global__ void append_token_kernel(const __half* __restrict__ k, const __half* __restrict__ v,
                                    __half* __restrict__ win_k, __half* __restrict__ win_v,
                                    SlotMap slots, int hkv, int cap, int dk, int dv, int nbh) {
  const int vk = dk / 8, vv = dv / 8;
  const int total = nbh * (vk + vv);
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += gridDim.x * blockDim.x) {
    const int bh = idx / (vk + vv), e = idx % (vk + vv);
    const int slot = slots.slot[bh / hkv];
    if (slot < 0) continue;
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
                                     __half* __restrict__ ret_k, __half* __restrict__ ret_v) {
  const int bh = blockIdx.x;
  for (int j = 0; j < ret.n; ++j) {
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
                                       __half* ret_v) {
  const int bh = blockIdx.x;
  for (int i = 0; i < up.n; ++i) {
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
__global__ void table_writes_kernel(int* __restrict__ table, TableWrites tw) {
  for (int i = threadIdx.x; i < tw.n; i += blockDim.x) table[tw.idx[i]] = tw.page[i];
}

inline int grid_for(long long items, int block) {
  long long g = (items + block - 1) / block;
  if (g > 148LL * 32) g = 148LL * 32;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

template <bool ROT>
cudaError_t launch_quantize_keys_t(const Dims& d, const __half* src, int src_rows, int g_begin,
                                   int n_groups, uint32_t* kcode, __half2* ksz, const int* table,
                                   cudaStream_t s) {
  const int gpb = d.dk >= 256 ? 1 : 256 / d.dk;
  dim3 block(d.dk, gpb);
  dim3 grid((n_groups + gpb - 1) / gpb, d.B * d.Hkv);
  const size_t smem = ROT ? static_cast<size_t>(gpb) * d.gk * d.dk * 2 : 0;
  auto kern = d.kb == 2 ? quantize_keys_kernel<2, ROT>
            : d.kb == 4 ? quantize_keys_kernel<4, ROT> : quantize_keys_kernel<8, ROT>;
  if (d.kb != 2 && d.kb != 4 && d.kb != 8) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, block, smem, s>>>(src, src_rows, d.dk, d.gk, g_begin, n_groups, d.lcap, kcode, ksz, table, d);
  return cudaGetLastError();
}

cudaError_t launch_quantize_keys(const Dims& d, const __half* src, int src_rows, int g_begin,
                                 int n_groups, uint32_t* kcode, __half2* ksz, const int* table,
                                 bool rotate, cudaStream_t s) {
  if (n_groups <= 0) return cudaSuccess;
  if (d.var) {
    if (rotate) return cudaErrorInvalidValue;
    const int smem = d.gk * d.kw * 4;       // <= 128 x 64 words
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(quantize_keys_var_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
    }
    quantize_keys_var_kernel<<<dim3(n_groups, d.B * d.Hkv), d.dk, smem, s>>>(src, src_rows, g_begin,
                                                                              kcode, ksz, table, d);
    return cudaGetLastError();
  }
  return rotate ? launch_quantize_keys_t<true>(d, src, src_rows, g_begin, n_groups, kcode, ksz, table, s)
                : launch_quantize_keys_t<false>(d, src, src_rows, g_begin, n_groups, kcode, ksz, table, s);
}

cudaError_t launch_table_writes(int* table, const TableWrites& tw, cudaStream_t s) {
  if (tw.n <= 0) return cudaSuccess;
  table_writes_kernel<<<1, 256, 0, s>>>(table, tw);
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
  if (d.var) {
    const long long rows = static_cast<long long>(nbh) * n_tokens;
    const long long blocks = (rows + 15) / 16;
    const int grid = static_cast<int>(blocks < 148 * 16 ? blocks : 148 * 16);
    quantize_values_var_kernel<<<grid, d.dv, 0, s>>>(src, src_rows, t_begin, n_tokens, vcode, vsz, table, d);
    return cudaGetLastError();
  }
  const long long items = static_cast<long long>(nbh) * n_tokens * d.nvg;
  const int block = 256;
  const int grid = grid_for(items, block);
  switch (d.vb) {
    case 2: quantize_values_kernel<2><<<grid, block, 0, s>>>(src, src_rows, d.dv, d.gv, t_begin, n_tokens, nbh, d.lcap, vcode, vsz, table, d); break;
    case 4: quantize_values_kernel<4><<<grid, block, 0, s>>>(src, src_rows, d.dv, d.gv, t_begin, n_tokens, nbh, d.lcap, vcode, vsz, table, d); break;
    case 8: quantize_values_kernel<8><<<grid, block, 0, s>>>(src, src_rows, d.dv, d.gv, t_begin, n_tokens, nbh, d.lcap, vcode, vsz, table, d); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_copy_rows(const __half* src, int src_rows, int src_base, __half* dst,
                             int dst_rows, int dst_base, int n, int d, int nbh, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const long long items = static_cast<long long>(nbh) * n * (d / 8);
  const int block = 256;
  copy_rows_kernel<<<grid_for(items, block), block, 0, s>>>(src, src_rows, src_base, dst, dst_rows,
                                                            dst_base, n, d, nbh);
  return cudaGetLastError();
}

cudaError_t launch_append_token(const Dims& d, const __half* k, const __half* v, __half* win_k,
                                __half* win_v, const SlotMap& slots, cudaStream_t s) {
  const int nbh = d.B * d.Hkv;
  const int total = nbh * (d.dk + d.dv) / 8;
  const int block = 256;
  append_token_kernel<<<(total + block - 1) / block, block, 0, s>>>(
      d.rot ? nullptr : k, v, win_k, win_v, slots, d.Hkv, d.cap, d.dk, d.dv, nbh);
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
  copy_retained_kernel<<<d.B * d.Hkv, 64, 0, s>>>(k, v, L, d.dk, d.dv, ret, ret_k, ret_v);
  return cudaGetLastError();
}

cudaError_t launch_update_retained(const Dims& d, const RetUpdate& up, __half* win_k,
                                   __half* win_v, __half* ret_k, __half* ret_v, cudaStream_t s) {
  if (up.n <= 0) return cudaSuccess;
  const int threads = ((d.dk > d.dv ? d.dk : d.dv) / 8 + 31) / 32 * 32;
  update_retained_kernel<<<d.B * d.Hkv, threads, 0, s>>>(up, d.cap, d.dk, d.dv, win_k, win_v,
                                                          ret_k, ret_v);
  return cudaGetLastError();
}

}  // namespace kvq
