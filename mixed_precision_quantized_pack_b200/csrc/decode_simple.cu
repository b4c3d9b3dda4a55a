// Generic decode-attention kernel on CUDA cores (any supported shape).
//
// Computes, for one (b, kv head) and one split of its tokens, the flash-decoding
// partial (m, l, o) of every query head sharing the kv head:
//   k_hat = code * s + z (key groups per channel, value groups per token), or the
//           fp16 copy for window and retained tokens ("LogQuant: Log-Distributed
//           2-Bit Quantization of KV Cache", §Méthodologie 2 and 3);
//   score = q . k_hat / sqrt(d_k) ("Thin Keys, Full Values", §2), kept in log2 units,
//           plus (U_h^T q) . z_hat for quantized tokens when the cache has a side code
//           ("HeadQ: Distortion visible par le modele et correction dans l'espace des
//           scores pour la quantification du cache KV", §3, step 3);
//   online softmax, o = sum_j 2^(score_j - m) v_hat_j.
// One warp per token: each lane holds d/32 channels, dot products reduce with
// warp shuffles.  The tensor-core kernel replaces this one on the shapes it
// supports; this one is the reference GPU path for everything else.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kMaxRep = 8;
constexpr int kMaxC = 8;      // d / 32, d <= 256
constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32)
decode_simple_kernel(Dims d, CacheBufs cb, DecodeWork w, const __half* __restrict__ q, Partials p) {
  __shared__ float sm_m[kWarps][kMaxRep];
  __shared__ float sm_l[kWarps][kMaxRep];
  __shared__ float sm_o[kWarps][kMaxRep][kMaxC * 32];
  __shared__ float sm_qt[kMaxRep][8];     // U_h^T q of each query head, times the score scale

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * d.Hkv + h;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nrep = d.n_rep, ck = d.dk / 32, cv = d.dv / 32;

  // query rows (lane holds channels lane + 32 j), rotated when the keys are, times the scale
  float qr[kMaxRep][kMaxC];
#pragma unroll
  for (int r = 0; r < kMaxRep; ++r) {
#pragma unroll
    for (int j = 0; j < kMaxC; ++j)
      qr[r][j] = (r < nrep && j < ck)
                     ? __half2float(q[(static_cast<size_t>(b) * d.Hq + h * nrep + r) * d.dk + lane + 32 * j])
                     : 0.0f;
    if (d.rot && r < nrep) {
      rotate_row_warp<kMaxC>(qr[r], ck, d.rot_signs, d.rot_inv_cq, lane);
#pragma unroll
      for (int j = 0; j < kMaxC; ++j) qr[r][j] = __half2float(__float2half_rn(qr[r][j]));
    }
#pragma unroll
    for (int j = 0; j < kMaxC; ++j) qr[r][j] *= w.score_scale;
  }
  float m[kMaxRep], l[kMaxRep], o[kMaxRep][kMaxC];
#pragma unroll
  for (int r = 0; r < kMaxRep; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.0f;
#pragma unroll
    for (int j = 0; j < kMaxC; ++j) o[r][j] = 0.0f;
  }

  if (d.sr) {
    // U_h^T q (of the rotated query, when keys are rotated), times the scale: warp 0
    if (warp == 0) {
      const float* u = cb.side_u + static_cast<size_t>(h) * d.dk * d.sr;
      for (int r = 0; r < nrep; ++r)
        for (int i = 0; i < d.sr; ++i) {
          float acc = 0.0f;
#pragma unroll
          for (int j = 0; j < kMaxC; ++j)
            if (j < ck) acc = fmaf(u[(lane + 32 * j) * d.sr + i], qr[r][j], acc);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
          if (lane == 0) sm_qt[r][i] = acc;
        }
    }
    __syncthreads();
  }

  const SeqWork sw = seq_work(w, b, d.gk, d.log_retain);   // this sequence's lengths
  const bool quant = split < w.splits_q;
  int begin, end;
  if (quant) {
    begin = static_cast<int>(static_cast<long long>(split) * sw.n_groups / w.splits_q) * d.gk;
    end = static_cast<int>(static_cast<long long>(split + 1) * sw.n_groups / w.splits_q) * d.gk;
  } else {
    const int f = split - w.splits_q;
    begin = static_cast<int>(static_cast<long long>(f) * sw.n_fp16 / w.splits_f);
    end = static_cast<int>(static_cast<long long>(f + 1) * sw.n_fp16 / w.splits_f);
  }
  const int perk = d.kb == 16 || d.var ? 1 : 32 / d.kb, perv = d.vb == 16 || d.var ? 1 : 32 / d.vb;
  const uint32_t maskk = (1u << (d.kb & 15)) - 1u, maskv = (1u << (d.vb & 15)) - 1u;
  // per-channel widths: each lane's channels' (word, shift, width), keys and values; a
  // dropped channel reads word 0 with an empty mask (its offset may be the row's end)
  uint32_t kvw[kMaxC], vvw[kMaxC];     // word index << 16 | shift << 8 | width
  auto pack_wsw = [](int wd, int off) -> uint32_t {
    return wd ? static_cast<uint32_t>(off / 32) << 16 | static_cast<uint32_t>(off % 32) << 8 | wd : 0u;
  };
#pragma unroll
  for (int j = 0; j < kMaxC; ++j) kvw[j] = vvw[j] = 0u;
  if (d.var) {
#pragma unroll
    for (int j = 0; j < kMaxC; ++j) {
      int wd = 0, off = 0;
      if (j < ck) channel_width(d.kcnt, lane + 32 * j, &wd, &off);
      kvw[j] = pack_wsw(wd, off);
      wd = off = 0;
      if (j < cv) channel_width(d.vcnt, lane + 32 * j, &wd, &off);
      vvw[j] = pack_wsw(wd, off);
    }
  }

  for (int i = begin + warp; i < end; i += kWarps) {
    float kh[kMaxC], vh[kMaxC];
    float zhat[8];                                              // side code, decoded
#pragma unroll
    for (int j = 0; j < 8; ++j) zhat[j] = 0.0f;
    if (quant) {
      // retained ({p < Q : p mod 2^floor(log2(Q - p)) == 0}): read from the fp16 list
      if (d.log_retain && (i & ((1 << (31 - __clz(sw.Q - i))) - 1)) == 0) continue;
      const bool tab_ok = KVQ_IN_BOUNDS(d, kSiteDecTable, i / d.gk, d.max_groups);
      size_t row = tab_ok ? group_row(d, cb.table, b, h, i / d.gk) + i % d.gk : 0;
      size_t gidx = tab_ok ? group_index(d, cb.table, b, h, i / d.gk) : 0;
      // (bounds-check builds) a token outside the buffers reads token 0 instead
      if (!KVQ_IN_BOUNDS(d, kSiteDecKCode, static_cast<long long>(row), quant_rows(d)) ||
          !KVQ_IN_BOUNDS(d, kSiteDecKMeta, static_cast<long long>(gidx), quant_groups(d)))
        row = gidx = 0;
      if (d.sr) {
        const uint8_t* zr = cb.zcode + row * d.zb;
        const uint32_t zrow = d.zb == 4 ? *reinterpret_cast<const uint32_t*>(zr)
                                        : *reinterpret_cast<const uint16_t*>(zr);
        const __half2* zs = cb.zsz + gidx * d.sr;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < d.sr) {
            const float2 sz = __half22float2(zs[j]);
            const uint32_t code = (zrow >> (j * d.sq)) & ((1u << d.sq) - 1u);
            zhat[j] = fmaf(static_cast<float>(code), sz.x, sz.y);
          }
      }
      const uint32_t* kr = cb.kcode + row * d.kw;
      const __half* ks = reinterpret_cast<const __half*>(cb.ksz) + gidx * 2 * d.dk;
      const uint32_t* vr = cb.vcode + row * d.vw;
      const __half2* vs = cb.vsz + row * d.nvg;
      if (d.var) {
        // per-channel widths: plain (scale, zero) pairs; dropped channels read 0
#pragma unroll
        for (int j = 0; j < kMaxC; ++j) {
          kh[j] = 0.0f;
          vh[j] = 0.0f;
          if (j < ck) {
            const int ch = lane + 32 * j;
            const uint32_t code = (kr[kvw[j] >> 16] >> ((kvw[j] >> 8) & 31u)) & ((1u << (kvw[j] & 15u)) - 1u);
            kh[j] = fmaf(static_cast<float>(code), __half2float(ks[2 * ch]), __half2float(ks[2 * ch + 1]));
          }
          if (j < cv) {
            const int ch = lane + 32 * j;
            const uint32_t code = (vr[vvw[j] >> 16] >> ((vvw[j] >> 8) & 31u)) & ((1u << (vvw[j] & 15u)) - 1u);
            const float2 sz = __half22float2(vs[ch / d.gv]);
            vh[j] = fmaf(static_cast<float>(code), sz.x, sz.y);
          }
        }
      } else {
#pragma unroll
      for (int j = 0; j < kMaxC; ++j) {
        kh[j] = 0.0f;
        vh[j] = 0.0f;
        if (j < ck) {
          const int ch = lane + 32 * j;
          const uint32_t code = (kr[ch / perk] >> ((ch % perk) * d.kb)) & maskk;
          // (scale, zero) of channel ch in the group's paired, quarter-interleaved block
          const int kwords = d.dk / perk, kq = kwords % 4 == 0 ? kwords / 4 : 0;
          const int kwd = ch / perk, kpos = kq ? (kwd % kq) * 4 + kwd / kq : kwd;
          const int slot = kpos * 2 * perk + (ch % perk % (perk / 2)) * 2 + (ch % perk) / (perk / 2);
          kh[j] = fmaf(static_cast<float>(code), __half2float(ks[slot]), __half2float(ks[slot + perk]));
        }
        if (j < cv) {
          const int ch = lane + 32 * j;
          const uint32_t code = (vr[ch / perv] >> ((ch % perv) * d.vb)) & maskv;
          const float2 sz = __half22float2(vs[ch / d.gv]);
          vh[j] = fmaf(static_cast<float>(code), sz.x, sz.y);
        }
      }
      }
    } else {
      const __half *kp, *vp;
      if (i < sw.n_ret) {
        size_t s = static_cast<size_t>(bh) * kMaxRetained + i;
        if (!KVQ_IN_BOUNDS(d, kSiteDecRetK, static_cast<long long>(s), ret_rows(d))) s = 0;
        kp = cb.ret_k + s * d.dk;
        vp = cb.ret_v + s * d.dv;
      } else {
        const int pos = sw.Q + (i - sw.n_ret);
        size_t s = static_cast<size_t>(bh) * d.cap + pos % d.cap;
        if (!KVQ_IN_BOUNDS(d, kSiteDecWinK, static_cast<long long>(s), win_rows(d))) s = 0;
        kp = cb.win_k + s * d.dk;
        vp = cb.win_v + s * d.dv;
      }
#pragma unroll
      for (int j = 0; j < kMaxC; ++j) {
        kh[j] = j < ck ? __half2float(kp[lane + 32 * j]) : 0.0f;
        vh[j] = j < cv ? __half2float(vp[lane + 32 * j]) : 0.0f;
      }
    }
#pragma unroll
    for (int r = 0; r < kMaxRep; ++r) {
      if (r >= nrep) break;
      float s = 0.0f;
#pragma unroll
      for (int j = 0; j < kMaxC; ++j) s = fmaf(qr[r][j], kh[j], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (d.sr) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < d.sr) s = fmaf(sm_qt[r][j], zhat[j], s);
      }
      const float mn = fmaxf(m[r], s);
      const float alpha = exp2f(m[r] - mn);
      const float pe = exp2f(s - mn);
      l[r] = fmaf(l[r], alpha, pe);
#pragma unroll
      for (int j = 0; j < kMaxC; ++j) o[r][j] = fmaf(o[r][j], alpha, pe * vh[j]);
      m[r] = mn;
    }
  }

  // merge the warps of this CTA, then write one partial per query head
#pragma unroll
  for (int r = 0; r < kMaxRep; ++r) {
    if (r < nrep) {
      if (lane == 0) {
        sm_m[warp][r] = m[r];
        sm_l[warp][r] = l[r];
      }
#pragma unroll
      for (int j = 0; j < kMaxC; ++j)
        if (j < cv) sm_o[warp][r][lane + 32 * j] = o[r][j];
    }
  }
  __syncthreads();
  for (int r = 0; r < nrep; ++r) {
    float M = -INFINITY;
    for (int k = 0; k < kWarps; ++k) M = fmaxf(M, sm_m[k][r]);
    const size_t part = (static_cast<size_t>(b) * d.Hq + h * nrep + r) * w.splits + split;
    if (!KVQ_IN_BOUNDS(d, kSiteDecPartial, static_cast<long long>(part), static_cast<long long>(d.B) * d.Hq * w.splits))
      continue;
    float wk[kWarps];
    float Lsum = 0.0f;
    for (int k = 0; k < kWarps; ++k) {
      wk[k] = (M == -INFINITY || sm_m[k][r] == -INFINITY) ? 0.0f : exp2f(sm_m[k][r] - M);
      Lsum = fmaf(wk[k], sm_l[k][r], Lsum);
    }
    if (threadIdx.x == 0) p.ml[part] = make_float2(M, Lsum);
    for (int c = threadIdx.x; c < d.dv; c += blockDim.x) {
      float acc = 0.0f;
      for (int k = 0; k < kWarps; ++k) acc = fmaf(wk[k], sm_o[k][r][c], acc);
      p.o[part * d.dv + c] = acc;
    }
  }
}

}  // namespace

cudaError_t launch_decode_simple(const Dims& d, const CacheBufs& c, const DecodeWork& w,
                                 const __half* q, const Partials& p, cudaStream_t s) {
  dim3 grid(w.splits, d.Hkv, d.B);
  decode_simple_kernel<<<grid, kWarps * 32, 0, s>>>(d, c, w, q, p);
  return cudaGetLastError();
}

}  // namespace kvq
