// Width-map decode: the host plan of a map, the shape check and the dispatch to the built
// instances of decode_var_kernel (decode_var.cuh; instances in decode_var_inst_gv*.cu).
#include <string.h>

#include <algorithm>
#include <vector>

#include "decode_var.cuh"

namespace kvq {
namespace var {

#define KVQ_VAR_DECL(NREP, GV, GK)                                                            \
  extern template cudaError_t launch_var<NREP, GV, GK>(const Dims&, const CacheBufs&,         \
                                                       const DecodeWork&, const VarPlan&,     \
                                                       const __half*, const Partials&, cudaStream_t);
#define KVQ_VAR_DECL_GV(GV)                                                                   \
  KVQ_VAR_DECL(1, GV, 16) KVQ_VAR_DECL(1, GV, 32) KVQ_VAR_DECL(1, GV, 64) KVQ_VAR_DECL(1, GV, 128) \
  KVQ_VAR_DECL(4, GV, 16) KVQ_VAR_DECL(4, GV, 32) KVQ_VAR_DECL(4, GV, 64) KVQ_VAR_DECL(4, GV, 128)
KVQ_VAR_DECL_GV(16)
KVQ_VAR_DECL_GV(32)
KVQ_VAR_DECL_GV(64)
KVQ_VAR_DECL_GV(128)
extern template cudaError_t launch_var<4, 32, 64, MapK3V2>(const Dims&, const CacheBufs&, const DecodeWork&,
                                                            const VarPlan&, const __half*, const Partials&,
                                                            cudaStream_t);
extern template cudaError_t launch_var<4, 64, 64, MapK8K2>(const Dims&, const CacheBufs&, const DecodeWork&,
                                                            const VarPlan&, const __half*, const Partials&,
                                                            cudaStream_t);

namespace {

// ----------------------------------------------------------------- host plan ----

struct Field {
  int ch, p, w;
};

uint32_t field_mask(const Field* f, int shift) {
  return f ? ((1u << f->w) - 1u) << (f->p + shift) : 0u;
}

// The couples of a key map.  Channel c (width w_c > 0, channels in order, packed LSB-first)
// sits at bit q_c = sum_{c' < c} w_c' of its row: word q_c / 32, byte (q_c / 8) mod 4, offset
// p = q_c mod 8 with p + w_c <= 8.  In each word the i-th fields of bytes 0 and 2 form register
// i of the first kind (masked in place), the i-th fields of bytes 1 and 3 register i of the second
// kind (masked after a shift by 8); couple i of the word is that pair of registers.
bool plan_keys(const Dims& d, VarPlan* vp) {
  std::vector<int> width;
  for (int i = 0; i < 4; ++i)
    for (int n = 0; n < d.kcnt[i]; ++n) width.push_back(8 >> i);
  if (static_cast<int>(width.size()) > kDK) return false;
  std::vector<std::vector<Field>> bytes(static_cast<size_t>(d.kw) * 4);
  int q = 0;
  for (int c = 0; c < static_cast<int>(width.size()); ++c) {
    const int wc = width[c];
    const Field f{c, q & 7, wc};
    if (f.p + wc > 8 || (q >> 3) >= d.kw * 4) return false;
    bytes[q >> 3].push_back(f);
    q += wc;
  }
  int n = 0;
  for (int wd = 0; wd < d.kw; ++wd) {
    const std::vector<Field>* by = &bytes[static_cast<size_t>(wd) * 4];
    const size_t cnt = std::max(std::max(by[0].size(), by[2].size()), std::max(by[1].size(), by[3].size()));
    for (size_t i = 0; i < cnt; ++i) {
      if (n >= kCouples) return false;
      const Field* f[4] = {i < by[0].size() ? &by[0][i] : nullptr, i < by[2].size() ? &by[2][i] : nullptr,
                           i < by[1].size() ? &by[1][i] : nullptr, i < by[3].size() ? &by[3][i] : nullptr};
      vp->kwo[n] = static_cast<uint32_t>(wd) * 4u;
      vp->kma[n] = field_mask(f[0], 0) | field_mask(f[1], 16);
      vp->kmb[n] = field_mask(f[2], 0) | field_mask(f[3], 16);
      for (int e = 0; e < 4; ++e) {
        vp->kch[n][e] = f[e] ? static_cast<unsigned char>(f[e]->ch) : kNone;
        vp->kpos[n][e] = f[e] ? static_cast<unsigned char>(f[e]->p) : 0;
      }
      ++n;
    }
  }
  for (int m = n; m < kCouples; ++m)
    for (int e = 0; e < 4; ++e) vp->kch[m][e] = kNone;
  vp->nks = (n + 3) / 4;
  return true;
}

bool make_plan(const Dims& d, VarPlan* vp) {
  memset(vp, 0, sizeof(*vp));
  if (!plan_keys(d, vp)) return false;
  if (d.nvg > 8) return false;
  // value groups: widths non-increasing over the channels, one width per group
  int bit = 0;
  for (int g = 0; g < d.nvg; ++g) {
    const int c = g * d.gv;
    int wdt = 0, first = 0;
    for (int i = 0; i < 4; ++i) {
      if (c < first + d.vcnt[i]) {
        wdt = 8 >> i;
        break;
      }
      first += d.vcnt[i];
    }
    vp->vbits[g] = wdt;
    vp->vbit0[g] = bit;
    bit += d.gv * wdt;
  }
  return bit <= d.vw * 32;
}


}  // namespace

bool supported(const Dims& d) {
  if (!d.var || d.dk != kDK || d.dv != kDV || (d.n_rep != 1 && d.n_rep != 4)) return false;
  if (d.gv != 16 && d.gv != 32 && d.gv != 64 && d.gv != 128) return false;
  if (d.gk != 16 && d.gk != 32 && d.gk != 64 && d.gk != 128) return false;
  VarPlan vp;
  if (!make_plan(d, &vp)) return false;
  const int stage = round128(var_stage_layout(d).bytes);
  return (kSmemPerCta - Smem::kStages) / stage >= 2 && (kSmemPerCta - Smem::kStages) / kRawStage >= 2 &&
         kWarps * 4 * kDV * 4 + kWarps * 4 * 8 <= kSmemPerCta - Smem::kStages;
}

namespace {

// The build-time instance of map M serves d when d has M's counts (its plan then has M's k-steps
// and row lengths).
template <class M>
bool map_matches(const Dims& d, const VarPlan& vp) {
  for (int i = 0; i < 4; ++i)
    if (d.kcnt[i] != M::kcnt(i) || d.vcnt[i] != M::vcnt(i)) return false;
  return vp.nks == M::NKS && d.kw == M::KW && d.vw == M::VW;
}

template <int NREP, int GV>
cudaError_t launch_gk(const Dims& d, const CacheBufs& c, const DecodeWork& w, const VarPlan& vp,
                      const __half* q, const Partials& p, cudaStream_t s) {
  switch (d.gk) {
    case 16: return launch_var<NREP, GV, 16>(d, c, w, vp, q, p, s);
    case 32: return launch_var<NREP, GV, 32>(d, c, w, vp, q, p, s);
    case 64: return launch_var<NREP, GV, 64>(d, c, w, vp, q, p, s);
    default: return launch_var<NREP, GV, 128>(d, c, w, vp, q, p, s);
  }
}

template <int NREP>
cudaError_t launch_gv(const Dims& d, const CacheBufs& c, const DecodeWork& w, const VarPlan& vp,
                      const __half* q, const Partials& p, cudaStream_t s) {
  switch (d.gv) {
    case 16: return launch_gk<NREP, 16>(d, c, w, vp, q, p, s);
    case 32: return launch_gk<NREP, 32>(d, c, w, vp, q, p, s);
    case 64: return launch_gk<NREP, 64>(d, c, w, vp, q, p, s);
    default: return launch_gk<NREP, 128>(d, c, w, vp, q, p, s);
  }
}

}  // namespace

cudaError_t launch(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                   const Partials& p, cudaStream_t s) {
  VarPlan vp;
  if (!supported(d) || !make_plan(d, &vp)) return cudaErrorNotSupported;
  if (d.n_rep == 4 && d.gk == 64 && d.gv == 32 && map_matches<MapK3V2>(d, vp))
    return launch_var<4, 32, 64, MapK3V2>(d, c, w, vp, q, p, s);
  if (d.n_rep == 4 && d.gk == 64 && d.gv == 64 && map_matches<MapK8K2>(d, vp))
    return launch_var<4, 64, 64, MapK8K2>(d, c, w, vp, q, p, s);
  return d.n_rep == 4 ? launch_gv<4>(d, c, w, vp, q, p, s) : launch_gv<1>(d, c, w, vp, q, p, s);
}

}  // namespace var

bool decode_var_supported(const Dims& d) { return var::supported(d); }

cudaError_t launch_decode_var(const Dims& d, const CacheBufs& c, const DecodeWork& w, const __half* q,
                              const Partials& p, cudaStream_t s) {
  return var::launch(d, c, w, q, p, s);
}

}  // namespace kvq
