// C ABI of libkvq: argument checks, buffer sizes, the host-side cache state
// (length L, quantized prefix Q, retained positions), the split planner and the
// kernel launches.  All state the kernels need is known on the host from the
// length alone, so no call ever waits for the device.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "../../include/kvq.h"
#include "kvq_internal.cuh"

struct kvq_cache {
  kvq::Dims d;
  kvq_buffers buf;
  std::vector<int> L;   // tokens of each sequence (0: empty)
  std::vector<int> Q;   // quantized prefix of each sequence (its retained set follows from it)
  std::vector<int> table;   // paged: host copy of the block table [B][max_groups]
  std::vector<int> free_pages;   // paged: pages not in use, the next one handed out last
  std::vector<int> held;         // paged: pages of each sequence, its table entries [0, held)
  int sm_count;
  int kernel;     // KVQ_KERNEL_*
  int centering;  // KVQ_CENTER_*
  bool stall_next;  // test hook armed by kvq_debug_stall_next_decode
  bool uniform() const {
    for (size_t b = 1; b < L.size(); ++b)
      if (L[b] != L[0]) return false;
    return true;
  }
  bool ready() const {   // every sequence holds at least one token
    for (int x : L)
      if (x < 1) return false;
    return true;
  }
};

namespace kvq {

#ifdef KVQ_DEBUG
// The bounds-check build's record of failed checks: one per device that loads the library
// (zero at load), found by the kernels through Dims::dbg.
static __device__ DebugRecord g_debug_record;
#endif

size_t workspace_bytes(const Dims& d, int splits) {
  const size_t rows = static_cast<size_t>(d.B) * d.Hq * splits;
  const size_t ml = (rows * sizeof(float2) + 255) / 256 * 256;
  return 256 + ml + rows * d.dv * sizeof(float);
}

Partials workspace_views(const Dims& d, int splits, void* ws) {
  const size_t rows = static_cast<size_t>(d.B) * d.Hq * splits;
  const size_t ml = (rows * sizeof(float2) + 255) / 256 * 256;
  char* base = static_cast<char*>(ws);
  Partials p;
  p.status = reinterpret_cast<unsigned int*>(base);
  p.ml = reinterpret_cast<float2*>(base + 256);
  p.o = reinterpret_cast<float*>(base + 256 + ml);
  return p;
}

}  // namespace kvq

namespace {

bool is_pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks a configuration and derives the sizes the kernels use.
int make_dims(const kvq_config* c, kvq::Dims* d) {
  if (!c || !d) return KVQ_ERR_INVALID_ARG;
  if (c->batch < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1 || c->max_context < 1 ||
      c->window < 0 || (c->log_retain != 0 && c->log_retain != 1))
    return KVQ_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads != 0) return KVQ_ERR_UNSUPPORTED;
  const int n_rep = c->n_q_heads / c->n_kv_heads;
  if (n_rep > 8) return KVQ_ERR_UNSUPPORTED;
  if (!is_pow2_in(c->d_k, 32, 256) || !is_pow2_in(c->d_v, 32, 256)) return KVQ_ERR_UNSUPPORTED;
  const bool raw = c->k_bits == 16 || c->v_bits == 16;
  const bool var = c->k_bits == 0 || c->v_bits == 0;
  int kcnt[4] = {0, 0, 0, 0}, vcnt[4] = {0, 0, 0, 0}, kbits = 0, vbits = 0;
  if (var) {
    // per-channel widths: both maps, each in {0, 1, 2, 4, 8} and non-increasing; a value
    // group's channels share one width
    if (c->k_bits != 0 || c->v_bits != 0) return KVQ_ERR_UNSUPPORTED;
    if (!is_pow2_in(c->group_k, 16, 128)) return KVQ_ERR_UNSUPPORTED;
    if (c->group_v < 8 || c->group_v > c->d_v || c->d_v % c->group_v != 0 || c->group_v % 8 != 0)
      return KVQ_ERR_UNSUPPORTED;
    auto class_of = [](int w) { return w == 8 ? 0 : w == 4 ? 1 : w == 2 ? 2 : w == 1 ? 3 : w == 0 ? 4 : -1; };
    auto read_map = [&](const unsigned char* wmap, int n, int* cnt, int* bits) {
      int prev = 0;
      for (int i = 0; i < n; ++i) {
        const int k = class_of(wmap[i]);
        if (k < 0 || k < prev) return false;
        prev = k;
        if (k < 4) ++cnt[k];
        *bits += wmap[i];
      }
      return true;
    };
    if (!read_map(c->k_widths, c->d_k, kcnt, &kbits) || !read_map(c->v_widths, c->d_v, vcnt, &vbits))
      return KVQ_ERR_UNSUPPORTED;
    for (int g = 0; g < c->d_v; g += c->group_v)
      for (int i = 1; i < c->group_v; ++i)
        if (c->v_widths[g + i] != c->v_widths[g]) return KVQ_ERR_UNSUPPORTED;
    if (c->side_rank != 0 || c->rot_keys != 0) return KVQ_ERR_UNSUPPORTED;
  } else if (raw) {
    if (c->k_bits != 16 || c->v_bits != 16) return KVQ_ERR_UNSUPPORTED;
  } else {
    auto okb = [](int b) { return b == 2 || b == 4 || b == 8; };
    if (!okb(c->k_bits) || !okb(c->v_bits)) return KVQ_ERR_UNSUPPORTED;
    if (!is_pow2_in(c->group_k, 16, 128)) return KVQ_ERR_UNSUPPORTED;
    if (c->group_v < 8 || c->group_v > c->d_v || c->d_v % c->group_v != 0 ||
        c->group_v % 8 != 0 || (c->group_v * c->v_bits) % 32 != 0)
      return KVQ_ERR_UNSUPPORTED;
  }
  // side code: rank 4 or 8, 4 or 8 bits, one 2- or 4-byte row per token, quantized keys
  if (c->side_rank != 0) {
    if (raw) return KVQ_ERR_UNSUPPORTED;
    if (c->side_rank != 4 && c->side_rank != 8) return KVQ_ERR_UNSUPPORTED;
    if (c->side_bits != 4 && c->side_bits != 8) return KVQ_ERR_UNSUPPORTED;
    const int row_bits = c->side_rank * c->side_bits;
    if (row_bits != 16 && row_bits != 32) return KVQ_ERR_UNSUPPORTED;
  }
  if (c->rot_keys != 0 && c->rot_keys != 1) return KVQ_ERR_INVALID_ARG;
  if (c->paged != 0 && c->paged != 1) return KVQ_ERR_INVALID_ARG;
  if (c->paged) {
    if (raw) return KVQ_ERR_UNSUPPORTED;
    if (c->n_pages < 1) return KVQ_ERR_INVALID_ARG;
    if (static_cast<long long>(c->n_pages) * c->n_kv_heads * c->group_k >= (1LL << 30))
      return KVQ_ERR_UNSUPPORTED;
  }
  // every element index must fit comfortably in 64 bits and every position in int
  const long long lcap = raw ? c->max_context
                             : (static_cast<long long>(c->max_context) + c->group_k - 1) /
                                   c->group_k * c->group_k;
  if (lcap > (1LL << 30)) return KVQ_ERR_UNSUPPORTED;
  // group indices (b, h, g) of an unpaged cache fit in 31 bits
  if (!raw && static_cast<long long>(c->batch) * c->n_kv_heads * (lcap / c->group_k) >= (1LL << 31))
    return KVQ_ERR_UNSUPPORTED;
  kvq::Dims x;
  x.B = c->batch;
  x.Hq = c->n_q_heads;
  x.Hkv = c->n_kv_heads;
  x.n_rep = n_rep;
  x.dk = c->d_k;
  x.dv = c->d_v;
  x.kb = c->k_bits;
  x.vb = c->v_bits;
  x.gk = raw ? 1 : c->group_k;
  x.gv = raw ? c->d_v : c->group_v;
  x.R = c->window;
  x.log_retain = raw ? 0 : c->log_retain;
  x.max_context = c->max_context;
  x.lcap = static_cast<int>(lcap);
  x.paged = c->paged;
  x.n_pages = c->paged ? c->n_pages : 0;
  x.sm_count = 148;
  x.dbg = nullptr;
  x.max_groups = static_cast<int>(lcap / x.gk);
  x.cap = raw ? c->max_context : c->window + c->group_k;
  x.kw = raw ? 0 : var ? std::max(1, (kbits + 31) / 32) : c->d_k * c->k_bits / 32;
  x.vw = raw ? 0 : var ? std::max(1, (vbits + 31) / 32) : c->d_v * c->v_bits / 32;
  x.var = var ? 1 : 0;
  for (int i = 0; i < 4; ++i) {
    x.kcnt[i] = kcnt[i];
    x.vcnt[i] = vcnt[i];
  }
  x.nvg = raw ? 1 : c->d_v / c->group_v;
  x.sr = c->side_rank;
  x.sq = c->side_rank ? c->side_bits : 0;
  x.zb = c->side_rank * x.sq / 8;
  x.rot = c->rot_keys;
  for (int i = 0; i < 8; ++i) x.rot_signs[i] = c->rot_keys ? c->rot_signs[i] : 0u;
  // c_k = 2^ceil(log2(d_k)/2), c_q = d_k / c_k: both powers of two, so 1/c is exact
  int log2d = 0;
  while ((1 << log2d) < x.dk) ++log2d;
  const int ck = 1 << ((log2d + 1) / 2);
  x.rot_inv_ck = 1.0f / static_cast<float>(ck);
  x.rot_inv_cq = static_cast<float>(ck) / static_cast<float>(x.dk);
  *d = x;
  return KVQ_OK;
}

int quantized_prefix(const kvq::Dims& d, int L) {
  if (!d.quantized()) return 0;
  const int over = L - d.R;
  return over > 0 ? over / d.gk * d.gk : 0;
}

// {p < Q : p mod 2^floor(log2(Q - p)) == 0}, ascending: one position per age octave.
std::vector<int> retained_positions(int Q) {
  std::vector<int> out;
  for (int l = 0; l < 31 && (1 << l) <= Q; ++l) {
    // ages a in [2^l, 2^(l+1)) are positions (Q - 2^(l+1), Q - 2^l]; keep the multiple of 2^l
    const int hi = Q - (1 << l);
    out.push_back(hi / (1 << l) * (1 << l));
  }
  std::sort(out.begin(), out.end());
  return out;
}

int split_cap(const kvq::Dims& d) {
  const int rows = d.B * d.Hkv;
  return std::min(256, std::max(2, 8192 / rows));
}

// CTAs per SM the planner's wave model assumes.  Both kernels are resident 4 per SM; for
// the tensor-core kernel the model uses 3, which picks the split counts measured fastest
// on the long-context workloads.
int ctas_per_sm(bool fast) { return fast ? 3 : 4; }

// Quantized groups and fp16 entries of a sequence of L tokens.
void seq_counts(const kvq::Dims& d, int L, int* nG, int* nF) {
  const int Q = quantized_prefix(d, L);
  *nG = Q / d.gk;
  *nF = (d.log_retain ? kvq::retained_count(Q) : 0) + (L - Q);
}

// Chooses the split counts: the number of CTAs per (b, kv head) over the quantized
// groups and over the fp16 tokens, trading wave quantization against per-CTA cost; nG and
// nF are those of the longest sequence.
// Value-code centring of the tensor-core kernel: on from this many quantized tokens (AUTO).  Its
// p.V products of unsigned codes accumulate in fp32 inside the MMA, which truncates; the
// accumulators grow with the tokens summed while the output (a softmax-weighted mean) shrinks,
// so the relative error grows with the context.  Centred codes keep the accumulators near zero
// at the cost of one fp16 subtraction per code register (measured: +7% decode time).
constexpr int kCenterFromTokens = 65536;

int plan_counts(const kvq::Dims& d, int nG, int nF, int sm_count, int num_splits, bool fast,
                kvq_plan* out, int centering = KVQ_CENTER_AUTO) {
  if (sm_count < 1 || num_splits < 0) return KVQ_ERR_INVALID_ARG;
  const int rows = d.B * d.Hkv;
  const int cap = split_cap(d);
  const long long slots = static_cast<long long>(sm_count) * ctas_per_sm(fast);
  // cost model in bytes read: per quantized group, per fp16 token, per CTA
  const double bq = d.quantized()
                        ? static_cast<double>(d.gk) * (d.kw * 4 + d.vw * 4 + d.nvg * 4 + d.zb) +
                              d.dk * 4.0 + d.sr * 4.0
                        : 0.0;
  const double bf = 2.0 * (d.dk + d.dv);
  const double cta_cost = 16384.0;
  // In a launch of a single wave a CTA's fixed work (query prologue, first copies, merge and
  // partial rows, its share of the combine) is not hidden behind other CTAs' streaming, so there
  // a split gets at least kMinSplitBytes of cache to read (measured on 4k-token caches: 3 splits
  // of 21 groups beat 6 of 11 and 9 of 7; multi-wave launches are left to the wave model).
  const double kMinSplitBytes = 112.0 * 1024.0;
  auto best_split = [&](int n_units, double unit_bytes, int forced) {
    if (n_units <= 0) return 0;
    const int hi = std::min(n_units, cap);
    if (forced > 0) return std::min(forced, hi);
    int best = 1;
    double best_t = 1e300;
    for (int s = 1; s <= hi; ++s) {
      const long long waves = (static_cast<long long>(rows) * s + slots - 1) / slots;
      const double per_cta = ((n_units + s - 1) / s) * unit_bytes + cta_cost;
      const double t = waves * per_cta;
      if (t < best_t * 0.999) {
        best_t = t;
        best = s;
      }
    }
    if (static_cast<long long>(rows) * best <= slots) {
      const int by_size = static_cast<int>(std::max(1.0, floor(n_units * unit_bytes / kMinSplitBytes)));
      best = std::min(best, by_size);
    }
    return best;
  };
  int sq = 0, sf = 0;
  if (nG > 0) {
    sq = best_split(nG, bq, num_splits);
    // fp16 CTAs get about as many bytes as a quantized CTA
    const double per_q = ((nG + sq - 1) / sq) * bq;
    int want = static_cast<int>(ceil(nF * bf / std::max(per_q, 1.0)));
    sf = std::max(1, std::min(want, std::min(cap, (nF + 15) / 16)));
  } else {
    sf = best_split((nF + 15) / 16, 16 * bf, num_splits);
  }
  if (nF == 0) sf = 0;
  out->splits_quant = sq;
  out->splits_fp16 = sf;
  out->n_groups = nG;
  out->n_fp16 = nF;
  out->fast_path = fast ? 1 : 0;
  out->centered = fast && d.quantized() && !d.var &&
                  (centering == KVQ_CENTER_ON ||
                   (centering == KVQ_CENTER_AUTO && static_cast<long long>(nG) * d.gk >= kCenterFromTokens))
                      ? 1 : 0;
  return KVQ_OK;
}

int plan_decode(const kvq::Dims& d, int L, int sm_count, int num_splits, bool fast, kvq_plan* out) {
  if (L < 1 || L > d.max_context) return KVQ_ERR_INVALID_ARG;
  int nG, nF;
  seq_counts(d, L, &nG, &nF);
  return plan_counts(d, nG, nF, sm_count, num_splits, fast, out);
}

// The plan of a cache: counts of its longest sequences.
int plan_cache(const kvq_cache* c, int num_splits, bool fast, kvq_plan* out) {
  int nG = 0, nF = 0;
  for (size_t b = 0; b < c->L.size(); ++b) {
    int g, f;
    seq_counts(c->d, c->L[b], &g, &f);
    nG = std::max(nG, g);
    nF = std::max(nF, f);
  }
  return plan_counts(c->d, nG, nF, c->sm_count, num_splits, fast, out, c->centering);
}

int check_cuda(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

bool tensor_kernel_built(const kvq::Dims& d) {
  return d.var ? kvq::decode_var_supported(d) : kvq::decode_mma_supported(d);
}

bool use_tensor_kernel(const kvq_cache* c) {
  return c->kernel != KVQ_KERNEL_GENERIC && tensor_kernel_built(c->d);
}

// Dims and buffers of sequence b alone (a batch of one over the same memory).
void sequence_view(const kvq_cache* c, int b, kvq::Dims* d1, kvq_buffers* b1) {
  const kvq::Dims& d = c->d;
  *d1 = d;
  d1->B = 1;
  const size_t bh = static_cast<size_t>(b) * d.Hkv;
  auto at = [](void* p, size_t bytes) -> void* { return p ? static_cast<char*>(p) + bytes : nullptr; };
  *b1 = c->buf;
  if (d.paged) {
    // the pools are shared; the view's block table is row b
    b1->block_table = at(c->buf.block_table, static_cast<size_t>(b) * d.max_groups * 4);
  } else {
    b1->kcode = at(c->buf.kcode, bh * d.lcap * d.kw * 4);
    b1->ksz = at(c->buf.ksz, bh * (d.lcap / d.gk) * d.dk * 4);
    b1->vcode = at(c->buf.vcode, bh * d.lcap * d.vw * 4);
    b1->vsz = at(c->buf.vsz, bh * d.lcap * d.nvg * 4);
    b1->zcode = at(c->buf.zcode, bh * d.lcap * d.zb);
    b1->zsz = at(c->buf.zsz, bh * (d.lcap / d.gk) * d.sr * 4);
  }
  b1->win_k = at(c->buf.win_k, bh * d.cap * d.dk * 2);
  b1->win_v = at(c->buf.win_v, bh * d.cap * d.dv * 2);
  b1->ret_k = at(c->buf.ret_k, bh * kvq::kMaxRetained * d.dk * 2);
  b1->ret_v = at(c->buf.ret_v, bh * kvq::kMaxRetained * d.dv * 2);
}

// ---- the page pool of a paged cache ----
// Pages sequence b holds (those of its quantized groups, once their launches are queued).
int pages_held(const kvq_cache* c, int b) { return c->d.paged ? c->held[b] : 0; }

void release_pages(kvq_cache* c, int b) {
  const int mg = c->d.max_groups;
  for (int g = pages_held(c, b) - 1; g >= 0; --g) {
    c->free_pages.push_back(c->table[b * mg + g]);
    c->table[b * mg + g] = -1;
  }
  if (c->d.paged) c->held[b] = 0;
}

// Collects block-table writes and launches them in batches of a launch parameter's size.
struct TableWriter {
  kvq_cache* c;
  cudaStream_t s;
  kvq::TableWrites tw;
  int rc = KVQ_OK;
  TableWriter(kvq_cache* c_, cudaStream_t s_) : c(c_), s(s_) { tw.n = 0; }
  int flush() {
    if (tw.n > 0 && !rc)
      rc = check_cuda(kvq::launch_table_writes(c->d, static_cast<int*>(c->buf.block_table), tw, s));
    tw.n = 0;
    return rc;
  }
  // hands sequence b the next free page for its next group (the caller checked there is one)
  void assign(int b) {
    const int page = c->free_pages.back();
    c->free_pages.pop_back();
    const int idx = b * c->d.max_groups + c->held[b]++;
    c->table[idx] = page;
    tw.idx[tw.n] = idx;
    tw.page[tw.n] = page;
    if (++tw.n == static_cast<int>(sizeof(tw.idx) / sizeof(tw.idx[0]))) flush();
  }
};

kvq::CacheBufs cache_bufs(const kvq_cache* c) {
  kvq::CacheBufs b;
  b.kcode = static_cast<const uint32_t*>(c->buf.kcode);
  b.ksz = static_cast<const __half2*>(c->buf.ksz);
  b.vcode = static_cast<const uint32_t*>(c->buf.vcode);
  b.vsz = static_cast<const __half2*>(c->buf.vsz);
  b.win_k = static_cast<const __half*>(c->buf.win_k);
  b.win_v = static_cast<const __half*>(c->buf.win_v);
  b.ret_k = static_cast<const __half*>(c->buf.ret_k);
  b.ret_v = static_cast<const __half*>(c->buf.ret_v);
  b.zcode = static_cast<const uint8_t*>(c->buf.zcode);
  b.zsz = static_cast<const __half2*>(c->buf.zsz);
  b.side_u = static_cast<const float*>(c->buf.side_u);
  b.table = static_cast<const int*>(c->buf.block_table);
  return b;
}

}  // namespace

extern "C" {

const char* kvq_strerror(int code) {
  switch (code) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported shape, bit width or group size";
    case KVQ_ERR_ALIGN: return "device pointer not 16-byte aligned";
    case KVQ_ERR_CAPACITY: return "cache capacity (max_context or page pool) exceeded";
    case KVQ_ERR_WORKSPACE: return "decode workspace too small";
    case KVQ_ERR_STATE: return "a sequence of the cache is empty";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown error";
  }
}

int kvq_buffer_sizes(const kvq_config* cfg, kvq_sizes* out) {
  if (!out) return KVQ_ERR_INVALID_ARG;
  kvq::Dims d;
  const int rc = make_dims(cfg, &d);
  if (rc) return rc;
  const size_t bh = static_cast<size_t>(d.B) * d.Hkv;
  kvq_sizes s;
  memset(&s, 0, sizeof(s));
  if (d.quantized()) {
    // token rows and groups of the quantized buffers: per (b, h) region, or per page
    const size_t groups = d.paged ? static_cast<size_t>(cfg->n_pages) * d.Hkv : bh * d.max_groups;
    const size_t rows = groups * d.gk;
    s.kcode = rows * d.kw * 4;
    s.ksz = groups * d.dk * 4;
    s.vcode = rows * d.vw * 4;
    s.vsz = rows * d.nvg * 4;
    s.ret_k = bh * kvq::kMaxRetained * d.dk * 2;
    s.ret_v = bh * kvq::kMaxRetained * d.dv * 2;
    if (d.sr) {
      s.zcode = rows * d.zb;
      s.zsz = groups * d.sr * 4;
      s.side_u = static_cast<size_t>(d.Hkv) * d.dk * d.sr * 4;
    }
    if (d.paged) s.block_table = static_cast<size_t>(d.B) * d.max_groups * 4;
  }
  s.win_k = bh * d.cap * d.dk * 2;
  s.win_v = bh * d.cap * d.dv * 2;
  s.workspace = kvq::workspace_bytes(d, 2 * split_cap(d));
  *out = s;
  return KVQ_OK;
}

int kvq_cache_init(const kvq_config* cfg, const kvq_buffers* bufs, kvq_cache** out) {
  if (!cfg || !bufs || !out) return KVQ_ERR_INVALID_ARG;
  kvq::Dims d;
  int rc = make_dims(cfg, &d);
  if (rc) return rc;
  const void* need[] = {bufs->win_k, bufs->win_v};
  for (const void* p : need)
    if (!p) return KVQ_ERR_INVALID_ARG;
  if (d.quantized()) {
    const void* q[] = {bufs->kcode, bufs->ksz, bufs->vcode, bufs->vsz, bufs->ret_k, bufs->ret_v};
    for (const void* p : q)
      if (!p) return KVQ_ERR_INVALID_ARG;
  }
  if (d.sr) {
    const void* z[] = {bufs->zcode, bufs->zsz, bufs->side_u};
    for (const void* p : z)
      if (!p) return KVQ_ERR_INVALID_ARG;
  }
  if (d.paged && !bufs->block_table) return KVQ_ERR_INVALID_ARG;
  const void* all[] = {bufs->kcode, bufs->ksz, bufs->vcode, bufs->vsz, bufs->win_k, bufs->win_v,
                       bufs->ret_k, bufs->ret_v, bufs->zcode, bufs->zsz, bufs->side_u,
                       bufs->block_table};
  for (const void* p : all)
    if (p && !aligned16(p)) return KVQ_ERR_ALIGN;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
#ifdef KVQ_DEBUG
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.dbg), kvq::g_debug_record) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
#endif
  kvq_cache* c = new (std::nothrow) kvq_cache;
  if (!c) return KVQ_ERR_INVALID_ARG;
  c->d = d;
  c->d.sm_count = sms;
  c->buf = *bufs;
  if (!d.paged) c->buf.block_table = nullptr;
  c->L.assign(d.B, 0);
  c->Q.assign(d.B, 0);
  if (d.paged) {
    c->table.assign(static_cast<size_t>(d.B) * d.max_groups, -1);
    c->held.assign(d.B, 0);
    // handed out from the back: a fresh pool gives pages 0, 1, 2, ... in order
    for (int p = cfg->n_pages - 1; p >= 0; --p) c->free_pages.push_back(p);
  }
  c->sm_count = sms;
  c->kernel = KVQ_KERNEL_AUTO;
  c->centering = KVQ_CENTER_AUTO;
  c->stall_next = false;
  *out = c;
  return KVQ_OK;
}

void kvq_cache_destroy(kvq_cache* cache) { delete cache; }

int kvq_allocate_bits(const double* weight, int n, int unit_bits, int budget, unsigned char* widths) {
  if (!weight || !widths || n < 1 || unit_bits < 1 || budget < 0) return KVQ_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (!(weight[i] >= 0.0) || !isfinite(weight[i])) return KVQ_ERR_INVALID_ARG;
  // the width steps 0->1->2->4->8 and their distortion drops per bit for weight 1:
  // (4^-b1 - 4^-b2) / (b2 - b1), exact binary fractions
  static const int kFrom[4] = {0, 1, 2, 4}, kTo[4] = {1, 2, 4, 8};
  static const double kDrop[4] = {0.75, 0.1875, 15.0 / 512.0, 255.0 / 262144.0};
  struct Step {
    double drop;
    int unit, from, to;
  };
  std::vector<Step> steps;
  steps.reserve(static_cast<size_t>(n) * 4);
  for (int i = 0; i < n; ++i)
    for (int k = 0; k < 4; ++k) {
      const double drop = weight[i] * kDrop[k];
      if (drop > 0.0) steps.push_back({drop, i, kFrom[k], kTo[k]});
    }
  std::stable_sort(steps.begin(), steps.end(), [](const Step& a, const Step& b) { return a.drop > b.drop; });
  std::vector<unsigned char> w(n, 0);
  long long used = 0;
  for (size_t i = 0; i < steps.size();) {
    size_t j = i;
    long long cost = 0;
    while (j < steps.size() && steps[j].drop == steps[i].drop) {
      cost += static_cast<long long>(steps[j].to - steps[j].from) * unit_bits;
      ++j;
    }
    if (used + cost > budget) break;
    for (size_t k = i; k < j; ++k) w[steps[k].unit] = static_cast<unsigned char>(steps[k].to);
    used += cost;
    i = j;
  }
  std::copy(w.begin(), w.end(), widths);
  return static_cast<int>(used);
}

int kvq_retained_positions(int Q, int* out, int cap) {
  if (Q < 0) return KVQ_ERR_INVALID_ARG;
  const std::vector<int> r = retained_positions(Q);
  if (r.empty()) return 0;
  if (!out || cap < static_cast<int>(r.size())) return KVQ_ERR_INVALID_ARG;
  std::copy(r.begin(), r.end(), out);
  return static_cast<int>(r.size());
}

}  // extern "C"

namespace {

// Prefill of the sequences of (d, buf): k, v [d.B][Hkv][src_rows][d], the first L rows valid.
int prefill_rows(const kvq::Dims& d, const kvq_buffers& buf, const __half* kh, const __half* vh,
                 int src_rows, int L, cudaStream_t s) {
  const int Q = quantized_prefix(d, L);
  const int nbh = d.B * d.Hkv;
  const int* table = static_cast<const int*>(buf.block_table);
  int rc = KVQ_OK;
  if (Q > 0) {
    rc = check_cuda(kvq::launch_quantize_keys(d, kh, src_rows, 0, Q / d.gk,
                                              static_cast<uint32_t*>(buf.kcode),
                                              static_cast<__half2*>(buf.ksz), table, d.rot != 0, s));
    if (!rc)
      rc = check_cuda(kvq::launch_quantize_side(
          d, kh, src_rows, 0, Q / d.gk, static_cast<const uint32_t*>(buf.kcode),
          static_cast<const __half2*>(buf.ksz), static_cast<const float*>(buf.side_u),
          static_cast<uint8_t*>(buf.zcode), static_cast<__half2*>(buf.zsz), table, d.rot != 0, s));
    if (!rc)
      rc = check_cuda(kvq::launch_quantize_values(d, vh, src_rows, 0, Q,
                                                  static_cast<uint32_t*>(buf.vcode),
                                                  static_cast<__half2*>(buf.vsz), table, s));
  }
  if (!rc)
    rc = check_cuda(d.rot ? kvq::launch_rotate_key_rows(d, kh, src_rows, Q, static_cast<__half*>(buf.win_k),
                                                        d.cap, Q, L - Q, nullptr, s)
                          : kvq::launch_copy_rows(d, kh, src_rows, Q, static_cast<__half*>(buf.win_k), d.cap,
                                                  Q, L - Q, d.dk, nbh, s));
  if (!rc)
    rc = check_cuda(kvq::launch_copy_rows(d, vh, src_rows, Q, static_cast<__half*>(buf.win_v), d.cap, Q,
                                          L - Q, d.dv, nbh, s));
  if (!rc && d.log_retain && Q > 0) {
    const std::vector<int> ret = retained_positions(Q);
    kvq::RetList rl;
    rl.n = static_cast<int>(ret.size());
    for (int i = 0; i < rl.n; ++i) rl.pos[i] = ret[i];
    rc = check_cuda(kvq::launch_copy_retained(d, d.rot ? nullptr : kh, vh, src_rows, rl,
                                              static_cast<__half*>(buf.ret_k),
                                              static_cast<__half*>(buf.ret_v), s));
    if (!rc && d.rot)
      rc = check_cuda(kvq::launch_rotate_key_rows(d, kh, src_rows, 0, static_cast<__half*>(buf.ret_k),
                                                  kvq::kMaxRetained, 0, rl.n, &rl, s));
  }
  return rc;
}

// The oldest group_k window tokens of the sequences of (d, buf), whose quantized prefix is
// Q, become one key group and group_k value rows; the retained set moves to that of Q + gk.
// The window already holds the cached (rotated, if so configured) keys.
int quantize_window_group(const kvq::Dims& d, const kvq_buffers& buf, int Q, cudaStream_t s) {
  __half* wk = static_cast<__half*>(buf.win_k);
  __half* wv = static_cast<__half*>(buf.win_v);
  const int* table = static_cast<const int*>(buf.block_table);
  int rc = check_cuda(kvq::launch_quantize_keys(d, wk, d.cap, Q / d.gk, 1,
                                                static_cast<uint32_t*>(buf.kcode),
                                                static_cast<__half2*>(buf.ksz), table, false, s));
  if (!rc)
    rc = check_cuda(kvq::launch_quantize_side(
        d, wk, d.cap, Q / d.gk, 1, static_cast<const uint32_t*>(buf.kcode),
        static_cast<const __half2*>(buf.ksz), static_cast<const float*>(buf.side_u),
        static_cast<uint8_t*>(buf.zcode), static_cast<__half2*>(buf.zsz), table, false, s));
  if (!rc)
    rc = check_cuda(kvq::launch_quantize_values(d, wv, d.cap, Q, d.gk, static_cast<uint32_t*>(buf.vcode),
                                                static_cast<__half2*>(buf.vsz), table, s));
  if (!rc && d.log_retain) {
    const std::vector<int> old_ret = retained_positions(Q);
    const std::vector<int> nr = retained_positions(Q + d.gk);
    kvq::RetUpdate up;
    up.n = static_cast<int>(nr.size());
    for (int i = 0; i < up.n; ++i) {
      const auto it = std::lower_bound(old_ret.begin(), old_ret.end(), nr[i]);
      if (it != old_ret.end() && *it == nr[i]) {
        up.from_window[i] = 0;
        up.index[i] = static_cast<int>(it - old_ret.begin());
      } else {
        up.from_window[i] = 1;
        up.index[i] = nr[i] % d.cap;
      }
    }
    rc = check_cuda(kvq::launch_update_retained(d, up, wk, wv, static_cast<__half*>(buf.ret_k),
                                                static_cast<__half*>(buf.ret_v), s));
  }
  return rc;
}

// Prefill of every sequence: k, v [B][Hkv][L_max][d], sequence b's first lengths[b] rows.
// A paged cache takes back all pages first and hands out Q_b / gk to each sequence.
int prefill_all(kvq_cache* c, const __half* kh, const __half* vh, int L_max, const int* lengths,
                cudaStream_t s) {
  const kvq::Dims& d = c->d;
  if (d.paged) {
    long long need = 0, avail = static_cast<long long>(c->free_pages.size());
    for (int b = 0; b < d.B; ++b) {
      need += quantized_prefix(d, lengths[b]) / d.gk;
      avail += pages_held(c, b);
    }
    if (need > avail) return KVQ_ERR_CAPACITY;
  }
  for (int b = 0; b < d.B; ++b) {
    release_pages(c, b);
    c->L[b] = c->Q[b] = 0;
  }
  if (d.paged) {
    TableWriter tw(c, s);
    for (int b = 0; b < d.B; ++b)
      for (int g = 0; g < quantized_prefix(d, lengths[b]) / d.gk; ++g) tw.assign(b);
    if (tw.flush()) return tw.rc;
  }
  bool same = true;
  for (int b = 1; b < d.B; ++b) same = same && lengths[b] == lengths[0];
  if (same) {
    const int rc = prefill_rows(d, c->buf, kh, vh, L_max, lengths[0], s);
    if (rc) return rc;
  } else {
    for (int b = 0; b < d.B; ++b) {
      kvq::Dims d1;
      kvq_buffers b1;
      sequence_view(c, b, &d1, &b1);
      const size_t off = static_cast<size_t>(b) * d.Hkv * L_max;
      const int rc = prefill_rows(d1, b1, kh + off * d.dk, vh + off * d.dv, L_max, lengths[b], s);
      if (rc) return rc;
    }
  }
  for (int b = 0; b < d.B; ++b) {
    c->L[b] = lengths[b];
    c->Q[b] = quantized_prefix(d, lengths[b]);
  }
  return KVQ_OK;
}

}  // namespace

extern "C" {

int kvq_quantize_prefill(kvq_cache* c, const void* k, const void* v, int L, void* stream) {
  if (!c || !k || !v) return KVQ_ERR_INVALID_ARG;
  if (L < 1 || L > c->d.max_context) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return KVQ_ERR_ALIGN;
  const std::vector<int> lengths(c->d.B, L);
  return prefill_all(c, static_cast<const __half*>(k), static_cast<const __half*>(v), L, lengths.data(),
                     static_cast<cudaStream_t>(stream));
}

int kvq_quantize_prefill_ragged(kvq_cache* c, const void* k, const void* v, int L_max,
                                const int* lengths, void* stream) {
  if (!c || !k || !v || !lengths) return KVQ_ERR_INVALID_ARG;
  const kvq::Dims& d = c->d;
  if (L_max < 1 || L_max > d.max_context) return KVQ_ERR_INVALID_ARG;
  for (int b = 0; b < d.B; ++b)
    if (lengths[b] < 1 || lengths[b] > L_max) return KVQ_ERR_INVALID_ARG;
  if (d.B > kvq::kMaxSeqs) {
    for (int b = 1; b < d.B; ++b)
      if (lengths[b] != lengths[0]) return KVQ_ERR_UNSUPPORTED;
  }
  if (!aligned16(k) || !aligned16(v)) return KVQ_ERR_ALIGN;
  return prefill_all(c, static_cast<const __half*>(k), static_cast<const __half*>(v), L_max, lengths,
                     static_cast<cudaStream_t>(stream));
}

int kvq_prefill_sequence(kvq_cache* c, int b, const void* k, const void* v, int L, void* stream) {
  if (!c || !k || !v) return KVQ_ERR_INVALID_ARG;
  const kvq::Dims& d = c->d;
  if (b < 0 || b >= d.B || L < 1 || L > d.max_context) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return KVQ_ERR_ALIGN;
  const int Q = quantized_prefix(d, L);
  if (d.paged && Q / d.gk > static_cast<int>(c->free_pages.size()) + pages_held(c, b))
    return KVQ_ERR_CAPACITY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  release_pages(c, b);
  c->L[b] = c->Q[b] = 0;
  if (d.paged) {
    TableWriter tw(c, s);
    for (int g = 0; g < Q / d.gk; ++g) tw.assign(b);
    if (tw.flush()) return tw.rc;
  }
  kvq::Dims d1;
  kvq_buffers b1;
  sequence_view(c, b, &d1, &b1);
  const int rc = prefill_rows(d1, b1, static_cast<const __half*>(k), static_cast<const __half*>(v), L, L, s);
  if (rc) return rc;
  c->L[b] = L;
  c->Q[b] = Q;
  return KVQ_OK;
}

int kvq_release_sequence(kvq_cache* c, int b) {
  if (!c || b < 0 || b >= c->d.B) return KVQ_ERR_INVALID_ARG;
  release_pages(c, b);
  c->L[b] = c->Q[b] = 0;
  return KVQ_OK;
}

int kvq_free_pages(const kvq_cache* c) {
  if (!c) return KVQ_ERR_INVALID_ARG;
  return static_cast<int>(c->free_pages.size());
}

int kvq_append_ragged(kvq_cache* c, const void* k_new, const void* v_new, const unsigned char* active,
                      void* stream) {
  if (!c || !k_new || !v_new) return KVQ_ERR_INVALID_ARG;
  const kvq::Dims& d = c->d;
  int crossing = 0;   // sequences whose window spills a group into the quantized prefix
  for (int b = 0; b < d.B; ++b) {
    if (active && !active[b]) continue;
    if (c->L[b] < 1) return KVQ_ERR_STATE;
    if (c->L[b] + 1 > d.max_context) return KVQ_ERR_CAPACITY;
    crossing += d.quantized() && c->L[b] + 1 - c->Q[b] == d.R + d.gk;
  }
  if (d.paged && crossing > static_cast<int>(c->free_pages.size())) return KVQ_ERR_CAPACITY;
  if (!aligned16(k_new) || !aligned16(v_new)) return KVQ_ERR_ALIGN;
  bool all = true;
  for (int b = 0; b < d.B && active; ++b) all = all && active[b];
  if (!all && d.B > kvq::kMaxSeqs) return KVQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool lockstep = all && c->uniform();
  kvq::SlotMap slots;
  if (lockstep) {
    slots.slot[0] = c->L[0] % d.cap;
    for (int b = 1; b < d.B && b < kvq::kMaxSeqs; ++b) slots.slot[b] = slots.slot[0];
  } else {
    for (int b = 0; b < d.B; ++b) slots.slot[b] = (!active || active[b]) ? c->L[b] % d.cap : -1;
  }
  int rc = KVQ_OK;
  if (lockstep && d.B > kvq::kMaxSeqs) {
    // more sequences than a slot map holds, all in the same slot: one launch per chunk
    for (int b0 = 0; b0 < d.B && !rc; b0 += kvq::kMaxSeqs) {
      kvq::Dims dc = d;
      dc.B = std::min(kvq::kMaxSeqs, d.B - b0);
      const size_t bh0 = static_cast<size_t>(b0) * d.Hkv;
      rc = check_cuda(kvq::launch_append_token(
          dc, static_cast<const __half*>(k_new) + bh0 * d.dk, static_cast<const __half*>(v_new) + bh0 * d.dv,
          static_cast<__half*>(c->buf.win_k) + bh0 * d.cap * d.dk,
          static_cast<__half*>(c->buf.win_v) + bh0 * d.cap * d.dv, slots, s));
    }
  } else {
    rc = check_cuda(kvq::launch_append_token(d, static_cast<const __half*>(k_new),
                                             static_cast<const __half*>(v_new),
                                             static_cast<__half*>(c->buf.win_k),
                                             static_cast<__half*>(c->buf.win_v), slots, s));
  }
  if (rc) return rc;
  // new pages for the groups that spill (paged caches), written before they are quantized
  if (d.paged && crossing) {
    TableWriter tw(c, s);
    for (int b = 0; b < d.B; ++b)
      if ((!active || active[b]) && c->L[b] + 1 - c->Q[b] == d.R + d.gk) tw.assign(b);
    if (tw.flush()) return tw.rc;
  }
  if (lockstep) {
    // every sequence in step: one launch per kernel for the whole batch
    const int L = c->L[0] + 1;
    if (d.quantized() && L - c->Q[0] == d.R + d.gk) {
      rc = quantize_window_group(d, c->buf, c->Q[0], s);
      if (rc) return rc;
      c->Q.assign(d.B, c->Q[0] + d.gk);
    }
    c->L.assign(d.B, L);
    return KVQ_OK;
  }
  for (int b = 0; b < d.B; ++b) {
    if (active && !active[b]) continue;
    c->L[b] += 1;
    if (d.quantized() && c->L[b] - c->Q[b] == d.R + d.gk) {
      kvq::Dims d1;
      kvq_buffers b1;
      sequence_view(c, b, &d1, &b1);
      rc = quantize_window_group(d1, b1, c->Q[b], s);
      if (rc) return rc;
      c->Q[b] += d.gk;
    }
  }
  return KVQ_OK;
}

int kvq_append(kvq_cache* c, const void* k_new, const void* v_new, void* stream) {
  return kvq_append_ragged(c, k_new, v_new, nullptr, stream);
}

int kvq_plan_decode(const kvq_config* cfg, int L, int sm_count, int num_splits, kvq_plan* out) {
  if (!out) return KVQ_ERR_INVALID_ARG;
  kvq::Dims d;
  const int rc = make_dims(cfg, &d);
  if (rc) return rc;
  return plan_decode(d, L, sm_count, num_splits, tensor_kernel_built(d), out);
}

int kvq_get_plan(const kvq_cache* c, int num_splits, kvq_plan* out) {
  if (!c || !out) return KVQ_ERR_INVALID_ARG;
  if (!c->ready()) return KVQ_ERR_STATE;
  return plan_cache(c, num_splits, use_tensor_kernel(c), out);
}

int kvq_decode_workspace_size(const kvq_cache* c, int num_splits, size_t* bytes) {
  if (!c || !bytes) return KVQ_ERR_INVALID_ARG;
  kvq_plan p;
  const int rc = kvq_get_plan(c, num_splits, &p);
  if (rc) return rc;
  *bytes = kvq::workspace_bytes(c->d, p.splits_quant + p.splits_fp16);
  return KVQ_OK;
}

int kvq_decode_attention(kvq_cache* c, const void* q, void* out, void* workspace,
                         size_t workspace_bytes, int num_splits, void* stream) {
  if (!c || !q || !out || !workspace || num_splits < 0) return KVQ_ERR_INVALID_ARG;
  if (!c->ready()) return KVQ_ERR_STATE;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return KVQ_ERR_ALIGN;
  const kvq::Dims& d = c->d;
  kvq_plan plan;
  int rc = plan_cache(c, num_splits, use_tensor_kernel(c), &plan);
  if (rc) return rc;
  kvq::DecodeWork w;
  w.uniform = c->uniform() ? 1 : 0;
  if (!w.uniform && d.B > kvq::kMaxSeqs) return KVQ_ERR_UNSUPPORTED;
  for (int b = 0; b < (w.uniform ? 1 : d.B); ++b) {
    w.L[b] = c->L[b];
    w.Q[b] = c->Q[b];
  }
  w.n_groups = plan.n_groups;
  w.n_fp16 = plan.n_fp16;
  w.splits_q = plan.splits_quant;
  w.splits_f = plan.splits_fp16;
  w.splits = plan.splits_quant + plan.splits_fp16;
  w.score_scale = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(d.dk)));
  w.stall = c->stall_next && plan.fast_path ? 1 : 0;
  w.center = plan.centered;
  c->stall_next = false;
  if (workspace_bytes < kvq::workspace_bytes(d, w.splits)) return KVQ_ERR_WORKSPACE;
  const kvq::Partials parts = kvq::workspace_views(d, w.splits, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __half* qh = static_cast<const __half*>(q);
  const kvq::CacheBufs cb = cache_bufs(c);
  if (plan.fast_path)
    rc = check_cuda(d.var ? kvq::launch_decode_var(d, cb, w, qh, parts, s)
                          : kvq::launch_decode_mma(d, cb, w, qh, parts, s));
  else
    rc = check_cuda(kvq::launch_decode_simple(d, cb, w, qh, parts, s));
  if (!rc) rc = check_cuda(kvq::launch_combine(d, w, parts, static_cast<__half*>(out), s));
  return rc;
}

int kvq_debug_stall_next_decode(kvq_cache* c) {
  if (!c) return KVQ_ERR_INVALID_ARG;
  c->stall_next = true;
  return KVQ_OK;
}

int kvq_set_value_centering(kvq_cache* c, int mode) {
  if (!c || mode < KVQ_CENTER_AUTO || mode > KVQ_CENTER_ON) return KVQ_ERR_INVALID_ARG;
  c->centering = mode;
  return KVQ_OK;
}

int kvq_set_decode_kernel(kvq_cache* c, int kernel) {
  if (!c || kernel < KVQ_KERNEL_AUTO || kernel > KVQ_KERNEL_TENSOR) return KVQ_ERR_INVALID_ARG;
  if (kernel == KVQ_KERNEL_TENSOR && !tensor_kernel_built(c->d)) return KVQ_ERR_UNSUPPORTED;
  c->kernel = kernel;
  return KVQ_OK;
}

int kvq_get_seq_state(const kvq_cache* c, int b, int* L, int* Q, int* n_retained, int* retained_idx) {
  if (!c || b < 0 || b >= c->d.B) return KVQ_ERR_INVALID_ARG;
  const std::vector<int> ret = c->d.log_retain ? retained_positions(c->Q[b]) : std::vector<int>();
  if (L) *L = c->L[b];
  if (Q) *Q = c->Q[b];
  if (n_retained) *n_retained = static_cast<int>(ret.size());
  if (retained_idx)
    for (size_t i = 0; i < ret.size(); ++i) retained_idx[i] = ret[i];
  return KVQ_OK;
}

int kvq_get_state(const kvq_cache* c, int* L, int* Q, int* n_retained, int* retained_idx) {
  return kvq_get_seq_state(c, 0, L, Q, n_retained, retained_idx);
}

int kvq_debug_build(void) {
#ifdef KVQ_DEBUG
  return 1;
#else
  return 0;
#endif
}

int kvq_debug_take_record(kvq_debug_record* out, void* stream) {
  if (!out) return KVQ_ERR_INVALID_ARG;
#ifdef KVQ_DEBUG
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  kvq::DebugRecord r;
  if (cudaStreamSynchronize(s) != cudaSuccess ||
      cudaMemcpyFromSymbol(&r, kvq::g_debug_record, sizeof(r)) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  const kvq::DebugRecord zero = {0u, 0u, 0, 0};
  if (cudaMemcpyToSymbol(kvq::g_debug_record, &zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  out->failures = r.failures;
  out->site = r.site;
  out->index = r.index;
  out->extent = r.extent;
  return KVQ_OK;
#else
  (void)stream;
  return KVQ_ERR_UNSUPPORTED;
#endif
}

const char* kvq_debug_site_name(unsigned int site) {
  static const char* const kNames[] = {
      "none", "quantize keys: source", "quantize keys: codes", "quantize keys: (scale, zero)",
      "quantize values: source", "quantize values: codes", "quantize values: (scale, zero)",
      "side code: source", "side code: key codes", "side code: key (scale, zero)", "side code: basis",
      "side code: codes", "side code: (scale, zero)", "row copy: source", "row copy: destination",
      "append: window slot", "rotated rows: source", "rotated rows: destination",
      "retained: source", "retained: destination", "retained update: source",
      "block table: entry", "block table: page", "decode: block table entry",
      "decode: quantized group", "decode: key (scale, zero) group", "decode: retained slot",
      "decode: window slot", "decode: partial row"};
  static_assert(sizeof(kNames) / sizeof(kNames[0]) == kvq::kSiteCount, "one name per site");
  return site < kvq::kSiteCount ? kNames[site] : "unknown";
}

int kvq_reset_status(void* workspace, void* stream) {
  if (!workspace) return KVQ_ERR_INVALID_ARG;
  return check_cuda(cudaMemsetAsync(workspace, 0, sizeof(unsigned int),
                                    static_cast<cudaStream_t>(stream)));
}

int kvq_read_status(const void* workspace, unsigned int* status, void* stream) {
  if (!workspace || !status) return KVQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
  return check_cuda(cudaMemcpy(status, workspace, sizeof(unsigned int), cudaMemcpyDeviceToHost));
}

}  // extern "C"
