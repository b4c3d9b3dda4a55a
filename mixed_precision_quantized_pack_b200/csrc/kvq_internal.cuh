// Internal declarations shared by the host API and the kernels of libkvq.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kvq {

constexpr int kMaxRetained = 32;

// The first failed bounds check of a bounds-check build (see KVQ_IN_BOUNDS below).
struct DebugRecord {
  unsigned int failures;   // failed checks since the record was last taken
  unsigned int site;       // DebugSite of the first one
  long long index;         // its index (elements of the buffer's type)
  long long extent;        // and the buffer's extent
};

// Where a bounds check sits: the data-dependent global-memory accesses of the kernels (rows
// and groups found through the length rules or the block table, window and retained slots,
// partial rows).  Accesses whose indices follow from the launch shape alone are not checked.
enum DebugSite : unsigned int {
  kSiteNone = 0,
  kSiteQKeySrc, kSiteQKeyCode, kSiteQKeyMeta,                 // key quantizers
  kSiteQValSrc, kSiteQValCode, kSiteQValMeta,                 // value quantizers
  kSiteSideSrc, kSiteSideCode, kSiteSideMeta, kSiteSideU, kSiteSideZCode, kSiteSideZMeta,
  kSiteCopySrc, kSiteCopyDst,                                 // window / retained copies
  kSiteAppendWin, kSiteRotSrc, kSiteRotDst,
  kSiteRetSrc, kSiteRetDst, kSiteRetUpd,
  kSiteTableIdx, kSiteTablePage,
  kSiteDecTable, kSiteDecKCode, kSiteDecKMeta, kSiteDecRetK, kSiteDecWinK, kSiteDecPartial,
  kSiteCount
};
constexpr int kMaxSeqs = 256;   // sequences of a cache whose lengths may differ (per-launch arrays)

// Derived sizes of one cache (see include/kvq.h for the layouts).
struct Dims {
  int B, Hq, Hkv, n_rep, dk, dv, kb, vb, gk, gv, R, log_retain, max_context;
  int lcap;   // quantized rows per (b, kv head): max_context rounded up to group_k
  int cap;    // window ring slots: R + group_k, or max_context at 16 bits
  int kw;     // u32 words per key row:   dk * kb / 32
  int vw;     // u32 words per value row: dv * vb / 32
  int nvg;    // value groups per token:  dv / gv
  int sr;     // side-code rank r (0: no side code)
  int sq;     // bits per side code
  int zb;     // bytes per side-code row: sr * sq / 8 (2 or 4)
  int rot;    // key-only rotation on/off
  unsigned int rot_signs[8];   // bit c set: sigma_c = -1
  float rot_inv_ck, rot_inv_cq;   // 1/c_k (keys), 1/c_q (queries): powers of two
  int paged;        // quantized groups in a pool of pages, located through a block table
  int max_groups;   // groups per sequence: lcap / gk (block-table row length)
  // per-channel widths (kb = vb = 0): widths are non-increasing over the channels, so a map
  // is the number of channels of width 8, 4, 2 and 1 (the rest are dropped, width 0)
  int var;
  int kcnt[4], vcnt[4];
  int n_pages;      // pages of a paged cache's pool (0 otherwise)
  int sm_count;     // SMs of the cache's device (persistent grids; set when the handle is made)
  DebugRecord* dbg; // bounds-check builds: the library's debug record on this device (else null)
  bool quantized() const { return kb != 16; }
};

// Extents of the cache buffers in elements of their types (token rows of the quantized
// buffers: a (b, kv head) region of lcap rows per sequence, or n_pages pages of Hkv * gk rows).
__host__ __device__ inline long long quant_rows(const Dims& d) {
  return d.paged ? static_cast<long long>(d.n_pages) * d.Hkv * d.gk
                 : static_cast<long long>(d.B) * d.Hkv * d.lcap;
}
__host__ __device__ inline long long quant_groups(const Dims& d) {
  return d.paged ? static_cast<long long>(d.n_pages) * d.Hkv
                 : static_cast<long long>(d.B) * d.Hkv * d.max_groups;
}
__host__ __device__ inline long long win_rows(const Dims& d) { return static_cast<long long>(d.B) * d.Hkv * d.cap; }
__host__ __device__ inline long long ret_rows(const Dims& d) { return static_cast<long long>(d.B) * d.Hkv * kMaxRetained; }

// Bounds checks of a bounds-check build (compiled with -DKVQ_DEBUG): every global index a
// kernel computes is compared with its buffer's extent; a failed check counts in the
// library's debug record (the first failure's site, index and extent are kept) and the
// caller skips the access or redirects it to the buffer's start.  No trap, no assert: the
// kernel runs on.  In other builds the checks compile to `true`.
#ifdef KVQ_DEBUG
__device__ __forceinline__ bool debug_in_bounds(const Dims& d, unsigned int site, long long idx,
                                                long long extent) {
  if (idx >= 0 && idx < extent) return true;
  if (d.dbg && atomicAdd(&d.dbg->failures, 1u) == 0u) {
    d.dbg->site = site;
    d.dbg->index = idx;
    d.dbg->extent = extent;
  }
  return false;
}
#define KVQ_IN_BOUNDS(d, site, idx, extent) ::kvq::debug_in_bounds((d), (site), (idx), (extent))
#else
#define KVQ_IN_BOUNDS(d, site, idx, extent) (static_cast<void>(idx), true)
#endif
// [idx, idx + len) inside [0, extent)
#define KVQ_RANGE_IN_BOUNDS(d, site, idx, len, extent) \
  (KVQ_IN_BOUNDS(d, site, idx, extent) && KVQ_IN_BOUNDS(d, site, (idx) + (len) - 1, extent))

// Width and bit offset in its packed row of channel c of a per-channel width map given by
// its class counts (channels of width 8, then 4, 2, 1, then 0): the offset is the sum of
// the widths before c.
__host__ __device__ inline void channel_width(const int* cnt, int c, int* width, int* offset) {
  int off = 0, base = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int w = 8 >> i;
    if (c < base + cnt[i]) {
      *width = w;
      *offset = off + (c - base) * w;
      return;
    }
    off += cnt[i] * w;
    base += cnt[i];
  }
  *width = 0;
  *offset = off;
}

// Where key group g of (b, kv head h) lives in the quantized buffers: the token row of its
// first token in the code arrays (rows of kw / vw words, of zb side bytes, of nvg value
// (scale, zero) pairs) and its index in the per-group arrays (key and side (scale, zero)).
// Unpaged: region (b, h) of lcap rows; paged: page table[b][g], laid out [page][h][gk].
__host__ __device__ inline size_t group_row(const Dims& d, const int* table, int b, int h, int g) {
  if (d.paged) return (static_cast<size_t>(table[b * d.max_groups + g]) * d.Hkv + h) * d.gk;
  return static_cast<size_t>(b * d.Hkv + h) * d.lcap + static_cast<size_t>(g) * d.gk;
}
__host__ __device__ inline size_t group_index(const Dims& d, const int* table, int b, int h, int g) {
  if (d.paged) return static_cast<size_t>(table[b * d.max_groups + g]) * d.Hkv + h;
  return static_cast<size_t>(b * d.Hkv + h) * d.max_groups + g;
}
// The same from the flat row bh = b * Hkv + h: a division only for a paged cache.
__host__ __device__ inline size_t group_row_bh(const Dims& d, const int* table, int bh, int g) {
  if (d.paged) return group_row(d, table, bh / d.Hkv, bh % d.Hkv, g);
  return static_cast<size_t>(bh) * d.lcap + static_cast<size_t>(g) * d.gk;
}
__host__ __device__ inline size_t group_index_bh(const Dims& d, const int* table, int bh, int g) {
  if (d.paged) return group_index(d, table, bh / d.Hkv, bh % d.Hkv, g);
  return static_cast<size_t>(bh) * d.max_groups + g;
}

// The rotation of one key or query row of d = 32 * M channels by a warp, lane l holding
// channels l + 32 m in x[m]: x <- FWHT(sigma * x) * inv_c in fp32, butterflies of span
// 1, 2, ..., d/2 in that order, each (x_i, x_{i+h}) -> (x_i + x_{i+h}, x_i - x_{i+h});
// spans below 32 pair lanes, longer spans pair registers.  (Randomized Hadamard key-only
// rotation: "Quantize What Counts: More for Keys, Less for Values", Intégration de la
// Rotation.)  m_count <= M is the number of valid registers (d / 32).
template <int M>
__device__ __forceinline__ void rotate_row_warp(float (&x)[M], int m_count, const unsigned int* signs,
                                                float inv_c, int lane) {
#pragma unroll
  for (int m = 0; m < M; ++m)
    if (m < m_count && ((signs[m] >> lane) & 1u)) x[m] = -x[m];
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float y = __shfl_xor_sync(0xffffffffu, x[m], h);
      x[m] = (lane & h) ? __fsub_rn(y, x[m]) : __fadd_rn(x[m], y);
    }
  }
#pragma unroll
  for (int hm = 1; hm < M; hm <<= 1) {
#pragma unroll
    for (int m = 0; m < M; ++m)
      if ((m & hm) == 0 && (m | hm) < m_count) {
        const float a = x[m], b = x[m | hm];
        x[m] = __fadd_rn(a, b);
        x[m | hm] = __fsub_rn(a, b);
      }
  }
#pragma unroll
  for (int m = 0; m < M; ++m) x[m] = __fmul_rn(x[m], inv_c);
}

// Positions of the retained tokens, ascending (kernel parameter by value).
struct RetList {
  int n;
  int pos[kMaxRetained];
};

// Where each entry of the new retained list comes from during an append.
struct RetUpdate {
  int n;
  int from_window[kMaxRetained];   // 1: window slot, 0: old retained slot
  int index[kMaxRetained];         // the slot
};

// Retained positions of a quantized prefix of Q tokens ({p < Q : p mod 2^floor(log2(Q-p)) == 0},
// one per age octave): how many, and the i-th in ascending order (octave floor(log2 Q) - i).
__host__ __device__ inline int retained_count(int Q) {
  int n = 0;
  while (n < 31 && (1 << n) <= Q) ++n;
  return n;
}
__host__ __device__ inline int retained_position(int Q, int i) {
  const int l = retained_count(Q) - 1 - i;
  return ((Q - (1 << l)) >> l) << l;
}

// The tokens one decode call reads, and how they are split over CTAs.  Sequence b holds L[b]
// tokens, Q[b] of them quantized (one entry for all sequences when `uniform`); its fp16 list
// is its retained entries, then window positions Q[b]..L[b]-1.
struct DecodeWork {
  int uniform;       // 1: every sequence has L[0], Q[0]
  int L[kMaxSeqs], Q[kMaxSeqs];
  int n_groups;      // quantized groups of the longest prefix (max over b of Q[b] / gk)
  int n_fp16;        // longest fp16 list
  int splits_q;      // CTAs per (b, kv head) over the groups
  int splits_f;      // CTAs per (b, kv head) over the fp16 list
  int splits;        // splits_q + splits_f (partials per (b, query head))
  float score_scale; // log2(e) / sqrt(d_k)
  int stall;         // test hook: CTA (0, 0, 0) asks for 16 bytes more than its first copy delivers
  int center;        // 1: the tensor-core kernel centres the value codes (long contexts)
};

// Lengths of sequence b in a decode call: L, Q, quantized groups (Q / gk; Q is 0 for an
// unquantized cache), retained entries and fp16 entries.
struct SeqWork {
  int L, Q, n_groups, n_ret, n_fp16;
};
__device__ __forceinline__ SeqWork seq_work(const DecodeWork& w, int b, int gk, int log_retain) {
  SeqWork s;
  s.L = w.uniform ? w.L[0] : w.L[b];
  s.Q = w.uniform ? w.Q[0] : w.Q[b];
  s.n_groups = s.Q / gk;
  s.n_ret = log_retain ? retained_count(s.Q) : 0;
  s.n_fp16 = s.n_ret + (s.L - s.Q);
  return s;
}

// Window slot each sequence's new token goes to on an append (-1: the sequence does not append).
struct SlotMap {
  int slot[kMaxSeqs];
};

// Device views of the cache buffers.
struct CacheBufs {
  const uint32_t* kcode;
  const __half2* ksz;
  const uint32_t* vcode;
  const __half2* vsz;
  const __half* win_k;
  const __half* win_v;
  const __half* ret_k;
  const __half* ret_v;
  const uint8_t* zcode;   // side codes (null without a side code)
  const __half2* zsz;     // side (scale, zero) per key group and coordinate
  const float* side_u;    // basis U_h, fp32 [Hkv][dk][sr]
  const int* table;       // block table of a paged cache, int32 [B][max_groups]
};

// Block-table entries to write (a launch parameter): table[idx[i]] = page[i].
struct TableWrites {
  int n;
  int idx[480];
  int page[480];
};

// Workspace layout: [status u32, padded to 256 B][(m, l) float2 per partial][o floats]
struct Partials {
  unsigned int* status;
  float2* ml;    // [B*Hq][splits]
  float* o;      // [B*Hq][splits][dv]
};

size_t workspace_bytes(const Dims& d, int splits);
Partials workspace_views(const Dims& d, int splits, void* ws);

// ---- launchers (return the launch error, cudaSuccess when fine) ----
// rotate: src holds unrotated keys that are rotated on the fly (prefill); otherwise src
// already holds the cached (rotated or not) keys (the window, on append)
cudaError_t launch_quantize_keys(const Dims& d, const __half* src, int src_rows, int g_begin,
                                 int n_groups, uint32_t* kcode, __half2* ksz, const int* table,
                                 bool rotate, cudaStream_t s);
cudaError_t launch_table_writes(const Dims& d, int* table, const TableWrites& tw, cudaStream_t s);

// Side codes of key groups [g_begin, g_begin + n_groups) whose base codes and (scale, zero)
// are already in kcode / ksz (same stream); keys read from src as for launch_quantize_keys.
cudaError_t launch_quantize_side(const Dims& d, const __half* src, int src_rows, int g_begin,
                                 int n_groups, const uint32_t* kcode, const __half2* ksz,
                                 const float* side_u, uint8_t* zcode, __half2* zsz, const int* table,
                                 bool rotate, cudaStream_t s);
cudaError_t launch_quantize_values(const Dims& d, const __half* src, int src_rows, int t_begin,
                                   int n_tokens, uint32_t* vcode, __half2* vsz, const int* table,
                                   cudaStream_t s);
cudaError_t launch_copy_rows(const Dims& d, const __half* src, int src_rows, int src_base, __half* dst,
                             int dst_rows, int dst_base, int n, int width, int nbh, cudaStream_t s);
// Rotated key rows (one warp per row): dst[bh][dst row i] = rotate(src[bh][src row i]) for
// i < n, rows (src_base + i) % src_rows -> (dst_base + i) % dst_rows, or, when `list` is
// given, rows list->pos[i] -> i.
cudaError_t launch_rotate_key_rows(const Dims& d, const __half* src, int src_rows, int src_base,
                                   __half* dst, int dst_rows, int dst_base, int n,
                                   const RetList* list, cudaStream_t s);
// The new token of every sequence b with slots.slot[b] >= 0 into window slot slots.slot[b]:
// the value row, and the key row (rotated when the cache rotates keys).
cudaError_t launch_append_token(const Dims& d, const __half* k, const __half* v, __half* win_k,
                                __half* win_v, const SlotMap& slots, cudaStream_t s);
// k may be null: only the value rows are copied
cudaError_t launch_copy_retained(const Dims& d, const __half* k, const __half* v, int L,
                                 const RetList& ret, __half* ret_k, __half* ret_v, cudaStream_t s);
cudaError_t launch_update_retained(const Dims& d, const RetUpdate& up, __half* win_k,
                                   __half* win_v, __half* ret_k, __half* ret_v, cudaStream_t s);
cudaError_t launch_decode_simple(const Dims& d, const CacheBufs& c, const DecodeWork& w,
                                 const __half* q, const Partials& p, cudaStream_t s);
bool decode_var_supported(const Dims& d);
cudaError_t launch_decode_var(const Dims& d, const CacheBufs& c, const DecodeWork& w,
                              const __half* q, const Partials& p, cudaStream_t s);
bool decode_mma_supported(const Dims& d);
cudaError_t launch_decode_mma(const Dims& d, const CacheBufs& c, const DecodeWork& w,
                              const __half* q, const Partials& p, cudaStream_t s);
cudaError_t launch_combine(const Dims& d, const DecodeWork& w, const Partials& p, __half* out,
                           cudaStream_t s);

}  // namespace kvq
