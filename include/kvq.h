/*
 * kvq.h — decode attention read straight from a packed, mixed-precision,
 * groupwise-quantized KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operation (one attention layer of autoregressive decoding):
 *   - the cache keeps every token ("LogQuant: Log-Distributed 2-Bit Quantization
 *     of KV Cache", §Méthodologie 3: quantize instead of evicting);
 *   - the most recent tokens stay fp16 (same page, §Comment LogQuant Fonctionne);
 *     optionally one older token per age octave stays fp16 too (same page,
 *     §Méthodologie 2, log-based filtering);
 *   - older keys are quantized per channel over groups of group_k tokens (same
 *     page, §5), older values per token over groups of group_v channels, keys
 *     with more bits than values ("Quantize What Counts: More for Keys, Less for
 *     Values", §La Solution, K4V2);
 *   - keys may be thinner than values, d_k < d_v ("Thin Keys, Full Values:
 *     Reducing KV Cache via Low-Dimensional Attention Selection", §2), and the
 *     score is q.k / sqrt(d_k);
 *   - the order in which tokens are visited is free (LogQuant §4, A.V = A_P.V_P).
 *
 * Quantizer (bit-exact contract; every step IEEE binary32, round to nearest even):
 *   s = fp16((max - min) / (2^bits - 1))   (+0 if that is zero)
 *   z = fp16(min)                          (+0 for a signed zero)
 *   code = s == 0 ? 0 : clamp(rint((x - z) / s), 0, 2^bits - 1)
 * Regions: with L tokens, Q = floor(max(L - window, 0) / group_k) * group_k
 * tokens are quantized and [Q, L) are fp16 (Q = 0 when the bit widths are 16).
 * Retained set (log_retain = 1): { p < Q : p mod 2^floor(log2(Q - p)) == 0 }.
 *
 * Optional side code (side_rank r > 0; "HeadQ: Distortion visible par le modele et
 * correction dans l'espace des scores pour la quantification du cache KV", §3):
 * with a caller-given basis U_h (fp32 [d_k][r] per kv head), each quantized key
 * group also stores, per token, the base residual projected on U_h and quantized:
 *   e = fl32(k - fl32(code * s + z))                  per channel
 *   y_i = sum_c U_h[c][i] * e_c                        fp32, c ascending from +0,
 *                                                      one rounded product and sum per c
 *   side codes: the quantizer above with side_bits, per coordinate i over the
 *   group's group_k tokens (z = fp16(min y_i) rounds to nearest)
 * and decode adds (U_h^T q) . z_hat_j / sqrt(d_k), z_hat = code * s + z, to the
 * score of every quantized token that is not retained.
 *
 * Optional key-only rotation (rot_keys = 1; "Quantize What Counts: More for Keys,
 * Less for Values", Intégration de la Rotation): every key is rotated before it is
 * cached and every query before it is used, by the randomized Hadamard transform
 *   k' = fp16(FWHT(sigma * k) / c_k),   q' = fp16(FWHT(sigma * q) / c_q)
 * with sigma_c = -1 where bit c of rot_signs is set, c_k = 2^ceil(log2(d_k)/2),
 * c_q = d_k / c_k (so q'.k' = q.k before the fp16 roundings), and FWHT the fp32
 * Walsh-Hadamard transform by butterflies of span 1, 2, ..., d_k/2, each
 * (x_i, x_{i+h}) -> (x_i + x_{i+h}, x_i - x_{i+h}).  The cache then holds k'
 * everywhere (codes, window, retained copies, side code).
 *
 * Buffer layouts (all caller-owned device memory, 256-byte aligned recommended,
 * 16-byte aligned required; sizes from kvq_buffer_sizes):
 *   kcode  u32  [B][Hkv][Lcap][d_k*k_bits/32]   token rows, channel c at word
 *               c/(32/k_bits), bit (c%(32/k_bits))*k_bits (LSB first)
 *   ksz    f16  [B][Hkv][Lcap/group_k][2*d_k]  (scale, zero) per key group and channel:
 *               for each packed word w of a key row (P = 32/k_bits channels, H = P/2)
 *               the scales of channels (wP+i, wP+i+H), i < H, then their zeros; with
 *               W = d_k*k_bits/32 words and 4 | W, word w's block is stored at
 *               position (w % (W/4))*4 + w/(W/4)
 *   vcode  u32  [B][Hkv][Lcap][d_v*v_bits/32]   same packing per token row
 *   vsz    f16  [B][Hkv][Lcap][d_v/group_v][2] (scale, zero) per token and value group
 *   win_k  f16  [B][Hkv][C][d_k]  token p in slot p % C, C = window + group_k
 *   win_v  f16  [B][Hkv][C][d_v]  (bits 16: C = max_context, the whole cache)
 *   ret_k  f16  [B][Hkv][32][d_k] retained tokens, ascending positions
 *   ret_v  f16  [B][Hkv][32][d_v]
 *   zcode  u8   [B][Hkv][Lcap][r*side_bits/8]  side codes of a token, coordinate i
 *               at bit i*side_bits of the little-endian row   (side_rank r > 0 only)
 *   zsz    f16  [B][Hkv][Lcap/group_k][r][2]   side (scale, zero) per key group and
 *               coordinate
 *   side_u f32  [Hkv][d_k][r]  the basis U_h; written by the caller before the first
 *               prefill, read by prefill, append and decode, never written here
 * with Lcap = max_context rounded up to a multiple of group_k.
 *
 * Paged caches (paged = 1; serving shapes, no counterpart on the pages): the six
 * quantized buffers hold a pool of n_pages pages instead of one Lcap-token region per
 * (b, kv head): page p is one key group of one sequence for every kv head, laid out
 *   kcode [n_pages][Hkv][group_k][d_k*k_bits/32]   ksz [n_pages][Hkv][2*d_k]
 *   vcode [n_pages][Hkv][group_k][d_v*v_bits/32]   vsz [n_pages][Hkv][group_k][d_v/group_v][2]
 *   zcode [n_pages][Hkv][group_k][r*side_bits/8]   zsz [n_pages][Hkv][r][2]
 * (each page is the (b, h) layout above restricted to one group), and block_table
 * int32 [B][Lcap/group_k] maps a sequence's group g to its page.  The library hands out
 * pages (prefill, and an append that quantizes a window group) and takes them back
 * (a new prefill of the sequence, kvq_release_sequence), and writes the table; the
 * window and retained buffers stay per sequence.  Needs quantized keys and values;
 * 1 <= n_pages, n_pages*Hkv*group_k < 2^30.
 *
 * Per-channel bit widths (k_bits = v_bits = 0; "Attention-Aware Transform Coding (AATC)",
 * §Méthodologie, Allocation de Bits): key channel c has k_widths[c] bits and value channel c
 * v_widths[c] bits, each in {0, 1, 2, 4, 8}, non-increasing over the channels (the
 * caller's decorrelating transform, folded into its projections, orders them by
 * strength); the channels of one value group share a width.  A channel of width 0 is
 * dropped: nothing is stored and it reads as 0.  Rows pack the codes channel after
 * channel, LSB-first, channel c at bit offset sum_{c'<c} width_c' (never straddling a
 * word), in W = max(1, ceil(sum of the widths / 32)) words:
 *   kcode u32 [B][Hkv][Lcap][Wk]    ksz f16 [B][Hkv][Lcap/group_k][d_k][2] (scale, zero)
 *   vcode u32 [B][Hkv][Lcap][Wv]    vsz as above; dropped channels / groups store (0, 0).
 * Not combined with side codes or rotation.  kvq_allocate_bits computes such a map.
 *
 * Conventions: every call is asynchronous on the caller's CUDA stream (passed as
 * void*, a cudaStream_t; NULL = legacy default stream); no call synchronizes or
 * copies device memory back to the host, except the status and record readers
 * (kvq_read_status, kvq_noalloc_read_status, kvq_debug_take_record).  The library
 * allocates nothing at call time; the only device memory it holds is the static
 * scratch array of kvq_decode_attention_noalloc (and, in a bounds-check build, its
 * debug record), one per GPU that loads it.  A cache handle must not be used from two host
 * threads or two streams at once.  Inputs must be finite; NaN or Inf in K, V or
 * q gives undefined (but memory-safe) results.  GQA: query head hq reads kv
 * head hq / (n_q_heads / n_kv_heads).  Every function returns KVQ_OK (0) or one
 * of the negative codes below and changes nothing when it fails argument checks.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_OK                 0
#define KVQ_ERR_INVALID_ARG   -1  /* null pointer, non-positive size, L > max_context */
#define KVQ_ERR_UNSUPPORTED   -2  /* shape / bit width / group outside the built set */
#define KVQ_ERR_ALIGN         -3  /* a device pointer is not 16-byte aligned */
#define KVQ_ERR_CAPACITY      -4  /* an append past max_context; a page pool too small */
#define KVQ_ERR_WORKSPACE     -5  /* workspace smaller than kvq_decode_workspace_size */
#define KVQ_ERR_STATE         -6  /* decode or append on an empty sequence */
#define KVQ_ERR_CUDA          -7  /* a CUDA runtime call or kernel launch failed */

#define KVQ_MAX_RETAINED      32

/* Device status bits, written into the first word of a decode workspace. */
#define KVQ_STATUS_TIMEOUT    1u  /* a bounded wait in the decode kernel gave up */

typedef struct kvq_config {
    int batch;          /* B, sequences (slots) of the cache */
    int n_q_heads;      /* Hq */
    int n_kv_heads;     /* Hkv; Hq % Hkv == 0 */
    int d_k;            /* key/query head dim: 32, 64, 128 or 256 */
    int d_v;            /* value head dim: 32, 64, 128 or 256 */
    int k_bits;         /* 2, 4, 8, 16 (= unquantized; then v_bits must be 16), or 0 */
    int v_bits;         /* 2, 4, 8, 16, or 0 (per-channel widths: both 0) */
    int group_k;        /* tokens per key group: 16, 32, 64 or 128 */
    int group_v;        /* channels per value group: divides d_v, >= 32/v_bits */
    int window;         /* R >= 0: fp16 recent tokens kept beside the quantized prefix */
    int log_retain;     /* 0/1: keep log-spaced older tokens in fp16 (ignored at 16 bits) */
    int max_context;    /* capacity in tokens, >= 1 */
    int side_rank;      /* r: 0 (no side code), 4 or 8; needs quantized keys */
    int side_bits;      /* bits per side code: 4 or 8, with side_rank*side_bits 16 or 32 */
    int rot_keys;       /* 0/1: key-only rotation */
    unsigned int rot_signs[8];  /* rotation signs: bit c (word c/32, bit c%32) set -> -1 */
    int paged;          /* 0/1: quantized groups live in a shared pool of pages (see below) */
    int n_pages;        /* pages in the pool (paged caches); one page = one key group */
    unsigned char k_widths[256];  /* k_bits = v_bits = 0: bits of key channel c (see below) */
    unsigned char v_widths[256];  /* k_bits = v_bits = 0: bits of value channel c */
} kvq_config;

typedef struct kvq_sizes {
    size_t kcode, ksz, vcode, vsz, win_k, win_v, ret_k, ret_v;
    size_t workspace;   /* a decode workspace large enough for any length and split count */
    size_t zcode, zsz, side_u;   /* side code buffers (0 without a side code) */
    size_t block_table; /* paged caches: int32 [B][max_context/group_k rounded up] */
} kvq_sizes;

typedef struct kvq_buffers {
    void *kcode, *ksz, *vcode, *vsz, *win_k, *win_v, *ret_k, *ret_v;
    void *zcode, *zsz, *side_u;  /* side code buffers (NULL without a side code) */
    void *block_table;           /* paged caches (NULL otherwise); written by the library */
} kvq_buffers;

typedef struct kvq_cache kvq_cache;   /* opaque host-side handle */

/* Split plan of one decode call (see kvq_plan_decode). */
typedef struct kvq_plan {
    int splits_quant;   /* CTAs per (b, kv head) over the quantized groups */
    int splits_fp16;    /* CTAs per (b, kv head) over window + retained tokens */
    int n_groups;       /* quantized groups, Q / group_k */
    int n_fp16;         /* fp16 tokens: retained + window */
    int fast_path;      /* 1: tensor-core kernel; 0: generic CUDA-core kernel */
    int centered;       /* 1: the tensor-core kernel centres the value codes (see below) */
} kvq_plan;

/* Bytes of each buffer for a configuration (see the layout above).  Host only.
 * Buffers a configuration does not use (e.g. kcode at 16 bits) get size 0 and
 * may be passed as NULL.  Errors: INVALID_ARG, UNSUPPORTED. */
int kvq_buffer_sizes(const kvq_config* cfg, kvq_sizes* out);

/* Create a handle over caller-owned device buffers (not touched here).  Queries
 * the current device's SM count.  The handle copies cfg and the pointers; the
 * buffers must outlive it.  Errors: INVALID_ARG, UNSUPPORTED, ALIGN, CUDA. */
int kvq_cache_init(const kvq_config* cfg, const kvq_buffers* bufs, kvq_cache** out);

/* Free the handle (not the buffers).  NULL is a no-op. */
void kvq_cache_destroy(kvq_cache* cache);

/* Fill an empty cache with L >= 1 tokens: k fp16 [B][Hkv][L][d_k], v fp16
 * [B][Hkv][L][d_v], contiguous device memory.  Quantizes [0, Q), copies [Q, L)
 * into the window and the retained tokens into ret_k/ret_v.  Resets any earlier
 * content.  Errors: INVALID_ARG (L < 1 or L > max_context), CAPACITY (a paged
 * pool with too few pages), ALIGN, CUDA. */
int kvq_quantize_prefill(kvq_cache* cache, const void* k, const void* v, int L, void* stream);

/* Append one token per sequence: k_new fp16 [B][Hkv][d_k], v_new fp16
 * [B][Hkv][d_v].  When the window reaches window + group_k tokens, its oldest
 * group_k tokens are quantized and the retained set is updated.
 * Errors: STATE (no prefill yet), CAPACITY, INVALID_ARG, ALIGN, CUDA. */
int kvq_append(kvq_cache* cache, const void* k_new, const void* v_new, void* stream);

/* Sequences of different lengths (serving batches; no counterpart on the pages, whose
 * rules apply to each sequence on its own: its window, quantized prefix and retained set
 * follow from its own length).
 *
 * kvq_quantize_prefill_ragged: k fp16 [B][Hkv][L_max][d_k], v fp16 [B][Hkv][L_max][d_v];
 * sequence b's first lengths[b] tokens are valid (lengths: host int[B], each in
 * [1, L_max], L_max <= max_context).  With more than KVQ_MAX_SEQS sequences the lengths
 * must be equal (UNSUPPORTED otherwise).
 * kvq_append_ragged: kvq_append for the sequences with active[b] != 0 (host bytes [B];
 * NULL = all); the rows of the others in k_new / v_new are ignored and their state is
 * unchanged.  A partial mask needs B <= KVQ_MAX_SEQS (UNSUPPORTED otherwise).
 * kvq_decode_attention then attends, for every sequence, over its own L_b tokens.
 * Errors as for kvq_quantize_prefill / kvq_append. */
#define KVQ_MAX_SEQS 256
int kvq_quantize_prefill_ragged(kvq_cache* cache, const void* k, const void* v, int L_max,
                                const int* lengths, void* stream);

int kvq_append_ragged(kvq_cache* cache, const void* k_new, const void* v_new,
                      const unsigned char* active, void* stream);

/* Slot management (serving; no counterpart on the pages).
 * kvq_prefill_sequence: prefill sequence b alone with 1 <= L <= max_context tokens,
 * k fp16 [Hkv][L][d_k], v fp16 [Hkv][L][d_v]; the other sequences are untouched.  A
 * paged cache first takes back b's old pages.
 * kvq_release_sequence: forget sequence b (a paged cache takes back its pages); its
 * length becomes 0.  Decode fails with STATE while any sequence is empty, and so does
 * an append that includes an empty sequence.
 * kvq_free_pages: pages of the pool not in use (0 for caches that are not paged).
 * With more than KVQ_MAX_SEQS sequences, decode needs their lengths equal (UNSUPPORTED).
 * Errors: INVALID_ARG (b or L out of range), CAPACITY (the pool has too few free pages;
 * nothing changes), ALIGN, CUDA. */
int kvq_prefill_sequence(kvq_cache* cache, int b, const void* k, const void* v, int L, void* stream);
int kvq_release_sequence(kvq_cache* cache, int b);
int kvq_free_pages(const kvq_cache* cache);

/* Reverse water-filling ("Attention-Aware Transform Coding (AATC)", §Méthodologie,
 * Allocation de Bits; host only): widths[i] in {0, 1, 2, 4, 8} for n units of weight
 * weight[i] >= 0 (a key channel, or a value group whose width bit costs unit_bits = group_v
 * bits), minimising sum_i weight[i] * 4^-widths[i] under `budget` bits per row.  Each
 * step of a unit's width (0->1->2->4->8) lowers that sum by weight * (4^-b1 - 4^-b2) for
 * (b2 - b1) * unit_bits bits; steps are taken in decreasing order of that drop per bit,
 * equal drops together, until the next set would exceed the budget; a step that lowers
 * nothing is never taken.  Units of larger weight get at least as many bits, so weights
 * sorted in decreasing order give a map kvq_config accepts.  Returns the bits spent, or
 * INVALID_ARG (n < 1, unit_bits < 1, budget < 0, a weight negative or not finite, null). */
int kvq_allocate_bits(const double* weight, int n, int unit_bits, int budget, unsigned char* widths);

/* Workspace bytes kvq_decode_attention needs at the cache's current length for
 * num_splits (0 = automatic).  Always <= kvq_sizes.workspace. */
int kvq_decode_workspace_size(const kvq_cache* cache, int num_splits, size_t* bytes);

/* Attention of one query token per sequence over all L cached tokens:
 * q fp16 [B][Hq][d_k] -> out fp16 [B][Hq][d_v].  Scores q.k/sqrt(d_k), fp32
 * softmax and accumulation, split over tokens (flash-decoding) and merged by a
 * log-sum-exp combine.  workspace: device scratch of workspace_bytes; its first
 * 4 bytes are a status word the kernel ORs KVQ_STATUS_* bits into (never
 * cleared by this call; see kvq_reset_status).  num_splits: 0 = automatic, else
 * the number of splits over the quantized groups (or over the fp16 tokens when
 * nothing is quantized), clamped to the available work.
 * Errors: STATE, INVALID_ARG, ALIGN, WORKSPACE, CUDA. */
int kvq_decode_attention(kvq_cache* cache, const void* q, void* out, void* workspace,
                         size_t workspace_bytes, int num_splits, void* stream);

/* Decode kernel selection for a cache (default KVQ_KERNEL_AUTO: the tensor-core
 * kernel where it is built for the shape, else the generic CUDA-core kernel).
 * KVQ_KERNEL_TENSOR fails with UNSUPPORTED on shapes it is not built for. */
#define KVQ_KERNEL_AUTO     0
#define KVQ_KERNEL_GENERIC  1
#define KVQ_KERNEL_TENSOR   2
int kvq_set_decode_kernel(kvq_cache* cache, int kernel);

/* Value-code centring of the tensor-core kernel on fixed-width caches (a numerical choice of
 * this library; no counterpart on the pages).  Its p.V products of unsigned value codes
 * accumulate in fp32 inside the tensor core, which truncates; the accumulated magnitude grows
 * with the tokens summed while the attention output shrinks, so the relative error grows with
 * the context.  Centred codes (code - 2^(v_bits-1), the offset added back through the zero-point
 * sum) keep the accumulators near zero, at about 7% more decode time.  KVQ_CENTER_AUTO (the
 * default) centres when the longest sequence has at least 65536 quantized tokens; ON and OFF
 * force it.  The plan's `centered` field reports the choice.  Errors: INVALID_ARG. */
#define KVQ_CENTER_AUTO     0
#define KVQ_CENTER_OFF      1
#define KVQ_CENTER_ON       2
int kvq_set_value_centering(kvq_cache* cache, int mode);

/* kvq_decode_attention without a workspace argument, for callers that cannot
 * allocate device memory: an engine that has reserved the device's memory for
 * its own pool, a plugin whose host offers no allocator, or a latency-critical
 * loop that must not pay for cudaMalloc/cudaFree.  (The pages have no
 * counterpart: this is a property of the library, not of the method.)
 * The split partials go to a scratch array of KVQ_NOALLOC_SCRATCH_BYTES that
 * lives in the library; every GPU that loads the library holds it until the
 * process exits.  Nothing is allocated at call time.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress, with that
 * device current); make that first call before any stream capture.  The array
 * is shared by every call and keeps the last call's contents; calls whose
 * executions overlap on the GPU race on it, so issue them on one stream or
 * otherwise serialize them.  Its first word is a status word like a workspace's:
 * zero when the library is loaded, ORed with KVQ_STATUS_* bits by any call whose
 * bounded waits gave up (that call's output is then undefined), never cleared by
 * a decode; read it with kvq_noalloc_read_status, clear it with
 * kvq_noalloc_reset_status (both for the current device).
 * num_splits: 0 = automatic, reduced if needed so that the partials fit in the
 * array; an explicit split count whose partials do not fit, or a cache so large
 * that even one split per (b, kv head) does not fit, returns KVQ_ERR_WORKSPACE.
 * Other errors as for kvq_decode_attention. */
#define KVQ_NOALLOC_SCRATCH_BYTES (8u << 20)
int kvq_decode_attention_noalloc(kvq_cache* cache, const void* q, void* out, int num_splits,
                                 void* stream);

/* Status word of the current device's scratch array (see kvq_decode_attention_noalloc):
 * kvq_noalloc_read_status waits for stream, then copies the word to *status (it
 * synchronizes, like kvq_read_status); kvq_noalloc_reset_status zeroes it,
 * asynchronously on stream.  Errors: INVALID_ARG (status NULL), CUDA. */
int kvq_noalloc_read_status(unsigned int* status, void* stream);
int kvq_noalloc_reset_status(void* stream);

/* The plan kvq_decode_attention would use now (host only, no launch); its counts are
 * those of the longest sequence. */
int kvq_get_plan(const kvq_cache* cache, int num_splits, kvq_plan* out);

/* Pure host planner behind kvq_get_plan, for a configuration, length L, SM count
 * and split request.  Errors: INVALID_ARG, UNSUPPORTED. */
int kvq_plan_decode(const kvq_config* cfg, int L, int sm_count, int num_splits, kvq_plan* out);

/* Host-side state of sequence 0 (of every sequence when all have the same length):
 * length L, quantized prefix Q, retained count and the ascending retained positions
 * (retained_idx: host int[32], may be NULL). */
int kvq_get_state(const kvq_cache* cache, int* L, int* Q, int* n_retained, int* retained_idx);

/* The same for sequence b (0 <= b < batch, else INVALID_ARG). */
int kvq_get_seq_state(const kvq_cache* cache, int b, int* L, int* Q, int* n_retained,
                      int* retained_idx);

/* The retention rule for a quantized prefix of Q tokens (host only): writes the
 * ascending positions into out[0..cap) and returns their count (>= 0), or
 * INVALID_ARG if out is NULL while Q > 0, or if cap is too small. */
int kvq_retained_positions(int Q, int* out, int cap);

/* Test hook for the timeout path (no counterpart on the pages).  Arms the next
 * kvq_decode_attention on this cache: when it runs the tensor-core kernel, one CTA
 * asks its first shared-memory copy for 16 bytes more than the copy delivers, so
 * that CTA's bounded waits give up after their 1 s limit; it then sets
 * KVQ_STATUS_TIMEOUT in the workspace status word and contributes nothing, and the
 * call's output is undefined.  Nothing faults or hangs, the context stays usable and
 * the following calls are normal.  Returns KVQ_OK or KVQ_ERR_INVALID_ARG. */
int kvq_debug_stall_next_decode(kvq_cache* cache);

/* Zero the status word of a decode workspace (asynchronous, on stream). */
int kvq_reset_status(void* workspace, void* stream);

/* Wait for stream, then copy the status word of a decode workspace to *status.
 * The only call that synchronizes. */
int kvq_read_status(const void* workspace, unsigned int* status, void* stream);

/* Static description of an error code. */
const char* kvq_strerror(int code);

/* Bounds-check build (a development aid; no counterpart on the pages).  The library built
 * with -DKVQ_DEBUG (libkvq_debug.so beside libkvq.so) compares every global-memory index its
 * kernels compute with the extent of the buffer it addresses; a failed check is counted in a
 * record the library keeps on each device (the first failure's site, index and extent), and
 * the access is skipped or redirected to the buffer's start.  Nothing traps.
 * kvq_debug_build: 1 in a bounds-check build, else 0.
 * kvq_debug_take_record: waits for stream, copies the current device's record to *out and
 * clears it.  Errors: INVALID_ARG (out NULL), UNSUPPORTED (not a bounds-check build), CUDA.
 * kvq_debug_site_name: static description of a record's site. */
typedef struct kvq_debug_record {
    unsigned int failures;   /* failed checks since the record was last taken */
    unsigned int site;       /* where the first one failed (kvq_debug_site_name) */
    long long index;         /* its index, in elements of the buffer's type */
    long long extent;        /* the buffer's extent in the same elements */
} kvq_debug_record;
int kvq_debug_build(void);
int kvq_debug_take_record(kvq_debug_record* out, void* stream);
const char* kvq_debug_site_name(unsigned int site);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
