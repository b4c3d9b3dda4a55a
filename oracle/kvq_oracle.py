"""CPU oracle for decode attention over a packed mixed-precision KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports this module: only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm
may call it.  It shares no code with the CUDA library; both sides are fed the
same fp16 tensors by ``mixed_precision_quantized_pack_b200.workloads``.

What it computes, step by step in the order the pages give it:

1. Regions.  A full-precision recent window stays fp16 ("LogQuant: Log-Distributed
   2-Bit Quantization of KV Cache", §Comment LogQuant Fonctionne / §Méthodologie 2);
   everything older is quantized, never evicted (same page, §Méthodologie 3).
   Reading: key groups need whole groups of G_k tokens, so the quantized prefix is
   Q = floor(max(L-R, 0) / G_k) * G_k and the window [Q, L) holds R..R+G_k-1
   tokens.  Bit width 16 means "not quantized": Q = 0.
2. Keys are quantized per channel over groups of G_k tokens (LogQuant, §5
   "par canal par Clé"; group sizes from "Quantize What Counts", §Sensibilité à
   la Taille de Groupe), with more bits than values (K4V2 by default; same page,
   §La Solution).  Values are quantized per token over groups of G_v channels.
3. The quantizer is asymmetric uniform min-max with an fp16 scale and zero per
   group (reading: the pages name Quanto/HQQ but print no formula):
       s16 = fp16(fl32(mx - mn) / fl32(2^b - 1)),  s16 == 0 -> +0
       z16 = fp16(mn)  (exact; -0 -> +0)
       code = 0 if s16 == 0 else clamp(rint(fl32(fl32(x - z16) / s16)), 0, 2^b-1)
   All arithmetic is IEEE binary32 with round-to-nearest-even, one operation at
   a time (numpy float32 ufuncs), rint is half-to-even.
4. Packing: within a token row, codes are packed channel by channel, least
   significant bits first, into little-endian uint32 words (channel c of a b-bit
   row lives in word c // (32/b) at bit (c % (32/b)) * b).  Value (scale, zero)
   pairs are stored as fp16 pairs.  The key (scale, zero) of one group follow the
   packed words of a key row: for word w (channels w*P .. w*P+P-1, P = 32/b,
   H = 16/b) come the P scales in the order (w*P+i, w*P+i+H) for i < H, then the
   P zeros in the same order.  When the row has W >= 4 words and 4 divides W,
   the blocks of the W words are stored quarter-interleaved: the block of word w
   sits at position (w mod W/4) * 4 + w div W/4 (key_meta_order).  The pages fix
   no memory layout; this one puts the two channels whose codes share a 32-bit
   word half by half next to each other, and the blocks that the four quarters of
   a key row need at the same time next to each other.
5. Log-spaced retention (LogQuant §Méthodologie 2, "density halves further
   back"; the printed text is garbled).  Reading: among the quantized positions
   p < Q, p is kept in fp16 iff p is a multiple of 2^floor(log2(Q - p)); this
   keeps exactly one token per age octave [2^l, 2^(l+1)), floor(log2 Q)+1 tokens
   in all, and as Q grows a token can only leave the set.
6. Attention (fp64) over every token: fp16 values for window and retained
   tokens, code*s16 + z16 otherwise; scores q.k/sqrt(d_k) ("Thin Keys, Full
   Values", §2, where d_k may be smaller than d_v; the score form of "HeadQ",
   §2.1), softmax with max subtraction, p.V.  Token order is irrelevant
   (LogQuant §4, A.V = A_P.V_P).  GQA: query head hq reads kv head hq // n_rep.
7. Optional side code ("HeadQ: ... correction dans l'espace des scores", §3,
   Aperçu de l'algorithme, steps 2 and 3), with a basis U_h of r columns per kv
   head (fp32 [d_k][r], given by the caller; the pages learn it by PCA over
   calibration queries).  When a key group is quantized, for each of its tokens:
       e = fl32(k - fl32(code * s16 + z16))           (the base residual)
       y_i = sum_c U_h[c, i] * e_c                      (fp32, c ascending from +0,
                                                         one product and one sum at a time)
   and the side quantizer Q_q (reading: the step-3 quantizer, per coordinate i
   over the group's G_k tokens, on the fp32 y; z16 = fp16(min) then rounds)
   gives side codes and one fp16 (scale, zero) per coordinate.  Decode adds
   (U_h^T q) . z_hat_j / sqrt(d_k), z_hat = code * s + z, to the score of every
   quantized token that is not retained; window and retained tokens are exact.
8. Optional key-only rotation ("Quantize What Counts", §Contributions Clés and
   §Résultats, Intégration de la Rotation: rotating the keys alone, as QuaRot
   does, recovers most of K4V4's accuracy at K4V2).  Reading: a randomized
   Hadamard rotation R = H_d diag(sigma) / sqrt(d) (Sylvester H_d, signs sigma
   given by the caller), applied to every key before it is cached (prefill and
   append) and to the query at decode, so that q'.k' = q.k.  To keep every step
   exact but the fp16 roundings, keys are scaled by 1/c_k and queries by 1/c_q,
   powers of two with c_k * c_q = d (c_k = 2^ceil(log2(d)/2)):
       k' = fp16(FWHT(sigma * k) / c_k),   q' = fp16(FWHT(sigma * q) / c_q)
   where FWHT is the Walsh-Hadamard transform in fp32 by butterflies of span
   1, 2, 4, ..., d/2, each (x_i, x_{i+h}) -> (x_i + x_{i+h}, x_i - x_{i+h}).
   The rotated keys are then cached exactly as unrotated ones would be.

9. Optional per-channel bit widths ("Attention-Aware Transform Coding (AATC)", §Méthodologie,
   Allocation de Bits: reverse water-filling gives each transformed channel its own number
   of bits, zero for the weakest, separately for keys and values).  Readings: the
   decorrelating transform is the caller's (folded into the projections), so the cache
   sees transformed keys and values; widths come from {0, 1, 2, 4, 8}; key channel c has
   width kw_c, non-increasing in c (the transform orders channels by strength); the
   channels of one value group share a width, non-increasing from group to group.  A
   width-b channel (b >= 1) goes through the quantizer of step 3 with b bits (keys per
   channel over G_k tokens, values per token over the group); a width-0 channel is
   dropped: nothing is stored and it reads as 0.  A token row packs the codes channel
   after channel, LSB-first: channel c at bit offset o_c = sum of the widths before it
   (a power-of-two width never straddles a word because every width before it is a
   multiple of it), in max(1, ceil(sum/32)) words.  Key (scale, zero) are stored plainly,
   [group][d_k][2]; dropped channels and groups store (0, 0).
   The allocation (allocate_bits) minimises sum_c w_c * 4^(-b_c) -- the high-rate
   distortion of a b-bit uniform quantizer on a channel of weight w_c (its attention-
   aware weight times its variance, from the caller's calibration), the whole w_c when
   dropped -- under a budget of bits per row, as reverse water-filling does: lowering a
   common slope ("water level"), every step of a channel's width (0->1->2->4->8) whose
   distortion drop per bit lies above the level is taken.  Steps of equal slope are taken
   together, zero-slope steps never, and the level stops at the first set of steps that
   would exceed the budget (so the result is optimal for the bits it spends).

Buffer formats mirror the CUDA library's so the tests can compare bytes:
  kcode u32 [B][Hkv][Lcap][d_k*kb/32]        ksz fp16 [B][Hkv][Lcap/Gk][2*d_k] (key_meta_order)
  vcode u32 [B][Hkv][Lcap][d_v*vb/32]        vsz fp16 [B][Hkv][Lcap][d_v/Gv][2]
  win_k/v fp16 [B][Hkv][C][d] with token p in slot p % C,
          C = R + G_k (quantized caches) or Lcap (bits 16)
  ret_k/v fp16 [B][Hkv][32][d] in ascending position order, ret_idx int32 list.
  zcode u8 [B][Hkv][Lcap][r*q/8]: the r side codes of a token, coordinate i at bit
        i*q of the little-endian row (pack_side); zsz fp16 [B][Hkv][Lcap/Gk][r][2].
  Per-channel widths (k_bits = v_bits = 0, step 9): kcode u32 [B][Hkv][Lcap][Wk],
        ksz fp16 [B][Hkv][Lcap/Gk][d_k][2], vcode u32 [B][Hkv][Lcap][Wv], vsz as above,
        W = max(1, ceil(sum of the widths / 32)).
"""
from __future__ import annotations

import math
from typing import List, Optional

import numpy as np

MAX_RETAINED = 32


# ---------------------------------------------------------------- regions -----
def quantized_prefix(L: int, window: int, group_k: int, k_bits: int) -> int:
    """Q: number of leading tokens held quantized (step 1 above)."""
    if k_bits == 16:
        return 0
    return max(L - window, 0) // group_k * group_k


def retained_positions(Q: int) -> List[int]:
    """Ascending list {p < Q : p mod 2^floor(log2(Q-p)) == 0} (step 5 above)."""
    if Q <= 0:
        return []
    p = np.arange(Q, dtype=np.int64)
    age = (Q - p).astype(np.float64)
    _, e = np.frexp(age)                 # age = m * 2^e, m in [0.5, 1): floor(log2 age) = e-1
    octave = (e - 1).astype(np.int64)
    keep = (p % (np.int64(1) << octave)) == 0
    return [int(x) for x in p[keep]]


# -------------------------------------------------------------- quantizer -----
def minmax_quantize(x: np.ndarray, bits: int, axis: int):
    """Asymmetric min-max quantizer of step 3 over groups laid along ``axis``.

    ``x`` holds fp16 values (any float dtype holding them exactly), or fp32 values
    (float32 dtype: the side coordinates of step 7, where z16 = fp16(min) rounds).
    Returns (codes uint32 with x's shape, s16 fp16, z16 fp16) where s16/z16 keep a
    length-1 ``axis``.
    """
    x = np.asarray(x)
    # fp32 data (the side quantizer's projections) is taken as it is; anything else
    # holds fp16 values and is read through fp16, which is exact
    x32 = x if x.dtype == np.float32 else x.astype(np.float16).astype(np.float32)
    mn = x32.min(axis=axis, keepdims=True)
    mx = x32.max(axis=axis, keepdims=True)
    levels = np.float32(2 ** bits - 1)
    s32 = (mx - mn) / levels
    s16 = s32.astype(np.float16)
    s16 = np.where(s16 == 0, np.float16(0.0), s16).astype(np.float16)   # canonical +0
    z16 = (mn + np.float32(0.0)).astype(np.float16)                     # exact, -0 -> +0
    sf = s16.astype(np.float32)
    zf = z16.astype(np.float32)
    diff = x32 - zf
    with np.errstate(divide="ignore", invalid="ignore"):
        quot = diff / sf
    code = np.rint(quot)
    code = np.where(sf == 0, np.float32(0.0), code)
    code = np.clip(code, 0, levels)
    return code.astype(np.uint32), s16, z16


def dequantize(codes: np.ndarray, s16: np.ndarray, z16: np.ndarray) -> np.ndarray:
    """code * s + z, exactly, in fp64."""
    return codes.astype(np.float64) * s16.astype(np.float64) + z16.astype(np.float64)


def key_residual(k: np.ndarray, codes: np.ndarray, s16: np.ndarray, z16: np.ndarray) -> np.ndarray:
    """Step 7: e = fl32(k - fl32(code * s16 + z16)), elementwise, fp32 (code*s16 is exact)."""
    k32 = np.asarray(k, np.float16).astype(np.float32)
    base = codes.astype(np.float32) * s16.astype(np.float32)
    base = base + z16.astype(np.float32)
    return k32 - base


def side_project(e: np.ndarray, U: np.ndarray) -> np.ndarray:
    """Step 7: y[n][i] = sum_c U[c][i] * e[n][c] in fp32, c ascending from +0, one
    rounded product and one rounded sum at a time.  e fp32 [n][d], U fp32 [d][r]."""
    e = np.asarray(e, np.float32)
    U = np.asarray(U, np.float32)
    y = np.zeros((e.shape[0], U.shape[1]), np.float32)
    for c in range(e.shape[1]):
        y = y + e[:, c:c + 1] * U[c][None, :]
    return y


def side_code_group(k: np.ndarray, kcodes: np.ndarray, ksz: np.ndarray, U: np.ndarray,
                    bits: int, group_k: int):
    """Side code of keys [n][d] (n a multiple of group_k) whose base codes [n][d] and
    per-group (scale, zero) ksz fp16 [n/group_k][d][2] are given: returns side codes
    uint32 [n][r] and side (scale, zero) fp16 [n/group_k][r][2] (step 7)."""
    n, d = k.shape
    s = np.repeat(ksz[:, :, 0], group_k, axis=0)
    z = np.repeat(ksz[:, :, 1], group_k, axis=0)
    y = side_project(key_residual(k, kcodes, s, z), U)                   # [n][r] fp32
    r = y.shape[1]
    codes, ss, sz = minmax_quantize(y.reshape(n // group_k, group_k, r), bits, axis=1)
    return codes.reshape(n, r), np.stack([ss[:, 0, :], sz[:, 0, :]], axis=-1)


def side_query(U: np.ndarray, q: np.ndarray) -> np.ndarray:
    """U^T q in fp64 (step 7): the query's coordinates in the side basis, U fp32 [d][r]."""
    return np.asarray(U, np.float64).T @ np.asarray(q, np.float64)


def pack_side(codes: np.ndarray, bits: int) -> np.ndarray:
    """[..., r] side codes -> [..., ceil(r*bits/8)] bytes: coordinate i at bit i*bits of
    the little-endian row, unused high bits 0."""
    r = codes.shape[-1]
    shifts = np.arange(r, dtype=np.uint64) * np.uint64(bits)
    row = (codes.astype(np.uint64) << shifts).sum(axis=-1)
    nbytes = -(-r * bits // 8)
    out = [(row >> np.uint64(8 * j)) & np.uint64(0xFF) for j in range(nbytes)]
    return np.stack(out, axis=-1).astype(np.uint8)


def unpack_side(rows: np.ndarray, bits: int, r: int) -> np.ndarray:
    """Inverse of pack_side."""
    acc = np.zeros(rows.shape[:-1], np.uint64)
    for j in range(rows.shape[-1]):
        acc |= rows[..., j].astype(np.uint64) << np.uint64(8 * j)
    shifts = np.arange(r, dtype=np.uint64) * np.uint64(bits)
    return ((acc[..., None] >> shifts) & np.uint64((1 << bits) - 1)).astype(np.uint32)


def fwht32(x: np.ndarray) -> np.ndarray:
    """Step 8: Walsh-Hadamard transform along the last axis in fp32, butterflies of span
    1, 2, ..., d/2, each pair (i, i+h) with i & h == 0 -> (x_i + x_{i+h}, x_i - x_{i+h})."""
    y = np.asarray(x, np.float32).copy()
    d = y.shape[-1]
    h = 1
    while h < d:
        for i in range(d):
            if i & h == 0:
                a = y[..., i].copy()
                b = y[..., i + h].copy()
                y[..., i] = a + b
                y[..., i + h] = a - b
        h *= 2
    return y


def rotation_scales(d: int):
    """(c_k, c_q): powers of two with c_k * c_q = d, c_k = 2^ceil(log2(d)/2)."""
    e = int(math.log2(d))
    ck = 2 ** ((e + 1) // 2)
    return ck, d // ck


def sign_vector(sign_bits, d: int) -> np.ndarray:
    """sigma_c = -1 where bit c of the little-endian words sign_bits is set, else +1."""
    return np.array([-1.0 if (sign_bits[c // 32] >> (c % 32)) & 1 else 1.0 for c in range(d)], np.float32)


def rotate_rows(x: np.ndarray, sigma: np.ndarray, c: int) -> np.ndarray:
    """Step 8: fp16(FWHT(sigma * x) / c) for fp16 rows x [..., d] (sigma*x and /c are exact)."""
    y = np.asarray(x, np.float16).astype(np.float32) * sigma
    return (fwht32(y) / np.float32(c)).astype(np.float16)


def quantize_keys(k: np.ndarray, group_k: int, bits: int):
    """Keys [n][d] with n a multiple of group_k -> codes [n][d], sz fp16 [n/group_k][d][2].

    One (scale, zero) per channel per group of group_k consecutive tokens.
    """
    n, d = k.shape
    assert n % group_k == 0
    g = k.reshape(n // group_k, group_k, d)
    codes, s, z = minmax_quantize(g, bits, axis=1)          # s, z: [ng][1][d]
    sz = np.stack([s[:, 0, :], z[:, 0, :]], axis=-1)
    return codes.reshape(n, d), sz


def quantize_values(v: np.ndarray, group_v: int, bits: int):
    """Values [n][d] -> codes [n][d], sz fp16 [n][d/group_v][2] (groups of channels per token)."""
    n, d = v.shape
    assert d % group_v == 0
    g = v.reshape(n, d // group_v, group_v)
    codes, s, z = minmax_quantize(g, bits, axis=2)          # s, z: [n][ng][1]
    sz = np.stack([s[:, :, 0], z[:, :, 0]], axis=-1)
    return codes.reshape(n, d), sz


# ---------------------------------------------------------------- packing -----
def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """[..., d] codes -> [..., d*bits/32] uint32 words, channels LSB-first (step 4)."""
    per = 32 // bits
    d = codes.shape[-1]
    assert d % per == 0
    c = codes.astype(np.uint64).reshape(codes.shape[:-1] + (d // per, per))
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    words = (c << shifts).sum(axis=-1)
    return words.astype(np.uint32)


def key_meta_order(d_k: int, bits: int):
    """Slot order of one key group's fp16 (scale, zero) block (step 4): for slot i of
    the 2*d_k slots, the channel it holds and whether it is the scale (0) or zero (1)."""
    per, half = 32 // bits, 16 // bits
    words = d_k // per
    quarter = words // 4 if words % 4 == 0 else 0
    chan, which = [], []
    for pos in range(words):
        w = (pos % 4) * quarter + pos // 4 if quarter else pos     # word stored at pos
        for part in (0, 1):                          # scales, then zeros
            for i in range(half):
                for c in (w * per + i, w * per + i + half):
                    chan.append(c)
                    which.append(part)
    return np.array(chan), np.array(which)


def pack_key_meta(sz: np.ndarray, bits: int) -> np.ndarray:
    """sz fp16 [..., d_k, 2] (scale, zero per channel) -> [..., 2*d_k] in key_meta_order."""
    chan, which = key_meta_order(sz.shape[-2], bits)
    return sz[..., chan, which]


def unpack_key_meta(block: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of pack_key_meta: [..., 2*d_k] -> [..., d_k, 2]."""
    d_k = block.shape[-1] // 2
    chan, which = key_meta_order(d_k, bits)
    out = np.empty(block.shape[:-1] + (d_k, 2), block.dtype)
    out[..., chan, which] = block
    return out


def unpack_codes(words: np.ndarray, bits: int) -> np.ndarray:
    per = 32 // bits
    w = words.astype(np.uint64)[..., None]
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    mask = np.uint64((1 << bits) - 1)
    c = (w >> shifts) & mask
    return c.reshape(words.shape[:-1] + (words.shape[-1] * per,)).astype(np.uint32)


# --------------------------------------------------- per-channel widths -----
WIDTHS = (0, 1, 2, 4, 8)
# distortion drop per bit of each width step of a channel of weight 1 (step 9):
# (4^-b1 - 4^-b2) / (b2 - b1) for 0->1, 1->2, 2->4, 4->8 (exact binary fractions)
STEP_SLOPES = ((0, 1, 0.75), (1, 2, 0.1875), (2, 4, 15.0 / 512.0), (4, 8, 255.0 / 262144.0))


def allocation_distortion(weight, widths) -> float:
    """sum_c w_c * 4^(-b_c), the objective of step 9's allocation."""
    w = np.asarray(weight, np.float64)
    b = np.asarray(widths, np.float64)
    return float((w * np.power(4.0, -b)).sum())


def allocate_bits(weight, budget: int, unit_bits: int = 1) -> np.ndarray:
    """Step 9: widths in WIDTHS for units of weight w >= 0 (a key channel, or a value group
    whose widening by one bit costs unit_bits = G_v bits) under `budget` bits per row, by
    reverse water-filling: width steps in decreasing order of w * slope, equal slopes
    together, until the next set does not fit; zero-slope steps are never taken."""
    w = np.asarray(weight, np.float64)
    steps = []
    for c in range(w.shape[0]):
        for b1, b2, f in STEP_SLOPES:
            slope = float(w[c] * f)
            if slope > 0.0:
                steps.append((slope, c, b1, b2))
    steps.sort(key=lambda e: -e[0])
    widths = np.zeros(w.shape[0], np.int64)
    used, i = 0, 0
    while i < len(steps):
        j = i
        while j < len(steps) and steps[j][0] == steps[i][0]:
            j += 1
        cost = unit_bits * sum(b2 - b1 for _, _, b1, b2 in steps[i:j])
        if used + cost > budget:
            break
        for _, c, b1, b2 in steps[i:j]:
            assert widths[c] == b1
            widths[c] = b2
        used += cost
        i = j
    return widths


def width_offsets(widths) -> np.ndarray:
    """Bit offset of each channel in a packed row (step 9): the sum of the widths before it."""
    w = np.asarray(widths, np.int64)
    return np.concatenate([[0], np.cumsum(w)[:-1]]).astype(np.int64)


def row_words(widths) -> int:
    """Words of a packed row of per-channel widths: max(1, ceil(sum / 32))."""
    return max(1, -(-int(np.sum(widths)) // 32))


def pack_var(codes: np.ndarray, widths) -> np.ndarray:
    """[..., d] codes -> [..., row_words] uint32, channel c at bit width_offsets[c] (step 9)."""
    off = width_offsets(widths)
    out = np.zeros(codes.shape[:-1] + (row_words(widths),), np.uint64)
    for c, b in enumerate(widths):
        if b:
            out[..., off[c] // 32] |= codes[..., c].astype(np.uint64) << np.uint64(off[c] % 32)
    return out.astype(np.uint32)


def unpack_var(words: np.ndarray, widths) -> np.ndarray:
    """Inverse of pack_var; dropped channels read code 0."""
    off = width_offsets(widths)
    out = np.zeros(words.shape[:-1] + (len(widths),), np.uint32)
    for c, b in enumerate(widths):
        if b:
            w = words[..., off[c] // 32].astype(np.uint64)
            out[..., c] = ((w >> np.uint64(off[c] % 32)) & np.uint64((1 << int(b)) - 1)).astype(np.uint32)
    return out


def quantize_keys_var(k: np.ndarray, group_k: int, widths):
    """Keys [n][d] -> codes [n][d], sz fp16 [n/group_k][d][2]: channel c through step 3 with
    widths[c] bits over each group of group_k tokens; dropped channels (0 bits) store 0."""
    n, d = k.shape
    assert n % group_k == 0
    codes = np.zeros((n, d), np.uint32)
    sz = np.zeros((n // group_k, d, 2), np.float16)
    for c, b in enumerate(widths):
        if b:
            cc, s, z = minmax_quantize(k[:, c].reshape(n // group_k, group_k), int(b), axis=1)
            codes[:, c] = cc.reshape(n)
            sz[:, c, 0] = s[:, 0]
            sz[:, c, 1] = z[:, 0]
    return codes, sz


def quantize_values_var(v: np.ndarray, group_v: int, widths):
    """Values [n][d] -> codes [n][d], sz fp16 [n][d/group_v][2]: value group g through step 3
    with the width of its channels; dropped groups store 0."""
    n, d = v.shape
    codes = np.zeros((n, d), np.uint32)
    sz = np.zeros((n, d // group_v, 2), np.float16)
    for g in range(d // group_v):
        b = int(widths[g * group_v])
        assert all(int(x) == b for x in widths[g * group_v:(g + 1) * group_v])
        if b:
            cc, s, z = minmax_quantize(v[:, g * group_v:(g + 1) * group_v], b, axis=1)
            codes[:, g * group_v:(g + 1) * group_v] = cc
            sz[:, g, 0] = s[:, 0]
            sz[:, g, 1] = z[:, 0]
    return codes, sz


# -------------------------------------------------------------- attention -----
def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
              extra: Optional[np.ndarray] = None) -> np.ndarray:
    """softmax((q.K^T + extra) * scale) V in fp64 for one query vector; ``extra`` is the
    per-token additive logit correction of step 7 (before the 1/sqrt(d) scale)."""
    q = np.asarray(q, dtype=np.float64)
    s = np.asarray(k, dtype=np.float64) @ q
    if extra is not None:
        s = s + extra
    s = s * scale
    p = np.exp(s - s.max())
    return (p @ np.asarray(v, dtype=np.float64)) / p.sum()


def buffer_bytes(cfg: dict) -> dict:
    """Bytes of each cache buffer, as laid out above."""
    B, H, dk, dv = cfg["batch"], cfg["n_kv_heads"], cfg["d_k"], cfg["d_v"]
    kb, vb, gk, gv, R = cfg["k_bits"], cfg["v_bits"], cfg["group_k"], cfg["group_v"], cfg["window"]
    if kb == 16:
        lcap = cfg["max_context"]
        cap = lcap
        return dict(kcode=0, ksz=0, vcode=0, vsz=0, win_k=B * H * cap * dk * 2,
                    win_v=B * H * cap * dv * 2, ret_k=0, ret_v=0, zcode=0, zsz=0)
    lcap = -(-cfg["max_context"] // gk) * gk
    cap = R + gk
    sr, sq = cfg.get("side_rank", 0), cfg.get("side_bits", 0)
    if kb == 0:      # per-channel widths (step 9)
        wk, wv = row_words(cfg["k_widths"][:dk]), row_words(cfg["v_widths"][:dv])
        return dict(kcode=B * H * lcap * wk * 4, ksz=B * H * (lcap // gk) * dk * 4,
                    vcode=B * H * lcap * wv * 4, vsz=B * H * lcap * (dv // gv) * 4,
                    win_k=B * H * cap * dk * 2, win_v=B * H * cap * dv * 2,
                    ret_k=B * H * MAX_RETAINED * dk * 2, ret_v=B * H * MAX_RETAINED * dv * 2,
                    zcode=0, zsz=0)
    return dict(kcode=B * H * lcap * dk * kb // 8, ksz=B * H * (lcap // gk) * dk * 4,
                vcode=B * H * lcap * dv * vb // 8, vsz=B * H * lcap * (dv // gv) * 4,
                win_k=B * H * cap * dk * 2, win_v=B * H * cap * dv * 2,
                ret_k=B * H * MAX_RETAINED * dk * 2, ret_v=B * H * MAX_RETAINED * dv * 2,
                zcode=B * H * lcap * sr * sq // 8, zsz=B * H * (lcap // gk) * sr * 4)


# ------------------------------------------------------------------ cache -----
class OracleCache:
    """The whole cache of one layer: prefill, append, decode (see module docstring).

    ``side_basis`` fp32 [Hkv][d_k][r] is required when cfg["side_rank"] = r > 0 (step 7).
    """

    def __init__(self, cfg: dict, side_basis: Optional[np.ndarray] = None):
        self.cfg = dict(cfg)
        self.sr = int(cfg.get("side_rank", 0))
        self.sq = int(cfg.get("side_bits", 0))
        self.rot = bool(cfg.get("rot_keys", 0))
        if self.rot:
            self.sigma = sign_vector(cfg["rot_signs"], cfg["d_k"])
            self.ck, self.cq = rotation_scales(cfg["d_k"])
        if self.sr:
            if cfg["k_bits"] == 16 or side_basis is None:
                raise ValueError("a side code needs quantized keys and a basis")
            self.U = np.asarray(side_basis, np.float32)
            assert self.U.shape == (cfg["n_kv_heads"], cfg["d_k"], self.sr)
        B, H = cfg["batch"], cfg["n_kv_heads"]
        self.B, self.H, self.Hq = B, H, cfg["n_q_heads"]
        self.dk, self.dv = cfg["d_k"], cfg["d_v"]
        self.kb, self.vb = cfg["k_bits"], cfg["v_bits"]
        self.gk, self.gv, self.R = cfg["group_k"], cfg["group_v"], cfg["window"]
        self.log_retain = bool(cfg["log_retain"]) and self.kb != 16
        self.max_context = cfg["max_context"]
        self.var = self.kb == 0          # per-channel widths (step 9)
        if self.var:
            assert self.vb == 0 and not self.sr and not self.rot
            self.kw = np.array(cfg["k_widths"][:self.dk], np.int64)
            self.vw = np.array(cfg["v_widths"][:self.dv], np.int64)
        if self.kb == 16:
            self.lcap = self.max_context
            self.cap = self.lcap
        elif self.var:
            self.lcap = -(-self.max_context // self.gk) * self.gk
            self.cap = self.R + self.gk
            self.kcode = np.zeros((B, H, self.lcap, row_words(self.kw)), np.uint32)
            self.ksz = np.zeros((B, H, self.lcap // self.gk, self.dk, 2), np.float16)
            self.vcode = np.zeros((B, H, self.lcap, row_words(self.vw)), np.uint32)
            self.vsz = np.zeros((B, H, self.lcap, self.dv // self.gv, 2), np.float16)
            self.ret_k = np.zeros((B, H, MAX_RETAINED, self.dk), np.float16)
            self.ret_v = np.zeros((B, H, MAX_RETAINED, self.dv), np.float16)
        else:
            self.lcap = -(-self.max_context // self.gk) * self.gk
            self.cap = self.R + self.gk
            self.kcode = np.zeros((B, H, self.lcap, self.dk * self.kb // 32), np.uint32)
            self.ksz = np.zeros((B, H, self.lcap // self.gk, 2 * self.dk), np.float16)
            self.vcode = np.zeros((B, H, self.lcap, self.dv * self.vb // 32), np.uint32)
            self.vsz = np.zeros((B, H, self.lcap, self.dv // self.gv, 2), np.float16)
            self.ret_k = np.zeros((B, H, MAX_RETAINED, self.dk), np.float16)
            self.ret_v = np.zeros((B, H, MAX_RETAINED, self.dv), np.float16)
            if self.sr:
                self.zcode = np.zeros((B, H, self.lcap, self.sr * self.sq // 8), np.uint8)
                self.zsz = np.zeros((B, H, self.lcap // self.gk, self.sr, 2), np.float16)
        self.win_k = np.zeros((B, H, self.cap, self.dk), np.float16)
        self.win_v = np.zeros((B, H, self.cap, self.dv), np.float16)
        self.ret_idx: List[int] = []
        self.L = 0
        self.Q = 0

    # -- write path -----------------------------------------------------------
    def _quantize_rows(self, b: int, h: int, t0: int, k_rows: np.ndarray, v_rows: np.ndarray):
        """Quantize tokens [t0, t0+n) (n a multiple of G_k) and store their codes."""
        n = k_rows.shape[0]
        if self.var:
            kc, ksz = quantize_keys_var(k_rows, self.gk, self.kw)
            vc, vsz = quantize_values_var(v_rows, self.gv, self.vw)
            self.kcode[b, h, t0:t0 + n] = pack_var(kc, self.kw)
            self.ksz[b, h, t0 // self.gk:(t0 + n) // self.gk] = ksz
            self.vcode[b, h, t0:t0 + n] = pack_var(vc, self.vw)
            self.vsz[b, h, t0:t0 + n] = vsz
            return
        kc, ksz = quantize_keys(k_rows, self.gk, self.kb)
        vc, vsz = quantize_values(v_rows, self.gv, self.vb)
        self.kcode[b, h, t0:t0 + n] = pack_codes(kc, self.kb)
        self.ksz[b, h, t0 // self.gk:(t0 + n) // self.gk] = pack_key_meta(ksz, self.kb)
        self.vcode[b, h, t0:t0 + n] = pack_codes(vc, self.vb)
        self.vsz[b, h, t0:t0 + n] = vsz
        if self.sr:
            zc, zsz = side_code_group(k_rows, kc, ksz, self.U[h], self.sq, self.gk)
            self.zcode[b, h, t0:t0 + n] = pack_side(zc, self.sq)
            self.zsz[b, h, t0 // self.gk:(t0 + n) // self.gk] = zsz

    def prefill(self, k: np.ndarray, v: np.ndarray):
        """k [B][Hkv][L][d_k], v [B][Hkv][L][d_v] fp16: the cache's first L tokens."""
        k = np.asarray(k, np.float16)
        if self.rot:
            k = rotate_rows(k, self.sigma, self.ck)
        v = np.asarray(v, np.float16)
        L = k.shape[2]
        if L > self.max_context:
            raise ValueError("context exceeds max_context")
        Q = quantized_prefix(L, self.R, self.gk, self.kb)
        for b in range(self.B):
            for h in range(self.H):
                if Q:
                    self._quantize_rows(b, h, 0, k[b, h, :Q], v[b, h, :Q])
                for p in range(Q, L):
                    self.win_k[b, h, p % self.cap] = k[b, h, p]
                    self.win_v[b, h, p % self.cap] = v[b, h, p]
        self.ret_idx = retained_positions(Q) if self.log_retain else []
        for j, p in enumerate(self.ret_idx):
            self.ret_k[:, :, j] = k[:, :, p]
            self.ret_v[:, :, j] = v[:, :, p]
        self.L, self.Q = L, Q

    def append(self, k_new: np.ndarray, v_new: np.ndarray):
        """One token per sequence: k_new [B][Hkv][d_k], v_new [B][Hkv][d_v]."""
        if self.L + 1 > self.max_context:
            raise ValueError("append past max_context")
        p = self.L
        k_new = np.asarray(k_new, np.float16)
        if self.rot:
            k_new = rotate_rows(k_new, self.sigma, self.ck)
        self.win_k[:, :, p % self.cap] = k_new
        self.win_v[:, :, p % self.cap] = np.asarray(v_new, np.float16)
        self.L += 1
        if self.kb != 16 and self.L - self.Q == self.R + self.gk:
            Q0, Q1 = self.Q, self.Q + self.gk
            slots = [t % self.cap for t in range(Q0, Q1)]
            for b in range(self.B):
                for h in range(self.H):
                    self._quantize_rows(b, h, Q0, self.win_k[b, h, slots], self.win_v[b, h, slots])
            if self.log_retain:
                new = retained_positions(Q1)
                old = {pos: j for j, pos in enumerate(self.ret_idx)}
                rk = np.zeros_like(self.ret_k)
                rv = np.zeros_like(self.ret_v)
                for j, pos in enumerate(new):
                    if pos in old:
                        rk[:, :, j] = self.ret_k[:, :, old[pos]]
                        rv[:, :, j] = self.ret_v[:, :, old[pos]]
                    else:                      # a token of the group being quantized now
                        assert Q0 <= pos < Q1
                        rk[:, :, j] = self.win_k[:, :, pos % self.cap]
                        rv[:, :, j] = self.win_v[:, :, pos % self.cap]
                n = len(new)
                self.ret_k[:, :, :n] = rk[:, :, :n]
                self.ret_v[:, :, :n] = rv[:, :, :n]
                self.ret_idx = new
            self.Q = Q1

    # -- read path ------------------------------------------------------------
    def decoded_kv(self, b: int, h: int):
        """(K_hat [L][d_k], V_hat [L][d_v]) in fp64, positions 0..L-1 in order."""
        L, Q = self.L, self.Q
        kh = np.empty((L, self.dk), np.float64)
        vh = np.empty((L, self.dv), np.float64)
        if Q:
            if self.var:
                kc = unpack_var(self.kcode[b, h, :Q], self.kw)
                ksz = self.ksz[b, h, :Q // self.gk]
            else:
                kc = unpack_codes(self.kcode[b, h, :Q], self.kb)                   # [Q][dk]
                ksz = unpack_key_meta(self.ksz[b, h, :Q // self.gk], self.kb)       # [ng][dk][2]
            ks = np.repeat(ksz[:, :, 0], self.gk, axis=0)
            kz = np.repeat(ksz[:, :, 1], self.gk, axis=0)
            kh[:Q] = dequantize(kc, ks, kz)
            if self.var:
                vc = unpack_var(self.vcode[b, h, :Q], self.vw)
            else:
                vc = unpack_codes(self.vcode[b, h, :Q], self.vb)                   # [Q][dv]
            vsz = self.vsz[b, h, :Q]                                            # [Q][ngv][2]
            vs = np.repeat(vsz[:, :, 0], self.gv, axis=1)
            vz = np.repeat(vsz[:, :, 1], self.gv, axis=1)
            vh[:Q] = dequantize(vc, vs, vz)
            for j, pos in enumerate(self.ret_idx):
                kh[pos] = self.ret_k[b, h, j]
                vh[pos] = self.ret_v[b, h, j]
        slots = [p % self.cap for p in range(Q, L)]
        kh[Q:] = self.win_k[b, h, slots]
        vh[Q:] = self.win_v[b, h, slots]
        return kh, vh

    def decoded_side(self, b: int, h: int) -> np.ndarray:
        """z_hat [L][r] in fp64 (step 7): code*s + z for quantized tokens that are not
        retained, 0 for retained and window tokens."""
        Q = self.Q
        zh = np.zeros((self.L, self.sr), np.float64)
        if Q:
            zc = unpack_side(self.zcode[b, h, :Q], self.sq, self.sr)          # [Q][r]
            zsz = self.zsz[b, h, :Q // self.gk]                                  # [ng][r][2]
            zs = np.repeat(zsz[:, :, 0], self.gk, axis=0)
            zz = np.repeat(zsz[:, :, 1], self.gk, axis=0)
            zh[:Q] = dequantize(zc, zs, zz)
            for pos in self.ret_idx:
                zh[pos] = 0.0
        return zh

    def decode(self, q: np.ndarray, rows: Optional[List[int]] = None,
               side_sign: float = 1.0) -> np.ndarray:
        """q [B][Hq][d_k] fp16 -> out [B][Hq][d_v] fp64 (rows: optional subset of b).
        ``side_sign`` = -1 flips the side correction (the pages' wrong-sign control)."""
        if self.L == 0:
            raise ValueError("decode before prefill")
        q = np.asarray(q, np.float16)
        if self.rot:
            q = rotate_rows(q, self.sigma, self.cq)
        q = q.astype(np.float64)
        n_rep = self.Hq // self.H
        out = np.full((self.B, self.Hq, self.dv), np.nan)
        scale = 1.0 / math.sqrt(self.dk)
        for b in (rows if rows is not None else range(self.B)):
            for h in range(self.H):
                kh, vh = self.decoded_kv(b, h)
                zh = self.decoded_side(b, h) if self.sr else None
                for r in range(n_rep):
                    hq = h * n_rep + r
                    extra = None
                    if zh is not None:
                        extra = side_sign * (zh @ side_query(self.U[h], q[b, hq]))
                    out[b, hq] = attention(q[b, hq], kh, vh, scale, extra)
        return out


def max_rel_error(out: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of max_c |out - ref| / max_c |ref| (rows = all leading dims)."""
    o = np.asarray(out, np.float64).reshape(-1, out.shape[-1])
    r = np.asarray(ref, np.float64).reshape(-1, ref.shape[-1])
    num = np.abs(o - r).max(axis=1)
    den = np.maximum(np.abs(r).max(axis=1), 1e-30)
    return float((num / den).max())
