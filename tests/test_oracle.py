"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: hand-derived
worked examples (tests/golden), closed forms (exact grids), library routines
(torch's scaled_dot_product_attention in fp64), invariants the pages state
(softmax invariance to a shared key translation: "HeadQ", §2.1; token-order
invariance A.V = A_P.V_P: "LogQuant", §4), brute force on tiny inputs, and byte
arithmetic ("Quantize What Counts", §Résultats: K4V2 saves 25% over K4V4).
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import kvq_oracle as O
from mixed_precision_quantized_pack_b200 import workloads as W


def f16bits(x):
    return int(np.asarray(x, np.float16).view(np.uint16))


# ------------------------------------------------------------ golden files ----
def test_golden_quantizer_examples():
    rows = read_golden("quantizer_worked.txt")
    assert len(rows) >= 6
    for bits, vals, codes, sbits, zbits in rows:
        x = np.array([float(v) for v in vals], np.float16)
        c, s, z = O.minmax_quantize(x, int(bits[0]), axis=0)
        assert [int(t) for t in c] == [int(t) for t in codes], (vals, c)
        assert f16bits(s[0]) == int(sbits[0], 16)
        assert f16bits(z[0]) == int(zbits[0], 16)


def test_golden_key_meta_order():
    """Slot order of a key group's (scale, zero) block, against a hand-written list."""
    for bits, order in read_golden("key_meta_worked.txt"):
        b = int(bits[0])
        d_k = len(order) // 2
        chan, which = O.key_meta_order(d_k, b)
        got = [("s" if w == 0 else "z") + str(c) for c, w in zip(chan, which)]
        assert got == order, (b, got)
        # pack/unpack are mutually inverse and place channel c's scale where the list says
        sz = np.arange(2 * d_k, dtype=np.float16).reshape(d_k, 2)
        blk = O.pack_key_meta(sz, b)
        for slot, name in enumerate(order):
            c = int(name[1:])
            assert blk[slot] == sz[c, 0 if name[0] == "s" else 1]
        assert np.array_equal(O.unpack_key_meta(blk, b), sz)


def test_golden_packing_examples():
    for bits, codes, words in read_golden("packing_worked.txt"):
        b = int(bits[0])
        c = np.array([[int(t) for t in codes]], np.uint32)
        w = O.pack_codes(c, b)
        assert [int(t) for t in w[0]] == [int(t, 16) for t in words]
        assert np.array_equal(O.unpack_codes(w, b), c)


def test_golden_retention_examples():
    for q, pos in read_golden("retention_worked.txt"):
        assert O.retained_positions(int(q[0])) == [int(p) for p in pos]


# --------------------------------------------------------------- quantizer ----
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_grid_inputs_give_exact_codes(bits):
    rng = np.random.default_rng(bits)
    for trial in range(50):
        e = int(rng.integers(-8, 0))
        step = 2.0 ** e
        levels = 2 ** bits - 1
        n = int(rng.integers(2, 70))
        k = rng.integers(0, levels + 1, size=n)
        k[rng.integers(0, n)] = 0
        k[(rng.integers(0, n - 1) + 1 + np.argmin(k)) % n] = levels
        if k.min() != 0 or k.max() != levels:
            continue
        z = float(rng.integers(-64, 64)) * step
        x = np.array([z + int(t) * step for t in k], np.float64)
        assert np.array_equal(x.astype(np.float16).astype(np.float64), x)   # exact in fp16
        c, s, zz = O.minmax_quantize(x.astype(np.float16), bits, axis=0)
        assert np.array_equal(c, k.astype(np.uint32))
        assert float(s[0]) == step and float(zz[0]) == z
        assert int(c[np.argmin(x)]) == 0 and int(c[np.argmax(x)]) == levels


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_reconstruction_error_bound(bits):
    # |x - (code*s + z)| <= s * (1/2 + 2^(b-22)): half a step, plus the fp32 rounding of
    # (x - z) and of the quotient (each <= 2^-24 relative on a quotient <= 2^b).
    x = W.random_fp16((400, 64), seed=7, scale=3.0, mean=1.0).numpy()
    for axis in (0, 1):
        c, s, z = O.minmax_quantize(x, bits, axis=axis)
        deq = O.dequantize(c, s, z)
        err = np.abs(x.astype(np.float64) - deq)
        bound = s.astype(np.float64) * (0.5 + 2.0 ** (bits - 22))
        assert np.all(err <= bound + 0.0)
        assert np.all(c <= 2 ** bits - 1)


@pytest.mark.parametrize("bits", [2, 4])
def test_codes_are_nearest_level_brute_force(bits):
    x = W.random_fp16((200, 8), seed=11, scale=2.0).numpy()
    c, s, z = O.minmax_quantize(x, bits, axis=1)
    levels = np.arange(2 ** bits, dtype=np.float64)
    for i in range(x.shape[0]):
        si, zi = float(s[i, 0]), float(z[i, 0])
        for j in range(x.shape[1]):
            d = np.abs(float(x[i, j]) - (levels * si + zi))
            best = np.sort(d)
            if best[1] - best[0] < 1e-5 * si:       # a near tie: either answer is right
                continue
            assert int(c[i, j]) == int(np.argmin(d))


def test_key_and_value_grouping_axes():
    # keys: one (s, z) per channel per group of G_k tokens; values: per token per G_v channels
    k = W.random_fp16((64, 16), seed=3, scale=2.0).numpy()
    kc, ksz = O.quantize_keys(k, 32, 4)
    assert ksz.shape == (2, 16, 2)
    for g in range(2):
        for ch in range(16):
            col = k[32 * g:32 * g + 32, ch].astype(np.float32)
            assert float(ksz[g, ch, 1]) == float(col.min())
    v = W.random_fp16((5, 64), seed=4).numpy()
    vc, vsz = O.quantize_values(v, 32, 2)
    assert vsz.shape == (5, 2, 2)
    for t in range(5):
        for g in range(2):
            assert float(vsz[t, g, 1]) == float(v[t, 32 * g:32 * g + 32].astype(np.float32).min())


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(5)
    for bits in (2, 4, 8):
        c = rng.integers(0, 2 ** bits, size=(7, 128)).astype(np.uint32)
        assert np.array_equal(O.unpack_codes(O.pack_codes(c, bits), bits), c)


# --------------------------------------------------------------- attention ----
def sdpa_fp64(q, k, v):
    """torch's attention in fp64; q [B][Hq][dk], k [B][Hkv][L][dk], v [B][Hkv][L][dv]."""
    q = torch.as_tensor(np.asarray(q, np.float64))
    k = torch.as_tensor(np.asarray(k, np.float64))
    v = torch.as_tensor(np.asarray(v, np.float64))
    rep = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(rep, dim=1)
    v = v.repeat_interleave(rep, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q[:, :, None, :], k, v)
    return o[:, :, 0, :].numpy()


def cfg_of(B, Hq, Hkv, dk, dv, kb, vb, gk, gv, R, log_retain, max_context):
    return dict(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, d_k=dk, d_v=dv, k_bits=kb, v_bits=vb,
                group_k=gk, group_v=gv, window=R, log_retain=log_retain, max_context=max_context)


@pytest.mark.parametrize("dk,dv", [(64, 64), (32, 128)])
def test_unquantized_cache_matches_library_attention(dk, dv):
    B, Hq, Hkv, L = 2, 4, 2, 200
    k = W.random_fp16((B, Hkv, L, dk), seed=21, scale=2.0).numpy()
    v = W.random_fp16((B, Hkv, L, dv), seed=22).numpy()
    q = W.random_fp16((B, Hq, dk), seed=23).numpy()
    c = O.OracleCache(cfg_of(B, Hq, Hkv, dk, dv, 16, 16, 64, 64, 128, 0, 256))
    c.prefill(k, v)
    assert c.Q == 0
    ref = sdpa_fp64(q, k, v)
    assert np.allclose(c.decode(q), ref, rtol=1e-12, atol=1e-12)


def test_whole_context_in_window_is_exact():
    B, Hq, Hkv, d, L = 1, 4, 1, 64, 100
    k = W.random_fp16((B, Hkv, L, d), seed=31, scale=3.0).numpy()
    v = W.random_fp16((B, Hkv, L, d), seed=32).numpy()
    q = W.random_fp16((B, Hq, d), seed=33).numpy()
    c = O.OracleCache(cfg_of(B, Hq, Hkv, d, d, 4, 2, 32, 32, 128, 1, 512))
    c.prefill(k, v)
    assert c.Q == 0 and c.ret_idx == []
    assert np.allclose(c.decode(q), sdpa_fp64(q, k, v), rtol=1e-12, atol=1e-12)


def grid_cache_inputs(B, H, L, dk, dv, kb, vb, gk, gv, seed):
    """fp16 K/V that the quantizer reproduces exactly: each key group-channel and each
    value token-group lies on z + k*2^e with both end codes present."""
    rng = np.random.default_rng(seed)

    def grid(shape_groups, n, bits):
        levels = 2 ** bits - 1
        codes = rng.integers(0, levels + 1, size=shape_groups + (n,))
        codes[..., 0] = 0
        codes[..., 1] = levels
        perm = np.argsort(rng.random(size=codes.shape), axis=-1)
        codes = np.take_along_axis(codes, perm, axis=-1)
        e = rng.integers(-6, -2, size=shape_groups + (1,)).astype(np.float64)
        step = 2.0 ** e
        z = rng.integers(-32, 32, size=shape_groups + (1,)) * step
        return z + codes * step

    ng = -(-L // gk)
    kg = grid((B, H, ng, dk), gk, kb)                      # [B][H][ng][dk][gk]
    k = kg.transpose(0, 1, 2, 4, 3).reshape(B, H, ng * gk, dk)[:, :, :L]
    vg = grid((B, H, L, dv // gv), gv, vb)                  # [B][H][L][ngv][gv]
    v = vg.reshape(B, H, L, dv)
    assert np.array_equal(k.astype(np.float16).astype(np.float64), k)
    assert np.array_equal(v.astype(np.float16).astype(np.float64), v)
    return k.astype(np.float16), v.astype(np.float16)


@pytest.mark.parametrize("kb,vb,gk,gv,dk,dv", [(4, 2, 32, 32, 64, 64), (8, 4, 16, 64, 32, 128),
                                              (2, 2, 64, 16, 64, 32)])
def test_lossless_grid_cache_decode_equals_exact_attention(kb, vb, gk, gv, dk, dv):
    # On grid inputs quantization is lossless, so the decode over codes must equal the
    # library's exact attention: pins dequantization, scale/zero indexing and packing.
    B, Hq, Hkv, R = 2, 4, 2, 16
    L = 6 * gk + R + 3
    k, v = grid_cache_inputs(B, Hkv, L, dk, dv, kb, vb, gk, gv, seed=kb * 10 + vb)
    q = W.random_fp16((B, Hq, dk), seed=41).numpy()
    c = O.OracleCache(cfg_of(B, Hq, Hkv, dk, dv, kb, vb, gk, gv, R, 0, L + 8))
    c.prefill(k, v)
    assert c.Q == (L - R) // gk * gk and c.Q > 0
    assert np.allclose(c.decode(q), sdpa_fp64(q, k, v), rtol=1e-11, atol=1e-12)


def test_retained_tokens_are_read_in_fp16():
    # Grid inputs except the retained positions, which are moved off-grid inside the
    # group's range: the decode is exact only if those tokens come from the fp16 copy.
    kb, vb, gk, gv, d, R = 4, 2, 32, 32, 64, 32
    B, Hq, Hkv = 1, 2, 1
    L = 10 * gk + R
    k, v = grid_cache_inputs(B, Hkv, L, d, d, kb, vb, gk, gv, seed=5)
    Q = O.quantized_prefix(L, R, gk, kb)
    ret = O.retained_positions(Q)
    kf = k.astype(np.float64)
    vf = v.astype(np.float64)
    rset = set(ret)
    for p in ret:
        g0 = p // gk * gk
        lo = kf[0, 0, g0:g0 + gk].min(axis=0)
        hi = kf[0, 0, g0:g0 + gk].max(axis=0)
        kf[0, 0, p] = lo + (hi - lo) * 0.37 + 2.0 ** -9
        vf[0, 0, p] = vf[0, 0, p] + 2.0 ** -9
        # keep each channel's group extremes on tokens that are not retained
        free = [t for t in range(g0, g0 + gk) if t not in rset]
        kf[0, 0, free[0]] = lo
        kf[0, 0, free[1]] = hi
    k2, v2 = kf.astype(np.float16), vf.astype(np.float16)
    q = W.random_fp16((B, Hq, d), seed=6, scale=2.0).numpy()
    exact = sdpa_fp64(q, k2, v2)
    with_ret = O.OracleCache(cfg_of(B, Hq, Hkv, d, d, kb, vb, gk, gv, R, 1, L + 8))
    with_ret.prefill(k2, v2)
    assert with_ret.ret_idx == ret
    assert np.allclose(with_ret.decode(q), exact, rtol=1e-11, atol=1e-12)
    without = O.OracleCache(cfg_of(B, Hq, Hkv, d, d, kb, vb, gk, gv, R, 0, L + 8))
    without.prefill(k2, v2)
    assert not np.allclose(without.decode(q), exact, rtol=1e-9, atol=1e-9)


def test_shared_key_translation_is_softmax_null():
    # "HeadQ", §2.1: adding one vector mu to every key adds q.mu to every score; softmax
    # ignores it.  Per-channel key quantization commutes with it when fp16 adds are exact.
    B, Hq, Hkv, d, L, gk, R = 1, 4, 1, 64, 32 * 6 + 40, 32, 32
    rng = np.random.default_rng(8)
    k = (rng.integers(-1024, 1024, size=(B, Hkv, L, d)) * 2.0 ** -6).astype(np.float16)
    mu = rng.integers(-8, 9, size=(d,)).astype(np.float64)
    k_mu = (k.astype(np.float64) + mu).astype(np.float16)
    assert np.array_equal(k_mu.astype(np.float64), k.astype(np.float64) + mu)
    v = W.random_fp16((B, Hkv, L, d), seed=9).numpy()
    q = W.random_fp16((B, Hq, d), seed=10).numpy()
    cfg = cfg_of(B, Hq, Hkv, d, d, 4, 2, gk, 32, R, 1, L)
    a, b = O.OracleCache(cfg), O.OracleCache(cfg)
    a.prefill(k, v)
    b.prefill(k_mu, v)
    assert np.array_equal(a.kcode, b.kcode)
    ng = a.Q // gk
    sa = O.unpack_key_meta(a.ksz[0, 0, :ng], 4)          # [ng][d][(scale, zero)]
    sb = O.unpack_key_meta(b.ksz[0, 0, :ng], 4)
    assert np.array_equal(sa[..., 0], sb[..., 0])
    assert np.array_equal(sb[..., 1].astype(np.float64), sa[..., 1].astype(np.float64) + mu)
    assert np.allclose(a.decode(q), b.decode(q), rtol=1e-11, atol=1e-12)


def test_token_order_invariance():
    # "LogQuant", §4: A.V = A_P.V_P for any permutation P of the tokens.
    rng = np.random.default_rng(12)
    k = rng.normal(size=(300, 32)) * 3
    v = rng.normal(size=(300, 48))
    q = rng.normal(size=32)
    perm = rng.permutation(300)
    a = O.attention(q, k, v, 1 / math.sqrt(32))
    b = O.attention(q, k[perm], v[perm], 1 / math.sqrt(32))
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)


def test_thin_key_scale_is_one_over_sqrt_dk():
    # "Thin Keys, Full Values", §2: softmax(Q K^T / sqrt(d_select)) V with d_select = d_k.
    rng = np.random.default_rng(13)
    k = rng.normal(size=(50, 32))
    v = rng.normal(size=(50, 128))
    q = rng.normal(size=32)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None], torch.tensor(k)[None], torch.tensor(v)[None])[0, 0].numpy()
    assert np.allclose(O.attention(q, k, v, 1 / math.sqrt(32)), ref, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------- retention ----
def retained_by_octaves(Q):
    """Independent enumeration: for each octave l the multiple of 2^l among ages [2^l, 2^(l+1))."""
    out = []
    l = 0
    while (1 << l) <= Q:
        lo = max(Q - (1 << (l + 1)) + 1, 0)
        hi = Q - (1 << l)
        cands = [p for p in range(lo, hi + 1) if p % (1 << l) == 0]
        assert len(cands) == 1
        out.append(cands[0])
        l += 1
    return sorted(out)


def test_retention_matches_octave_enumeration_and_count():
    for Q in list(range(1, 300)) + [32640, 32704, 130944, 131008]:
        r = O.retained_positions(Q)
        assert r == retained_by_octaves(Q)
        assert len(r) == int(math.floor(math.log2(Q))) + 1
        assert len(r) <= O.MAX_RETAINED
    assert len(O.retained_positions(32640)) == 15          # ~log2(L) at the 32k workload


def test_retention_only_shrinks_as_q_grows():
    gk = 64
    for Q in range(gk, 40 * gk, gk):
        old, new = set(O.retained_positions(Q)), set(O.retained_positions(Q + gk))
        assert all(p in old or Q <= p < Q + gk for p in new)


# ------------------------------------------------------ append vs prefill ----
@pytest.mark.parametrize("log_retain", [0, 1])
def test_appends_reach_the_same_state_as_one_prefill(log_retain):
    B, Hq, Hkv, d, gk, gv, R = 2, 4, 2, 32, 16, 16, 24
    L0, n_app = 70, 90
    k = W.random_fp16((B, Hkv, L0 + n_app, d), seed=51, scale=4.0).numpy()
    v = W.random_fp16((B, Hkv, L0 + n_app, d), seed=52).numpy()
    cfg = cfg_of(B, Hq, Hkv, d, d, 4, 2, gk, gv, R, log_retain, 256)
    a = O.OracleCache(cfg)
    a.prefill(k[:, :, :L0], v[:, :, :L0])
    events = 0
    for t in range(L0, L0 + n_app):
        q_before = a.Q
        old_ret = set(a.ret_idx)
        a.append(k[:, :, t], v[:, :, t])
        assert R <= a.L - a.Q < R + gk
        if a.Q != q_before:
            events += 1
            assert a.Q == q_before + gk
            assert all(p in old_ret or q_before <= p < a.Q for p in a.ret_idx)
    assert events >= 4
    b = O.OracleCache(cfg)
    b.prefill(k, v)
    assert (a.L, a.Q, a.ret_idx) == (b.L, b.Q, b.ret_idx)
    for name in ("kcode", "ksz", "vcode", "vsz", "win_k", "win_v", "ret_k", "ret_v"):
        x, y = getattr(a, name), getattr(b, name)
        if name.startswith("win"):
            slots = [p % a.cap for p in range(a.Q, a.L)]
            x, y = x[:, :, slots], y[:, :, slots]
        if name.startswith("ret"):
            x, y = x[:, :, :len(a.ret_idx)], y[:, :, :len(a.ret_idx)]
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), name


def test_window_sizes_of_the_workloads():
    for key, want in (("tiny", 64), ("gqa4k", 128), ("long32k", 128), ("thin16k", 64)):
        w = W.WORKLOADS[key]
        Q = O.quantized_prefix(w.context, w.window, w.group_k, w.k_bits)
        assert w.context - Q == want


# ------------------------------------------------------------------- bytes ----
def test_k4v2_saves_a_quarter_of_k4v4_code_bytes():
    # "Quantize What Counts", §Résultats / §Contributions: K4V2 uses 25% less KV memory
    # than K4V4 (code bytes: 4+2 bits vs 4+4 bits per K/V pair of elements).
    base = cfg_of(8, 32, 8, 128, 128, 4, 4, 64, 64, 128, 0, 4096)
    a = O.buffer_bytes(base)
    b = O.buffer_bytes(dict(base, v_bits=2))
    assert (b["kcode"] + b["vcode"]) / (a["kcode"] + a["vcode"]) == 0.75


def test_algorithmic_bytes_per_token_k4v2_g64():
    # codes + (scale, zero) per token per kv head at d=128, K4 G64 / V2 G64: 64+8+32+8 = 112 B
    cfg = cfg_of(1, 1, 1, 128, 128, 4, 2, 64, 64, 128, 0, 64 * 100)
    bb = O.buffer_bytes(cfg)
    lcap = 64 * 100
    assert (bb["kcode"] + bb["ksz"] + bb["vcode"] + bb["vsz"]) / lcap == 112


# ------------------------------------------------------- HeadQ side code ----
# "HeadQ: Distortion visible par le modele et correction dans l'espace des scores pour la
# quantification du cache KV", §3 (Apercu de l'algorithme): base key, residual, side code
# Q_q(U^T e), and the additive logit correction q^T U z_hat / sqrt(d).
from fractions import Fraction


def _golden_headq():
    rows = {}
    for fields in read_golden("headq_worked.txt"):
        name = fields[0][0]
        rows.setdefault(name, []).append(fields[1:])
    return rows


def test_golden_headq_worked_example():
    g = _golden_headq()
    num = lambda xs: [float(x) for x in xs]
    k = np.array([num(r[1]) for r in sorted(g["K"], key=lambda r: int(r[0][0]))], np.float16)
    U = np.array([num(r[1]) for r in sorted(g["U"], key=lambda r: int(r[0][0]))], np.float32)
    gk = k.shape[0]
    kc, ksz = O.quantize_keys(k, gk, 2)
    for ch, sz, codes in g["base"]:
        c = int(ch[0])
        assert [float(ksz[0, c, 0]), float(ksz[0, c, 1])] == num(sz)
        assert [int(x) for x in kc[:, c]] == [int(x) for x in codes]
    s = np.repeat(ksz[:, :, 0], gk, axis=0)
    z = np.repeat(ksz[:, :, 1], gk, axis=0)
    e = O.key_residual(k, kc, s, z)
    for t, vals in g["residual"]:
        assert list(e[int(t[0])]) == num(vals)
    y = O.side_project(e, U)
    for t, vals in g["y"]:
        assert list(y[int(t[0])]) == num(vals)
    zc, zsz = O.side_code_group(k, kc, ksz, U, 2, gk)
    for i, sz, codes in g["side"]:
        c = int(i[0])
        assert [float(zsz[0, c, 0]), float(zsz[0, c, 1])] == num(sz)
        assert [int(x) for x in zc[:, c]] == [int(x) for x in codes]
    packed = O.pack_side(zc, 2)
    assert [int(x) for x in packed[:, 0]] == [int(x, 16) for x in g["packed"][0][0]]
    assert np.array_equal(O.unpack_side(packed, 2, 2), zc)
    zh = O.dequantize(zc, np.repeat(zsz[:, :, 0], gk, axis=0), np.repeat(zsz[:, :, 1], gk, axis=0))
    for t, vals in g["zhat"]:
        assert list(zh[int(t[0])]) == num(vals)
    q = np.array(num(g["q"][0][0]))
    qt = O.side_query(U, q)
    assert list(qt) == num(g["qt"][0][0])
    assert list(zh @ qt) == num(g["correction"][0][0])
    kh = O.dequantize(kc, s, z)
    assert list(kh @ q) == num(g["base_dot"][0][0])
    assert list(k.astype(np.float64) @ q) == num(g["exact_dot"][0][0])


# IEEE binary formats emulated on exact rationals (independent of numpy's float32)
def _round(x: Fraction, mant: int, emin: int) -> Fraction:
    """Round-to-nearest-even of x to a binary float with `mant` significant bits and
    minimum normal exponent `emin` (subnormals below it)."""
    if x == 0:
        return Fraction(0)
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - mant + 1)
    n = a / ulp
    m, rem = divmod(n.numerator, n.denominator)
    if 2 * rem > n.denominator or (2 * rem == n.denominator and m % 2 == 1):
        m += 1
    return (m * ulp) if x > 0 else -(m * ulp)


def r32(x):
    return _round(Fraction(x), 24, -126)


def r16(x):
    return _round(Fraction(x), 11, -14)


def _rint_even(x: Fraction) -> int:
    m, rem = divmod(x.numerator, x.denominator)
    if 2 * rem > x.denominator or (2 * rem == x.denominator and m % 2 == 1):
        m += 1
    return m


@pytest.mark.parametrize("side_bits", [4, 8])
def test_side_code_matches_exact_rational_ieee_emulation(side_bits):
    """Residual, projection and side quantizer against the same steps on exact rationals,
    each operation rounded by an independent IEEE emulation."""
    n, d, r, gk, kb = 16, 16, 4, 8, 4
    k = W.random_fp16((n, d), seed=91, scale=3.0, mean=0.5).numpy()
    rng = np.random.default_rng(92)
    U = rng.standard_normal((d, r)).astype(np.float32)
    kc, ksz = O.quantize_keys(k, gk, kb)
    zc, zsz = O.side_code_group(k, kc, ksz, U, side_bits, gk)
    levels = 2 ** side_bits - 1
    for g in range(n // gk):
        y = [[None] * r for _ in range(gk)]
        for t in range(gk):
            row = g * gk + t
            e = []
            for c in range(d):
                base = r32(Fraction(int(kc[row, c])) * Fraction(float(ksz[g, c, 0])) +
                           Fraction(float(ksz[g, c, 1])))
                e.append(r32(Fraction(float(k[row, c])) - base))
            for i in range(r):
                acc = Fraction(0)
                for c in range(d):
                    acc = r32(acc + r32(Fraction(float(U[c, i])) * e[c]))
                y[t][i] = acc
        for i in range(r):
            col = [y[t][i] for t in range(gk)]
            mn, mx = min(col), max(col)
            s16 = r16(r32(r32(mx - mn) / levels))
            z16 = r16(mn)
            assert Fraction(float(zsz[g, i, 0])) == s16
            assert Fraction(float(zsz[g, i, 1])) == z16
            for t in range(gk):
                if s16 == 0:
                    want = 0
                else:
                    want = min(max(_rint_even(r32(r32(col[t] - z16) / s16)), 0), levels)
                assert int(zc[g * gk + t, i]) == want, (g, t, i)


def test_side_projection_sums_channels_in_ascending_order():
    # fp32: (2^24 + 1) rounds to 2^24 (tie to even), so the ascending sum is 0 and the
    # descending one is 1; the definition fixes the ascending order.
    ones = np.ones((3, 1), np.float32)
    up = np.array([[2.0 ** 24, 1.0, -2.0 ** 24]], np.float32)
    assert float(O.side_project(up, ones)[0, 0]) == 0.0
    assert float(O.side_project(up[:, ::-1].copy(), ones)[0, 0]) == 1.0


def side_cfg(B, Hq, Hkv, d, kb, vb, gk, gv, R, log_retain, max_context, sr, sq):
    return dict(cfg_of(B, Hq, Hkv, d, d, kb, vb, gk, gv, R, log_retain, max_context),
                side_rank=sr, side_bits=sq)


def test_standard_basis_side_code_is_a_per_channel_residual_correction():
    """U_h = columns of the identity (channels ch_h): y = e[:, ch_h] exactly, so the decode
    equals plain attention over keys k_hat + z_hat placed on those channels."""
    B, Hq, Hkv, d, gk, R, L = 2, 8, 2, 32, 16, 24, 200
    k = W.random_fp16((B, Hkv, L, d), seed=61, scale=4.0, mean=1.0).numpy()
    v = W.random_fp16((B, Hkv, L, d), seed=62).numpy()
    q = W.random_fp16((B, Hq, d), seed=63).numpy()
    chans = [[3, 17, 0, 30], [9, 1, 22, 14]]
    U = np.zeros((Hkv, d, 4), np.float32)
    for h in range(Hkv):
        for i, c in enumerate(chans[h]):
            U[h, c, i] = 1.0
    cfg = side_cfg(B, Hq, Hkv, d, 2, 4, gk, 16, R, 1, 256, 4, 8)
    oc = O.OracleCache(cfg, side_basis=U)
    oc.prefill(k, v)
    assert oc.Q > 0 and oc.ret_idx
    got = oc.decode(q)
    keff = np.empty((B, Hkv, L, d))
    veff = np.empty((B, Hkv, L, d))
    for b in range(B):
        for h in range(Hkv):
            kh, vh = oc.decoded_kv(b, h)
            veff[b, h] = vh
            Q = oc.Q
            kc = O.unpack_codes(oc.kcode[b, h, :Q], 2)
            ksz = O.unpack_key_meta(oc.ksz[b, h, :Q // gk], 2)
            e = O.key_residual(k[b, h, :Q], kc, np.repeat(ksz[:, :, 0], gk, 0), np.repeat(ksz[:, :, 1], gk, 0))
            for i, c in enumerate(chans[h]):
                col = e[:, c].reshape(Q // gk, gk)
                codes, s, z = O.minmax_quantize(col, 8, axis=1)
                zh = O.dequantize(codes, s, z).reshape(Q)
                zh[oc.ret_idx] = 0.0
                kh[:Q, c] += zh
            keff[b, h] = kh
    want = sdpa_fp64(q.astype(np.float64), keff, veff)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_zero_residual_gives_a_null_side_code():
    """Keys on the base grid: e = 0, y = 0, every side scale and zero 0, output unchanged."""
    B, Hq, Hkv, d, gk, R, L = 1, 4, 1, 32, 16, 16, 96
    rng = np.random.default_rng(71)
    k = rng.integers(0, 16, size=(B, Hkv, L, d)).astype(np.float16)
    k[:, :, ::gk, :] = 0          # every (group, channel) holds 0 and 15: s = 1, z = 0
    k[:, :, 1::gk, :] = 15
    v = W.random_fp16((B, Hkv, L, d), seed=72).numpy()
    q = W.random_fp16((B, Hq, d), seed=73).numpy()
    U = np.linalg.qr(rng.standard_normal((d, 4)))[0].astype(np.float32)[None]
    base = O.OracleCache(cfg_of(B, Hq, Hkv, d, d, 4, 2, gk, 16, R, 0, 128))
    side = O.OracleCache(side_cfg(B, Hq, Hkv, d, 4, 2, gk, 16, R, 0, 128, 4, 4), side_basis=U)
    base.prefill(k, v)
    side.prefill(k, v)
    assert side.Q > 0
    assert not side.zsz[:, :, :side.Q // gk].any() and not side.zcode[:, :, :side.Q].any()
    assert np.array_equal(side.decode(q), base.decode(q))


def test_side_correction_recovers_scores_in_the_basis_and_wrong_sign_hurts():
    """q in span(U_h): the score error of the corrected keys is the side quantizer's own
    (small) error; flipping the correction's sign (the pages' wrong-sign control) is worse
    than no correction at all."""
    B, Hq, Hkv, d, gk, R, L = 1, 4, 2, 64, 32, 32, 600
    rng = np.random.default_rng(81)
    k = W.random_fp16((B, Hkv, L, d), seed=82, scale=2.0, mean=0.5).numpy()
    v = W.random_fp16((B, Hkv, L, d), seed=83).numpy()
    U = np.stack([np.linalg.qr(rng.standard_normal((d, 4)))[0] for _ in range(Hkv)]).astype(np.float32)
    a = rng.standard_normal((B, Hq, 4)) * 2.0
    q = np.einsum("qdr,bqr->bqd", U[np.arange(Hq) // (Hq // Hkv)].astype(np.float64), a)
    q = q.astype(np.float16)
    cfg = cfg_of(B, Hq, Hkv, d, d, 2, 8, gk, 16, R, 0, 1024)
    base = O.OracleCache(cfg)
    side = O.OracleCache(dict(cfg, side_rank=4, side_bits=8), side_basis=U)
    base.prefill(k, v)
    side.prefill(k, v)
    # exact keys with the same decoded values isolate the score error
    vd = np.stack([np.stack([side.decoded_kv(b, h)[1] for h in range(Hkv)]) for b in range(B)])
    ref = sdpa_fp64(q.astype(np.float64), k.astype(np.float64), vd)
    e_base = O.max_rel_error(base.decode(q), ref)
    e_side = O.max_rel_error(side.decode(q), ref)
    e_flip = O.max_rel_error(side.decode(q, side_sign=-1.0), ref)
    assert e_side < 0.05 * e_base, (e_side, e_base)
    assert e_flip > e_base, (e_flip, e_base)


def test_side_appends_reach_the_same_state_as_one_prefill():
    B, Hq, Hkv, d, gk, gv, R = 2, 4, 2, 32, 16, 16, 24
    L0, n_app = 70, 60
    k = W.random_fp16((B, Hkv, L0 + n_app, d), seed=95, scale=4.0).numpy()
    v = W.random_fp16((B, Hkv, L0 + n_app, d), seed=96).numpy()
    U = np.random.default_rng(97).standard_normal((Hkv, d, 8)).astype(np.float32)
    cfg = side_cfg(B, Hq, Hkv, d, 4, 2, gk, gv, R, 1, 256, 8, 4)
    a = O.OracleCache(cfg, side_basis=U)
    a.prefill(k[:, :, :L0], v[:, :, :L0])
    for t in range(L0, L0 + n_app):
        a.append(k[:, :, t], v[:, :, t])
    b = O.OracleCache(cfg, side_basis=U)
    b.prefill(k, v)
    assert (a.L, a.Q) == (b.L, b.Q) and a.Q > L0
    for name in ("zcode", "zsz"):
        assert np.array_equal(getattr(a, name).view(np.uint8), getattr(b, name).view(np.uint8)), name


def test_side_code_bytes_per_token():
    # r*q/8 code bytes per token and one fp16 (scale, zero) per coordinate per key group
    for sr, sq, per_tok in ((4, 4, 2 + 16 / 64), (4, 8, 4 + 16 / 64), (8, 4, 4 + 32 / 64)):
        cfg = dict(cfg_of(1, 1, 1, 128, 128, 2, 2, 64, 64, 128, 0, 64 * 100), side_rank=sr, side_bits=sq)
        bb = O.buffer_bytes(cfg)
        assert (bb["zcode"] + bb["zsz"]) / (64 * 100) == per_tok


# ------------------------------------------------------ key-only rotation ----
# "Quantize What Counts", §Contributions Clés and §Résultats (Intégration de la Rotation).
def sylvester(d):
    H = np.array([[1.0]])
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def test_golden_rotation_examples():
    for name, bits, d, k, kr, q, qr, dot in read_golden("rotation_worked.txt"):
        d = int(d[0])
        sigma = O.sign_vector([int(bits[0], 16)], d)
        ck, cq = O.rotation_scales(d)
        assert ck * cq == d
        got_k = O.rotate_rows(np.array([[float(x) for x in k]], np.float16), sigma, ck)[0]
        got_q = O.rotate_rows(np.array([[float(x) for x in q]], np.float16), sigma, cq)[0]
        assert [float(x) for x in got_k] == [float(x) for x in kr], name
        assert [float(x) for x in got_q] == [float(x) for x in qr], name
        assert float(got_k.astype(np.float64) @ got_q.astype(np.float64)) == float(dot[0])


@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128, 256])
def test_fwht_is_the_sylvester_hadamard_product(d):
    rng = np.random.default_rng(d)
    x = rng.integers(-50, 50, size=(5, d)).astype(np.float32)     # sums stay exact in fp32
    assert np.array_equal(O.fwht32(x).astype(np.float64), x.astype(np.float64) @ sylvester(d).T)
    ck, cq = O.rotation_scales(d)
    assert ck * cq == d and ck in (cq, 2 * cq)


def test_fwht_rounding_matches_exact_rational_ieee_emulation():
    """The butterflies on random fp16 data, each add/sub rounded by the independent emulation."""
    d = 32
    x = W.random_fp16((6, d), seed=121, scale=100.0).numpy().astype(np.float32)
    x[0, 0] = 2.0 ** 24                     # force roundings that depend on the order
    x[0, 1] = 1.0
    x[0, 3] = -(2.0 ** 24)
    got = O.fwht32(x)
    for row in range(x.shape[0]):
        y = [Fraction(float(v)) for v in x[row]]
        h = 1
        while h < d:
            for i in range(d):
                if i & h == 0:
                    a, b = y[i], y[i + h]
                    y[i], y[i + h] = r32(a + b), r32(a - b)
            h *= 2
        assert [Fraction(float(v)) for v in got[row]] == y, row


def test_rotation_preserves_scores_up_to_the_fp16_roundings():
    d = 128
    k = W.random_fp16((300, d), seed=131, scale=4.0, mean=1.0).numpy()
    q = W.random_fp16((7, d), seed=132).numpy()
    for bits in ([0] * 4, [0x9E3779B9, 0x7F4A7C15, 0x12345678, 0xDEADBEEF]):
        sigma = O.sign_vector(bits, d)
        ck, cq = O.rotation_scales(d)
        kr = O.rotate_rows(k, sigma, ck).astype(np.float64)
        qr = O.rotate_rows(q, sigma, cq).astype(np.float64)
        exact = q.astype(np.float64) @ k.astype(np.float64).T
        rot = qr @ kr.T
        # each rotated coordinate is rounded once to fp16 (2^-11 relative) and |R x| = |x|
        bound = 2.0 ** -10 * np.linalg.norm(q.astype(np.float64), axis=1)[:, None] * \
            np.linalg.norm(k.astype(np.float64), axis=1)[None, :] * 1.01
        assert np.all(np.abs(rot - exact) <= bound)
        assert np.allclose(np.linalg.norm(kr, axis=1) * ck / math.sqrt(d),
                           np.linalg.norm(k.astype(np.float64), axis=1), rtol=2e-3)


def rot_cfg(B, Hq, Hkv, d, kb, vb, gk, gv, R, log_retain, max_context, bits):
    return dict(cfg_of(B, Hq, Hkv, d, d, kb, vb, gk, gv, R, log_retain, max_context),
                rot_keys=1, rot_signs=list(bits))


def test_rotated_unquantized_cache_matches_library_attention():
    B, Hq, Hkv, d, L = 2, 8, 2, 64, 150
    k = W.random_fp16((B, Hkv, L, d), seed=141, scale=3.0).numpy()
    v = W.random_fp16((B, Hkv, L, d), seed=142).numpy()
    q = W.random_fp16((B, Hq, d), seed=143).numpy()
    bits = [0x0F0F1234, 0x89ABCDEF]
    oc = O.OracleCache(rot_cfg(B, Hq, Hkv, d, 16, 16, 64, 64, 0, 0, 256, bits))
    oc.prefill(k, v)
    got = oc.decode(q)
    sigma = O.sign_vector(bits, d)
    ck, cq = O.rotation_scales(d)
    want = sdpa_fp64(O.rotate_rows(q, sigma, cq), O.rotate_rows(k, sigma, ck), v)
    assert np.allclose(got, want, rtol=0, atol=1e-12)
    plain = sdpa_fp64(q, k, v)
    assert O.max_rel_error(got, plain) < 2e-2          # the fp16 roundings of the rotation only


def test_rotated_appends_reach_the_same_state_as_one_prefill():
    B, Hq, Hkv, d, gk, gv, R = 2, 4, 2, 32, 16, 16, 24
    L0, n_app = 70, 60
    k = W.random_fp16((B, Hkv, L0 + n_app, d), seed=161, scale=4.0).numpy()
    v = W.random_fp16((B, Hkv, L0 + n_app, d), seed=162).numpy()
    cfg = rot_cfg(B, Hq, Hkv, d, 4, 2, gk, gv, R, 1, 256, [0xC0FFEE11])
    a = O.OracleCache(cfg)
    a.prefill(k[:, :, :L0], v[:, :, :L0])
    for t in range(L0, L0 + n_app):
        a.append(k[:, :, t], v[:, :, t])
    b = O.OracleCache(cfg)
    b.prefill(k, v)
    assert (a.L, a.Q, a.ret_idx) == (b.L, b.Q, b.ret_idx)
    for name in ("kcode", "ksz", "ret_k"):
        assert np.array_equal(getattr(a, name).view(np.uint8), getattr(b, name).view(np.uint8)), name
    q = W.random_fp16((B, Hq, d), seed=163).numpy()
    assert np.array_equal(a.decode(q), b.decode(q))


# ------------------------------------------------------- per-channel widths ----
def test_golden_aatc_allocations_and_packing():
    n_alloc = n_pack = 0
    for row in read_golden("aatc_worked.txt"):
        if row[0] == ["alloc"]:
            w = [float(x) for x in row[1]]
            got = O.allocate_bits(w, int(row[3][0]), int(row[2][0]))
            assert [int(x) for x in got] == [int(x) for x in row[4]], row
            n_alloc += 1
        else:
            widths = [int(x) for x in row[1]]
            codes = np.array([[int(x) for x in row[2]]], np.uint32)
            words = O.pack_var(codes, widths)
            assert [int(x) for x in words[0]] == [int(x, 16) for x in row[3]], row
            assert np.array_equal(O.unpack_var(words, widths), codes)
            n_pack += 1
    assert n_alloc >= 10 and n_pack >= 4


def _all_allocations(n):
    import itertools
    return itertools.product(O.WIDTHS, repeat=n)


@pytest.mark.parametrize("seed", range(6))
def test_allocation_is_optimal_for_the_bits_it_spends_brute_force(seed):
    """No width vector that spends at most as many bits has a lower distortion (tiny n)."""
    rng = np.random.default_rng(seed)
    n = 3 if seed % 2 else 4
    w = rng.lognormal(0.0, 1.5, size=n)
    if seed == 5:
        w[1] = w[2]                                     # a tie
    for budget in range(0, 8 * n + 2):
        got = O.allocate_bits(w, budget)
        spent = int(got.sum())
        assert spent <= budget
        d = O.allocation_distortion(w, got)
        for cand in _all_allocations(n):
            if sum(cand) <= spent:
                assert O.allocation_distortion(w, cand) >= d - 1e-12 * max(d, 1.0), (budget, cand, got)


def test_allocation_is_monotone_and_permutation_equivariant():
    rng = np.random.default_rng(7)
    w = rng.lognormal(0.0, 2.0, size=64)
    for budget in (0, 17, 64, 150, 256, 511, 512, 600):
        got = O.allocate_bits(w, budget)
        order = np.argsort(-w, kind="stable")
        assert np.all(np.diff(got[order]) <= 0)                 # more weight, at least as many bits
        perm = rng.permutation(64)
        assert np.array_equal(O.allocate_bits(w[perm], budget), got[perm])
        assert got.sum() <= budget
    assert np.array_equal(O.allocate_bits(w, 10 ** 6), np.full(64, 8))
    assert np.array_equal(O.allocate_bits(w, 0), np.zeros(64))


def test_continuous_water_filling_is_bracketed():
    """The allocation is a water level: every step whose drop per bit lies above the lowest
    drop taken is taken, so a channel gets bits exactly when its first step (0 -> 1, drop
    3w/4) lies above that level."""
    rng = np.random.default_rng(11)
    w = rng.lognormal(0.0, 2.0, size=128)
    got = O.allocate_bits(w, 3 * 128)
    # the level: the smallest drop per bit that was taken
    taken = [w[c] * f for c in range(128) for b1, b2, f in O.STEP_SLOPES if got[c] >= b2]
    lam = min(taken)
    for c in range(128):
        for b1, b2, f in O.STEP_SLOPES:
            if w[c] * f > lam:
                assert got[c] >= b2
            elif w[c] * f < lam:
                assert got[c] <= b1
    assert np.all(got[w * 0.75 < lam] == 0)
    assert np.all(got[w * 0.75 > lam] >= 1)


def test_uniform_widths_reduce_to_the_fixed_width_quantizer():
    """A map of one width b everywhere gives the fixed-width codes, (scale, zero) and packed
    words of steps 3-4."""
    rng = np.random.default_rng(3)
    for b in (2, 4, 8):
        k = (rng.standard_normal((128, 64)) * 3).astype(np.float16)
        v = rng.standard_normal((128, 64)).astype(np.float16)
        kc, ksz = O.quantize_keys_var(k, 32, [b] * 64)
        kc0, ksz0 = O.quantize_keys(k, 32, b)
        assert np.array_equal(kc, kc0) and np.array_equal(ksz.view(np.uint16), ksz0.view(np.uint16))
        assert np.array_equal(O.pack_var(kc, [b] * 64), O.pack_codes(kc0, b))
        vc, vsz = O.quantize_values_var(v, 16, [b] * 64)
        vc0, vsz0 = O.quantize_values(v, 16, b)
        assert np.array_equal(vc, vc0) and np.array_equal(vsz.view(np.uint16), vsz0.view(np.uint16))


def test_packing_matches_big_integer_arithmetic():
    """Each row, read as one little-endian integer, is sum_c code_c << offset_c."""
    rng = np.random.default_rng(5)
    for widths in ([8] * 3 + [4] * 5 + [2] * 7 + [1] * 9 + [0] * 8, [4] * 16 + [1] * 16, [1] * 32,
                   [8, 8, 2, 2, 2, 2, 1, 1, 1, 1, 0, 0]):
        codes = np.array([[rng.integers(0, 2 ** b) if b else 0 for b in widths] for _ in range(5)],
                         np.uint32)
        words = O.pack_var(codes, widths)
        for r in range(5):
            big = sum(int(codes[r, c]) << int(sum(widths[:c])) for c in range(len(widths)))
            got = sum(int(words[r, j]) << (32 * j) for j in range(words.shape[1]))
            assert got == big
        assert words.shape[1] == max(1, -(-sum(widths) // 32))


def var_cfg(B, Hq, Hkv, dk, dv, gk, gv, R, log_retain, max_context, kw, vw):
    return dict(cfg_of(B, Hq, Hkv, dk, dv, 0, 0, gk, gv, R, log_retain, max_context),
                k_widths=list(kw), v_widths=list(vw))


def test_lossless_grid_cache_with_dropped_channels_equals_exact_attention():
    """Inputs on each channel's (group's) grid quantize losslessly, and dropped channels read 0:
    the decode must equal exact attention over keys and values with those channels zeroed."""
    B, Hq, Hkv, dk, dv, gk, gv, R = 2, 4, 2, 64, 64, 32, 16, 16
    kw = [8] * 8 + [4] * 24 + [2] * 16 + [1] * 8 + [0] * 8
    vw = [4] * 16 + [2] * 16 + [1] * 16 + [0] * 16
    L = 5 * gk + R + 3
    rng = np.random.default_rng(21)
    ng = -(-L // gk)
    k = np.zeros((B, Hkv, ng * gk, dk))
    for c, b in enumerate(kw):
        kk, _ = grid_cache_inputs(B, Hkv, ng * gk, 32, 32, max(b, 1), 2, gk, 32, seed=100 + c)
        k[:, :, :, c] = kk[:, :, :, 0]
    k = k[:, :, :L].astype(np.float16)
    v = np.zeros((B, Hkv, L, dv))
    for g in range(dv // gv):
        _, vv = grid_cache_inputs(B, Hkv, L, 32, gv, 2, max(vw[g * gv], 1), gk, gv, seed=200 + g)
        v[:, :, :, g * gv:(g + 1) * gv] = vv
    v = v.astype(np.float16)
    q = W.random_fp16((B, Hq, dk), seed=42).numpy()
    c = O.OracleCache(var_cfg(B, Hq, Hkv, dk, dv, gk, gv, R, 0, L + 8, kw, vw))
    c.prefill(k, v)
    assert c.Q > 0
    kz, vz = k.astype(np.float64).copy(), v.astype(np.float64).copy()
    kz[:, :, :c.Q, np.array(kw) == 0] = 0.0
    vz[:, :, :c.Q, np.array(vw) == 0] = 0.0
    assert np.allclose(c.decode(q), sdpa_fp64(q, kz, vz), rtol=1e-11, atol=1e-12)
    # and without the zeroing the decode differs (the dropped channels carry signal)
    assert not np.allclose(c.decode(q), sdpa_fp64(q, k, v), rtol=1e-6, atol=1e-6)


def test_dropped_channels_do_not_influence_the_quantized_tokens():
    B, Hq, Hkv, dk, dv, gk, gv, R = 1, 2, 1, 32, 32, 16, 8, 8
    kw = [4] * 16 + [0] * 16
    vw = [2] * 16 + [0] * 16
    L = 4 * gk + R
    k = W.random_fp16((B, Hkv, L, dk), seed=1).numpy()
    v = W.random_fp16((B, Hkv, L, dv), seed=2).numpy()
    q = W.random_fp16((B, Hq, dk), seed=3).numpy()
    cfg = var_cfg(B, Hq, Hkv, dk, dv, gk, gv, R, 1, L + 8, kw, vw)
    a, b2 = O.OracleCache(cfg), O.OracleCache(cfg)
    a.prefill(k, v)
    k2, v2 = k.copy(), v.copy()
    Q = a.Q
    keep = set(a.ret_idx)
    rows = [p for p in range(Q) if p not in keep]
    k2[:, :, rows, 16:] = 7.0                       # dropped key channels of non-retained quantized tokens
    v2[:, :, rows, 16:] = -3.0
    b2.prefill(k2, v2)
    assert np.array_equal(a.decode(q), b2.decode(q))


def test_variable_width_appends_reach_the_same_state_as_one_prefill():
    B, Hq, Hkv, dk, dv, gk, gv, R = 2, 4, 2, 64, 32, 16, 8, 8
    kw = [8] * 4 + [4] * 20 + [2] * 30 + [0] * 10
    vw = [4] * 8 + [1] * 16 + [0] * 8
    L0, n = 40, 45
    k = W.random_fp16((B, Hkv, L0 + n, dk), seed=4).numpy()
    v = W.random_fp16((B, Hkv, L0 + n, dv), seed=5).numpy()
    cfg = var_cfg(B, Hq, Hkv, dk, dv, gk, gv, R, 1, L0 + n + 8, kw, vw)
    a, b2 = O.OracleCache(cfg), O.OracleCache(cfg)
    a.prefill(k[:, :, :L0], v[:, :, :L0])
    for t in range(L0, L0 + n):
        a.append(k[:, :, t], v[:, :, t])
    b2.prefill(k, v)
    assert (a.L, a.Q, a.ret_idx) == (b2.L, b2.Q, b2.ret_idx)
    for name in ("kcode", "ksz", "vcode", "vsz"):
        x, y = getattr(a, name)[:, :, :a.Q // (gk if name == "ksz" else 1)], \
            getattr(b2, name)[:, :, :b2.Q // (gk if name == "ksz" else 1)]
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), name


def test_variable_width_bytes_per_token():
    """A K(8x16, 4x64, 2x32, 0x16) / V(4, 2 over two 64-channel groups) row is 14+12 words of
    codes: 26 * 4 = 104 B per token vs 112 B for K4V2 (plus the (scale, zero))."""
    kw = [8] * 16 + [4] * 64 + [2] * 32 + [0] * 16
    vw = [4] * 64 + [2] * 64
    cfg = var_cfg(1, 4, 1, 128, 128, 64, 64, 128, 0, 4096, kw, vw)
    bb = O.buffer_bytes(cfg)
    assert bb["kcode"] == 4096 * 4 * 14 and bb["vcode"] == 4096 * 4 * 12
    assert bb["ksz"] == 64 * 128 * 4 and bb["vsz"] == 4096 * 2 * 4
