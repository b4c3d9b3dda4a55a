"""Host-side pieces of bench.py on CPU: the algorithmic bytes of a decode call (the roofline's
numerator) against the cache layout, and the lookup of the committed ncu traffic figures."""
import hashlib
import os
import re

import pytest

import bench
from oracle import kvq_oracle as O
from mixed_precision_quantized_pack_b200 import kvq as K
from mixed_precision_quantized_pack_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("key", list(W.WORKLOADS))
def test_decode_bytes_are_the_layouts_bytes_read_once(key):
    """Quantized tokens cost their rows of codes and value (scale, zero) plus their key group's
    (scale, zero); retained and window tokens their fp16 rows; then q (and block-table entries)."""
    w = W.WORKLOADS[key]
    c = w.kvq_config()
    L = w.context + 1
    got = bench.decode_bytes(c, L)
    B, H, Hq, dk, dv = w.batch, w.n_kv_heads, w.n_q_heads, w.d_k, w.d_v
    if w.k_bits == 16:
        assert got == B * H * L * (dk + dv) * 2 + B * Hq * dk * 2
        return
    bb = O.buffer_bytes(dict(c, batch=1, n_kv_heads=1))
    lcap = -(-c["max_context"] // w.group_k) * w.group_k
    per_tok = (bb["kcode"] + bb["vcode"] + bb["vsz"] + bb["zcode"]) // lcap
    per_group = (bb["ksz"] + bb["zsz"]) // (lcap // w.group_k)
    Q = O.quantized_prefix(L, w.window, w.group_k, w.k_bits)
    nret = len(O.retained_positions(Q)) if w.log_retain else 0
    want = B * H * (Q * per_tok + (Q // w.group_k) * per_group + (L - Q + nret) * (dk + dv) * 2)
    want += B * Hq * dk * 2
    if w.paged:
        want += B * (Q // w.group_k) * 4
    assert got == want


def test_every_profile_summary_names_a_source_and_its_traffic():
    """Each committed summary gives the kernel source it was taken on and the traffic per launch;
    bench reports that traffic only while the source is unchanged."""
    prof = os.path.join(ROOT, "profiles")
    names = [f for f in os.listdir(prof) if f.startswith("decode_") and f.endswith("_ncu.md")]
    assert {"decode_long32k_ncu.md", "decode_paged32k_ncu.md", "decode_aatc32k_ncu.md"} <= set(names)
    for f in names:
        text = open(os.path.join(prof, f)).read()
        sha = re.search(r"decode_source_sha256:\s*([0-9a-f]+)", text).group(1)
        src = re.search(r"decode_source:\s*([\w.]+)", text)
        src = src.group(1) if src else "decode_mma.cuh"
        cur = hashlib.sha256(open(os.path.join(ROOT, "mixed_precision_quantized_pack_b200", "csrc", src),
                                  "rb").read()).hexdigest()
        key = f[len("decode_"):-len("_ncu.md")]
        t = bench.profile_traffic(key)
        if cur.startswith(sha):
            assert t is not None and t > 0
        else:
            assert t is None


def test_width_map_rows_are_counted_in_words():
    c = W.WORKLOADS["aatc32k"].kvq_config()
    sizes = K.kvq_buffer_sizes(c)
    lcap = -(-c["max_context"] // 64) * 64
    assert sizes["kcode"] == 32 * 8 * lcap * 14 * 4 and sizes["vcode"] == 32 * 8 * lcap * 9 * 4


@pytest.mark.parametrize("key", list(W.WORKLOADS) + ["sweep-b8-k8v4", "sweep-b1-k16v16"])
def test_prefill_bytes_read_the_inputs_once_and_write_the_layout_once(key):
    w = W.by_key(key)
    c = w.kvq_config()
    L = w.context
    B, H, dk, dv = w.batch, w.n_kv_heads, w.d_k, w.d_v
    got = bench.prefill_bytes(c, L)
    read = B * H * L * (dk + dv) * 2
    if w.k_bits == 16:
        assert got == 2 * read
        return
    bb = O.buffer_bytes(dict(c, batch=1, n_kv_heads=1))
    lcap = -(-c["max_context"] // w.group_k) * w.group_k
    per_tok = (bb["kcode"] + bb["vcode"] + bb["vsz"] + bb["zcode"]) // lcap
    per_group = (bb["ksz"] + bb["zsz"]) // (lcap // w.group_k)
    Q = O.quantized_prefix(L, w.window, w.group_k, w.k_bits)
    nret = len(O.retained_positions(Q)) if w.log_retain else 0
    want = read + B * H * (Q * per_tok + (Q // w.group_k) * per_group + (L - Q + nret) * (dk + dv) * 2)
    if w.paged:
        want += B * (Q // w.group_k) * 4
    assert got == want


def test_every_sweep_point_has_a_key():
    keys = set(W.SWEEP_KEYS)
    assert len(keys) == 16
    for b in W.SWEEP_BATCHES:
        for kb, vb in W.SWEEP_BITS:
            w = W.by_key(f"sweep-b{b}-k{kb}v{vb}")
            assert (w.batch, w.k_bits, w.v_bits, w.context) == (b, kb, vb, 131072)
            assert w.per_seq == 1
    with pytest.raises(KeyError):
        W.by_key("sweep-b3-k4v2")


def test_step_plan_counts_the_group_quantize_launches():
    """A step whose append makes the window R + G_k long also quantizes one group: keys, values
    (and retained set, side code, table entries when the cache has them)."""
    w = W.WORKLOADS["long32k"]
    c = w.kvq_config(max_context=w.context + 200)
    L0 = w.context
    plan = bench.step_plan(c, L0, 0, 130)
    crossing = [i for i in range(130) if (L0 + i + 1 - 128) // 64 != (L0 + i - 128) // 64]
    assert crossing
    for i, (nbytes, n) in enumerate(plan):
        assert nbytes == bench.decode_bytes(c, L0 + i + 1)
        assert n == 3 + (3 if i in crossing else 0)
