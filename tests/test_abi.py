"""Host-side checks of the C ABI: no kernel launches, so these run without a GPU."""
import ctypes
import os
import subprocess
import sys
import re

import pytest

from oracle import kvq_oracle as O
from mixed_precision_quantized_pack_b200 import kvq as K
from mixed_precision_quantized_pack_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(kvq_\w+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_function():
    lib = K.lib()
    names = header_functions()
    assert "kvq_decode_attention" in names and "kvq_quantize_prefill" in names
    for n in names:
        assert hasattr(lib, n), n
        assert n in K._SIGNATURES, f"binding lacks {n}"


def cfg(**kw):
    base = dict(batch=2, n_q_heads=8, n_kv_heads=2, d_k=128, d_v=128, k_bits=4, v_bits=2,
                group_k=64, group_v=64, window=128, log_retain=1, max_context=4096)
    base.update(kw)
    return base


@pytest.mark.parametrize("w", [x for x in W.WORKLOADS.values() if not x.paged] +
                         [W.sweep_workload(b, kb, vb) for b in (1, 64) for kb, vb in W.SWEEP_BITS])
def test_buffer_sizes_match_the_oracle_layout(w):
    c = w.kvq_config()
    got = K.kvq_buffer_sizes(c)
    want = O.buffer_bytes(c)
    for n in K.BUFFER_FIELDS:
        assert got[n] == want[n], n
    assert got["workspace"] > 0


def test_retention_rule_matches_the_oracle():
    for Q in list(range(0, 600)) + [32640, 65536, 131008, (1 << 30) - 64]:
        assert K.kvq_retained_positions(Q) == O.retained_positions(Q) if Q < 200000 else \
            len(K.kvq_retained_positions(Q)) == 30


@pytest.mark.parametrize("bad,code", [
    (dict(n_q_heads=6, n_kv_heads=4), K.KVQ_ERR_UNSUPPORTED),
    (dict(n_q_heads=32, n_kv_heads=2), K.KVQ_ERR_UNSUPPORTED),       # n_rep 16
    (dict(d_k=96), K.KVQ_ERR_UNSUPPORTED),
    (dict(k_bits=3), K.KVQ_ERR_UNSUPPORTED),
    (dict(k_bits=16, v_bits=2), K.KVQ_ERR_UNSUPPORTED),
    (dict(group_k=48), K.KVQ_ERR_UNSUPPORTED),
    (dict(group_v=24), K.KVQ_ERR_UNSUPPORTED),
    (dict(group_v=8, v_bits=2), K.KVQ_ERR_UNSUPPORTED),              # word spans two groups
    (dict(batch=0), K.KVQ_ERR_INVALID_ARG),
    (dict(window=-1), K.KVQ_ERR_INVALID_ARG),
    (dict(log_retain=2), K.KVQ_ERR_INVALID_ARG),
    (dict(max_context=0), K.KVQ_ERR_INVALID_ARG),
    (dict(rot_keys=2), K.KVQ_ERR_INVALID_ARG),
])
def test_invalid_configurations_are_rejected(bad, code):
    with pytest.raises(K.KVQError) as e:
        K.kvq_buffer_sizes(cfg(**bad))
    assert e.value.code == code


def test_misaligned_buffers_are_rejected_before_any_device_call():
    c = cfg()
    ptrs = {n: 4096 * (i + 1) for i, n in enumerate(K.BUFFER_FIELDS)}
    ptrs["vsz"] += 8
    with pytest.raises(K.KVQError) as e:
        K.kvq_cache_init(c, ptrs)
    assert e.value.code == K.KVQ_ERR_ALIGN
    ptrs = {n: 4096 * (i + 1) for i, n in enumerate(K.BUFFER_FIELDS)}
    ptrs["ret_k"] = 0
    with pytest.raises(K.KVQError) as e:
        K.kvq_cache_init(c, ptrs)
    assert e.value.code == K.KVQ_ERR_INVALID_ARG


def test_null_arguments_are_errors_not_crashes():
    lib = K.lib()
    assert lib.kvq_quantize_prefill(None, None, None, 1, None) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_append(None, None, None, None) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_decode_attention(None, None, None, None, 0, 0, None) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_get_state(None, None, None, None, None) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_reset_status(None, None) == K.KVQ_ERR_INVALID_ARG
    lib.kvq_cache_destroy(None)


def test_strerror_covers_every_code():
    codes = [K.KVQ_OK, K.KVQ_ERR_INVALID_ARG, K.KVQ_ERR_UNSUPPORTED, K.KVQ_ERR_ALIGN,
             K.KVQ_ERR_CAPACITY, K.KVQ_ERR_WORKSPACE, K.KVQ_ERR_STATE, K.KVQ_ERR_CUDA]
    msgs = [K.kvq_strerror(c) for c in codes]
    assert len(set(msgs)) == len(msgs) and "unknown" in K.kvq_strerror(-99)


@pytest.mark.parametrize("key", list(W.WORKLOADS))
def test_planner_covers_the_work(key):
    w = W.WORKLOADS[key]
    c = w.kvq_config()
    L = w.context + w.appends
    Q = O.quantized_prefix(L, w.window, w.group_k, w.k_bits)
    nret = len(O.retained_positions(Q)) if w.log_retain else 0
    for sms in (1, 148):
        for req in (0, 1, 3, 1000):
            p = K.kvq_plan_decode(c, L, sms, req)
            assert p["n_groups"] == Q // w.group_k
            assert p["n_fp16"] == nret + L - Q
            assert 1 <= p["splits_quant"] <= max(1, p["n_groups"])
            assert 1 <= p["splits_fp16"] <= p["n_fp16"]
            if req:
                assert p["splits_quant"] == min(req, p["n_groups"], p["splits_quant"] if req == 1000 else req)
            ws = K.kvq_buffer_sizes(c)["workspace"]
            rows = w.batch * w.n_q_heads * (p["splits_quant"] + p["splits_fp16"])
            assert ws >= 256 + rows * 8 + rows * w.d_v * 4


def test_planner_unquantized_cache_splits_the_fp16_tokens():
    w = W.sweep_workload(1, 16, 16)
    p = K.kvq_plan_decode(w.kvq_config(), 131072, 148, 0)
    assert p["n_groups"] == 0 and p["splits_quant"] == 0
    assert p["n_fp16"] == 131072 and p["splits_fp16"] > 8


def test_planner_rejects_lengths_outside_the_cache():
    c = cfg(max_context=1000)
    for L in (0, 1001):
        with pytest.raises(K.KVQError):
            K.kvq_plan_decode(c, L, 148, 0)


# ---------------------------------------------------------------- side code ----
@pytest.mark.parametrize("sr,sq", [(4, 4), (4, 8), (8, 4)])
def test_side_buffer_sizes_match_the_oracle_layout(sr, sq):
    for w in (W.WORKLOADS["headq32k"], W.WORKLOADS["long32k"].with_(side_rank=sr, side_bits=sq)):
        c = dict(w.kvq_config(), side_rank=sr, side_bits=sq)
        got = K.kvq_buffer_sizes(c)
        want = O.buffer_bytes(c)
        for n in K.BUFFER_FIELDS + ("zcode", "zsz"):
            assert got[n] == want[n], n
        assert got["side_u"] == c["n_kv_heads"] * c["d_k"] * sr * 4


@pytest.mark.parametrize("bad", [
    dict(side_rank=3, side_bits=4), dict(side_rank=4, side_bits=2), dict(side_rank=8, side_bits=8),
    dict(side_rank=16, side_bits=2), dict(side_rank=4, side_bits=4, k_bits=16, v_bits=16),
])
def test_invalid_side_codes_are_rejected(bad):
    with pytest.raises(K.KVQError) as e:
        K.kvq_buffer_sizes(cfg(**bad))
    assert e.value.code == K.KVQ_ERR_UNSUPPORTED


def test_side_code_buffers_are_required_and_aligned():
    c = cfg(side_rank=4, side_bits=4)
    fields = K.BUFFER_FIELDS + K.SIDE_FIELDS
    ptrs = {n: 4096 * (i + 1) for i, n in enumerate(fields)}
    ptrs["side_u"] = 0
    with pytest.raises(K.KVQError) as e:
        K.kvq_cache_init(c, ptrs)
    assert e.value.code == K.KVQ_ERR_INVALID_ARG
    ptrs = {n: 4096 * (i + 1) for i, n in enumerate(fields)}
    ptrs["zsz"] += 4
    with pytest.raises(K.KVQError) as e:
        K.kvq_cache_init(c, ptrs)
    assert e.value.code == K.KVQ_ERR_ALIGN


def test_ragged_calls_check_their_arguments():
    lib = K.lib()
    assert lib.kvq_quantize_prefill_ragged(None, None, None, 1, None, None) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_append_ragged(None, None, None, None, None) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_get_seq_state(None, 0, None, None, None, None) == K.KVQ_ERR_INVALID_ARG


# ------------------------------------------------------------ paged layout ----
@pytest.mark.parametrize("sr", [0, 4])
def test_paged_pool_sizes_are_pages_of_the_unpaged_layout(sr):
    """A pool of n_pages pages holds n_pages (b, group) blocks of the unpaged layout; the
    block table is int32 [B][Lcap/group_k]."""
    base = cfg(max_context=1000, side_rank=sr, side_bits=4 if sr else 0)
    flat = K.kvq_buffer_sizes(base)
    groups = base["batch"] * -(-1000 // base["group_k"])
    for n_pages in (1, 7, groups, 3 * groups):
        got = K.kvq_buffer_sizes(dict(base, paged=1, n_pages=n_pages))
        for n in ("kcode", "ksz", "vcode", "vsz") + (("zcode", "zsz") if sr else ()):
            assert got[n] * groups == flat[n] * n_pages, n
        for n in ("win_k", "win_v", "ret_k", "ret_v", "workspace", "side_u"):
            assert got[n] == flat[n], n
        assert got["block_table"] == groups * 4
    assert flat["block_table"] == 0


@pytest.mark.parametrize("bad,code", [
    (dict(paged=2, n_pages=8), K.KVQ_ERR_INVALID_ARG),
    (dict(paged=1, n_pages=0), K.KVQ_ERR_INVALID_ARG),
    (dict(paged=1, n_pages=-3), K.KVQ_ERR_INVALID_ARG),
    (dict(paged=1, n_pages=8, k_bits=16, v_bits=16), K.KVQ_ERR_UNSUPPORTED),
    (dict(paged=1, n_pages=(1 << 30) // (2 * 64)), K.KVQ_ERR_UNSUPPORTED),   # 2^30 rows
])
def test_invalid_paged_configurations_are_rejected(bad, code):
    with pytest.raises(K.KVQError) as e:
        K.kvq_buffer_sizes(cfg(**bad))
    assert e.value.code == code


def test_paged_caches_need_a_block_table():
    c = cfg(paged=1, n_pages=16)
    ptrs = {n: 4096 * (i + 1) for i, n in enumerate(K.POINTER_FIELDS)}
    ptrs["block_table"] = 0
    with pytest.raises(K.KVQError) as e:
        K.kvq_cache_init(c, ptrs)
    assert e.value.code == K.KVQ_ERR_INVALID_ARG
    ptrs = {n: 4096 * (i + 1) for i, n in enumerate(K.POINTER_FIELDS)}
    ptrs["block_table"] += 4
    with pytest.raises(K.KVQError) as e:
        K.kvq_cache_init(c, ptrs)
    assert e.value.code == K.KVQ_ERR_ALIGN


def test_sequence_calls_check_their_arguments():
    lib = K.lib()
    assert lib.kvq_prefill_sequence(None, 0, None, None, 1, None) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_release_sequence(None, 0) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_free_pages(None) == K.KVQ_ERR_INVALID_ARG


def test_unpaged_group_indices_must_fit_31_bits():
    # B * Hkv * Lcap / group_k >= 2^31 groups
    with pytest.raises(K.KVQError) as e:
        K.kvq_buffer_sizes(cfg(batch=1 << 14, n_kv_heads=8, n_q_heads=8, group_k=16,
                               max_context=1 << 18))
    assert e.value.code == K.KVQ_ERR_UNSUPPORTED


# ------------------------------------------------------ per-channel widths ----
def var(**kw):
    base = cfg(k_bits=0, v_bits=0, group_v=32, k_widths=[8] * 16 + [4] * 64 + [2] * 32 + [0] * 16,
               v_widths=[4] * 32 + [2] * 64 + [1] * 32)
    base.update(kw)
    return base


@pytest.mark.parametrize("seed", range(12))
def test_allocator_matches_the_oracle(seed):
    import numpy as np
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 200))
    w = rng.lognormal(0.0, 2.0, size=n)
    if seed % 3 == 0:
        w[rng.integers(0, n, size=n // 3)] = w[0]            # ties
    if seed % 4 == 1:
        w[rng.integers(0, n, size=n // 4)] = 0.0              # zero weights
    if seed % 5 == 2:
        w = np.round(w * 4) / 4                                # many exact ties
    unit = int(rng.choice([1, 8, 16, 64]))
    for budget in (0, 1, unit * n // 2, unit * 3 * n, unit * 8 * n, 10 ** 7):
        got, spent = K.kvq_allocate_bits(list(w), budget, unit)
        want = O.allocate_bits(w, budget, unit)
        assert got == [int(x) for x in want], (seed, budget)
        assert spent == unit * int(np.sum(want)) <= budget


def test_allocator_rejects_bad_arguments():
    for args in (([], 4, 1), ([1.0, -1.0], 4, 1), ([1.0, float("nan")], 4, 1), ([1.0, float("inf")], 4, 1),
                 ([1.0], -1, 1), ([1.0], 4, 0)):
        with pytest.raises(K.KVQError) as e:
            K.kvq_allocate_bits(*args)
        assert e.value.code == K.KVQ_ERR_INVALID_ARG
    lib = K.lib()
    assert lib.kvq_allocate_bits(None, 1, 1, 1, None) == K.KVQ_ERR_INVALID_ARG


def test_allocation_of_sorted_weights_is_a_valid_width_map():
    import numpy as np
    rng = np.random.default_rng(9)
    kw_ = sorted(rng.lognormal(0.0, 2.0, size=128), reverse=True)
    vw_ = sorted(rng.lognormal(0.0, 1.0, size=4), reverse=True)
    kmap, _ = K.kvq_allocate_bits(kw_, 3 * 128)
    gmap, _ = K.kvq_allocate_bits(vw_, 2 * 128, unit_bits=32)
    vmap = [w for w in gmap for _ in range(32)]
    sizes = K.kvq_buffer_sizes(var(k_widths=kmap, v_widths=vmap))
    c = var(k_widths=kmap, v_widths=vmap)
    assert sizes["kcode"] == O.buffer_bytes(c)["kcode"]


@pytest.mark.parametrize("kw_,vw_", [
    ([4] * 64 + [8] * 64, [2] * 128),                        # keys increase
    ([3] * 128, [2] * 128),                                  # width 3
    ([4] * 128, [2] * 16 + [1] * 112),                       # a value group of 32 split 16/16
    ([4] * 128, [1] * 32 + [2] * 96),                        # values increase
    ([16] * 128, [2] * 128),                                 # width 16
])
def test_invalid_width_maps_are_rejected(kw_, vw_):
    with pytest.raises(K.KVQError) as e:
        K.kvq_buffer_sizes(var(k_widths=kw_, v_widths=vw_))
    assert e.value.code == K.KVQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("bad", [dict(v_bits=2), dict(k_bits=4), dict(side_rank=4, side_bits=4),
                                 dict(rot_keys=1), dict(group_k=48), dict(group_v=12)])
def test_width_maps_do_not_combine_with_other_modes(bad):
    with pytest.raises(K.KVQError) as e:
        K.kvq_buffer_sizes(var(**bad))
    assert e.value.code == K.KVQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw_,vw_,gv,fast", [
    ([8] * 16 + [4] * 64 + [2] * 32 + [0] * 16, [4] * 32 + [2] * 64 + [1] * 32, 32, 1),
    ([0] * 128, [0] * 128, 64, 1),                           # everything dropped: 1-word rows
    ([1] * 128, [8] * 8 + [1] * 120, 8, 0),                  # value groups below 16 channels
    ([8] * 128, [4] * 128, 128, 1),
    ([8] * 12 + [4] * 116, [2] * 128, 32, 0),                # 3 + 28 + 2 = 33 couples > 32
    ([8] * 14 + [4] * 84 + [0] * 30, [2] * 128, 32, 1),      # word 3 mixes widths: 25 couples
    ([4] * 128, [1] * 128, 16, 1),                           # 1-bit value groups of 16
    ([4] * 128, [1] * 128, 8, 0),                            # value groups of 8
])
def test_width_map_sizes_match_the_oracle_layout(kw_, vw_, gv, fast):
    c = var(k_widths=kw_, v_widths=vw_, group_v=gv)
    got, want = K.kvq_buffer_sizes(c), O.buffer_bytes(c)
    for n in K.BUFFER_FIELDS:
        assert got[n] == want[n], n
    # the planner counts the packed rows; the tensor-core kernel takes the maps it is built for
    p = K.kvq_plan_decode(c, 3000, 148, 0)
    assert p["fast_path"] == fast and p["n_groups"] == (3000 - 128) // 64
    assert K.kvq_plan_decode(dict(c, d_k=64), 3000, 148, 0)["fast_path"] == 0 if len(kw_) == 128 else True


def test_release_build_has_no_bounds_checks():
    """The in-tree libkvq.so is the release build: kvq_debug_take_record is UNSUPPORTED there
    (no device call is made), and every check site has a name."""
    lib = K.lib()
    assert lib.kvq_debug_build() == 0
    rec = K.kvq_debug_record()
    assert lib.kvq_debug_take_record(ctypes.byref(rec), None) == K.KVQ_ERR_UNSUPPORTED
    assert lib.kvq_debug_take_record(None, None) == K.KVQ_ERR_INVALID_ARG
    names = [lib.kvq_debug_site_name(i).decode() for i in range(64)]
    assert names[0] == "none" and "unknown" in names
    known = names[:names.index("unknown")]
    assert len(set(known)) == len(known) > 20


def test_bounds_check_build_reports_itself():
    """libkvq_debug.so (built with -DKVQ_DEBUG from the same sources) says so."""
    path = os.path.join(ROOT, "mixed_precision_quantized_pack_b200", "libkvq_debug.so")
    if not os.path.exists(path):
        pytest.skip("bounds-check library not built")
    code = ("import ctypes,sys; l=ctypes.CDLL(sys.argv[1]); l.kvq_debug_build.restype=ctypes.c_int; "
            "print(l.kvq_debug_build())")
    out = subprocess.run([sys.executable, "-c", code, path], capture_output=True, text=True, timeout=120)
    assert out.stdout.strip() == "1", out.stderr


def test_value_centering_policy():
    """The tensor-core kernel centres value codes from 65536 quantized tokens (AUTO); the plan
    reports it, and never for the generic kernel, unquantized or per-channel-width caches."""
    w = W.sweep_workload(8, 4, 2)
    cfg = w.kvq_config()
    assert K.kvq_plan_decode(cfg, 131072, 148, 0)["centered"] == 1
    assert K.kvq_plan_decode(cfg, 65536 + 128, 148, 0)["centered"] == 1       # Q = 65536
    assert K.kvq_plan_decode(cfg, 65536 + 127, 148, 0)["centered"] == 0       # Q = 65472
    assert K.kvq_plan_decode(W.WORKLOADS["long32k"].kvq_config(), 32768, 148, 0)["centered"] == 0
    assert K.kvq_plan_decode(W.sweep_workload(8, 16, 16).kvq_config(), 131072, 148, 0)["centered"] == 0
    assert K.kvq_plan_decode(W.WORKLOADS["aatc32k"].with_(context=131072).kvq_config(), 131072, 148, 0)["centered"] == 0
    generic = W.WORKLOADS["gqa4k"].with_(n_q_heads=64, context=131072)
    assert K.kvq_plan_decode(generic.kvq_config(), 131072, 148, 0) == dict(
        K.kvq_plan_decode(generic.kvq_config(), 131072, 148, 0), fast_path=0, centered=0)
    lib = K.lib()
    assert lib.kvq_set_value_centering(None, K.KVQ_CENTER_ON) == K.KVQ_ERR_INVALID_ARG
