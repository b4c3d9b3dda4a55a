"""CUDA path vs the CPU oracle, through the C ABI.

Packed codes, (scale, zero) pairs, window slots, retained tokens and retained
positions must match the oracle bit for bit; attention outputs must be within
2e-3 of the oracle's fp64 result, measured per (b, query head) as
max_c |o - o*| / max_c |o*|.
"""
import numpy as np
import pytest
import torch

from oracle import kvq_oracle as O
from mixed_precision_quantized_pack_b200 import kvq as K
from mixed_precision_quantized_pack_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL = 2e-3
AATC = W.WORKLOADS["aatc32k"]
# AUTO picks the tensor-core kernel wherever it is built for the shape; GENERIC is
# the CUDA-core kernel.  Both are checked against the oracle.
KERNELS = (K.KVQ_KERNEL_AUTO, K.KVQ_KERNEL_GENERIC)


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def np16(t):
    return t.detach().cpu().numpy()


def compare_state(gc: K.KVCache, oc: O.OracleCache, b_rows=None, where="", seq=None):
    """Bit-exact comparison of every valid byte of the cache, rows b in b_rows (the state of
    sequence `seq` when the sequences' lengths differ)."""
    L, Q, ret = gc.state() if seq is None else gc.seq_state(seq)
    assert (L, Q, ret) == (oc.L, oc.Q, oc.ret_idx), where
    rows = list(range(gc.B)) if b_rows is None else list(b_rows)
    c = gc.cfg
    if c["k_bits"] != 16 and Q:
        gk = c["group_k"]
        pairs = [("kcode", slice(0, Q)), ("ksz", slice(0, Q // gk)), ("vcode", slice(0, Q)),
                 ("vsz", slice(0, Q))]
        if c.get("side_rank", 0):
            pairs += [("zcode", slice(0, Q)), ("zsz", slice(0, Q // gk))]
        for name, sl in pairs:
            if c.get("paged"):     # the sequence's pages, gathered through the block table
                g = np.stack([gc.sequence_view(name, b).cpu().numpy() for b in rows])
            else:
                g = gc.view(name)[rows][:, :, sl].cpu().numpy()
            o = getattr(oc, name)[:, :, sl]
            if b_rows is None:
                o = o[rows]
            assert np.array_equal(g.view(np.uint8), np.ascontiguousarray(o).view(np.uint8)), \
                f"{where}: {name} differs"
    slots = [p % oc.cap for p in range(Q, L)]
    for name in ("win_k", "win_v"):
        g = gc.view(name)[rows][:, :, slots].cpu().numpy()
        o = getattr(oc, name)[:, :, slots]
        if b_rows is None:
            o = o[rows]
        assert np.array_equal(g.view(np.uint16), o.view(np.uint16)), f"{where}: {name} differs"
    if ret:
        n = len(ret)
        for name in ("ret_k", "ret_v"):
            g = gc.view(name)[rows][:, :, :n].cpu().numpy()
            o = getattr(oc, name)[:, :, :n]
            if b_rows is None:
                o = o[rows]
            assert np.array_equal(g.view(np.uint16), o.view(np.uint16)), f"{where}: {name} differs"


def make_caches(cfg, inp, batch=None):
    """A GPU cache and an oracle cache of one configuration (with the inputs' side basis)."""
    U = inp.side_basis
    gc = K.KVCache(cfg, side_basis=U)
    ocfg = cfg if batch is None else dict(cfg, batch=batch)
    oc = O.OracleCache(ocfg, side_basis=None if U is None else U.cpu().numpy())
    return gc, oc


def run_small(w: W.Workload, num_splits=(0,), steps=None, centering=None):
    """Prefill + (appends) + decodes of a workload small enough for the full oracle."""
    need_gpu()
    inp = W.Inputs(w, device="cpu")
    cfg = w.kvq_config()
    gc, oc = make_caches(cfg, inp)
    if centering is not None:
        gc.set_centering(centering)
    gc.prefill(inp.k.cuda(), inp.v.cuda())
    oc.prefill(np16(inp.k), np16(inp.v))
    if centering == K.KVQ_CENTER_ON:
        assert gc.plan()["centered"] == 1
    compare_state(gc, oc, where="prefill")
    worst = 0.0
    n_dec = len(inp.q)
    for i in range(n_dec):
        if w.appends:
            gc.append(inp.k_app[i].cuda(), inp.v_app[i].cuda())
            oc.append(np16(inp.k_app[i]), np16(inp.v_app[i]))
        if steps is not None and i not in steps:
            continue
        compare_state(gc, oc, where=f"step {i}")
        ref = oc.decode(np16(inp.q[i]))
        for kern in KERNELS:
            gc.set_kernel(kern)
            for s in num_splits:
                out = gc.decode(inp.q[i].cuda(), num_splits=s)
                err = O.max_rel_error(out.float().cpu().numpy(), ref)
                worst = max(worst, err)
                assert err <= TOL, f"step {i} kernel {kern} splits {s}: max rel error {err:.3e}"
        gc.set_kernel(K.KVQ_KERNEL_AUTO)
    assert gc.status() == 0
    return worst


def tensor_kernel_built(w: W.Workload) -> bool:
    return K.kvq_plan_decode(w.kvq_config(), w.context, 148, 0)["fast_path"] == 1


@pytest.mark.parametrize("key", list(W.WORKLOADS))
def test_tensor_kernel_covers_the_named_workloads(key):
    assert tensor_kernel_built(W.WORKLOADS[key])
    for b in W.SWEEP_BATCHES:
        for kb, vb in W.SWEEP_BITS:
            assert tensor_kernel_built(W.sweep_workload(b, kb, vb))


def test_tiny_single_head():
    run_small(W.WORKLOADS["tiny"], num_splits=(0, 1, 2, 5))


def test_gqa_4k_with_append():
    run_small(W.WORKLOADS["gqa4k"], num_splits=(0, 1, 3))


def test_thin_keys_16k():
    run_small(W.WORKLOADS["thin16k"].with_(batch=2), num_splits=(0, 1))


@pytest.mark.parametrize("kb,vb", [(8, 4), (4, 2), (2, 2), (4, 4), (8, 8), (2, 4)])
def test_bit_widths(kb, vb):
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=1500, k_bits=kb, v_bits=vb, appends=70,
                                   log_retain=1, seed=77)
    run_small(w, num_splits=(0, 2), steps={0, 1, 57, 58, 69})


@pytest.mark.parametrize("kb,vb,gv,gk", [(4, 2, 64, 64), (4, 2, 32, 32), (8, 4, 64, 64), (8, 4, 32, 32),
                                         (2, 2, 64, 64), (4, 4, 64, 64)])
def test_centred_value_codes(kb, vb, gv, gk):
    """The tensor-core kernel with centred value codes (forced on at these short contexts; the
    library turns it on by itself from 65536 quantized tokens) matches the oracle."""
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=1500, k_bits=kb, v_bits=vb, group_v=gv, group_k=gk,
                                   appends=66, log_retain=1, seed=71 + kb + gv)
    assert tensor_kernel_built(w)
    need_gpu()
    run_small(w, num_splits=(0, 2), steps={0, 64, 65}, centering=K.KVQ_CENTER_ON)


def test_unquantized_fp16_cache():
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=3000, k_bits=16, v_bits=16, appends=3,
                                   seed=78)
    run_small(w, num_splits=(0, 1, 4))


@pytest.mark.parametrize("n_q,n_kv", [(8, 8), (16, 8), (64, 8)])
def test_gqa_group_sizes(n_q, n_kv):
    w = W.WORKLOADS["gqa4k"].with_(batch=1, n_q_heads=n_q, n_kv_heads=n_kv, context=777, seed=79)
    run_small(w, num_splits=(0, 1))


@pytest.mark.parametrize("gk,gv,R", [(16, 16, 0), (32, 128, 32), (128, 64, 5), (64, 32, 300)])
def test_group_sizes_and_windows(gk, gv, R):
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=1111, group_k=gk, group_v=gv, window=R,
                                   log_retain=1, appends=2 * gk + 3, seed=80 + gk)
    run_small(w, num_splits=(0, 3), steps={0, gk - 1, gk, 2 * gk + 2})


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (256, 256), (32, 32)])
def test_head_dims(dk, dv):
    w = W.WORKLOADS["gqa4k"].with_(batch=1, n_q_heads=8, n_kv_heads=2, d_k=dk, d_v=dv,
                                   context=900, group_v=32, seed=81)
    run_small(w, num_splits=(0,))


@pytest.mark.parametrize("L", [1, 5, 127, 128, 129, 191, 192, 193, 256])
def test_short_contexts(L):
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=L, appends=0, log_retain=1, seed=90 + L)
    run_small(w, num_splits=(0, 1))


def test_split_invariance():
    need_gpu()
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=6000, log_retain=1, seed=91)
    inp = W.Inputs(w)
    gc = K.KVCache(w.kvq_config())
    gc.prefill(inp.k.cuda(), inp.v.cuda())
    q = inp.q[0].cuda()
    outs = [gc.decode(q, num_splits=s).float() for s in (1, 2, 3, 7, 16, 0)]
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 2e-3 * outs[0].abs().max().item()


@pytest.mark.parametrize("case", ["fixed", "paged", "widths"])
def test_a_wait_that_runs_out_sets_the_timeout_status(case):
    """The tensor-core kernels' waits are bounded: when one gives up (the test hook makes one
    copy stage ask for 16 bytes more than it receives) the call sets KVQ_STATUS_TIMEOUT
    within seconds, and the context and the cache stay usable for the next call."""
    need_gpu()
    import time
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=1024, appends=0, seed=91)
    if case == "paged":
        w = w.with_(paged=1)
    elif case == "widths":
        w = AATC.with_(batch=2, context=1024, appends=0, seed=92)
    inp = W.Inputs(w, device="cpu")
    cfg = w.kvq_config()
    gc = K.KVCache(cfg)
    oc = O.OracleCache(cfg)
    gc.prefill(inp.k.cuda(), inp.v.cuda())
    oc.prefill(np16(inp.k), np16(inp.v))
    assert gc.plan()["fast_path"] == 1
    ref = oc.decode(np16(inp.q[0]))
    q = inp.q[0].cuda()
    assert O.max_rel_error(gc.decode(q).float().cpu().numpy(), ref) <= TOL
    assert gc.status() == 0
    K.kvq_debug_stall_next_decode(gc.handle)
    t0 = time.time()
    gc.decode(q)
    status = gc.status()
    assert status & K.KVQ_STATUS_TIMEOUT
    assert time.time() - t0 < 30
    gc.reset_status()
    out = gc.decode(q)
    assert gc.status() == 0
    assert O.max_rel_error(out.float().cpu().numpy(), ref) <= TOL


def test_error_paths():
    need_gpu()
    w = W.WORKLOADS["tiny"].with_(context=100)
    gc = K.KVCache(w.kvq_config(max_context=101))
    q = torch.zeros((1, 1, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(K.KVQError) as e:
        gc.decode(q)
    assert e.value.code == K.KVQ_ERR_STATE
    kv = torch.zeros((1, 1, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(K.KVQError) as e:
        gc.append(kv, kv)
    assert e.value.code == K.KVQ_ERR_STATE
    inp = W.Inputs(w)
    gc.prefill(inp.k.cuda(), inp.v.cuda())
    gc.append(kv, kv)
    with pytest.raises(K.KVQError) as e:
        gc.append(kv, kv)
    assert e.value.code == K.KVQ_ERR_CAPACITY
    need = K.kvq_decode_workspace_size(gc.handle, 0)
    out = torch.empty((1, 1, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(K.KVQError) as e:
        K.kvq_decode_attention(gc.handle, q.data_ptr(), out.data_ptr(), gc.workspace.data_ptr(),
                               need - 1, 0, K._stream())
    assert e.value.code == K.KVQ_ERR_WORKSPACE
    with pytest.raises(K.KVQError) as e:
        K.kvq_decode_attention(gc.handle, q.data_ptr() + 2, out.data_ptr(),
                               gc.workspace.data_ptr(), need, 0, K._stream())
    assert e.value.code == K.KVQ_ERR_ALIGN
    with pytest.raises(K.KVQError) as e:
        gc.prefill(inp.k.cuda()[:, :, :0], inp.v.cuda()[:, :, :0])
    assert e.value.code == K.KVQ_ERR_INVALID_ARG


# ----------------------------------------------------------------- full sizes ----
def sampled_full_size(w: W.Workload, rows, steps=(0,)):
    """Full-size workload on the GPU; the oracle recomputes sampled sequences b."""
    need_gpu()
    inp = W.Inputs(w, device="cuda")
    gc = K.KVCache(w.kvq_config(), side_basis=inp.side_basis)
    gc.prefill(inp.k, inp.v)
    U = None if inp.side_basis is None else inp.side_basis.cpu().numpy()
    ocs = {}
    for b in rows:
        sub = dict(w.kvq_config(), batch=1)
        oc = O.OracleCache(sub, side_basis=U)
        oc.prefill(np16(inp.k[b:b + 1]), np16(inp.v[b:b + 1]))
        ocs[b] = oc
    n_dec = len(inp.q)
    for i in range(n_dec):
        if w.appends:
            gc.append(inp.k_app[i], inp.v_app[i])
            for b, oc in ocs.items():
                oc.append(np16(inp.k_app[i][b:b + 1]), np16(inp.v_app[i][b:b + 1]))
        if i not in steps:
            continue
        out = gc.decode(inp.q[i]).float().cpu().numpy()
        for b, oc in ocs.items():
            compare_state(gc, oc, b_rows=[b], where=f"b={b} step {i}")
            ref = oc.decode(np16(inp.q[i][b:b + 1]))
            err = O.max_rel_error(out[b:b + 1], ref)
            assert err <= TOL, f"b={b} step {i}: {err:.3e}"
    assert gc.status() == 0
    del gc, inp
    torch.cuda.empty_cache()


def test_full_size_long_32k_logretain():
    w = W.WORKLOADS["long32k"]
    sampled_full_size(w, rows=(0, 31))


def test_full_size_gqa_4k():
    sampled_full_size(W.WORKLOADS["gqa4k"], rows=(3,))


def test_full_size_thin_16k():
    sampled_full_size(W.WORKLOADS["thin16k"], rows=(0, 15))


# ------------------------------------------------------- HeadQ side code ----
@pytest.mark.parametrize("kb", [4, 2])
@pytest.mark.parametrize("sr,sq", [(4, 4), (4, 8), (8, 4)])
def test_side_code_tensor_kernel(kb, sr, sq):
    """Side codes bit-exact after prefill and across appends that quantize new groups;
    outputs of both kernels within the bound (the tensor-core kernel is built for these)."""
    w = W.WORKLOADS["headq32k"].with_(batch=2, context=1500, k_bits=kb, side_rank=sr,
                                      side_bits=sq, appends=70, seed=101 + sr + sq)
    assert tensor_kernel_built(w)
    run_small(w, num_splits=(0, 3), steps={0, 1, 57, 58, 69})


@pytest.mark.parametrize("shape", [
    dict(n_q_heads=8, n_kv_heads=8, d_k=128, group_k=64),     # n_rep 1
    dict(n_q_heads=8, n_kv_heads=2, d_k=64, d_v=64, group_k=32, group_v=32),
    dict(n_q_heads=8, n_kv_heads=2, d_k=256, d_v=128, group_k=128, k_bits=8, v_bits=4),
])
def test_side_code_generic_kernel_shapes(shape):
    w = W.WORKLOADS["headq32k"].with_(batch=2, context=900, appends=2, seed=111, **shape)
    assert not tensor_kernel_built(w)
    run_small(w, num_splits=(0, 2))


def test_full_size_headq_32k():
    sampled_full_size(W.WORKLOADS["headq32k"], rows=(0, 31))


# ------------------------------------------------------ key-only rotation ----
@pytest.mark.parametrize("kb,vb", [(4, 2), (2, 2), (8, 4)])
def test_rotation_tensor_kernel(kb, vb):
    """Rotated keys: codes, window and retained copies bit-exact across appends; outputs of
    both kernels within the bound."""
    w = W.WORKLOADS["rot32k"].with_(batch=2, context=1500, k_bits=kb, v_bits=vb, appends=70,
                                    seed=171 + kb)
    assert tensor_kernel_built(w)
    run_small(w, num_splits=(0, 3), steps={0, 1, 57, 58, 69})


def test_rotation_with_side_code():
    w = W.WORKLOADS["headq32k"].with_(batch=2, context=1200, appends=66, rot_keys=1, rot_seed=5,
                                      seed=181)
    run_small(w, num_splits=(0, 2), steps={0, 63, 64, 65})


@pytest.mark.parametrize("dk,dv", [(32, 128), (64, 64), (256, 128)])
def test_rotation_head_dims(dk, dv):
    w = W.WORKLOADS["rot32k"].with_(batch=1, n_q_heads=8, n_kv_heads=2, d_k=dk, d_v=dv, context=900,
                                    group_k=32, group_v=32, window=64, appends=34, seed=191)
    run_small(w, num_splits=(0, 2), steps={0, 33})


def test_rotation_unquantized_cache():
    w = W.WORKLOADS["rot32k"].with_(batch=2, context=700, k_bits=16, v_bits=16, appends=3, seed=201)
    run_small(w, num_splits=(0, 3))


def test_full_size_rot_32k():
    sampled_full_size(W.WORKLOADS["rot32k"], rows=(0, 31))


# ------------------------------------------- sequences of different lengths ----
def run_ragged(w: W.Workload, lengths, n_app, steps, seed, num_splits=(0, 2)):
    """Ragged prefill, then appends where random sequences sit out: every sequence's cache
    bytes and outputs match an oracle cache of that sequence alone."""
    need_gpu()
    L_max = max(lengths)
    inp = W.Inputs(w.with_(context=L_max, appends=n_app), device="cpu")
    cfg = w.kvq_config(max_context=L_max + n_app + 64)
    gc = K.KVCache(cfg, side_basis=inp.side_basis)
    gc.prefill_ragged(inp.k.cuda(), inp.v.cuda(), lengths)
    U = None if inp.side_basis is None else inp.side_basis.numpy()
    ocs = []
    for b, Lb in enumerate(lengths):
        oc = O.OracleCache(dict(cfg, batch=1), side_basis=U)
        oc.prefill(np16(inp.k[b:b + 1, :, :Lb]), np16(inp.v[b:b + 1, :, :Lb]))
        ocs.append(oc)
    rng = np.random.default_rng(seed)
    for i in range(n_app):
        active = [True] * len(lengths) if i % 3 == 0 else [bool(x) for x in rng.integers(0, 2, len(lengths))]
        gc.append(inp.k_app[i].cuda(), inp.v_app[i].cuda(), active=active)
        for b, oc in enumerate(ocs):
            if active[b]:
                oc.append(np16(inp.k_app[i][b:b + 1]), np16(inp.v_app[i][b:b + 1]))
        if i not in steps:
            continue
        for b, oc in enumerate(ocs):
            assert gc.seq_state(b) == (oc.L, oc.Q, oc.ret_idx), (i, b)
            compare_state(gc, oc, b_rows=[b], where=f"step {i} b={b}", seq=b)
        for kern in KERNELS:
            gc.set_kernel(kern)
            for ns in num_splits:
                out = gc.decode(inp.q[i].cuda(), num_splits=ns).float().cpu().numpy()
                for b, oc in enumerate(ocs):
                    err = O.max_rel_error(out[b:b + 1], oc.decode(np16(inp.q[i][b:b + 1])))
                    assert err <= TOL, f"step {i} b={b} kernel {kern} splits {ns}: {err:.3e}"
        gc.set_kernel(K.KVQ_KERNEL_AUTO)
    assert gc.status() == 0


def test_ragged_batch_tensor_kernel():
    w = W.WORKLOADS["long32k"].with_(batch=5, seed=211)
    run_ragged(w, [1500, 700, 64, 1111, 129], n_app=70, steps={0, 5, 40, 69}, seed=212)


def test_ragged_batch_with_side_code_and_rotation():
    w = W.WORKLOADS["headq32k"].with_(batch=3, rot_keys=1, rot_seed=9, seed=221)
    run_ragged(w, [900, 333, 1280], n_app=66, steps={1, 64, 65}, seed=222)


def test_ragged_batch_generic_shapes():
    w = W.WORKLOADS["gqa4k"].with_(batch=3, n_q_heads=6, n_kv_heads=3, d_k=64, d_v=64, group_k=32,
                                   group_v=32, window=48, log_retain=1, seed=231)
    run_ragged(w, [400, 81, 257], n_app=40, steps={0, 17, 39}, seed=232)


def test_uniform_lengths_through_the_ragged_calls_match_the_plain_ones():
    need_gpu()
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=1000, appends=5, log_retain=1, seed=241)
    inp = W.Inputs(w, device="cpu")
    cfg = w.kvq_config()
    a, b = K.KVCache(cfg), K.KVCache(cfg)
    a.prefill(inp.k.cuda(), inp.v.cuda())
    b.prefill_ragged(inp.k.cuda(), inp.v.cuda(), [1000, 1000])
    for i in range(5):
        a.append(inp.k_app[i].cuda(), inp.v_app[i].cuda())
        b.append(inp.k_app[i].cuda(), inp.v_app[i].cuda(), active=[True, True])
    assert a.state() == b.state() == b.seq_state(1)
    for name in ("kcode", "ksz", "vcode", "vsz", "ret_k", "ret_v"):
        assert torch.equal(a.buffers[name], b.buffers[name]), name
    assert torch.equal(a.decode(inp.q[-1].cuda()), b.decode(inp.q[-1].cuda()))


# ------------------------------------------------------------------ paged caches ----
def paged_twins(w: W.Workload, max_context: int, n_pages: int, side_basis):
    """A paged cache and an unpaged one of the same configuration."""
    cfg = w.kvq_config(max_context=max_context)
    paged = K.KVCache(dict(cfg, paged=1, n_pages=n_pages), side_basis=side_basis)
    flat = K.KVCache(dict(cfg, paged=0, n_pages=0), side_basis=side_basis)
    return cfg, paged, flat


def run_paged(w: W.Workload, lengths, n_app, steps, seed, restart=None, num_splits=(0, 2)):
    """Paged cache under ragged prefill, masked appends and (at step `restart`) a release and
    a new prefill of sequence 1 with other tokens: every sequence's pages hold the oracle's
    bytes, outputs match the oracle, and they equal the unpaged cache's outputs bit for bit."""
    need_gpu()
    L_max = max(lengths)
    inp = W.Inputs(w.with_(context=L_max, appends=n_app), device="cpu")
    mc = L_max + n_app + 64
    gk = w.group_k
    groups = len(lengths) * -(-mc // gk)
    cfg, gp, gf = paged_twins(w, mc, groups + 3, inp.side_basis)
    gp.prefill_ragged(inp.k.cuda(), inp.v.cuda(), lengths)
    gf.prefill_ragged(inp.k.cuda(), inp.v.cuda(), lengths)
    U = None if inp.side_basis is None else inp.side_basis.numpy()

    def oracle_of(k, v):
        oc = O.OracleCache(dict(cfg, batch=1), side_basis=U)
        oc.prefill(np16(k), np16(v))
        return oc

    ocs = [oracle_of(inp.k[b:b + 1, :, :Lb], inp.v[b:b + 1, :, :Lb]) for b, Lb in enumerate(lengths)]
    held = sum(oc.Q // gk for oc in ocs)
    assert gp.free_pages() == groups + 3 - held
    rng = np.random.default_rng(seed)
    for i in range(n_app):
        if i == restart:
            # sequence 1 starts over with the first Lr tokens of sequence 0's prefill
            Lr = lengths[0] - 3
            k1 = inp.k[0, :, :Lr].contiguous()
            v1 = inp.v[0, :, :Lr].contiguous()
            before = gp.free_pages()
            gp.release(1)
            assert gp.free_pages() == before + ocs[1].Q // gk
            gp.prefill_sequence(1, k1.cuda(), v1.cuda())
            gf.prefill_sequence(1, k1.cuda(), v1.cuda())
            ocs[1] = oracle_of(k1[None], v1[None])
        active = [True] * len(lengths) if i % 3 == 0 else [bool(x) for x in rng.integers(0, 2, len(lengths))]
        for c in (gp, gf):
            c.append(inp.k_app[i].cuda(), inp.v_app[i].cuda(), active=active)
        for b, oc in enumerate(ocs):
            if active[b]:
                oc.append(np16(inp.k_app[i][b:b + 1]), np16(inp.v_app[i][b:b + 1]))
        assert gp.free_pages() == groups + 3 - sum(oc.Q // gk for oc in ocs)
        if i not in steps:
            continue
        for b, oc in enumerate(ocs):
            compare_state(gp, oc, b_rows=[b], where=f"paged step {i} b={b}", seq=b)
        table = gp.view("block_table").cpu()
        used = [int(p) for b, oc in enumerate(ocs) for p in table[b, :oc.Q // gk]]
        assert len(set(used)) == len(used), "a page is held twice"
        for kern in KERNELS:
            gp.set_kernel(kern)
            gf.set_kernel(kern)
            # the same kernel on both layouts gives the same bits (the tensor-core kernel has
            # no paged instances for side codes: there the paged cache runs the generic one)
            same = gp.plan()["fast_path"] == gf.plan()["fast_path"]
            for ns in num_splits:
                out = gp.decode(inp.q[i].cuda(), num_splits=ns)
                if same:
                    assert torch.equal(out, gf.decode(inp.q[i].cuda(), num_splits=ns)), (i, kern, ns)
                out = out.float().cpu().numpy()
                for b, oc in enumerate(ocs):
                    err = O.max_rel_error(out[b:b + 1], oc.decode(np16(inp.q[i][b:b + 1])))
                    assert err <= TOL, f"paged step {i} b={b} kernel {kern} splits {ns}: {err:.3e}"
        gp.set_kernel(K.KVQ_KERNEL_AUTO)
        gf.set_kernel(K.KVQ_KERNEL_AUTO)
    assert gp.status() == 0 and gf.status() == 0
    return gp


def test_paged_cache_tensor_kernel():
    w = W.WORKLOADS["paged32k"].with_(batch=4, seed=251)
    gp = run_paged(w, [1500, 700, 64, 1111], n_app=70, steps={0, 20, 21, 69}, seed=252, restart=20)
    assert gp.plan()["fast_path"] == 1


def test_paged_cache_with_side_code_and_rotation():
    w = W.WORKLOADS["headq32k"].with_(batch=3, rot_keys=1, rot_seed=9, seed=261, paged=1)
    assert tensor_kernel_built(w)
    run_paged(w, [900, 333, 1280], n_app=66, steps={1, 10, 64, 65}, seed=262, restart=10)


@pytest.mark.parametrize("kb,sr,sq", [(2, 4, 4), (4, 8, 4), (4, 4, 8)])
def test_paged_cache_with_side_code_tensor_kernel(kb, sr, sq):
    """Paged caches with a side code run on the tensor-core kernel (the paged side-code
    instances), against the oracle and bit for bit against their unpaged twins."""
    w = W.WORKLOADS["headq32k"].with_(batch=2, k_bits=kb, side_rank=sr, side_bits=sq,
                                      seed=263 + sr + sq, paged=1)
    assert tensor_kernel_built(w)
    run_paged(w, [1000, 555], n_app=66, steps={0, 65}, seed=264)


def test_paged_cache_generic_shapes():
    w = W.WORKLOADS["gqa4k"].with_(batch=3, n_q_heads=6, n_kv_heads=3, d_k=64, d_v=64, group_k=32,
                                   group_v=32, window=48, log_retain=1, seed=271, paged=1)
    run_paged(w, [400, 81, 257], n_app=40, steps={0, 5, 39}, seed=272, restart=5)


@pytest.mark.parametrize("kb,vb", [(8, 4), (2, 2), (4, 4)])
def test_paged_cache_bit_widths(kb, vb):
    w = W.WORKLOADS["paged32k"].with_(batch=2, k_bits=kb, v_bits=vb, seed=281 + kb)
    run_paged(w, [1000, 555], n_app=66, steps={0, 65}, seed=282)


def test_full_size_paged_32k():
    sampled_full_size(W.WORKLOADS["paged32k"], rows=(0, 31))


def test_full_size_headq_paged_32k():
    assert tensor_kernel_built(W.WORKLOADS["headq-paged32k"])
    sampled_full_size(W.WORKLOADS["headq-paged32k"], rows=(0, 31))


def test_page_pool_exhaustion_changes_nothing():
    need_gpu()
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=600, appends=80, seed=291, paged=1)
    inp = W.Inputs(w, device="cpu")
    gk, R = w.group_k, w.window
    q600 = (600 - R) // gk          # groups of a 600-token prefill: 7
    cfg = w.kvq_config(max_context=800)
    c = K.KVCache(dict(cfg, n_pages=2 * q600), side_basis=None)
    k, v = inp.k.cuda(), inp.v.cuda()
    c.prefill(k, v)
    assert c.free_pages() == 0
    with pytest.raises(K.KVQError) as e:          # the pool is full: no room for a bigger prefill
        c.prefill_sequence(0, torch.cat([k[0], k[1]], 1)[:, :700].contiguous(),
                           torch.cat([v[0], v[1]], 1)[:, :700].contiguous())
    assert e.value.code == K.KVQ_ERR_CAPACITY and c.seq_state(0)[:2] == (600, q600 * gk)
    # appends until the window spills a group: that append needs a page and fails whole
    n = 0
    while True:
        L = 600 + n
        if L + 1 - q600 * gk == R + gk:
            break
        c.append(inp.k_app[n].cuda(), inp.v_app[n].cuda())
        n += 1
    s0, s1 = c.seq_state(0), c.seq_state(1)
    with pytest.raises(K.KVQError) as e:
        c.append(inp.k_app[n].cuda(), inp.v_app[n].cuda())
    assert e.value.code == K.KVQ_ERR_CAPACITY
    assert (c.seq_state(0), c.seq_state(1), c.free_pages()) == (s0, s1, 0)
    # sequence 1 leaves: decode refuses an empty sequence, sequence 0 alone appends and
    # takes one of the freed pages
    c.release(1)
    assert c.free_pages() == q600
    with pytest.raises(K.KVQError) as e:
        c.decode(inp.q[0].cuda())
    assert e.value.code == K.KVQ_ERR_STATE
    with pytest.raises(K.KVQError) as e:
        c.append(inp.k_app[n].cuda(), inp.v_app[n].cuda())
    assert e.value.code == K.KVQ_ERR_STATE
    c.append(inp.k_app[n].cuda(), inp.v_app[n].cuda(), active=[True, False])
    assert c.free_pages() == q600 - 1 and c.seq_state(0)[1] == (q600 + 1) * gk
    # sequence 1 comes back and the cache decodes again, matching the oracle
    c.prefill_sequence(1, k[1, :, :300].contiguous(), v[1, :, :300].contiguous())
    oc0 = O.OracleCache(dict(cfg, batch=1))
    oc0.prefill(np16(inp.k[0:1]), np16(inp.v[0:1]))
    for i in range(n + 1):
        oc0.append(np16(inp.k_app[i][0:1]), np16(inp.v_app[i][0:1]))
    oc1 = O.OracleCache(dict(cfg, batch=1))
    oc1.prefill(np16(inp.k[1:2, :, :300]), np16(inp.v[1:2, :, :300]))
    compare_state(c, oc0, b_rows=[0], seq=0, where="after refill b=0")
    compare_state(c, oc1, b_rows=[1], seq=1, where="after refill b=1")
    out = c.decode(inp.q[1].cuda()).float().cpu().numpy()
    for b, oc in enumerate((oc0, oc1)):
        assert O.max_rel_error(out[b:b + 1], oc.decode(np16(inp.q[1][b:b + 1]))) <= TOL


# ------------------------------------------------------------ per-channel widths ----


@pytest.mark.parametrize("shape", [
    dict(),                                                                  # the bench map
    dict(k_widths=(0,) * 128, v_widths=(0,) * 128, group_v=64),              # everything dropped
    dict(k_widths=(1,) * 128, v_widths=(1,) * 128, group_v=8),
    dict(d_k=64, d_v=256, group_k=16, group_v=128,
         k_widths=(8,) * 8 + (4,) * 8 + (2,) * 16 + (1,) * 16 + (0,) * 16, v_widths=(8,) * 128 + (2,) * 128),
    dict(d_k=32, d_v=32, group_k=128, group_v=8, window=5, k_widths=(4,) * 32,
         v_widths=(8,) * 8 + (4,) * 8 + (0,) * 16),
    dict(d_k=256, group_v=16, n_q_heads=8, n_kv_heads=8,
         k_widths=(8,) * 32 + (4,) * 96 + (2,) * 64 + (1,) * 32 + (0,) * 32,
         v_widths=(8,) * 16 + (4,) * 48 + (2,) * 32 + (1,) * 16 + (0,) * 16),
    dict(k_widths=(8,) * 128, v_widths=(8,) * 128, group_v=128, log_retain=0),
    dict(n_q_heads=8, n_kv_heads=8, group_k=16),                               # tensor cores, GQA 1
    dict(group_k=128, group_v=16, v_widths=(8,) * 16 + (4,) * 32 + (2,) * 80),  # tensor cores
    # a key word holding 8- and 4-bit fields; 1-bit value groups of 16 (two-bit runs)
    dict(group_v=16, k_widths=(8,) * 14 + (4,) * 84 + (0,) * 30, v_widths=(4,) * 16 + (2,) * 32 + (1,) * 80),
    dict(group_v=64, k_widths=(8,) * 32 + (2,) * 96, v_widths=(4,) * 64 + (2,) * 64),
])
def test_width_maps(shape):
    w = AATC.with_(batch=2, context=1500, appends=70, seed=301 + len(str(shape)), **shape)
    run_small(w, num_splits=(0, 3), steps={0, 1, 57, 58, 69})


def test_width_map_kernel_choice():
    """The tensor-core kernel serves d 128 maps with value groups of 16-128 channels whose key
    fields fit in 32 couples; the others run on the generic kernel."""
    assert tensor_kernel_built(AATC)
    assert tensor_kernel_built(AATC.with_(n_q_heads=8, n_kv_heads=8))
    assert tensor_kernel_built(AATC.with_(group_v=16, k_widths=(8,) * 14 + (4,) * 84 + (0,) * 30,
                                          v_widths=(4,) * 16 + (2,) * 32 + (1,) * 80))
    assert not tensor_kernel_built(AATC.with_(d_k=64, k_widths=(4,) * 64))
    assert not tensor_kernel_built(AATC.with_(group_v=8))
    assert not tensor_kernel_built(AATC.with_(k_widths=(8,) * 12 + (4,) * 116))   # 33 couples


def test_width_maps_ragged_batch():
    run_ragged(AATC.with_(batch=4, seed=311), [1300, 64, 777, 1029], n_app=66, steps={0, 33, 65}, seed=312)


def test_width_maps_paged():
    run_paged(AATC.with_(batch=3, seed=321, paged=1), [900, 333, 1280], n_app=66, steps={1, 10, 65},
              seed=322, restart=10)


def test_full_size_aatc_32k():
    sampled_full_size(AATC, rows=(0, 31))


def test_full_size_aatc_32k_second_map():
    assert tensor_kernel_built(W.WORKLOADS["aatc32k-k8k2"])
    sampled_full_size(W.WORKLOADS["aatc32k-k8k2"], rows=(0, 31))


def test_full_size_aatc_32k_run_time_map():
    """A map with no build-time instance: the run-time plan at full size."""
    assert tensor_kernel_built(W.WORKLOADS["aatc32k-k4k2"])
    sampled_full_size(W.WORKLOADS["aatc32k-k4k2"], rows=(0, 31))
