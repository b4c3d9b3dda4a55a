"""The allocation-free decode entry point, called through the C ABI.

kvq_decode_attention_noalloc serves callers that cannot allocate device memory
(an engine that owns the device's memory pool, a plugin without an allocator, a
latency-critical loop that must not call cudaMalloc): instead of a caller
workspace it writes the split partials to a fixed scratch array inside the
library.  Its output must match kvq_decode_attention on the same cache, on two
calls in a row (the array keeps the previous call's contents), also when the
automatic split count has to shrink for the partials to fit; and the array's
status word must report a wait that gave up.  This file is collected last and
also runs on its own in a fresh process.
"""
import time

import numpy as np
import pytest
import torch

from mixed_precision_quantized_pack_b200 import kvq as K
from mixed_precision_quantized_pack_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL = 2e-3        # the tolerance of the parity tests: max_c|o - o*| / max_c|o*| per row


def rel_err(out: torch.Tensor, ref: torch.Tensor) -> float:
    o = out.float().reshape(-1, out.shape[-1])
    r = ref.float().reshape(-1, ref.shape[-1])
    return float(((o - r).abs().amax(1) / r.abs().amax(1).clamp_min(1e-30)).max())


def noalloc(cache: K.KVCache, q: torch.Tensor, num_splits: int = 0) -> torch.Tensor:
    out = torch.empty((cache.cfg["batch"], cache.cfg["n_q_heads"], cache.cfg["d_v"]),
                      dtype=torch.float16, device=q.device)
    K.kvq_decode_attention_noalloc(cache.handle, q.data_ptr(), out.data_ptr(), num_splits,
                                   K._stream())
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("w", [
    W.WORKLOADS["gqa4k"].with_(batch=4, appends=2, log_retain=1, seed=301),
    W.WORKLOADS["long32k"].with_(batch=4, appends=1, seed=302),
    W.WORKLOADS["thin16k"].with_(batch=2, appends=1, seed=303),
    W.WORKLOADS["gqa4k"].with_(batch=2, k_bits=16, v_bits=16, appends=1, seed=304),
], ids=["gqa4k", "long32k", "thin16k", "fp16"])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = W.Inputs(w, device="cuda")
    cache = K.KVCache(w.kvq_config())
    cache.prefill(inp.k, inp.v)
    for step in range(len(inp.q)):
        cache.append(inp.k_app[step], inp.v_app[step])
        ref = cache.decode(inp.q[step])
        torch.cuda.synchronize()
        first = noalloc(cache, inp.q[step])
        second = noalloc(cache, inp.q[step])
        assert rel_err(first, ref) <= TOL
        assert rel_err(second, ref) <= TOL
        assert torch.isfinite(second.float()).all()


def test_noalloc_rejects_a_split_count_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.WORKLOADS["gqa4k"].with_(batch=8, context=8192, seed=305)
    inp = W.Inputs(w, device="cuda")
    cache = K.KVCache(w.kvq_config())
    cache.prefill(inp.k, inp.v)
    splits = 100                     # 8 x 32 x 101 partials of 130 floats > 8 MiB
    assert K.kvq_decode_workspace_size(cache.handle, splits) > K.KVQ_NOALLOC_SCRATCH_BYTES
    with pytest.raises(K.KVQError) as e:
        noalloc(cache, inp.q[0], num_splits=splits)
    assert e.value.code == K.KVQ_ERR_WORKSPACE
    ref = cache.decode(inp.q[0], num_splits=splits)
    assert rel_err(noalloc(cache, inp.q[0]), ref) <= TOL


def test_noalloc_shrinks_the_automatic_split_count_to_fit():
    """A cache whose automatic plan needs more than the scratch array: 32 sequences of
    8192 tokens with 64 query heads (2048 partial rows of d_v + 2 floats per split)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.WORKLOADS["gqa4k"].with_(batch=32, context=8192, n_q_heads=64, appends=1, seed=306)
    inp = W.Inputs(w, device="cuda")
    cache = K.KVCache(w.kvq_config())
    cache.prefill(inp.k, inp.v)
    del inp.k, inp.v
    cache.append(inp.k_app[0], inp.v_app[0])
    assert K.kvq_decode_workspace_size(cache.handle, 0) > K.KVQ_NOALLOC_SCRATCH_BYTES
    auto = cache.plan()
    # the largest split count whose partials fit, as the entry point chooses it
    fits = [s for s in range(1, auto["splits_quant"])
            if K.kvq_decode_workspace_size(cache.handle, s) <= K.KVQ_NOALLOC_SCRATCH_BYTES]
    assert fits, "no split count fits the scratch array"
    ref = cache.decode(inp.q[0], num_splits=max(fits))
    torch.cuda.synchronize()
    for _ in range(2):
        out = noalloc(cache, inp.q[0])
        assert rel_err(out, ref) <= TOL
        assert torch.equal(out, ref)        # same kernels, same split count: same bits


def test_noalloc_status_reports_a_wait_that_gave_up():
    """The test hook makes one copy stage of the next decode ask for 16 bytes more than it
    receives, so that CTA's bounded waits give up after 1 s: the scratch array's status word
    must then carry KVQ_STATUS_TIMEOUT, and after a reset the next call is clean and correct."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.WORKLOADS["gqa4k"].with_(batch=2, context=1024, appends=0, seed=307)
    inp = W.Inputs(w, device="cuda")
    cache = K.KVCache(w.kvq_config())
    cache.prefill(inp.k, inp.v)
    assert cache.plan()["fast_path"] == 1
    ref = cache.decode(inp.q[0])
    s = K._stream()
    K.kvq_noalloc_reset_status(s)
    assert rel_err(noalloc(cache, inp.q[0]), ref) <= TOL
    assert K.kvq_noalloc_read_status(s) == 0
    K.kvq_debug_stall_next_decode(cache.handle)
    t0 = time.time()
    noalloc(cache, inp.q[0])
    assert K.kvq_noalloc_read_status(s) & K.KVQ_STATUS_TIMEOUT
    assert time.time() - t0 < 30
    noalloc(cache, inp.q[0])                 # a decode never clears the word
    assert K.kvq_noalloc_read_status(s) & K.KVQ_STATUS_TIMEOUT
    K.kvq_noalloc_reset_status(s)
    out = noalloc(cache, inp.q[0])
    assert K.kvq_noalloc_read_status(s) == 0
    assert rel_err(out, ref) <= TOL
