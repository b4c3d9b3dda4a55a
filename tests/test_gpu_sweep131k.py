"""The 131072-token sweep at full size, every precision, against the CPU oracle.

32 query / 8 kv heads, d = 128, groups of 64, window 128; 64 sequences of 131072 tokens are
prefilled on the GPU and then take 256 append + decode steps.  For two sampled sequences (the
first and the last) the oracle builds the cache of that sequence alone, in spawned worker
processes while the GPU runs, and at steps 0, 1, 63, 64, 65 and 255 (they include the appends
that quantize a window group: a group of 64 spills every 64 steps) the sequence's packed codes,
(scale, zero) pairs and window slots must equal the oracle's byte for byte (compared through
SHA-256 digests of every valid byte) and its attention output must lie within 2e-3 of the
oracle's fp64 result.  Precisions: K8V4, K4V2, K2V2 and the unquantized fp16 cache ("Quantize
What Counts: More for Keys, Less for Values", §La Solution and §Sensibilité à la Taille de
Groupe; "LogQuant", §5 Implémentation for 2-bit).
"""
import hashlib
import multiprocessing as mp
import os
import tempfile

import numpy as np
import pytest
import torch

from oracle import kvq_oracle as O
from mixed_precision_quantized_pack_b200 import kvq as K
from mixed_precision_quantized_pack_b200 import workloads as W

import sweep_oracle_jobs as J

pytestmark = pytest.mark.gpu
TOL = 2e-3
BATCH = 64
STEPS = (0, 1, 63, 64, 65, 255)
ROWS = (0, BATCH - 1)


def gpu_digests(gc: K.KVCache, b: int) -> dict:
    """The same digests as the oracle's, over the GPU cache's bytes of sequence b."""
    L, Q, ret = gc.state()
    out = {"L": L, "Q": Q, "ret": list(ret)}
    c = gc.cfg
    if c["k_bits"] != 16 and Q:
        gk = c["group_k"]
        for name, sl in (("kcode", slice(0, Q)), ("ksz", slice(0, Q // gk)),
                         ("vcode", slice(0, Q)), ("vsz", slice(0, Q))):
            a = np.ascontiguousarray(gc.view(name)[b, :, sl].cpu().numpy())
            out[name] = hashlib.sha256(a.view(np.uint8)).hexdigest()
    cap = gc.view("win_k").shape[2]
    slots = torch.tensor([p % cap for p in range(Q, L)], device="cuda")
    for name in ("win_k", "win_v"):
        a = np.ascontiguousarray(gc.view(name)[b].index_select(1, slots).cpu().numpy())
        out[name] = hashlib.sha256(a.view(np.uint8)).hexdigest()
    return out


def test_sweep_131k_full_size_every_precision():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    n_steps = max(STEPS) + 1
    base = W.sweep_workload(BATCH, 4, 2, appends=n_steps)
    inp = W.Inputs(base, device="cuda")          # the same draws serve every precision
    precisions = [(8, 4), (4, 2), (2, 2), (16, 16)]
    with tempfile.TemporaryDirectory() as tmp:
        for b in ROWS:
            np.save(os.path.join(tmp, f"k_{b}.npy"), inp.k[b].cpu().numpy())
            np.save(os.path.join(tmp, f"v_{b}.npy"), inp.v[b].cpu().numpy())
            np.save(os.path.join(tmp, f"k_app_{b}.npy"), torch.stack([x[b] for x in inp.k_app]).cpu().numpy())
            np.save(os.path.join(tmp, f"v_app_{b}.npy"), torch.stack([x[b] for x in inp.v_app]).cpu().numpy())
            np.save(os.path.join(tmp, f"q_{b}.npy"), torch.stack([x[b] for x in inp.q]).cpu().numpy())
        jobs, keys = [], []
        for kb, vb in precisions:
            w = base.with_(k_bits=kb, v_bits=vb)
            for b in ROWS:
                jobs.append({"cfg": dict(w.kvq_config(), batch=1), "dir": tmp, "b": b,
                             "steps": set(STEPS)})
                keys.append((kb, vb, b))
        workers = max(1, min(len(jobs), os.cpu_count() or 1))
        with mp.get_context("spawn").Pool(workers) as pool:
            pending = pool.map_async(J.run_job, jobs, chunksize=1)
            gpu = {}
            for kb, vb in precisions:
                w = base.with_(k_bits=kb, v_bits=vb)
                gc = K.KVCache(w.kvq_config())
                gc.prefill(inp.k, inp.v)
                for i in range(n_steps):
                    gc.append(inp.k_app[i], inp.v_app[i])
                    if i not in STEPS:
                        gc.decode(inp.q[i])
                        continue
                    out = gc.decode(inp.q[i]).float().cpu().numpy()
                    for b in ROWS:
                        gpu[(kb, vb, b, i)] = (gpu_digests(gc, b), out[b:b + 1])
                assert gc.status() == 0
                plan = gc.plan()
                assert plan["fast_path"] == 1
                # past 65536 quantized tokens the tensor-core kernel centres the value codes
                assert plan["centered"] == (1 if kb != 16 else 0)
                del gc
                torch.cuda.empty_cache()
            results = pending.get(timeout=1500)
    worst = {}
    for (kb, vb, b), res in zip(keys, results):
        for i in STEPS:
            o_dig, o_out = res[i]
            g_dig, g_out = gpu[(kb, vb, b, i)]
            where = f"K{kb}V{vb} b={b} step {i}"
            assert (g_dig["L"], g_dig["Q"], g_dig["ret"]) == (o_dig["L"], o_dig["Q"], o_dig["ret"]), where
            for name in o_dig:
                if name not in ("L", "Q", "ret"):
                    assert g_dig.get(name) == o_dig[name], f"{where}: {name} differs from the oracle"
            err = O.max_rel_error(g_out, o_out)
            worst[(kb, vb)] = max(worst.get((kb, vb), 0.0), err)
            assert err <= TOL, f"{where}: max relative error {err:.3e}"
    print("worst max relative error per precision:",
          {f"K{kb}V{vb}": f"{e:.3e}" for (kb, vb), e in worst.items()})
