"""Oracle side of the full-size 131072-token sweep test, run in spawned worker processes.

One job = one sequence of one precision: the oracle cache of that sequence alone is prefilled,
appended to step by step, and at the checked steps it reports a SHA-256 digest of every valid
byte of its state (codes, (scale, zero), window slots, retained copies) and its decode output.
The worker imports numpy and the oracle only (no torch, no CUDA), and reads its inputs from
.npy files the test wrote, so nothing large crosses the process pipe.
"""
from __future__ import annotations

import hashlib
import os

import numpy as np


def state_digests(oc, b: int) -> dict:
    """SHA-256 of the valid bytes of sequence b's cache state (the oracle's buffer layout)."""
    out = {"L": oc.L, "Q": oc.Q, "ret": list(oc.ret_idx)}
    Q, L = oc.Q, oc.L
    names = []
    if oc.kb != 16 and Q:
        gk = oc.gk
        names += [("kcode", slice(0, Q)), ("ksz", slice(0, Q // gk)), ("vcode", slice(0, Q)),
                  ("vsz", slice(0, Q))]
    for name, sl in names:
        a = np.ascontiguousarray(getattr(oc, name)[b, :, sl])
        out[name] = hashlib.sha256(a.view(np.uint8)).hexdigest()
    slots = [p % oc.cap for p in range(Q, L)]
    for name in ("win_k", "win_v"):
        a = np.ascontiguousarray(getattr(oc, name)[b][:, slots])
        out[name] = hashlib.sha256(a.view(np.uint8)).hexdigest()
    if oc.ret_idx:
        n = len(oc.ret_idx)
        for name in ("ret_k", "ret_v"):
            a = np.ascontiguousarray(getattr(oc, name)[b, :, :n])
            out[name] = hashlib.sha256(a.view(np.uint8)).hexdigest()
    return out


def run_job(job: dict) -> dict:
    """job: cfg (batch 1), the .npy directory, the precision tag, the sequence b and the checked
    steps.  Returns {step: (digests, decode output [1][Hq][d_v] fp64)}."""
    import threadpoolctl
    from oracle import kvq_oracle as O

    with threadpoolctl.threadpool_limits(1):
        d = job["dir"]
        b = job["b"]
        k = np.load(os.path.join(d, f"k_{b}.npy"))[None]
        v = np.load(os.path.join(d, f"v_{b}.npy"))[None]
        k_app = np.load(os.path.join(d, f"k_app_{b}.npy"))       # [steps][Hkv][d_k]
        v_app = np.load(os.path.join(d, f"v_app_{b}.npy"))
        q = np.load(os.path.join(d, f"q_{b}.npy"))               # [steps][Hq][d_k]
        oc = O.OracleCache(job["cfg"])
        oc.prefill(k, v)
        del k, v
        res = {}
        last = max(job["steps"])
        for i in range(last + 1):
            oc.append(k_app[i][None], v_app[i][None])
            if i in job["steps"]:
                res[i] = (state_digests(oc, 0), oc.decode(q[i][None]))
        return res
