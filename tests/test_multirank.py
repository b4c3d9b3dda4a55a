"""The multi-GPU path on CPU: world size 2 over gloo.

Every (b, kv head) of the cache is an independent unit, so ranks decode their own
batches with no collective on the data path; the only collectives are the barrier
and the max over ranks of the timings.  These tests run that host logic with the
CPU oracle standing in for the device.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from oracle import kvq_oracle as O
from mixed_precision_quantized_pack_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        base = W.WORKLOADS["tiny"].with_(batch=2, n_q_heads=4, n_kv_heads=2, context=300)
        w = bench.rank_workload(base, rank, steps=2)
        inp = W.Inputs(w)
        oc = O.OracleCache(w.kvq_config())
        oc.prefill(inp.k.numpy(), inp.v.numpy())
        outs = []
        for i in range(2):
            oc.append(inp.k_app[i].numpy(), inp.v_app[i].numpy())
            outs.append(oc.decode(inp.q[i].numpy()))
        fake_ms = [10.0 + rank, 3.0 * (world - rank)]
        red = bench.max_over_ranks(fake_ms, dist)
        np.save(os.path.join(outdir, f"out{rank}.npy"), np.stack(outs))
        np.save(os.path.join(outdir, f"k{rank}.npy"), inp.k.numpy())
        np.save(os.path.join(outdir, f"red{rank}.npy"), np.array(red))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_decode_independent_batches(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    k0, k1 = np.load(tmp_path / "k0.npy"), np.load(tmp_path / "k1.npy")
    assert k0.shape == k1.shape and not np.array_equal(k0, k1)        # own sequences
    red = [np.load(tmp_path / f"red{r}.npy") for r in range(world)]
    assert np.array_equal(red[0], red[1]) and list(red[0]) == [11.0, 6.0]
    # a rank's result equals what a single process computes for that rank's batch
    base = W.WORKLOADS["tiny"].with_(batch=2, n_q_heads=4, n_kv_heads=2, context=300)
    for r in range(world):
        w = bench.rank_workload(base, r, steps=2)
        inp = W.Inputs(w)
        oc = O.OracleCache(w.kvq_config())
        oc.prefill(inp.k.numpy(), inp.v.numpy())
        for i in range(2):
            oc.append(inp.k_app[i].numpy(), inp.v_app[i].numpy())
            ref = oc.decode(inp.q[i].numpy())
            assert np.array_equal(np.load(tmp_path / f"out{r}.npy")[i], ref)


def test_sharding_the_batch_does_not_change_results():
    # weak scaling splits sequences over ranks: decoding rows [0,1) and [1,2) separately
    # equals decoding the batch of two
    w = W.WORKLOADS["tiny"].with_(batch=2, n_q_heads=4, n_kv_heads=2, context=260)
    inp = W.Inputs(w)
    full = O.OracleCache(w.kvq_config())
    full.prefill(inp.k.numpy(), inp.v.numpy())
    ref = full.decode(inp.q[0].numpy())
    for b in range(2):
        one = O.OracleCache(dict(w.kvq_config(), batch=1))
        one.prefill(inp.k.numpy()[b:b + 1], inp.v.numpy()[b:b + 1])
        assert np.array_equal(one.decode(inp.q[0].numpy()[b:b + 1])[0], ref[b])
