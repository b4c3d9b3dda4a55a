"""Decode-attention throughput over a packed mixed-precision KV cache on B200.

One step = one generation step of every sequence in the batch: append the new
token's K/V (window write; every group_k steps the oldest window group is
quantized and the retained set updated) and decode attention of one query token
per query head over the whole cache (split-K decode kernel + log-sum-exp combine).
The default workload is the 32k long-context case: batch 32, 32 query / 8 KV heads,
d = 128, K4/V2 with groups of 64, fp16 window 128, log-spaced retention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs its own
batch (weak scaling, no collective on the data path); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import re
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixed_precision_quantized_pack_b200 import kvq as K  # noqa: E402
from mixed_precision_quantized_pack_b200 import workloads as W  # noqa: E402

METRIC = "decode attn tokens/s and achieved HBM GB/s over packed KV (K4V2, ctx 32k)"
UNIT = "tokens/s"
def profile_summary(workload_key: str) -> str:
    """The committed ncu summary of the decode kernel on a workload."""
    return os.path.join(ROOT, "profiles", f"decode_{workload_key}_ncu.md")


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def decode_bytes(cfg: dict, L: int) -> int:
    """Algorithmic bytes one decode reads: packed codes and (scale, zero) of the quantized
    tokens (retained slots included), fp16 window and retained tokens, q, and (paged caches)
    the block-table entries of the quantized groups."""
    B, H, dk, dv = cfg["batch"], cfg["n_kv_heads"], cfg["d_k"], cfg["d_v"]
    kb, vb, gk, gv, R = cfg["k_bits"], cfg["v_bits"], cfg["group_k"], cfg["group_v"], cfg["window"]
    if kb == 16:
        return B * H * L * (dk + dv) * 2 + B * cfg["n_q_heads"] * dk * 2
    Q = max(L - R, 0) // gk * gk
    nret = len(K.kvq_retained_positions(Q)) if cfg["log_retain"] else 0
    sr, sq = cfg.get("side_rank", 0), cfg.get("side_bits", 0)
    if kb == 0:       # per-channel widths: rows of max(1, ceil(bits / 32)) words
        kbytes = 4 * max(1, -(-sum(cfg["k_widths"][:dk]) // 32))
        vbytes = 4 * max(1, -(-sum(cfg["v_widths"][:dv]) // 32))
    else:
        kbytes, vbytes = dk * kb // 8, dv * vb // 8
    per_tok = kbytes + vbytes + (dv // gv) * 4 + sr * sq // 8
    quant = Q * per_tok + (Q // gk) * (dk * 4 + sr * 4)
    fp16 = (L - Q + nret) * (dk + dv) * 2
    table = B * (Q // gk) * 4 if cfg.get("paged") else 0
    return B * H * (quant + fp16) + B * cfg["n_q_heads"] * dk * 2 + table


CLOCK_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


def _clock_sampler_main(uuid, index, conn, stop):
    """Child process: poll the SM clock and the clock-event reasons every 0.5 ms (read-only
    NVML queries) until `stop` is set, then send [(monotonic time, MHz, reasons)] and the
    maximum SM clock back through `conn`."""
    samples, max_mhz = [], None
    try:
        import pynvml as nv
        nv.nvmlInit()
        try:
            h = nv.nvmlDeviceGetHandleByUUID(uuid)
        except Exception:
            h = nv.nvmlDeviceGetHandleByIndex(index)
        max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        conn.send("ready")
        while not stop.is_set():         # back-to-back queries (each takes a fraction of a ms)
            samples.append((time.monotonic(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                            get_reasons(h) if get_reasons else 0))
    except Exception:
        conn.send("ready")
    conn.send((samples, max_mhz))


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled by a separate process (so that it
    never competes with the launching thread for the interpreter) every ~0.5 ms; the samples
    kept are those taken between mark_start() and mark_end(), the host-side window in which
    the GPU ran the timed steps."""

    def __init__(self, device_index: int):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            uuid = ""
        self.conn, child = ctx.Pipe()
        self.stop_evt = ctx.Event()
        self.proc = ctx.Process(target=_clock_sampler_main,
                                args=(uuid, device_index, child, self.stop_evt), daemon=True)
        self.proc.start()
        self.ready = self.conn.poll(60) and self.conn.recv() == "ready"
        self.t_start = self.t_end = None

    def mark_start(self):
        self.t_start = time.monotonic()

    def mark_end(self):
        self.t_end = time.monotonic()

    def stop(self):
        self.stop_evt.set()
        samples, max_mhz = self.conn.recv() if self.conn.poll(10) else ([], None)
        self.proc.join(timeout=5)
        window = "timed region"
        if self.t_start is not None and self.t_end is not None:
            inside = [x for x in samples if self.t_start <= x[0] <= self.t_end]
            if not inside:
                # a short timed region can fall between two queries: take those within 100 ms of
                # it (the warm-up and the following steps run the same kernels)
                inside = [x for x in samples if self.t_start - 0.1 <= x[0] <= self.t_end + 0.1]
                window = "within 100 ms of the timed region"
            samples = inside
        if not samples:
            return None
        reasons = set()
        for _, _, r in samples:
            for bit, name in CLOCK_REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for _, m, _ in samples), "sm_max_mhz": max_mhz,
                "reasons": sorted(reasons), "samples": len(samples),
                "source": "nvml, separate process", "window": window}


def profile_traffic(workload_key: str):
    """dram bytes per decode launch from the committed ncu summary of the workload, if it was
    taken on the current kernel source (else None)."""
    try:
        text = open(profile_summary(workload_key)).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"decode_source_sha256:\s*([0-9a-f]+)", text)
    f = re.search(r"decode_source:\s*([\w.]+)", text)
    if not m or not h:
        return None
    import hashlib
    src = os.path.join(ROOT, "mixed_precision_quantized_pack_b200", "csrc", f.group(1) if f else "decode_mma.cuh")
    try:
        cur = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    return float(m.group(1)) if cur.startswith(h.group(1)) else None


# ------------------------------------------------------------------ ranks ---------
def rank_workload(w: W.Workload, rank: int, steps: int) -> W.Workload:
    """The batch a rank decodes: same shapes, its own seed (independent sequences)."""
    return w.with_(appends=steps, seed=w.seed + 7919 * rank)


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a group)."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


# ------------------------------------------------------------------ CPU oracle ----
def oracle_decode_sample(w: W.Workload, budget_s: float, steps: int = 1):
    """Times the CPU oracle's append+decode on whole sequences of the workload until
    about budget_s seconds of decode work; returns (tokens/s, seconds, sequences, threads)."""
    from oracle import kvq_oracle as O
    import threadpoolctl
    inp = W.Inputs(w.with_(batch=1, appends=max(steps, 1)), device="cpu")
    oc = O.OracleCache(dict(w.kvq_config(max_context=w.context + steps + 64), batch=1),
                       side_basis=None if inp.side_basis is None else inp.side_basis.numpy())
    oc.prefill(inp.k.numpy(), inp.v.numpy())
    spent, done = 0.0, 0
    for i in range(steps):
        t0 = time.perf_counter()
        oc.append(inp.k_app[i].numpy(), inp.v_app[i].numpy())
        oc.decode(inp.q[i].numpy())
        spent += time.perf_counter() - t0
        done += 1
        if spent >= budget_s:
            break
    threads = max([x.get("num_threads", 1) for x in threadpoolctl.threadpool_info()] or [1])
    return done / spent, spent, done, threads


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    times = []
    import threadpoolctl
    from oracle import kvq_oracle as O
    steps = args.steps + args.warmup
    inp = W.Inputs(w.with_(batch=1, appends=steps), device="cpu")
    oc = O.OracleCache(dict(w.kvq_config(max_context=w.context + steps + 64), batch=1),
                       side_basis=None if inp.side_basis is None else inp.side_basis.numpy())
    oc.prefill(inp.k.numpy(), inp.v.numpy())
    for i in range(steps):
        t0 = time.perf_counter()
        oc.append(inp.k_app[i].numpy(), inp.v_app[i].numpy())
        oc.decode(inp.q[i].numpy())
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    t = sum(times) / len(times)
    value = 1.0 / t          # one sequence's token per step, same workload
    threads = max([x.get("num_threads", 1) for x in threadpoolctl.threadpool_info()] or [1])
    sample = (f"CPU oracle (numpy, fp64 attention) append+decode of 1 of {w.batch} sequences "
              f"(all {w.n_kv_heads} kv heads) per step at context {w.context}")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------ GPU arm -------
def step_plan(cfg: dict, L0: int, first: int, count: int):
    """Per append+decode step i in [first, first+count): (algorithmic bytes of its decode,
    launches of this library's kernels), computed on the host before anything is timed."""
    gk, R = cfg["group_k"], cfg["window"]

    def q_of(L):          # quantized prefix after L tokens (the window rule of the cache)
        return 0 if cfg["k_bits"] == 16 else max(L - R, 0) // gk * gk

    out = []
    for i in range(first, first + count):
        L = L0 + i + 1
        # append (one copy kernel for K and V; rotated keys take a second one), decode, combine
        n = (2 if cfg.get("rot_keys") else 1) + 2
        if q_of(L) != q_of(L - 1):
            # a window group was quantized: keys, values, side code, retained set, and (paged)
            # the new page's block-table entries
            n += 2 + (1 if cfg.get("side_rank") else 0) + (1 if cfg["log_retain"] else 0)
            n += 1 if cfg.get("paged") else 0
        out.append((decode_bytes(cfg, L), n))
    return out


def prefill_bytes(cfg: dict, L: int) -> int:
    """Algorithmic bytes of a prefill of L tokens per sequence: every input key and value
    read once; codes, (scale, zero), side codes, the fp16 window and the retained copies
    written once (and, paged, the block-table entries)."""
    B, H, dk, dv = cfg["batch"], cfg["n_kv_heads"], cfg["d_k"], cfg["d_v"]
    kb, gk, gv, R = cfg["k_bits"], cfg["group_k"], cfg["group_v"], cfg["window"]
    read = B * H * L * (dk + dv) * 2
    if kb == 16:
        return read + B * H * L * (dk + dv) * 2
    Q = max(L - R, 0) // gk * gk
    nret = len(K.kvq_retained_positions(Q)) if cfg["log_retain"] else 0
    sr, sq = cfg.get("side_rank", 0), cfg.get("side_bits", 0)
    if kb == 0:
        kbytes = 4 * max(1, -(-sum(cfg["k_widths"][:dk]) // 32))
        vbytes = 4 * max(1, -(-sum(cfg["v_widths"][:dv]) // 32))
    else:
        kbytes, vbytes = dk * kb // 8, dv * cfg["v_bits"] // 8
    per_tok = kbytes + vbytes + (dv // gv) * 4 + sr * sq // 8
    written = Q * per_tok + (Q // gk) * (dk * 4 + sr * 4) + (L - Q + nret) * (dk + dv) * 2
    table = B * (Q // gk) * 4 if cfg.get("paged") else 0
    return read + B * H * written + table


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default="long32k", choices=W.ALL_KEYS)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    args = ap.parse_args()
    w = W.by_key(args.workload)
    if args.batch:
        w = w.with_(batch=args.batch)
    if args.impl == "reference":
        return run_reference(args, w)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    steps, warm = args.steps, max(args.warmup, 3)
    wl = rank_workload(w, rank, steps + warm)
    cfg = wl.kvq_config(max_context=wl.context + steps + warm + 64)
    inp = W.Inputs(wl, device=dev)
    cache = K.KVCache(cfg, device=dev, side_basis=inp.side_basis)
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = peaks()

    # prefill: three calls on the same inputs (each one resets the cache), median of the
    # last two; the first is reported as well
    torch.cuda.synchronize(dev)
    pre_ms = []
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cache.prefill(inp.k, inp.v)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        pre_ms.append(e0.elapsed_time(e1))
    pre_bytes = prefill_bytes(cfg, wl.context)
    pre_med = statistics.median(pre_ms[1:])
    del inp.k, inp.v
    torch.cuda.empty_cache()

    out = torch.empty((wl.batch, wl.n_q_heads, wl.d_v), dtype=torch.float16, device=dev)
    n_ev = steps + warm
    step_start = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    L0, _, _ = cache.state()
    plan_steps = step_plan(cfg, L0, warm, steps)
    bytes_read = [b for b, _ in plan_steps]
    launches = sum(n for _, n in plan_steps)

    # a decode whose bytes are not well above the L2 size would find part of them in L2 at
    # the next step: then L2 is flushed (a write of twice its size) before every step,
    # outside the step's events, and the step time is the mean of the steps' own events
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20) or (126 << 20))
    flush = bytes_read[0] < 4 * l2
    flush_buf = torch.empty(2 * l2, dtype=torch.uint8, device=dev) if flush else None

    def step(i):
        if flush:
            flush_buf.zero_()
        step_start[i].record(stream)
        cache.append(inp.k_app[i], inp.v_app[i])
        starts[i].record(stream)
        cache.decode(inp.q[i], out=out)
        ends[i].record(stream)

    for i in range(warm):
        step(i)
    clocks = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(warm, warm + steps):
        step(i)
    t1.record(stream)
    while not t1.query():
        time.sleep(0.0002)
    clocks.mark_end()
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    clk = clocks.stop()
    region_ms = t0.elapsed_time(t1)
    step_ms = [step_start[i].elapsed_time(ends[i]) for i in range(warm, warm + steps)]
    dec_ms = [starts[i].elapsed_time(ends[i]) for i in range(warm, warm + steps)]
    total_ms = sum(step_ms) if flush else region_ms
    dec_avg = sum(dec_ms) / len(dec_ms)
    dec_med = statistics.median(dec_ms)
    status = cache.status()
    total_ms, dec_avg, dec_med = max_over_ranks([total_ms, dec_avg, dec_med], dist, dev)
    ms_step = total_ms / steps
    value = world * wl.batch / (ms_step / 1e3)
    achieved = (sum(bytes_read) / len(bytes_read)) / (dec_avg / 1e3) / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = e2e_leg(wl, cfg, inp, out, steps, dev, stream, dist, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, spent, seqs, threads = oracle_decode_sample(w, args.cpu_budget, steps=8)
        cpu = {"value": v_cpu, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{seqs} append+decode steps of 1 of {w.batch} sequences "
                         f"(all {w.n_kv_heads} kv heads, context {w.context}) in {spent:.1f} s"}

    if rank == 0:
        plan = cache.plan()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": warm, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded; keys N(0,1)*sigma_c+mu_c with log-uniform sigma, values/q N(0,1))",
            "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "n_q_heads": wl.n_q_heads,
                       "n_kv_heads": wl.n_kv_heads, "d_k": wl.d_k, "d_v": wl.d_v,
                       "context": wl.context, "k_bits": wl.k_bits, "v_bits": wl.v_bits,
                       "group_k": wl.group_k, "group_v": wl.group_v, "window": wl.window,
                       "log_retain": wl.log_retain, "parallelism": f"dp{world} (independent batches)",
                       "l2": ("flushed before every step (write of %d MB, outside the step's events); "
                              "each decode reads %.1f MB" % (2 * l2 >> 20, bytes_read[0] / 1e6)) if flush
                             else "no flush: each decode reads %.0f MB > 4 x L2" % (bytes_read[0] / 1e6),
                       "timing": "mean of the steps' own events" if flush
                                 else "events around the whole timed region",
                       "step": "append 1 token + decode, per sequence",
                       "plan": plan},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak,
                         "traffic": None if args.batch else profile_traffic(args.workload),
                         "peak_kind": f"{peak_kind} HBM copy bandwidth",
                         "kernel": "decode (split-K kernel + combine), CUDA events per launch",
                         "decode_ms": dec_avg, "decode_ms_median": dec_med,
                         "bytes_per_launch": bytes_read[0]},
            "decode_tokens_per_s": world * wl.batch / (dec_avg / 1e3),
            "prefill": {"ms": pre_med, "ms_first_call": pre_ms[0], "tokens": wl.batch * wl.context,
                        "bytes": pre_bytes, "achieved_gbs": pre_bytes / (pre_med / 1e3) / 1e9,
                        "frac": pre_bytes / (pre_med / 1e3) / 1e9 / peak,
                        "note": "algorithmic bytes: K and V read once, cache written once; "
                                "median of calls 2 and 3"},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    del cache
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def e2e_leg(wl, cfg, inp, out, steps, dev, stream, dist, world):
    """End to end through the public API: every step copies its inputs from pinned host memory
    and its output back to pinned host memory.  The copies run on two copy streams with
    double-buffered device tensors, so step i's input copy overlaps step i-1's decode and step
    i's output copy overlaps step i+1's; every copy still lies inside the timed region."""
    h_q = [x.cpu().pin_memory() for x in inp.q[:steps]]
    h_k = [x.cpu().pin_memory() for x in inp.k_app[:steps]]
    h_v = [x.cpu().pin_memory() for x in inp.v_app[:steps]]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    d_q = [torch.empty_like(inp.q[0]) for _ in range(2)]
    d_k = [torch.empty_like(inp.k_app[0]) for _ in range(2)]
    d_v = [torch.empty_like(inp.v_app[0]) for _ in range(2)]
    d_out = [torch.empty_like(out) for _ in range(2)]
    inp2 = W.Inputs(wl.with_(appends=1), device=dev)
    e2e_cache = K.KVCache(cfg, device=dev, side_basis=inp2.side_basis)
    e2e_cache.prefill(inp2.k, inp2.v)
    del inp2
    torch.cuda.empty_cache()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]       # inputs of the slot uploaded
    ev_used = [torch.cuda.Event() for _ in range(2)]     # decode done with the slot
    ev_down = [torch.cuda.Event() for _ in range(2)]     # output of the slot downloaded
    for e in ev_used + ev_down:
        e.record(stream)

    def e2e_step(i):
        j = i % 2
        s_in.wait_event(ev_used[j])
        with torch.cuda.stream(s_in):
            d_q[j].copy_(h_q[i], non_blocking=True)
            d_k[j].copy_(h_k[i], non_blocking=True)
            d_v[j].copy_(h_v[i], non_blocking=True)
        ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        stream.wait_event(ev_down[j])
        e2e_cache.append(d_k[j], d_v[j])
        e2e_cache.decode(d_q[j], out=d_out[j])
        ev_used[j].record(stream)
        s_out.wait_event(ev_used[j])
        with torch.cuda.stream(s_out):
            h_out[j].copy_(d_out[j], non_blocking=True)
        ev_down[j].record(s_out)

    for i in range(3):
        e2e_step(i)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = min(steps, len(h_q)) - 3
    a.record(stream)
    s_in.wait_event(a)
    s_out.wait_event(a)
    for i in range(3, 3 + n_e2e):
        e2e_step(i)
    for e in ev_down:
        stream.wait_event(e)
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = a.elapsed_time(b) / max(n_e2e, 1)
    (e2e_ms,) = max_over_ranks([e2e_ms], dist, dev)
    h2d = (d_q[0].numel() + d_k[0].numel() + d_v[0].numel()) * 2
    d2h = out.numel() * 2
    del e2e_cache
    torch.cuda.empty_cache()
    return {"value": world * wl.batch / (e2e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "copies": "pinned host <-> device every step, on two copy streams that "
                      "overlap the neighbouring steps' decodes"}


if __name__ == "__main__":
    main()
