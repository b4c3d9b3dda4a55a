"""Workload shapes and seeded synthetic inputs for packed KV-cache decode attention.

This module only draws random numbers; it holds none of the method's arithmetic
(no quantization, packing, retention or attention).  Both the CUDA path and the
CPU oracle are fed from here, so that they see the very same fp16 tensors.

Distributions (the workloads of "Quantize What Counts: More for Keys, Less for
Values", §Méthodologie, are real model caches we do not have; these synthetic
stand-ins keep the property the pages stress: keys carry per-channel outliers,
values do not):

* keys   k[b,h,t,c] = N(0,1) * sigma[h,c] + mu[h,c], with sigma log-uniform on
  [0.5, 8] and mu ~ N(0, variance 2), both drawn per (kv head, channel) and
  shared by every sequence and token;
* values and queries ~ N(0, 1);
* thin keys ("Thin Keys, Full Values", §2): 128-dim keys drawn as above and
  projected to d_k dims by P with N(0, std 1/sqrt(128)) entries, in fp32;
* side-code workloads ("HeadQ", §3): per kv head a basis U_h, the orthonormal
  factor of a Gaussian d_k x r matrix, standing in for the PCA basis of calibration
  queries; their queries put a fraction f of their energy in span(U_h):
  q = sqrt(1-f) n + sqrt(f d_k / r) U_h a with n, a ~ N(0, I), so |q|^2 ~ d_k as
  for plain queries.

Everything is drawn in fp32 from one ``torch.Generator`` seeded per workload and
rounded once to fp16.  The generator lives on the device the tensors are made on,
so a CPU and a CUDA draw of the same seed differ; each test or benchmark uses
one of them and copies across as needed.  Workloads with ``per_seq`` set (the
131072-token sweep) draw each sequence's prefill keys and values from a
generator of its own, seeded with (seed, b), so a batch of 64 such sequences
is made one sequence at a time and any one sequence can be drawn alone.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    d_k: int
    d_v: int
    context: int          # tokens written by the prefill
    k_bits: int
    v_bits: int
    group_k: int          # tokens per key group
    group_v: int          # channels per value group
    window: int           # R, the fp16 recent window
    log_retain: int
    appends: int          # append+decode steps after the prefill (0: one decode only)
    thin_from: int = 0    # >0: keys are a projection of thin_from-dim keys
    seed: int = 0
    side_rank: int = 0    # >0: a side code of this rank ...
    side_bits: int = 0    # ... and bits per code
    q_in_basis: float = 0.0   # side workloads: fraction of query energy in span(U_h)
    rot_keys: int = 0     # key-only rotation, with signs drawn from rot_seed
    rot_seed: int = 0
    paged: int = 0        # quantized groups in a page pool just large enough for max_context
    k_widths: tuple = ()  # k_bits = v_bits = 0: per-channel key widths ...
    v_widths: tuple = ()  # ... and value widths (data, given with the workload)
    per_seq: int = 0      # 1: prefill K/V drawn per sequence from generators seeded (seed, b)

    @property
    def n_rep(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def max_context(self) -> int:
        return self.context + max(self.appends, 1) + 64

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def kvq_config(self, max_context: Optional[int] = None) -> dict:
        mc = max_context if max_context is not None else self.max_context
        return dict(batch=self.batch, n_q_heads=self.n_q_heads, n_kv_heads=self.n_kv_heads,
                    d_k=self.d_k, d_v=self.d_v, k_bits=self.k_bits, v_bits=self.v_bits,
                    group_k=self.group_k, group_v=self.group_v, window=self.window,
                    log_retain=self.log_retain, max_context=mc,
                    side_rank=self.side_rank, side_bits=self.side_bits, rot_keys=self.rot_keys,
                    rot_signs=rotation_signs(self.rot_seed) if self.rot_keys else [0] * 8,
                    paged=self.paged,
                    n_pages=self.batch * -(-mc // self.group_k) if self.paged else 0,
                    k_widths=list(self.k_widths), v_widths=list(self.v_widths))


def rotation_signs(seed: int) -> List[int]:
    """Eight random 32-bit words (the rotation's sign bits), from their own seeded generator."""
    gen = torch.Generator()
    gen.manual_seed(seed)
    return [int(x) for x in torch.randint(0, 2 ** 32, (8,), generator=gen, dtype=torch.int64)]


def _base(**kw) -> Workload:
    return Workload(**kw)


# The five workloads named with the metric.  Shapes, bit widths, group sizes and
# windows as stated there; seeds are 1000 + index.
WORKLOADS: Dict[str, Workload] = {
    "tiny": _base(name="tiny-1h-512", batch=1, n_q_heads=1, n_kv_heads=1, d_k=128, d_v=128,
                  context=512, k_bits=4, v_bits=2, group_k=32, group_v=32, window=64,
                  log_retain=0, appends=0, seed=1000),
    "gqa4k": _base(name="gqa-b8-32/8-4k-k4v2", batch=8, n_q_heads=32, n_kv_heads=8, d_k=128,
                   d_v=128, context=4096, k_bits=4, v_bits=2, group_k=64, group_v=64,
                   window=128, log_retain=0, appends=1, seed=1001),
    "long32k": _base(name="long-b32-32/8-32k-k4v2-logretain", batch=32, n_q_heads=32,
                     n_kv_heads=8, d_k=128, d_v=128, context=32768, k_bits=4, v_bits=2,
                     group_k=64, group_v=64, window=128, log_retain=1, appends=0, seed=1002),
    "thin16k": _base(name="thin-b16-32/8-dk32-dv128-16k-k4v2", batch=16, n_q_heads=32,
                     n_kv_heads=8, d_k=32, d_v=128, context=16384, k_bits=4, v_bits=2,
                     group_k=32, group_v=32, window=64, log_retain=0, appends=0,
                     thin_from=128, seed=1003),
    # the 32k case with 2-bit keys and a rank-4, 4-bit side code ("HeadQ", §5: rank 4 on
    # the 2-bit rows it repairs most)
    "headq32k": _base(name="headq-b32-32/8-32k-k2v2-r4q4-logretain", batch=32, n_q_heads=32,
                      n_kv_heads=8, d_k=128, d_v=128, context=32768, k_bits=2, v_bits=2,
                      group_k=64, group_v=64, window=128, log_retain=1, appends=0, seed=1005,
                      side_rank=4, side_bits=4, q_in_basis=0.9),
    # the 32k case with the keys rotated ("Quantize What Counts", rotation of the keys only)
    "rot32k": _base(name="rot-b32-32/8-32k-k4v2-logretain", batch=32, n_q_heads=32, n_kv_heads=8,
                    d_k=128, d_v=128, context=32768, k_bits=4, v_bits=2, group_k=64, group_v=64,
                    window=128, log_retain=1, appends=0, seed=1006, rot_keys=1, rot_seed=77),
    # the 32k case with per-channel widths ("Attention-Aware Transform Coding", bit
    # allocation): keys 16 x 8, 64 x 4, 32 x 2 bits and 16 dropped channels (448 bits per
    # row, 3.5 on average); values in groups of 32 channels at 4, 2, 2 and 1 bits (288 bits)
    "aatc32k": _base(name="aatc-b32-32/8-32k-kvar3.5-vvar2.25-logretain", batch=32, n_q_heads=32,
                     n_kv_heads=8, d_k=128, d_v=128, context=32768, k_bits=0, v_bits=0,
                     group_k=64, group_v=32, window=128, log_retain=1, appends=0, seed=1008,
                     k_widths=(8,) * 16 + (4,) * 64 + (2,) * 32 + (0,) * 16,
                     v_widths=(4,) * 32 + (2,) * 64 + (1,) * 32),
    # the 32k case with its quantized groups in a page pool, found through a block table
    "paged32k": _base(name="paged-b32-32/8-32k-k4v2-logretain", batch=32, n_q_heads=32,
                      n_kv_heads=8, d_k=128, d_v=128, context=32768, k_bits=4, v_bits=2,
                      group_k=64, group_v=64, window=128, log_retain=1, appends=0, seed=1007,
                      paged=1),
    # a second width map at 32k: keys 32 x 8 and 96 x 2 bits (3.5 on average), values in
    # groups of 64 channels at 4 and 2 bits (3)
    "aatc32k-k8k2": _base(name="aatc-b32-32/8-32k-k8x32-k2x96-v4x64-v2x64-logretain", batch=32,
                          n_q_heads=32, n_kv_heads=8, d_k=128, d_v=128, context=32768, k_bits=0,
                          v_bits=0, group_k=64, group_v=64, window=128, log_retain=1, appends=0,
                          seed=1009, k_widths=(8,) * 32 + (2,) * 96, v_widths=(4,) * 64 + (2,) * 64),
    # a third width map, not built in: it runs through the run-time plan of the map (keys 64 x 4
    # and 64 x 2 bits, values in groups of 32 channels at 4, 4, 2 and 2 bits)
    "aatc32k-k4k2": _base(name="aatc-b32-32/8-32k-k4x64-k2x64-v4x64-v2x64-logretain", batch=32,
                          n_q_heads=32, n_kv_heads=8, d_k=128, d_v=128, context=32768, k_bits=0,
                          v_bits=0, group_k=64, group_v=32, window=128, log_retain=1, appends=0,
                          seed=1011, k_widths=(4,) * 64 + (2,) * 64, v_widths=(4,) * 64 + (2,) * 64),
    # the HeadQ case on a paged cache
    "headq-paged32k": _base(name="headq-paged-b32-32/8-32k-k2v2-r4q4-logretain", batch=32,
                            n_q_heads=32, n_kv_heads=8, d_k=128, d_v=128, context=32768, k_bits=2,
                            v_bits=2, group_k=64, group_v=64, window=128, log_retain=1, appends=0,
                            seed=1010, side_rank=4, side_bits=4, q_in_basis=0.9, paged=1),
}

SWEEP_BATCHES = (1, 8, 32, 64)
SWEEP_BITS = ((8, 4), (4, 2), (2, 2), (16, 16))


def sweep_workload(batch: int, k_bits: int, v_bits: int, appends: int = 256) -> Workload:
    """Context-131072 sweep point: 32/8 heads, d=128, group 64, window 128."""
    return _base(name=f"sweep-b{batch}-k{k_bits}v{v_bits}-128k", batch=batch, n_q_heads=32,
                 n_kv_heads=8, d_k=128, d_v=128, context=131072, k_bits=k_bits, v_bits=v_bits,
                 group_k=64, group_v=64, window=128, log_retain=0, appends=appends,
                 seed=1004, per_seq=1)


def sweep_key(batch: int, k_bits: int, v_bits: int) -> str:
    return f"sweep-b{batch}-k{k_bits}v{v_bits}"


SWEEP_KEYS = [sweep_key(b, kb, vb) for b in SWEEP_BATCHES for kb, vb in SWEEP_BITS]
ALL_KEYS = list(WORKLOADS) + SWEEP_KEYS


def by_key(key: str) -> Workload:
    """A named workload, or a sweep point "sweep-b<B>-k<kb>v<vb>"."""
    if key in WORKLOADS:
        return WORKLOADS[key]
    for b in SWEEP_BATCHES:
        for kb, vb in SWEEP_BITS:
            if key == sweep_key(b, kb, vb):
                return sweep_workload(b, kb, vb)
    raise KeyError(f"unknown workload {key!r}; known: {', '.join(ALL_KEYS)}")


def sequence_generator(w: Workload, b: int, device) -> torch.Generator:
    """The generator of sequence b's prefill keys and values (per_seq workloads)."""
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(w.seed * 1_000_003 + b)
    return gen


def _keys(gen: torch.Generator, device, batch: int, heads: int, tokens: int, d: int,
          sigma: torch.Tensor, mu: torch.Tensor) -> torch.Tensor:
    x = torch.randn((batch, heads, tokens, d), generator=gen, device=device, dtype=torch.float32)
    return x * sigma[None, :, None, :] + mu[None, :, None, :]


def key_stats(gen: torch.Generator, device, heads: int, d: int):
    """Per (kv head, channel) outlier scale (log-uniform [0.5, 8]) and mean (N(0, 2))."""
    u = torch.rand((heads, d), generator=gen, device=device, dtype=torch.float32)
    sigma = torch.exp(math.log(0.5) + u * (math.log(8.0) - math.log(0.5)))
    mu = torch.randn((heads, d), generator=gen, device=device, dtype=torch.float32) * math.sqrt(2.0)
    return sigma, mu


class Inputs:
    """Seeded fp16 tensors for one workload.

    ``k``, ``v``: [B][Hkv][context][d]; ``q``: list of [B][Hq][d_k] (one per decode
    step); ``k_app``/``v_app``: list of [B][Hkv][d] (one per append step).
    """

    def __init__(self, w: Workload, device="cpu", batch_slice: Optional[slice] = None):
        self.w = w
        dev = torch.device(device)
        gen = torch.Generator(device=dev)
        gen.manual_seed(w.seed)
        d_src = w.thin_from if w.thin_from else w.d_k
        sigma, mu = key_stats(gen, dev, w.n_kv_heads, d_src)
        proj = None
        if w.thin_from:
            proj = torch.randn((w.thin_from, w.d_k), generator=gen, device=dev,
                               dtype=torch.float32) / math.sqrt(w.thin_from)
        self.sigma, self.mu, self.proj = sigma, mu, proj

        def keys(batch, tokens, g=gen):
            k = _keys(g, dev, batch, w.n_kv_heads, tokens, d_src, sigma, mu)
            if proj is not None:
                k = k @ proj
            return k.to(torch.float16)

        def normal(shape, g=gen):
            return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.float16)

        B = w.batch
        rows = range(B) if batch_slice is None else range(B)[batch_slice]
        if w.per_seq:
            # sequence by sequence (only the sequences of batch_slice are drawn)
            self.k = torch.empty((len(rows), w.n_kv_heads, w.context, w.d_k), dtype=torch.float16, device=dev)
            self.v = torch.empty((len(rows), w.n_kv_heads, w.context, w.d_v), dtype=torch.float16, device=dev)
            for i, b in enumerate(rows):
                g = sequence_generator(w, b, dev)
                self.k[i] = keys(1, w.context, g)[0]
                self.v[i] = normal((w.n_kv_heads, w.context, w.d_v), g)
        else:
            self.k = keys(B, w.context)
            self.v = normal((B, w.n_kv_heads, w.context, w.d_v))
        self.side_basis: Optional[torch.Tensor] = None
        if w.side_rank:
            g = torch.randn((w.n_kv_heads, w.d_k, w.side_rank), generator=gen, device=dev,
                            dtype=torch.float32)
            self.side_basis = torch.linalg.qr(g.cpu().double())[0].float().to(dev)

        def query(batch):
            n = torch.randn((batch, w.n_q_heads, w.d_k), generator=gen, device=dev, dtype=torch.float32)
            if not w.side_rank:
                return n.to(torch.float16)
            a = torch.randn((batch, w.n_q_heads, w.side_rank), generator=gen, device=dev,
                            dtype=torch.float32)
            U = self.side_basis.repeat_interleave(w.n_rep, dim=0)          # [Hq][d_k][r]
            f = w.q_in_basis
            q = math.sqrt(1.0 - f) * n + math.sqrt(f * w.d_k / w.side_rank) * torch.einsum("hdr,bhr->bhd", U, a)
            return q.to(torch.float16)

        n_dec = max(w.appends, 1)
        self.q: List[torch.Tensor] = []
        self.k_app: List[torch.Tensor] = []
        self.v_app: List[torch.Tensor] = []
        for _ in range(n_dec):
            self.q.append(query(B))
            if w.appends:
                self.k_app.append(keys(B, 1)[:, :, 0, :].contiguous())
                self.v_app.append(normal((B, w.n_kv_heads, w.d_v)))
        if batch_slice is not None:
            if not w.per_seq:
                self.k = self.k[batch_slice].contiguous()
                self.v = self.v[batch_slice].contiguous()
            self.q = [x[batch_slice].contiguous() for x in self.q]
            self.k_app = [x[batch_slice].contiguous() for x in self.k_app]
            self.v_app = [x[batch_slice].contiguous() for x in self.v_app]


def random_fp16(shape, seed: int, device="cpu", scale: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    """Plain N(mean, scale^2) fp16 tensor from its own seeded generator (small test cases)."""
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(seed)
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * scale + mean
    return x.to(torch.float16)
