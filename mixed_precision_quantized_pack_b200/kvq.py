"""Python binding of libkvq (ctypes): argument marshalling only.

Every computation runs in the library's CUDA kernels; PyTorch only provides
device memory (``torch.empty`` buffers) and the current CUDA stream.  The
functions keep the C names (``kvq_quantize_prefill`` ...); ``KVCache`` bundles
the buffers and the handle for convenience.  Loading fails loudly when the
library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# The library to load: the in-tree libkvq.so, or (KVQ_LIBRARY=debug) its bounds-check build
# libkvq_debug.so, built from the same sources with -DKVQ_DEBUG.
LIB_PATH = os.path.join(_HERE, "libkvq_debug.so" if os.environ.get("KVQ_LIBRARY") == "debug" else "libkvq.so")

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = -1
KVQ_ERR_UNSUPPORTED = -2
KVQ_ERR_ALIGN = -3
KVQ_ERR_CAPACITY = -4
KVQ_ERR_WORKSPACE = -5
KVQ_ERR_STATE = -6
KVQ_ERR_CUDA = -7
KVQ_MAX_RETAINED = 32
KVQ_KERNEL_AUTO = 0
KVQ_KERNEL_GENERIC = 1
KVQ_KERNEL_TENSOR = 2
KVQ_CENTER_AUTO = 0
KVQ_CENTER_OFF = 1
KVQ_CENTER_ON = 2
KVQ_STATUS_TIMEOUT = 1
KVQ_NOALLOC_SCRATCH_BYTES = 8 << 20
KVQ_MAX_SEQS = 256

CONFIG_FIELDS = ("batch", "n_q_heads", "n_kv_heads", "d_k", "d_v", "k_bits", "v_bits", "group_k",
                 "group_v", "window", "log_retain", "max_context", "side_rank", "side_bits",
                 "rot_keys")
OPTIONAL_CONFIG = ("side_rank", "side_bits", "rot_keys")   # default 0: no side code, no rotation
PAGE_CONFIG = ("paged", "n_pages")                          # default 0: one region per sequence
BUFFER_FIELDS = ("kcode", "ksz", "vcode", "vsz", "win_k", "win_v", "ret_k", "ret_v")
SIDE_FIELDS = ("zcode", "zsz", "side_u")
PAGE_FIELDS = ("block_table",)
SIZE_FIELDS = BUFFER_FIELDS + ("workspace",) + SIDE_FIELDS + PAGE_FIELDS
POINTER_FIELDS = BUFFER_FIELDS + SIDE_FIELDS + PAGE_FIELDS


class kvq_config(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_int) for n in CONFIG_FIELDS] + [("rot_signs", ctypes.c_uint * 8)] +
                [(n, ctypes.c_int) for n in PAGE_CONFIG] +
                [("k_widths", ctypes.c_ubyte * 256), ("v_widths", ctypes.c_ubyte * 256)])


class kvq_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in SIZE_FIELDS]


class kvq_debug_record(ctypes.Structure):
    _fields_ = [("failures", ctypes.c_uint), ("site", ctypes.c_uint), ("index", ctypes.c_longlong),
                ("extent", ctypes.c_longlong)]


class kvq_buffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in POINTER_FIELDS]


class kvq_plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("splits_quant", "splits_fp16", "n_groups", "n_fp16",
                                            "fast_path", "centered")]


class KVQError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {kvq_strerror(code)} ({code})")


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int

# name -> (restype, argtypes)
_SIGNATURES = {
    "kvq_buffer_sizes": (_I, [ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_sizes)]),
    "kvq_cache_init": (_I, [ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_buffers),
                            ctypes.POINTER(_P)]),
    "kvq_cache_destroy": (None, [_P]),
    "kvq_quantize_prefill": (_I, [_P, _P, _P, _I, _P]),
    "kvq_append": (_I, [_P, _P, _P, _P]),
    "kvq_quantize_prefill_ragged": (_I, [_P, _P, _P, _I, ctypes.POINTER(_I), _P]),
    "kvq_append_ragged": (_I, [_P, _P, _P, ctypes.POINTER(ctypes.c_ubyte), _P]),
    "kvq_get_seq_state": (_I, [_P, _I, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I),
                               ctypes.POINTER(_I)]),
    "kvq_decode_workspace_size": (_I, [_P, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "kvq_decode_attention": (_I, [_P, _P, _P, _P, ctypes.c_size_t, _I, _P]),
    "kvq_decode_attention_noalloc": (_I, [_P, _P, _P, _I, _P]),
    "kvq_noalloc_read_status": (_I, [ctypes.POINTER(ctypes.c_uint), _P]),
    "kvq_noalloc_reset_status": (_I, [_P]),
    "kvq_debug_build": (_I, []),
    "kvq_debug_take_record": (_I, [ctypes.POINTER(kvq_debug_record), _P]),
    "kvq_debug_site_name": (ctypes.c_char_p, [ctypes.c_uint]),
    "kvq_get_plan": (_I, [_P, _I, ctypes.POINTER(kvq_plan)]),
    "kvq_set_decode_kernel": (_I, [_P, _I]),
    "kvq_set_value_centering": (_I, [_P, _I]),
    "kvq_debug_stall_next_decode": (_I, [_P]),
    "kvq_plan_decode": (_I, [ctypes.POINTER(kvq_config), _I, _I, _I, ctypes.POINTER(kvq_plan)]),
    "kvq_get_state": (_I, [_P, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I),
                           ctypes.POINTER(_I)]),
    "kvq_retained_positions": (_I, [_I, ctypes.POINTER(_I), _I]),
    "kvq_reset_status": (_I, [_P, _P]),
    "kvq_read_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint), _P]),
    "kvq_strerror": (ctypes.c_char_p, [_I]),
    "kvq_prefill_sequence": (_I, [_P, _I, _P, _P, _I, _P]),
    "kvq_release_sequence": (_I, [_P, _I]),
    "kvq_free_pages": (_I, [_P]),
    "kvq_allocate_bits": (_I, [ctypes.POINTER(ctypes.c_double), _I, _I, _I, ctypes.POINTER(ctypes.c_ubyte)]),
}


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libkvq.so not found at {LIB_PATH}; build it with "
                               "`python -m mixed_precision_quantized_pack_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(rc: int, where: str) -> int:
    if rc < 0:
        raise KVQError(rc, where)
    return rc


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_config(cfg: Dict[str, int]) -> kvq_config:
    """cfg: the kvq_config fields by name; "rot_signs" is a list of up to 8 uint32 words."""
    c = kvq_config(*[int(cfg.get(n, 0) if n in OPTIONAL_CONFIG else cfg[n]) for n in CONFIG_FIELDS])
    for i, word in enumerate(list(cfg.get("rot_signs", ()))[:8]):
        c.rot_signs[i] = int(word) & 0xFFFFFFFF
    for n in PAGE_CONFIG:
        setattr(c, n, int(cfg.get(n, 0)))
    for n in ("k_widths", "v_widths"):
        for i, w in enumerate(list(cfg.get(n, ()))[:256]):
            getattr(c, n)[i] = int(w)
    return c


# ---- the C entry points, same names -----------------------------------------
def kvq_strerror(code: int) -> str:
    return lib().kvq_strerror(int(code)).decode()


def kvq_buffer_sizes(cfg: Dict[str, int]) -> Dict[str, int]:
    out = kvq_sizes()
    _check(lib().kvq_buffer_sizes(ctypes.byref(make_config(cfg)), ctypes.byref(out)),
           "kvq_buffer_sizes")
    return {n: int(getattr(out, n)) for n in SIZE_FIELDS}


def kvq_plan_decode(cfg: Dict[str, int], L: int, sm_count: int, num_splits: int = 0) -> Dict[str, int]:
    out = kvq_plan()
    _check(lib().kvq_plan_decode(ctypes.byref(make_config(cfg)), int(L), int(sm_count),
                                 int(num_splits), ctypes.byref(out)), "kvq_plan_decode")
    return {n: int(getattr(out, n)) for n, _ in kvq_plan._fields_}


def kvq_allocate_bits(weight, budget: int, unit_bits: int = 1) -> Tuple[List[int], int]:
    """Per-unit widths by reverse water-filling, and the bits they spend."""
    n = len(weight)
    w = (ctypes.c_double * n)(*[float(x) for x in weight])
    out = (ctypes.c_ubyte * n)()
    spent = _check(lib().kvq_allocate_bits(w, n, int(unit_bits), int(budget), out), "kvq_allocate_bits")
    return [int(out[i]) for i in range(n)], spent


def kvq_retained_positions(Q: int) -> List[int]:
    buf = (ctypes.c_int * KVQ_MAX_RETAINED)()
    n = _check(lib().kvq_retained_positions(int(Q), buf, KVQ_MAX_RETAINED), "kvq_retained_positions")
    return [int(buf[i]) for i in range(n)]


def kvq_cache_init(cfg: Dict[str, int], ptrs: Dict[str, int]) -> int:
    bufs = kvq_buffers(*[ptrs.get(n) or None for n in POINTER_FIELDS])
    h = _P()
    _check(lib().kvq_cache_init(ctypes.byref(make_config(cfg)), ctypes.byref(bufs), ctypes.byref(h)),
           "kvq_cache_init")
    return h.value


def kvq_cache_destroy(handle: int) -> None:
    lib().kvq_cache_destroy(handle)


def kvq_quantize_prefill(handle: int, k_ptr: int, v_ptr: int, L: int, stream: int) -> None:
    _check(lib().kvq_quantize_prefill(handle, k_ptr, v_ptr, int(L), stream), "kvq_quantize_prefill")


def kvq_append(handle: int, k_ptr: int, v_ptr: int, stream: int) -> None:
    _check(lib().kvq_append(handle, k_ptr, v_ptr, stream), "kvq_append")


def kvq_quantize_prefill_ragged(handle: int, k_ptr: int, v_ptr: int, L_max: int, lengths, stream: int) -> None:
    arr = (_I * len(lengths))(*[int(x) for x in lengths])
    _check(lib().kvq_quantize_prefill_ragged(handle, k_ptr, v_ptr, int(L_max), arr, stream),
           "kvq_quantize_prefill_ragged")


def kvq_append_ragged(handle: int, k_ptr: int, v_ptr: int, active, stream: int) -> None:
    mask = None if active is None else (ctypes.c_ubyte * len(active))(*[1 if a else 0 for a in active])
    _check(lib().kvq_append_ragged(handle, k_ptr, v_ptr, mask, stream), "kvq_append_ragged")


def kvq_prefill_sequence(handle: int, b: int, k_ptr: int, v_ptr: int, L: int, stream: int) -> None:
    _check(lib().kvq_prefill_sequence(handle, int(b), k_ptr, v_ptr, int(L), stream), "kvq_prefill_sequence")


def kvq_release_sequence(handle: int, b: int) -> None:
    _check(lib().kvq_release_sequence(handle, int(b)), "kvq_release_sequence")


def kvq_free_pages(handle: int) -> int:
    return _check(lib().kvq_free_pages(handle), "kvq_free_pages")


def kvq_get_seq_state(handle: int, b: int) -> Tuple[int, int, List[int]]:
    L, Q, n = _I(), _I(), _I()
    idx = (ctypes.c_int * KVQ_MAX_RETAINED)()
    _check(lib().kvq_get_seq_state(handle, int(b), ctypes.byref(L), ctypes.byref(Q), ctypes.byref(n), idx),
           "kvq_get_seq_state")
    return L.value, Q.value, [int(idx[i]) for i in range(n.value)]


def kvq_decode_workspace_size(handle: int, num_splits: int = 0) -> int:
    n = ctypes.c_size_t()
    _check(lib().kvq_decode_workspace_size(handle, int(num_splits), ctypes.byref(n)),
           "kvq_decode_workspace_size")
    return int(n.value)


def kvq_decode_attention(handle: int, q_ptr: int, out_ptr: int, ws_ptr: int, ws_bytes: int,
                         num_splits: int, stream: int) -> None:
    _check(lib().kvq_decode_attention(handle, q_ptr, out_ptr, ws_ptr, int(ws_bytes),
                                      int(num_splits), stream), "kvq_decode_attention")


def kvq_decode_attention_noalloc(handle: int, q_ptr: int, out_ptr: int, num_splits: int,
                                 stream: int) -> None:
    """Decode without a workspace: the partials go to the library's own scratch array."""
    _check(lib().kvq_decode_attention_noalloc(handle, q_ptr, out_ptr, int(num_splits), stream),
           "kvq_decode_attention_noalloc")


def kvq_noalloc_read_status(stream: int) -> int:
    """Status word of the library's scratch array on the current device (waits for stream)."""
    st = ctypes.c_uint()
    _check(lib().kvq_noalloc_read_status(ctypes.byref(st), stream), "kvq_noalloc_read_status")
    return int(st.value)


def kvq_noalloc_reset_status(stream: int) -> None:
    _check(lib().kvq_noalloc_reset_status(stream), "kvq_noalloc_reset_status")


def kvq_get_plan(handle: int, num_splits: int = 0) -> Dict[str, int]:
    out = kvq_plan()
    _check(lib().kvq_get_plan(handle, int(num_splits), ctypes.byref(out)), "kvq_get_plan")
    return {n: int(getattr(out, n)) for n, _ in kvq_plan._fields_}


def kvq_set_decode_kernel(handle: int, kernel: int) -> None:
    _check(lib().kvq_set_decode_kernel(handle, int(kernel)), "kvq_set_decode_kernel")


def kvq_set_value_centering(handle: int, mode: int) -> None:
    _check(lib().kvq_set_value_centering(handle, int(mode)), "kvq_set_value_centering")


def kvq_debug_build() -> bool:
    """True when the loaded library is the bounds-check build."""
    return bool(lib().kvq_debug_build())


def kvq_debug_take_record(stream: int) -> Dict[str, object]:
    """The bounds-check build's record of failed checks on the current device (then cleared)."""
    r = kvq_debug_record()
    _check(lib().kvq_debug_take_record(ctypes.byref(r), stream), "kvq_debug_take_record")
    return {"failures": int(r.failures), "site": lib().kvq_debug_site_name(r.site).decode(),
            "index": int(r.index), "extent": int(r.extent)}


def kvq_debug_stall_next_decode(handle: int) -> None:
    _check(lib().kvq_debug_stall_next_decode(handle), "kvq_debug_stall_next_decode")


def kvq_get_state(handle: int) -> Tuple[int, int, List[int]]:
    L, Q, n = _I(), _I(), _I()
    idx = (ctypes.c_int * KVQ_MAX_RETAINED)()
    _check(lib().kvq_get_state(handle, ctypes.byref(L), ctypes.byref(Q), ctypes.byref(n), idx),
           "kvq_get_state")
    return L.value, Q.value, [int(idx[i]) for i in range(n.value)]


def kvq_reset_status(ws_ptr: int, stream: int) -> None:
    _check(lib().kvq_reset_status(ws_ptr, stream), "kvq_reset_status")


def kvq_read_status(ws_ptr: int, stream: int) -> int:
    st = ctypes.c_uint()
    _check(lib().kvq_read_status(ws_ptr, ctypes.byref(st), stream), "kvq_read_status")
    return int(st.value)


# ---- convenience: buffers + handle over torch tensors ------------------------
def _fp16_cuda(t: torch.Tensor, shape, name: str) -> torch.Tensor:
    if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: need a contiguous CUDA fp16 tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")
    return t


class KVCache:
    """One attention layer's packed KV cache in device memory owned by PyTorch.

    With cfg["side_rank"] = r > 0 the cache keeps a side code and ``side_basis`` (fp32
    [Hkv][d_k][r], any device) is copied into the cache's basis buffer.  With cfg["paged"]
    = 1 the quantized groups live in a pool of cfg["n_pages"] pages."""

    def __init__(self, cfg: Dict[str, int], device=None, side_basis: Optional[torch.Tensor] = None):
        self.cfg = dict(cfg)
        self.device = torch.device(device or "cuda")
        self.sizes = kvq_buffer_sizes(self.cfg)
        self.buffers: Dict[str, Optional[torch.Tensor]] = {}
        for n in POINTER_FIELDS:
            sz = self.sizes[n]
            self.buffers[n] = torch.zeros(sz, dtype=torch.uint8, device=self.device) if sz else None
        r = int(self.cfg.get("side_rank", 0))
        if r:
            shape = (self.cfg["n_kv_heads"], self.cfg["d_k"], r)
            if side_basis is None or tuple(side_basis.shape) != shape:
                raise ValueError(f"side_basis: need an fp32 tensor of shape {shape}")
            self.view("side_u").copy_(side_basis.to(torch.float32))
        ptrs = {n: (b.data_ptr() if b is not None else 0) for n, b in self.buffers.items()}
        self.handle = kvq_cache_init(self.cfg, ptrs)
        self.workspace = torch.empty(self.sizes["workspace"], dtype=torch.uint8, device=self.device)
        kvq_reset_status(self.workspace.data_ptr(), _stream())

    def close(self):
        if getattr(self, "handle", None):
            kvq_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # shapes
    @property
    def B(self):
        return self.cfg["batch"]

    def prefill(self, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
        c = self.cfg
        L = k.shape[2]
        _fp16_cuda(k, (c["batch"], c["n_kv_heads"], L, c["d_k"]), "k")
        _fp16_cuda(v, (c["batch"], c["n_kv_heads"], L, c["d_v"]), "v")
        kvq_quantize_prefill(self.handle, k.data_ptr(), v.data_ptr(), L, _stream(stream))

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None, active=None) -> None:
        """One token per sequence; `active` (B bools) limits the append to some sequences."""
        c = self.cfg
        _fp16_cuda(k_new, (c["batch"], c["n_kv_heads"], c["d_k"]), "k_new")
        _fp16_cuda(v_new, (c["batch"], c["n_kv_heads"], c["d_v"]), "v_new")
        if active is None:
            kvq_append(self.handle, k_new.data_ptr(), v_new.data_ptr(), _stream(stream))
        else:
            if len(active) != c["batch"]:
                raise ValueError("active: one flag per sequence")
            kvq_append_ragged(self.handle, k_new.data_ptr(), v_new.data_ptr(), list(active), _stream(stream))

    def prefill_ragged(self, k: torch.Tensor, v: torch.Tensor, lengths, stream=None) -> None:
        """k, v [B][Hkv][L_max][d]; sequence b's first lengths[b] tokens are its context."""
        c = self.cfg
        L_max = k.shape[2]
        _fp16_cuda(k, (c["batch"], c["n_kv_heads"], L_max, c["d_k"]), "k")
        _fp16_cuda(v, (c["batch"], c["n_kv_heads"], L_max, c["d_v"]), "v")
        if len(lengths) != c["batch"]:
            raise ValueError("lengths: one per sequence")
        kvq_quantize_prefill_ragged(self.handle, k.data_ptr(), v.data_ptr(), L_max, list(lengths),
                                    _stream(stream))

    def prefill_sequence(self, b: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
        """k, v [Hkv][L][d]: sequence b alone (re)starts with these L tokens."""
        c = self.cfg
        L = k.shape[1]
        _fp16_cuda(k, (c["n_kv_heads"], L, c["d_k"]), "k")
        _fp16_cuda(v, (c["n_kv_heads"], L, c["d_v"]), "v")
        kvq_prefill_sequence(self.handle, b, k.data_ptr(), v.data_ptr(), L, _stream(stream))

    def release(self, b: int) -> None:
        kvq_release_sequence(self.handle, b)

    def free_pages(self) -> int:
        return kvq_free_pages(self.handle)

    def seq_state(self, b: int) -> Tuple[int, int, List[int]]:
        return kvq_get_seq_state(self.handle, b)

    def decode(self, q: torch.Tensor, out: Optional[torch.Tensor] = None, num_splits: int = 0,
               stream=None) -> torch.Tensor:
        c = self.cfg
        _fp16_cuda(q, (c["batch"], c["n_q_heads"], c["d_k"]), "q")
        if out is None:
            out = torch.empty((c["batch"], c["n_q_heads"], c["d_v"]), dtype=torch.float16,
                              device=q.device)
        _fp16_cuda(out, (c["batch"], c["n_q_heads"], c["d_v"]), "out")
        kvq_decode_attention(self.handle, q.data_ptr(), out.data_ptr(), self.workspace.data_ptr(),
                             self.workspace.numel(), num_splits, _stream(stream))
        return out

    def status(self, stream=None) -> int:
        return kvq_read_status(self.workspace.data_ptr(), _stream(stream))

    def reset_status(self, stream=None) -> None:
        kvq_reset_status(self.workspace.data_ptr(), _stream(stream))

    def state(self) -> Tuple[int, int, List[int]]:
        return kvq_get_state(self.handle)

    def set_kernel(self, kernel: int) -> None:
        kvq_set_decode_kernel(self.handle, kernel)

    def set_centering(self, mode: int) -> None:
        kvq_set_value_centering(self.handle, mode)

    def plan(self, num_splits: int = 0) -> Dict[str, int]:
        return kvq_get_plan(self.handle, num_splits)

    # typed views of the buffers, in the layouts of include/kvq.h
    def view(self, name: str) -> torch.Tensor:
        c = self.cfg
        B, H, dk, dv = c["batch"], c["n_kv_heads"], c["d_k"], c["d_v"]
        kb, vb, gk, gv = c["k_bits"], c["v_bits"], c["group_k"], c["group_v"]
        buf = self.buffers[name]
        if buf is None:
            raise ValueError(f"{name} is not used by this configuration")
        if kb == 16:
            cap = c["max_context"]
            lcap = cap
        else:
            lcap = -(-c["max_context"] // gk) * gk
            cap = c["window"] + gk
        # quantized buffers: [B][H][Lcap] regions, or a pool [n_pages][H][group_k]
        paged = bool(c.get("paged", 0))
        rows = (c["n_pages"], H, gk) if paged else (B, H, lcap)
        groups = (c["n_pages"], H) if paged else (B, H, lcap // gk)
        if kb == 0:        # per-channel widths: rows of max(1, ceil(sum / 32)) words
            kwords = max(1, -(-sum(int(x) for x in c["k_widths"][:dk]) // 32))
            vwords = max(1, -(-sum(int(x) for x in c["v_widths"][:dv]) // 32))
            ksz_shape = groups + (dk, 2)
        else:
            kwords, vwords = dk * kb // 32, dv * vb // 32
            ksz_shape = groups + (2 * dk,)
        shapes = {
            "kcode": (torch.int32, rows + (kwords,)),
            "ksz": (torch.float16, ksz_shape),
            "vcode": (torch.int32, rows + (vwords,)),
            "vsz": (torch.float16, rows + (dv // gv, 2)),
            "block_table": (torch.int32, (B, lcap // gk)),
            "win_k": (torch.float16, (B, H, cap, dk)),
            "win_v": (torch.float16, (B, H, cap, dv)),
            "ret_k": (torch.float16, (B, H, KVQ_MAX_RETAINED, dk)),
            "ret_v": (torch.float16, (B, H, KVQ_MAX_RETAINED, dv)),
        }
        r, sq = int(c.get("side_rank", 0)), int(c.get("side_bits", 0))
        if r:
            shapes.update({
                "zcode": (torch.uint8, rows + (r * sq // 8,)),
                "zsz": (torch.float16, groups + (r, 2)),
                "side_u": (torch.float32, (H, dk, r)),
            })
        dt, shape = shapes[name]
        return buf.view(dt).view(shape)

    def sequence_view(self, name: str, b: int) -> torch.Tensor:
        """Quantized buffer `name` of sequence b in the unpaged layout [H][Q_b/group_k...]:
        for a paged cache, its pages gathered through the block table (a copy)."""
        L, Q, _ = self.seq_state(b)
        gk = self.cfg["group_k"]
        t = self.view(name)
        if not self.cfg.get("paged", 0):
            return t[b, :, :Q] if name not in ("ksz", "zsz") else t[b, :, :Q // gk]
        pages = self.view("block_table")[b, :Q // gk].long()
        g = t[pages]                                   # [n_groups][H][...]
        if name in ("ksz", "zsz"):
            return g.transpose(0, 1).contiguous()
        # [n][H][gk][...] -> [H][n*gk][...]
        return g.transpose(0, 1).reshape((g.shape[1], -1) + tuple(g.shape[3:])).contiguous()
