"""ctypes binding of libmoeq4.so: the C ABI of include/moeq4.h, same names.

Argument marshalling only: torch tensors are passed as raw device pointers and
streams as their CUDA handles; every step of the path runs in the library's
kernels.  There is no fallback: if the shared library is missing or cannot be
loaded, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .config import MoeConfig

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoeq4.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_ALIGNMENT = -2
MOE_ERR_UNSUPPORTED_SHAPE = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_CACHE_STATE = -6
MOE_PRENORM = 1
MOE_DEVICE_FILL = 2
MOE_MAX_SLOTS = 32

EXPORTS = ("moe_ctx_create", "moe_ctx_destroy", "moe_ctx_check", "moe_ctx_trace", "moe_ctx_info",
           "moe_last_error", "moe_blob_bytes",
           "moe_router_topk", "moe_expert_ffn_q4", "moe_combine", "moe_lfu_init",
           "moe_ep_dispatch", "moe_ffn_rows", "moe_shared_ffn", "moe_ep_unpermute",
           "moe_cache_lookup_lfu", "moe_layer_decode", "moe_stack_decode",
           "moe_router_topk_noalloc", "moe_set_mma_min_tokens", "moe_set_wait_ns",
           "moe_store_stride", "moe_store_open", "moe_store_close", "moe_store_read",
           "moe_store_stats")


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moeq4 error {code}: {msg}")
        self.code = code


class CMoeConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("inter_shared", ctypes.c_int32), ("n_slots", ctypes.c_int32),
                ("renorm", ctypes.c_int32), ("gelu", ctypes.c_int32),
                ("rms_eps", ctypes.c_double)]


class CMoeLayer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "router_w", "router_scale", "router_bias", "shared_blob", "experts",
        "host_store", "slots", "lfu", "store")] + [
        ("store_layer", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class CMoeLayerOut(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("y", "topk_idx", "topk_w", "slot_of", "x_norm")]


class CMoeLfuTable(ctypes.Structure):
    _fields_ = [("expert", ctypes.c_int32 * MOE_MAX_SLOTS),
                ("count", ctypes.c_int64 * MOE_MAX_SLOTS),
                ("seq", ctypes.c_int64 * MOE_MAX_SLOTS),
                ("counter", ctypes.c_int64), ("hits", ctypes.c_int64),
                ("misses", ctypes.c_int64), ("n_slots", ctypes.c_int32),
                ("valid", ctypes.c_int32)]


LFU_TABLE_BYTES = ctypes.sizeof(CMoeLfuTable)
PAIR_BYTES = 16   # MoeFfnPair: blob pointer, int32 inter, int32 token
TRACE_WORDS = 160  # per CTA trace record of the fused layer kernel

_lib = None


def load() -> ctypes.CDLL:
    """Load libmoeq4.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "bit_quantized_expert_int8_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32 = ctypes.c_void_p, ctypes.c_int
    sig = {
        "moe_ctx_create": ([ctypes.POINTER(CMoeConfig), i32, ctypes.POINTER(P)], i32),
        "moe_ctx_destroy": ([P], i32),
        "moe_ctx_check": ([P, P], i32),
        "moe_ctx_trace": ([P, i32, P, i32], i32),
        "moe_ctx_info": ([P, ctypes.c_char_p, i32], i32),
        "moe_set_mma_min_tokens": ([P, i32], i32),
        "moe_set_wait_ns": ([P, ctypes.c_ulonglong], i32),
        "moe_last_error": ([], ctypes.c_char_p),
        "moe_blob_bytes": ([i32, i32], ctypes.c_size_t),
        "moe_router_topk": ([P, P, P, P, P, i32, P, P, P, P], i32),
        "moe_expert_ffn_q4": ([P, P, i32, P, i32, P, P], i32),
        "moe_combine": ([P, P, P, P, i32, P, P, P], i32),
        "moe_ep_dispatch": ([P, P, i32, i32, P, P, P, P, P, P], i32),
        "moe_ffn_rows": ([P, P, i32, P, i32, P, P, P], i32),
        "moe_shared_ffn": ([P, P, P, i32, P, P], i32),
        "moe_ep_unpermute": ([P, P, P, i32, P, P], i32),
        "moe_lfu_init": ([P, P, i32, P], i32),
        "moe_cache_lookup_lfu": ([P, P, P, i32, P, P, P, P], i32),
        "moe_layer_decode": ([P, ctypes.POINTER(CMoeLayer), P, i32,
                              ctypes.POINTER(CMoeLayerOut), i32, P, P], i32),
        "moe_stack_decode": ([P, P, i32, P, i32, P, P], i32),
        "moe_router_topk_noalloc": ([i32, i32, i32, i32, P, P, P, P, i32, P, P, P], i32),
        "moe_store_stride": ([ctypes.c_size_t], ctypes.c_size_t),
        "moe_store_open": ([ctypes.c_char_p, i32, i32, ctypes.c_size_t, i32, i32, ctypes.POINTER(P)], i32),
        "moe_store_close": ([P], i32),
        "moe_store_read": ([P, i32, P, i32, P], i32),
        "moe_store_stats": ([P, ctypes.POINTER(ctypes.c_ulonglong), ctypes.POINTER(ctypes.c_double),
                             ctypes.POINTER(ctypes.c_int)], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int):
    if rc != MOE_OK:
        raise MoeError(rc, load().moe_last_error().decode())


def last_error() -> str:
    return load().moe_last_error().decode()


def blob_bytes(hidden: int, inter: int) -> int:
    return int(load().moe_blob_bytes(hidden, inter))


class Context:
    """moe_ctx_create / moe_ctx_destroy."""

    def __init__(self, cfg: MoeConfig, max_tokens: int = 1):
        lib = load()
        self.cfg = cfg
        self.max_tokens = max_tokens
        self._c = CMoeConfig(cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is, cfg.S,
                             cfg.renorm, cfg.gelu, cfg.rms_eps)
        h = ctypes.c_void_p()
        _check(lib.moe_ctx_create(ctypes.byref(self._c), max_tokens, ctypes.byref(h)))
        self.handle = h.value

    def close(self):
        if self.handle:
            load().moe_ctx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_ctx_check(ctx, stream=None):
    """Synchronise and raise MoeError(MOE_ERR_TIMEOUT) if a bounded device
    wait of this context gave up since the last check."""
    _check(load().moe_ctx_check(ctx.handle, _stream(stream)))


def moe_ctx_info(ctx) -> str:
    """moe_ctx_info: which kernels serve single-token layers, and their
    shared memory and registers."""
    buf = ctypes.create_string_buffer(512)
    _check(load().moe_ctx_info(ctx.handle, buf, 512))
    return buf.value.decode()


def moe_set_mma_min_tokens(ctx, min_tokens: int):
    """moe_set_mma_min_tokens: bucket size from which multi-token steps run
    an expert on the tensor cores (0: never)."""
    _check(load().moe_set_mma_min_tokens(ctx.handle, int(min_tokens)))


def moe_set_wait_ns(ctx, ns: int):
    """moe_set_wait_ns: bound of every device wait of the context (ns)."""
    _check(load().moe_set_wait_ns(ctx.handle, int(ns)))


def moe_ctx_trace(ctx, enable=-1, read=False):
    """Switch phase tracing of the fused layer kernel (1 on, 0 off, -1 keep);
    with read=True return the last launch's records as an int64 array
    [n_ctas, 16] (see moeq4.h)."""
    import numpy as np
    n = 1024 * TRACE_WORDS
    buf = np.zeros(n, dtype=np.uint64) if read else None
    rc = load().moe_ctx_trace(ctx.handle, int(enable),
                              buf.ctypes.data if read else None, n if read else 0)
    if rc < 0:
        _check(rc)
    return buf[:rc].reshape(-1, TRACE_WORDS) if read else None


def moe_router_topk(ctx, Wr, row_scale, bias, x, T, topk_idx, topk_w, logits=None, stream=None):
    _check(load().moe_router_topk(ctx.handle, _ptr(Wr), _ptr(row_scale), _ptr(bias), _ptr(x), T,
                                  _ptr(topk_idx), _ptr(topk_w), _ptr(logits), _stream(stream)))


def moe_router_topk_noalloc(n_experts, hidden, top_k, renorm, Wr, row_scale, bias, x, T,
                            topk_idx, topk_w, stream=None):
    """Router without a context for callers that cannot allocate device
    memory; its scratch is a static device array (limits in include/moeq4.h)."""
    _check(load().moe_router_topk_noalloc(n_experts, hidden, top_k, renorm, _ptr(Wr),
                                          _ptr(row_scale), _ptr(bias), _ptr(x), T,
                                          _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def make_pairs(entries, device="cuda"):
    """Pack [(blob_ptr, inter, token), ...] into a device MoeFfnPair array."""
    buf = torch.empty((len(entries), PAIR_BYTES), dtype=torch.uint8)
    for i, (p, inter, tok) in enumerate(entries):
        buf[i, :8] = torch.tensor([p], dtype=torch.int64).view(torch.uint8)
        buf[i, 8:] = torch.tensor([inter, tok], dtype=torch.int32).view(torch.uint8)
    return buf.to(device)


def moe_expert_ffn_q4(ctx, pairs, n_pairs, x, T, y, stream=None):
    _check(load().moe_expert_ffn_q4(ctx.handle, _ptr(pairs), n_pairs, _ptr(x), T, _ptr(y),
                                    _stream(stream)))


def moe_combine(ctx, y_routed, y_shared, topk_w, T, y_out, residual=None, stream=None):
    _check(load().moe_combine(ctx.handle, _ptr(y_routed), _ptr(y_shared), _ptr(topk_w), T,
                              _ptr(y_out), _ptr(residual), _stream(stream)))


def moe_ep_dispatch(ctx, topk_idx, T, n_ranks, x, send_x, send_expert, send_order, send_counts,
                    stream=None):
    _check(load().moe_ep_dispatch(ctx.handle, _ptr(topk_idx), T, n_ranks, _ptr(x), _ptr(send_x),
                                  _ptr(send_expert), _ptr(send_order), _ptr(send_counts),
                                  _stream(stream)))


def moe_ffn_rows(ctx, experts, n_experts, expert_of_row, R, x_rows, y_rows, stream=None):
    _check(load().moe_ffn_rows(ctx.handle, _ptr(experts), n_experts, _ptr(expert_of_row), R,
                               _ptr(x_rows), _ptr(y_rows), _stream(stream)))


def moe_shared_ffn(ctx, shared_blob, x, T, y, stream=None):
    _check(load().moe_shared_ffn(ctx.handle, _ptr(shared_blob), _ptr(x), T, _ptr(y), _stream(stream)))


def moe_ep_unpermute(ctx, y_sorted, send_order, n, y_pairs, stream=None):
    _check(load().moe_ep_unpermute(ctx.handle, _ptr(y_sorted), _ptr(send_order), n, _ptr(y_pairs),
                                   _stream(stream)))


def new_lfu_table(device="cuda"):
    """Device buffer large enough for one MoeLfuTable."""
    return torch.zeros(LFU_TABLE_BYTES, dtype=torch.uint8, device=device)


def read_lfu_table(table) -> CMoeLfuTable:
    raw = table.cpu().numpy().tobytes()
    return CMoeLfuTable.from_buffer_copy(raw)


def moe_lfu_init(ctx, table, n_slots, stream=None):
    _check(load().moe_lfu_init(ctx.handle, _ptr(table), n_slots, _stream(stream)))


def moe_cache_lookup_lfu(ctx, table, topk_idx, T, slot_of, miss_list, n_miss, stream=None):
    _check(load().moe_cache_lookup_lfu(ctx.handle, _ptr(table), _ptr(topk_idx), T,
                                       _ptr(slot_of), _ptr(miss_list), _ptr(n_miss),
                                       _stream(stream)))


class Layer:
    """A layer's buffers (torch tensors) as the C MoeLayer struct."""

    def __init__(self, router_w, router_scale, router_bias=None, shared=None, experts=None,
                 host_store=None, slots=None, lfu=None, store=None, store_layer=0):
        self.keep = (router_w, router_scale, router_bias, shared, experts, host_store, slots, lfu,
                     store)
        self.c = CMoeLayer(_ptr(router_w), _ptr(router_scale), _ptr(router_bias), _ptr(shared),
                           _ptr(experts), _ptr(host_store), _ptr(slots), _ptr(lfu),
                           None if store is None else store.handle, int(store_layer), 0)

    @classmethod
    def from_dict(cls, d, **kw):
        return cls(d["router_w"], d["router_scale"], d.get("router_bias"), d["shared"],
                   d.get("experts"), **kw)


def moe_layer_decode(ctx, layer: Layer, x, T, y, topk_idx=None, topk_w=None, slot_of=None,
                     x_norm=None, flags=0, stream=None, copy_stream=None):
    out = CMoeLayerOut(_ptr(y), _ptr(topk_idx), _ptr(topk_w), _ptr(slot_of), _ptr(x_norm))
    cs = None if copy_stream is None else _stream(copy_stream)
    _check(load().moe_layer_decode(ctx.handle, ctypes.byref(layer.c), _ptr(x), T,
                                   ctypes.byref(out), flags, _stream(stream), cs))


def moe_stack_decode(ctx, layers, h, T, y_last=None, stream=None):
    arr = (CMoeLayer * len(layers))(*[l.c for l in layers])
    _check(load().moe_stack_decode(ctx.handle, ctypes.cast(arr, ctypes.c_void_p), len(layers),
                                   _ptr(h), T, _ptr(y_last), _stream(stream)))


def store_stride(blob_bytes: int) -> int:
    """moe_store_stride: bytes per blob in an expert file (padded to 4 KiB)."""
    return int(load().moe_store_stride(int(blob_bytes)))


class Store:
    """moe_store_open / moe_store_close: an expert file read with parallel pread."""

    def __init__(self, path, n_layers, n_experts, blob_bytes, n_threads=8, n_staging=16):
        h = ctypes.c_void_p()
        _check(load().moe_store_open(str(path).encode(), n_layers, n_experts, blob_bytes, n_threads,
                                     n_staging, ctypes.byref(h)))
        self.handle = h.value
        self.blob_bytes = blob_bytes

    def read(self, layer, experts, dst):
        """moe_store_read into the host arrays dst[i] (numpy uint8, blob_bytes each)."""
        import numpy as np
        ex = np.ascontiguousarray(np.asarray(experts, np.int32))
        ptrs = (ctypes.c_void_p * len(dst))(*[d.ctypes.data for d in dst])
        _check(load().moe_store_read(self.handle, int(layer), ex.ctypes.data, len(ex),
                                     ctypes.cast(ptrs, ctypes.c_void_p)))

    def stats(self):
        """moe_store_stats: (bytes read, seconds reading, O_DIRECT in use)."""
        b, t, d = ctypes.c_ulonglong(), ctypes.c_double(), ctypes.c_int()
        _check(load().moe_store_stats(self.handle, ctypes.byref(b), ctypes.byref(t), ctypes.byref(d)))
        return int(b.value), float(t.value), bool(d.value)

    def close(self):
        if self.handle:
            load().moe_store_close(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def write_expert_file(path, layers_experts, blob_bytes):
    """Writes an expert file in the store's format: for each layer (a uint8
    array or tensor [E][blob_bytes]) each blob padded to store_stride bytes."""
    import numpy as np
    stride = store_stride(blob_bytes)
    pad = np.zeros(stride - blob_bytes, np.uint8)
    with open(path, "wb") as f:
        for ex in layers_experts:
            a = ex.cpu().numpy() if hasattr(ex, "cpu") else np.asarray(ex)
            for e in range(a.shape[0]):
                f.write(a[e].tobytes())
                f.write(pad.tobytes())
