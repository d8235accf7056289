"""CPU oracle for the MoE decode hot path (fp64, scalar, slow).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / reference leg may import this package.  It
shares no code with the CUDA library in ``bit_quantized_expert_int8_b200``
and never imports it; the two meet only on the byte buffers produced by the
seeded input generators.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64 accumulation, one
weight at a time, compiled with ``-ffp-contract=off``); this module is
argument marshalling over numpy arrays.  Each wrapper names the function of
the C file that it calls; the C file cites the passages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no CUDA involved)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i32, i64, dbl, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_half_to_double.restype = dbl
    lib.oracle_double_to_half.argtypes = [dbl]
    lib.oracle_double_to_half.restype = ctypes.c_uint16
    lib.oracle_dequant.argtypes = [P, P, P, i32, i32, i32]
    lib.oracle_dequant.restype = dbl
    lib.oracle_blob_bytes.argtypes = [i32, i32]
    lib.oracle_blob_bytes.restype = sz
    lib.oracle_gelu.argtypes = [dbl, i32]
    lib.oracle_gelu.restype = dbl
    lib.oracle_expert_ffn.argtypes = [P, i32, i32, i32, P, P, P]
    lib.oracle_expert_ffn.restype = None
    lib.oracle_router_logits.argtypes = [P, P, P, P, i32, i32, P]
    lib.oracle_router_logits.restype = None
    lib.oracle_topk.argtypes = [P, i32, i32, P]
    lib.oracle_topk.restype = None
    lib.oracle_softmax.argtypes = [P, i32, P]
    lib.oracle_softmax.restype = None
    lib.oracle_topk_weights.argtypes = [P, P, i32, i32, P]
    lib.oracle_topk_weights.restype = None
    lib.oracle_combine.argtypes = [P, P, P, i32, i32, P]
    lib.oracle_combine.restype = None
    lib.oracle_moe_layer.argtypes = [i32, i32, i32, i32, i32, i32, i32,
                                     P, P, P, P, P, sz, P, P, P, P, P, P, P]
    lib.oracle_moe_layer.restype = None
    lib.oracle_rmsnorm.argtypes = [P, i32, dbl, P]
    lib.oracle_rmsnorm.restype = None
    lib.oracle_residual_add.argtypes = [P, P, i32]
    lib.oracle_residual_add.restype = None
    lib.oracle_lfu_token.argtypes = [i32, P, P, P, P, P, i32, P, P, P, P, P, P]
    lib.oracle_lfu_token.restype = i32
    lib.oracle_lfu_chunk.argtypes = [i32, P, P, P, P, P, i32, i32, P, P, P, P, P, P, P, P, P]
    lib.oracle_lfu_chunk.restype = i32
    lib.oracle_set_threads.argtypes = [i32]
    lib.oracle_set_threads.restype = i32
    _lib = lib
    return lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def set_threads(n: int = 0) -> int:
    """OpenMP threads for the row loops of the FFN (0: leave as is)."""
    return _load().oracle_set_threads(int(n))


def half_to_double(bits: int) -> float:
    return _load().oracle_half_to_double(int(bits))


def double_to_half(v: float) -> int:
    return _load().oracle_double_to_half(float(v))


def blob_bytes(H: int, I: int) -> int:
    return int(_load().oracle_blob_bytes(H, I))


def dequant(q, scale, bias, K: int, r: int, c: int) -> float:
    """``oracle_dequant``: one weight of a q4 matrix (q uint32, scale/bias
    as uint16 fp16 bits)."""
    q = _c(q, np.uint32); s = _c(scale, np.uint16); b = _c(bias, np.uint16)
    return _load().oracle_dequant(_p(q), _p(s), _p(b), K, r, c)


def gelu(g: float, variant: int = 0) -> float:
    return _load().oracle_gelu(float(g), int(variant))


def expert_ffn(blob, H: int, I: int, x, gelu_variant: int = 0):
    """``oracle_expert_ffn``: returns (y[H], h[I]) in fp64; x is fp64[H]."""
    blob = _c(blob, np.uint8)
    x = _c(np.asarray(x, dtype=np.float64), np.float64)
    y = np.zeros(H, np.float64)
    h = np.zeros(I, np.float64)
    _load().oracle_expert_ffn(_p(blob), H, I, gelu_variant, _p(x), _p(h), _p(y))
    return y, h


def router_logits(W, scale, bias, x16, E: int, H: int):
    """``oracle_router_logits``: W int8 [E,H], scale uint16 [E], bias
    float32 [E] or None, x16 uint16 [H] -> float64 [E]."""
    W = _c(W, np.int8); s = _c(scale, np.uint16); x16 = _c(x16, np.uint16)
    b = None if bias is None else _c(bias, np.float32)
    out = np.zeros(E, np.float64)
    _load().oracle_router_logits(_p(W), _p(s), _p(b), _p(x16), E, H, _p(out))
    return out


def topk(logits, k: int):
    logits = _c(np.asarray(logits, np.float64), np.float64)
    idx = np.zeros(k, np.int32)
    _load().oracle_topk(_p(logits), logits.size, k, _p(idx))
    return idx


def softmax(logits):
    logits = _c(np.asarray(logits, np.float64), np.float64)
    p = np.zeros_like(logits)
    _load().oracle_softmax(_p(logits), logits.size, _p(p))
    return p


def topk_weights(p, idx, renorm: int = 1):
    p = _c(np.asarray(p, np.float64), np.float64)
    idx = _c(np.asarray(idx, np.int32), np.int32)
    w = np.zeros(idx.size, np.float64)
    _load().oracle_topk_weights(_p(p), _p(idx), idx.size, int(renorm), _p(w))
    return w


def combine(y_shared, y_routed, w):
    """``oracle_combine``: y_shared [H], y_routed [k,H], w [k] -> y [H]."""
    ys = _c(np.asarray(y_shared, np.float64), np.float64)
    yr = _c(np.asarray(y_routed, np.float64), np.float64)
    w = _c(np.asarray(w, np.float64), np.float64)
    k, H = yr.shape
    y = np.zeros(H, np.float64)
    _load().oracle_combine(_p(ys), _p(yr), _p(w), k, H, _p(y))
    return y


def moe_layer(cfg, layer, x16):
    """``oracle_moe_layer`` for one token.

    cfg: object with H, E, k, I, Is, gelu, renorm.  layer: dict of numpy
    arrays router_w (int8 [E,H]), router_scale (uint16 [E]), router_bias
    (float32 [E] or None), shared (uint8 blob), experts (uint8 [E, blob]).
    Returns dict(idx, w, logits, y, y_shared, y_routed).
    """
    lib = _load()
    H, E, k = cfg.H, cfg.E, cfg.k
    Wr = _c(layer["router_w"], np.int8)
    rs = _c(layer["router_scale"], np.uint16)
    rb = layer.get("router_bias")
    rb = None if rb is None else _c(rb, np.float32)
    sh = _c(layer["shared"], np.uint8)
    ex = _c(layer["experts"], np.uint8)
    x16 = _c(x16, np.uint16)
    idx = np.zeros(k, np.int32)
    w = np.zeros(k, np.float64)
    logits = np.zeros(E, np.float64)
    y = np.zeros(H, np.float64)
    ysh = np.zeros(H, np.float64)
    yr = np.zeros((k, H), np.float64)
    lib.oracle_moe_layer(H, E, k, cfg.I, cfg.Is, cfg.gelu, cfg.renorm,
                         _p(Wr), _p(rs), _p(rb), _p(sh), _p(ex),
                         ex.shape[1], _p(x16), _p(idx), _p(w), _p(logits),
                         _p(y), _p(ysh), _p(yr))
    return dict(idx=idx, w=w, logits=logits, y=y, y_shared=ysh, y_routed=yr)


def rmsnorm(h16, eps: float):
    h16 = _c(h16, np.uint16)
    x = np.zeros_like(h16)
    _load().oracle_rmsnorm(_p(h16), h16.size, float(eps), _p(x))
    return x


def residual_add(h16, y):
    h16 = np.array(h16, dtype=np.uint16, copy=True)
    y = _c(np.asarray(y, np.float64), np.float64)
    _load().oracle_residual_add(_p(h16), _p(y), h16.size)
    return h16


class LfuCache:
    """One layer's LFU cache state, driven by ``oracle_lfu_token``."""

    def __init__(self, n_slots: int):
        self.S = n_slots
        self.expert = np.full(n_slots, -1, np.int32)
        self.count = np.zeros(n_slots, np.int64)
        self.seq = np.zeros(n_slots, np.int64)
        self.counter = np.zeros(1, np.int64)
        self.hits = np.zeros(1, np.int64)
        self.misses = np.zeros(1, np.int64)

    def token(self, idx):
        """Look up one token's experts; returns (slot_of, [(expert, slot)])."""
        idx = _c(np.asarray(idx, np.int32), np.int32)
        k = idx.size
        slot_of = np.full(k, -1, np.int32)
        me = np.zeros(k, np.int32)
        ms = np.zeros(k, np.int32)
        nm = np.zeros(1, np.int32)
        rc = _load().oracle_lfu_token(self.S, _p(self.expert), _p(self.count),
                                      _p(self.seq), _p(self.counter), _p(idx),
                                      k, _p(slot_of), _p(me), _p(ms), _p(nm),
                                      _p(self.hits), _p(self.misses))
        if rc != 0:
            raise ValueError("oracle_lfu_token: no victim or repeated expert")
        n = int(nm[0])
        return slot_of, list(zip(me[:n].tolist(), ms[:n].tolist()))

    def chunk(self, idx):
        """Look up a chunk of tokens (``idx`` [T, k]) at once, expert by
        expert in batches that fit the slots (``oracle_lfu_chunk``).  Returns
        (slot_of [T, k], batch_of [T, k], [(batch, expert, slot)], n_batch)."""
        idx = _c(np.asarray(idx, np.int32).reshape(-1, np.asarray(idx).shape[-1]), np.int32)
        T, k = idx.shape
        slot_of = np.full((T, k), -1, np.int32)
        batch_of = np.full((T, k), -1, np.int32)
        n_max = T * k
        mb = np.zeros(n_max, np.int32)
        me = np.zeros(n_max, np.int32)
        ms = np.zeros(n_max, np.int32)
        nm = np.zeros(1, np.int32)
        nb = np.zeros(1, np.int32)
        rc = _load().oracle_lfu_chunk(self.S, _p(self.expert), _p(self.count),
                                      _p(self.seq), _p(self.counter), _p(idx), T, k,
                                      _p(slot_of), _p(batch_of), _p(mb), _p(me), _p(ms),
                                      _p(nm), _p(nb), _p(self.hits), _p(self.misses))
        if rc != 0:
            raise ValueError("oracle_lfu_chunk: repeated expert, S <= k or bad size")
        n = int(nm[0])
        return slot_of, batch_of, list(zip(mb[:n].tolist(), me[:n].tolist(), ms[:n].tolist())), int(nb[0])
