"""Host-side checks of the C-ABI library that need no GPU: it builds, loads,
exports every function that include/*.h declares, and rejects bad shapes
before touching CUDA."""
import ctypes
import glob
import os
import re

import pytest

from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER, TINY

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moeq4.load()


def declared_functions():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", text, re.M):
            names.add(m.group(1))
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("moe_router_topk", "moe_expert_ffn_q4", "moe_combine", "moe_cache_lookup_lfu",
              "moe_layer_decode", "moe_ctx_create", "moe_ctx_destroy", "moe_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value
    for n in moeq4.EXPORTS:
        assert n in declared_functions()


def test_blob_bytes_agree_with_generator(lib):
    for cfg in (TINY, LAYER):
        assert moeq4.blob_bytes(cfg.H, cfg.I) == synth.blob_bytes(cfg.H, cfg.I)
        assert moeq4.blob_bytes(cfg.H, cfg.Is) == synth.blob_bytes(cfg.H, cfg.Is)
    assert moeq4.blob_bytes(2816, 704) == 3345408
    assert moeq4.blob_bytes(2816, 2112) == 10036224
    assert moeq4.blob_bytes(100, 64) == 0


@pytest.mark.parametrize("bad", [dict(H=100), dict(I=96), dict(k=9), dict(E=300),
                                 dict(S=8), dict(S=33), dict(gelu=3), dict(renorm=2)])
def test_ctx_create_rejects_bad_config_without_cuda(lib, bad):
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.Context(LAYER.with_(**bad), 1)
    assert ei.value.code in (moeq4.MOE_ERR_UNSUPPORTED_SHAPE, moeq4.MOE_ERR_INVALID_ARG)
    assert moeq4.last_error()


def test_lfu_table_struct_size_matches_c_layout(lib):
    # int32[32] + int64[32] * 2 + 3 int64 + 2 int32
    assert moeq4.LFU_TABLE_BYTES == 128 + 256 + 256 + 24 + 8
