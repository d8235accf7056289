"""Chunked prefill in streaming mode: a chunk of T > 1 tokens through one
layer whose routed experts live in pinned host memory behind the 16-slot LFU
cache ("Gemma 4 26B : Comment faire tourner un LLM en 2 Go de RAM", section
04 "Chunked Prefill": one expert fetched from storage serves every row of the
chunk that uses it).

The chunk is one cache lookup: its distinct experts are served in batches
that fit the slots, each expert copied at most once, and the kernels of a
resident multi-token step (tensor cores, or the CUDA-core grouped kernels at
threshold 0) serve each batch's (token, choice) pairs from the slots.

Checks at the layer shape (hidden 2816, 128 experts, top-8, 16 slots, router
bias N(0, 1.5)), two layers, a 96-token prompt with RMSNorm and the fp16
residual, both fill modes:
- streaming output equals the resident batched output bit for bit, y and the
  residual, with both on the tensor cores (default threshold) and both on
  the CUDA-core grouped kernels (threshold 0);
- the slot of every (token, choice), each layer's table and its hit and miss
  totals equal the oracle's chunk model run on the GPU's routing, and no
  expert is copied twice in a chunk;
- y is within tolerance of the oracle at sampled tokens (the oracle runs on
  the GPU's normalised layer input).
A tiny shape (5 slots for 16 experts) runs chunks of several sizes, one token
included, on one cache.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER, TINY
from gpu_util import assert_y_close, np_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moeq4.load()
    assert torch.cuda.is_available()
    yield
    torch.cuda.synchronize()


def _stack(cfg, n_layers, seed, bias_std):
    nb = synth.blob_bytes(cfg.H, cfg.I)
    out = []
    for l in range(n_layers):
        d = synth.layer_weights(cfg, seed, l, DEV, bias_std=bias_std)
        store = torch.empty((cfg.E, nb), dtype=torch.uint8, pin_memory=True)
        store.copy_(d["experts"])
        slots = torch.zeros((cfg.S, nb), dtype=torch.uint8, device=DEV)
        table = moeq4.new_lfu_table()
        host = {k: np_of(d[k]) for k in ("router_w", "router_scale", "router_bias", "shared")}
        host["experts"] = store.numpy()
        out.append(dict(d=d, store=store, slots=slots, table=table, host=host,
                        st=moeq4.Layer(d["router_w"], d["router_scale"], d["router_bias"],
                                       d["shared"], None, store, slots, table),
                        rs=moeq4.Layer.from_dict(d)))
    return out


def _table_state(table, S):
    tb = moeq4.read_lfu_table(table)
    return (list(tb.expert)[:S], list(tb.count)[:S], list(tb.seq)[:S], tb.hits, tb.misses, tb.valid)


def _oracle_state(c):
    return (c.expert.tolist(), c.count.tolist(), c.seq.tolist(), int(c.hits[0]), int(c.misses[0]), 1)


@pytest.mark.parametrize("fill,tau", [("host", None), ("device", None), ("host", 0)])
def test_chunk_layer_shape_resident_oracle_and_cache(fill, tau):
    cfg, T, n_layers = LAYER, 96, 2
    stack = _stack(cfg, n_layers, seed=17, bias_std=1.5)
    flags = moeq4.MOE_PRENORM | (moeq4.MOE_DEVICE_FILL if fill == "device" else 0)
    ctx_st, ctx_rs = moeq4.Context(cfg, T), moeq4.Context(cfg, T)
    if tau is not None:                                   # both sides on the grouped kernels
        moeq4.moe_set_mma_min_tokens(ctx_st, tau)
        moeq4.moe_set_mma_min_tokens(ctx_rs, tau)
    cs = torch.cuda.Stream()
    caches = [oracle.LfuCache(cfg.S) for _ in stack]
    for s in stack:
        moeq4.moe_lfu_init(ctx_st, s["table"], cfg.S)
    h0 = synth.tokens(T, cfg.H, seed=18, device=DEV)
    h_st, h_rs = h0.clone(), h0.clone()
    y_st = torch.empty((T, cfg.H), device=DEV)
    y_rs = torch.empty((T, cfg.H), device=DEV)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    so = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    xn = torch.empty((T, cfg.H), dtype=torch.float16, device=DEV)
    n_batches = 0
    for l, s in enumerate(stack):
        moeq4.moe_layer_decode(ctx_st, s["st"], h_st, T, y_st, idx, slot_of=so, x_norm=xn,
                               flags=flags, copy_stream=cs)
        moeq4.moe_layer_decode(ctx_rs, s["rs"], h_rs, T, y_rs, flags=moeq4.MOE_PRENORM)
        torch.cuda.synchronize()
        moeq4.moe_ctx_check(ctx_st)
        assert torch.equal(y_st, y_rs), l
        assert torch.equal(h_st, h_rs), l
        # the cache against the oracle's chunk model on the GPU's routing
        so_ref, _, miss, nb = caches[l].chunk(idx.cpu().numpy())
        n_batches += nb
        assert len({e for _, e, _ in miss}) == len(miss)
        np.testing.assert_array_equal(so.cpu().numpy(), so_ref)
        assert _table_state(s["table"], cfg.S) == _oracle_state(caches[l]), l
        # outputs against the oracle on the layer's own normalised input
        xs = np_of(xn)
        for t in (0, 1, 47, T - 1):
            ref = oracle.moe_layer(cfg, s["host"], xs[t])
            assert idx[t].cpu().tolist() == ref["idx"].tolist(), (l, t)
            assert_y_close(y_st[t].cpu().numpy(), ref["y"], f"layer {l} token {t}")
    # the chunks' experts did not fit the slots at once
    assert n_batches > n_layers
    ctx_st.close()
    ctx_rs.close()


@pytest.mark.parametrize("fill", ["host", "device"])
def test_chunks_of_several_sizes_tiny(fill):
    cfg = TINY.with_(S=5)                  # fewer slots than experts: chunks need several batches
    stack = _stack(cfg, 1, seed=23, bias_std=1.0)
    s = stack[0]
    flags = moeq4.MOE_PRENORM | (moeq4.MOE_DEVICE_FILL if fill == "device" else 0)
    ctx_st, ctx_rs = moeq4.Context(cfg, 40), moeq4.Context(cfg, 40)
    cs = torch.cuda.Stream()
    moeq4.moe_lfu_init(ctx_st, s["table"], cfg.S)
    cache = oracle.LfuCache(cfg.S)
    h = synth.tokens(100, cfg.H, seed=24, device=DEV)
    pos = 0
    for T in (7, 1, 40, 3, 1, 33, 15):
        hc = h[pos:pos + T]
        h_st, h_rs = hc.clone(), hc.clone()
        y_st = torch.empty((T, cfg.H), device=DEV)
        y_rs = torch.empty((T, cfg.H), device=DEV)
        idx = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
        so = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
        moeq4.moe_layer_decode(ctx_st, s["st"], h_st, T, y_st, idx, slot_of=so, flags=flags,
                               copy_stream=cs)
        moeq4.moe_layer_decode(ctx_rs, s["rs"], h_rs, T, y_rs, flags=moeq4.MOE_PRENORM)
        torch.cuda.synchronize()
        moeq4.moe_ctx_check(ctx_st)
        assert torch.equal(y_st, y_rs), T
        assert torch.equal(h_st, h_rs), T
        so_ref, _, _, _ = cache.chunk(idx.cpu().numpy())
        np.testing.assert_array_equal(so.cpu().numpy(), so_ref)
        assert _table_state(s["table"], cfg.S) == _oracle_state(cache), T
        pos += T
    ctx_st.close()
    ctx_rs.close()
