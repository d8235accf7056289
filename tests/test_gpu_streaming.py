"""Expert streaming at the layer shape: hidden 2816, 128 experts, top-8,
16 cache slots per layer, 4 layers with skewed router bias N(0, 1.5), 64
tokens decoded one after another with RMSNorm and the fp16 residual.

Both ways of filling a miss are covered: copies issued by the host after it
reads the miss list, and MOE_DEVICE_FILL, where a kernel reads the miss list
in device memory and pulls the blobs from pinned host memory.

Checks (the streaming configuration of the benchmark, at fewer layers and
tokens so that the oracle finishes in seconds):
- streaming output equals resident output bit for bit at every layer and
  token (same kernels, same bytes: the cache only moves where they are read);
- oracle-forced decode: every layer runs on the oracle's own residual stream;
  routing indices, the slot of every selected expert and the miss list match
  the oracle's LFU model bit for bit, y is within tolerance, and at the end
  each layer's table (expert, count, insertion number per slot) and its hit
  and miss totals equal the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER
from gpu_util import assert_y_close, np_of

pytestmark = pytest.mark.gpu
DEV = "cuda"
CFG = LAYER                 # S = 16
N_LAYERS, T = 4, 64


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moeq4.load()
    assert torch.cuda.is_available()
    yield
    torch.cuda.synchronize()


@pytest.fixture(scope="module")
def stack():
    nb = synth.blob_bytes(CFG.H, CFG.I)
    out = []
    for l in range(N_LAYERS):
        d = synth.layer_weights(CFG, 5, l, DEV, bias_std=1.5)
        store = torch.empty((CFG.E, nb), dtype=torch.uint8, pin_memory=True)
        store.copy_(d["experts"])
        slots = torch.zeros((CFG.S, nb), dtype=torch.uint8, device=DEV)
        table = moeq4.new_lfu_table()
        host = {k: np_of(d[k]) for k in ("router_w", "router_scale", "router_bias", "shared")}
        host["experts"] = store.numpy()                 # the very bytes the copies read
        out.append(dict(d=d, store=store, slots=slots, table=table, host=host,
                        st=moeq4.Layer(d["router_w"], d["router_scale"], d["router_bias"],
                                       d["shared"], None, store, slots, table),
                        rs=moeq4.Layer.from_dict(d)))
    return out


@pytest.mark.parametrize("fill", ["host", "device"])
def test_streaming_equals_resident_bitwise(stack, fill):
    flags = moeq4.MOE_PRENORM | (moeq4.MOE_DEVICE_FILL if fill == "device" else 0)
    ctx = moeq4.Context(CFG, 1)
    cs = torch.cuda.Stream()
    for s in stack:
        moeq4.moe_lfu_init(ctx, s["table"], CFG.S)
    h0 = synth.tokens(T, CFG.H, seed=55, device=DEV)
    h_st, h_rs = h0.clone(), h0.clone()
    y_st = torch.empty((1, CFG.H), device=DEV)
    y_rs = torch.empty((1, CFG.H), device=DEV)
    for t in range(T):
        for s in stack:
            moeq4.moe_layer_decode(ctx, s["st"], h_st[t:t + 1], 1, y_st,
                                   flags=flags, copy_stream=cs)
            moeq4.moe_layer_decode(ctx, s["rs"], h_rs[t:t + 1], 1, y_rs,
                                   flags=moeq4.MOE_PRENORM)
            torch.cuda.synchronize()
            assert torch.equal(y_st, y_rs), t
    moeq4.moe_ctx_check(ctx)
    assert torch.equal(h_st, h_rs)
    hits = sum(moeq4.read_lfu_table(s["table"]).hits for s in stack)
    misses = sum(moeq4.read_lfu_table(s["table"]).misses for s in stack)
    assert hits + misses == N_LAYERS * T * CFG.k
    assert hits > 0 and misses > CFG.S      # evictions happened
    ctx.close()


@pytest.mark.parametrize("fill", ["host", "device"])
def test_streaming_oracle_forced_cache_and_outputs(stack, fill):
    flags = moeq4.MOE_PRENORM | (moeq4.MOE_DEVICE_FILL if fill == "device" else 0)
    ctx = moeq4.Context(CFG, 1)
    cs = torch.cuda.Stream()
    for s in stack:
        moeq4.moe_lfu_init(ctx, s["table"], CFG.S)
    caches = [oracle.LfuCache(CFG.S) for _ in stack]
    h0 = np_of(synth.tokens(T, CFG.H, seed=56, device=DEV))
    y = torch.empty((1, CFG.H), device=DEV)
    idx = torch.empty((1, CFG.k), dtype=torch.int32, device=DEV)
    so = torch.empty((1, CFG.k), dtype=torch.int32, device=DEV)
    xn = torch.empty((1, CFG.H), dtype=torch.float16, device=DEV)
    for t in range(T):
        h_or = h0[t].copy()
        for l, s in enumerate(stack):
            x_or = oracle.rmsnorm(h_or, CFG.rms_eps)
            ref = oracle.moe_layer(CFG, s["host"], x_or)
            so_ref, _ = caches[l].token(ref["idx"])
            hg = torch.from_numpy(h_or.view(np.int16).copy()).view(torch.float16).to(DEV)[None]
            moeq4.moe_layer_decode(ctx, s["st"], hg, 1, y, idx, slot_of=so, x_norm=xn,
                                   flags=flags, copy_stream=cs)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(np_of(xn)[0], x_or)
            assert idx[0].cpu().tolist() == ref["idx"].tolist(), (t, l)
            assert so[0].cpu().tolist() == so_ref.tolist(), (t, l)
            assert_y_close(y[0].cpu().numpy(), ref["y"], f"token {t} layer {l}")
            h_or = oracle.residual_add(h_or, ref["y"])
    moeq4.moe_ctx_check(ctx)
    for l, s in enumerate(stack):
        tb = moeq4.read_lfu_table(s["table"])
        c = caches[l]
        assert (tb.hits, tb.misses) == (int(c.hits[0]), int(c.misses[0])), l
        assert list(tb.expert)[:CFG.S] == c.expert.tolist()
        assert list(tb.count)[:CFG.S] == c.count.tolist()
        assert list(tb.seq)[:CFG.S] == c.seq.tolist()
        assert tb.valid == 1
    ctx.close()
