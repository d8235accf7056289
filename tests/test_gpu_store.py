"""The storage tier on the GPU: streaming layers whose misses are read from an
expert file (parallel pread into pinned staging, one copy per blob) against
the same layers streaming from pinned host memory, at the layer shape (hidden
2816, 128 experts, top-8, 16 slots, router bias N(0, 1.5)), two layers with
RMSNorm and the fp16 residual: one token at a time, then a 64-token chunk.
The file holds the very bytes of the host store, so y, the residual, the slot
of every pair and the tables must be equal bit for bit."""
import numpy as np
import pytest
import torch

from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER

pytestmark = pytest.mark.gpu
DEV = "cuda"
CFG = LAYER


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moeq4.load()
    assert torch.cuda.is_available()
    yield
    torch.cuda.synchronize()


def test_store_streaming_equals_host_store(tmp_path):
    n_layers, T, C = 2, 24, 64
    nb = synth.blob_bytes(CFG.H, CFG.I)
    layers = [synth.layer_weights(CFG, 29, l, DEV, bias_std=1.5) for l in range(n_layers)]
    stores = []
    for d in layers:
        st = torch.empty((CFG.E, nb), dtype=torch.uint8, pin_memory=True)
        st.copy_(d["experts"])
        stores.append(st)
    path = tmp_path / "experts.bin"
    moeq4.write_expert_file(path, stores, nb)
    fst = moeq4.Store(path, n_layers, CFG.E, nb, n_threads=8, n_staging=CFG.S)
    sides = []
    for use_file in (False, True):
        objs = []
        for l, d in enumerate(layers):
            slots = torch.zeros((CFG.S, nb), dtype=torch.uint8, device=DEV)
            table = moeq4.new_lfu_table()
            lay = moeq4.Layer(d["router_w"], d["router_scale"], d["router_bias"], d["shared"], None,
                              None if use_file else stores[l], slots, table,
                              store=fst if use_file else None, store_layer=l)
            objs.append((lay, slots, table))
        sides.append(objs)
    ctx = moeq4.Context(CFG, C)
    cs = torch.cuda.Stream()
    h0 = synth.tokens(T + C, CFG.H, seed=30, device=DEV)
    outs = []
    for objs in sides:
        for (_, _, table) in objs:
            moeq4.moe_lfu_init(ctx, table, CFG.S)
        h = h0.clone()
        ys, sos = [], []
        y = torch.empty((C, CFG.H), device=DEV)
        so = torch.empty((C, CFG.k), dtype=torch.int32, device=DEV)
        for t in range(T):                                 # one token at a time
            for (lay, _, _) in objs:
                moeq4.moe_layer_decode(ctx, lay, h[t:t + 1], 1, y[:1], slot_of=so[:1],
                                       flags=moeq4.MOE_PRENORM, copy_stream=cs)
                torch.cuda.synchronize()
                ys.append(y[:1].clone())
                sos.append(so[:1].clone())
        for (lay, _, _) in objs:                           # then a chunk
            moeq4.moe_layer_decode(ctx, lay, h[T:], C, y, slot_of=so, flags=moeq4.MOE_PRENORM,
                                   copy_stream=cs)
            torch.cuda.synchronize()
            ys.append(y.clone())
            sos.append(so.clone())
        moeq4.moe_ctx_check(ctx)
        tables = [moeq4.read_lfu_table(t) for (_, _, t) in objs]
        outs.append((h, ys, sos, tables))
    (h_a, ys_a, so_a, tb_a), (h_b, ys_b, so_b, tb_b) = outs
    assert torch.equal(h_a, h_b)
    for a, b in zip(ys_a, ys_b):
        assert torch.equal(a, b)
    for a, b in zip(so_a, so_b):
        assert torch.equal(a, b)
    for a, b in zip(tb_a, tb_b):
        assert (list(a.expert), list(a.count), list(a.seq), a.hits, a.misses) == \
               (list(b.expert), list(b.count), list(b.seq), b.hits, b.misses)
        assert b.misses > CFG.S                            # the file really was read
    nbytes, secs, direct = fst.stats()
    assert nbytes == sum(t.misses for t in tb_b) * nb
    fst.close()
    ctx.close()


def test_store_refuses_device_fill(tmp_path):
    nb = synth.blob_bytes(CFG.H, CFG.I)
    d = synth.layer_weights(CFG, 31, 0, DEV, bias_std=1.5)
    path = tmp_path / "one.bin"
    moeq4.write_expert_file(path, [d["experts"].cpu()], nb)
    fst = moeq4.Store(path, 1, CFG.E, nb, n_threads=2, n_staging=4)
    slots = torch.zeros((CFG.S, nb), dtype=torch.uint8, device=DEV)
    table = moeq4.new_lfu_table()
    lay = moeq4.Layer(d["router_w"], d["router_scale"], d["router_bias"], d["shared"], None, None,
                      slots, table, store=fst, store_layer=0)
    ctx = moeq4.Context(CFG, 1)
    moeq4.moe_lfu_init(ctx, table, CFG.S)
    x = synth.tokens(1, CFG.H, seed=32, device=DEV)
    y = torch.empty((1, CFG.H), device=DEV)
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_layer_decode(ctx, lay, x, 1, y, flags=moeq4.MOE_DEVICE_FILL,
                               copy_stream=torch.cuda.Stream())
    assert ei.value.code == moeq4.MOE_ERR_INVALID_ARG
    fst.close()
    ctx.close()
