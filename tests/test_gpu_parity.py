"""GPU parity: every entry point of libmoeq4.so against the CPU oracle.

Routing indices, cache slots and hit/miss counts must match bit for bit;
fp outputs must satisfy rel L2 <= 1e-3 and max abs <= 2e-3 (gpu_util).
All calls go through the C ABI (ctypes binding).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER, TINY, MoeConfig
from gpu_util import (assert_half_close, assert_y_close, make_layer, np_layer, np_of)

pytestmark = pytest.mark.gpu
DEV = "cuda"

SMALL = MoeConfig(H=320, E=40, k=5, I=192, Is=128, S=11)   # ragged shapes


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moeq4.load()
    assert torch.cuda.is_available()
    yield
    torch.cuda.synchronize()


def ctx_for(cfg, T=1):
    return moeq4.Context(cfg, T)


# ---------------------------------------------------------------- router ----

# T >= 40 runs the batched router (CTA per token pair and block of experts:
# 4 blocks of 32 at T = 40 and 64, 2 of 64 at T = 131, one of 128 at T = 256);
# 131 tokens leave a CTA with one token; TINY's 16 experts fill part of a block.
@pytest.mark.parametrize("cfg,T,bias", [(TINY, 1, None), (TINY, 7, 1.5), (SMALL, 3, 0.7),
                                        (LAYER, 4, None), (LAYER, 2, 1.5), (TINY, 33, 1.5),
                                        (LAYER, 39, None), (LAYER, 40, 1.5), (LAYER, 64, None),
                                        (LAYER, 131, 1.5), (TINY, 128, None), (LAYER, 256, 1.5)])
def test_router_parity(cfg, T, bias):
    L = make_layer(cfg, seed=3, bias_std=bias)
    x = synth.tokens(T, cfg.H, seed=5, device=DEV)
    ctx = ctx_for(cfg, T)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=DEV)
    lg = torch.empty((T, cfg.E), dtype=torch.float64, device=DEV)
    moeq4.moe_router_topk(ctx, L["router_w"], L["router_scale"], L["router_bias"], x, T,
                          idx, w, lg)
    torch.cuda.synchronize()
    Ln = np_layer(L)
    xn = np_of(x)
    for t in range(T):
        ref = oracle.router_logits(Ln["router_w"], Ln["router_scale"], Ln["router_bias"],
                                   xn[t], cfg.E, cfg.H)
        np.testing.assert_array_equal(lg[t].cpu().numpy(), ref)        # exact
        ridx = oracle.topk(ref, cfg.k)
        assert idx[t].cpu().tolist() == ridx.tolist()
        rw = oracle.topk_weights(oracle.softmax(ref), ridx, cfg.renorm)
        np.testing.assert_allclose(w[t].cpu().numpy(), rw, rtol=2e-6, atol=1e-7)


def test_router_ties_go_to_lower_index():
    cfg = TINY
    L = make_layer(cfg, seed=1)
    Wr = L["router_w"].clone()
    sc = L["router_scale"].clone()
    sc[3] = sc[11]
    x = synth.tokens(1, cfg.H, seed=2, device=DEV)
    # experts 3 and 11 tie exactly and win: identical rows aligned with
    # sign(x), identical scales
    sgn = torch.sign(x[0].float()).to(torch.int8)
    Wr[3] = sgn * 100
    Wr[11] = sgn * 100
    ctx = ctx_for(cfg)
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((1, cfg.k), dtype=torch.float32, device=DEV)
    moeq4.moe_router_topk(ctx, Wr, sc, None, x, 1, idx, w)
    assert idx[0].tolist()[:2] == [3, 11]
    # all-zero router: every logit 0 -> experts 0..k-1, uniform weights
    moeq4.moe_router_topk(ctx, torch.zeros_like(Wr), sc, None, x, 1, idx, w)
    assert idx[0].tolist() == list(range(cfg.k))
    np.testing.assert_allclose(w[0].cpu().numpy(), 1.0 / cfg.k, rtol=1e-7)


# ------------------------------------------------------------ expert FFN ----

@pytest.mark.parametrize("cfg", [TINY, SMALL, LAYER])
def test_expert_ffn_parity(cfg):
    L = make_layer(cfg, seed=7)
    T = 3
    x = synth.tokens(T, cfg.H, seed=8, device=DEV)
    nb = synth.blob_bytes(cfg.H, cfg.I)
    base = L["experts"].data_ptr()
    entries = [(L["shared"].data_ptr(), cfg.Is, 0), (base + 5 * nb, cfg.I, 1),
               (base + 0 * nb, cfg.I, 2), (L["shared"].data_ptr(), cfg.Is, 2),
               (base + (cfg.E - 1) * nb, cfg.I, 0)]
    pairs = moeq4.make_pairs(entries)
    ctx = ctx_for(cfg, T)
    y = torch.empty((len(entries), cfg.H), dtype=torch.float32, device=DEV)
    moeq4.moe_expert_ffn_q4(ctx, pairs, len(entries), x, T, y)
    torch.cuda.synchronize()
    Ln = np_layer(L)
    xd = np_of(x).view(np.float16).astype(np.float64)
    blobs = [Ln["shared"], Ln["experts"][5], Ln["experts"][0], Ln["shared"],
             Ln["experts"][cfg.E - 1]]
    for p, (blob, (_, inter, tok)) in enumerate(zip(blobs, entries)):
        ref, _ = oracle.expert_ffn(blob, cfg.H, inter, xd[tok], cfg.gelu)
        assert_y_close(y[p].cpu().numpy(), ref, f"pair {p}")


# --------------------------------------------------------------- combine ----

def test_combine_parity_and_residual():
    cfg = LAYER
    T, k, H = 3, cfg.k, cfg.H
    g = torch.Generator(device="cpu").manual_seed(4)
    yr = torch.randn((T, k, H), generator=g).to(DEV)
    ys = torch.randn((T, H), generator=g).to(DEV)
    w = torch.softmax(torch.randn((T, k), generator=g), -1).to(DEV)
    h = (torch.randn((T, H), generator=g) * 4).half().to(DEV)
    h0 = np_of(h)
    y = torch.empty((T, H), device=DEV)
    ctx = ctx_for(cfg, T)
    moeq4.moe_combine(ctx, yr, ys, w, T, y, h)
    torch.cuda.synchronize()
    for t in range(T):
        ref = oracle.combine(ys[t].cpu().double().numpy(), yr[t].cpu().double().numpy(),
                             w[t].cpu().double().numpy())
        assert_y_close(y[t].cpu().numpy(), ref)
        href = oracle.residual_add(h0[t], ref)
        assert_half_close(np_of(h)[t], href)


# ------------------------------------------------------------------- LFU ----

def _lfu_run(cfg, seq, per_call):
    ctx = ctx_for(cfg, max(per_call, 1))
    tb = moeq4.new_lfu_table()
    moeq4.moe_lfu_init(ctx, tb, cfg.S)
    T = seq.shape[0]
    slot_of = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    misses = []
    ml = torch.empty((per_call * cfg.k, 2), dtype=torch.int32, device=DEV)
    nm = torch.empty(1, dtype=torch.int32, device=DEV)
    sd = seq.to(DEV)
    for t0 in range(0, T, per_call):
        n = min(per_call, T - t0)
        moeq4.moe_cache_lookup_lfu(ctx, tb, sd[t0:t0 + n], n, slot_of[t0:t0 + n], ml, nm)
        cnt = int(nm.item())
        misses += [tuple(r) for r in ml[:cnt].cpu().tolist()]
    return slot_of.cpu().numpy(), misses, moeq4.read_lfu_table(tb)


@pytest.mark.parametrize("k,S,E,per_call", [(8, 16, 128, 1), (8, 16, 128, 64), (2, 4, 9, 1),
                                            (5, 11, 40, 7)])
def test_lfu_parity(k, S, E, per_call):
    cfg = LAYER.with_(k=k, S=S, E=E)
    seq = synth.routing_sequence(300, E, k, seed=k * 100 + S)
    slot_of, misses, tb = _lfu_run(cfg, seq, per_call)
    ref = oracle.LfuCache(S)
    ref_misses = []
    for t in range(seq.shape[0]):
        so, ms = ref.token(seq[t].numpy())
        assert slot_of[t].tolist() == so.tolist(), t
        ref_misses += ms
    assert misses == ref_misses
    assert tb.hits == int(ref.hits[0]) and tb.misses == int(ref.misses[0])
    assert list(tb.expert)[:S] == ref.expert.tolist()
    assert list(tb.count)[:S] == ref.count.tolist()
    assert list(tb.seq)[:S] == ref.seq.tolist()


def test_lfu_hand_trace_on_gpu():
    cfg = TINY.with_(k=2, S=4, E=8)
    seq = torch.tensor([[1, 2], [1, 3], [4, 5], [1, 2]], dtype=torch.int32)
    slot_of, misses, tb = _lfu_run(cfg, seq, 1)
    assert [(tb.expert[s], tb.count[s], tb.seq[s]) for s in range(4)] == \
        [(1, 3, 1), (5, 1, 5), (2, 1, 6), (4, 1, 4)]
    assert (tb.hits, tb.misses) == (2, 6)
    assert misses == [(1, 0), (2, 1), (3, 2), (4, 3), (5, 1), (2, 2)]


# -------------------------------------------------------------- full layer ----

def _oracle_layer(cfg, Ln, x16):
    return oracle.moe_layer(cfg, Ln, x16)


@pytest.mark.parametrize("cfg,T,bias", [(TINY, 1, None), (TINY, 5, 1.5), (SMALL, 4, None),
                                        (LAYER, 1, None), (LAYER, 3, 1.5)])
def test_layer_resident_parity(cfg, T, bias):
    L = make_layer(cfg, seed=0, bias_std=bias)
    x = synth.tokens(T, cfg.H, seed=0, device=DEV)
    ctx = ctx_for(cfg, T)
    y = torch.empty((T, cfg.H), device=DEV)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, cfg.k), device=DEV)
    moeq4.moe_layer_decode(ctx, moeq4.Layer.from_dict(L), x, T, y, idx, w)
    torch.cuda.synchronize()
    Ln = np_layer(L)
    xn = np_of(x)
    for t in range(T):
        ref = _oracle_layer(cfg, Ln, xn[t])
        assert idx[t].cpu().tolist() == ref["idx"].tolist()
        np.testing.assert_allclose(w[t].cpu().numpy(), ref["w"], rtol=2e-6, atol=1e-7)
        assert_y_close(y[t].cpu().numpy(), ref["y"], f"token {t}")


@pytest.mark.parametrize("cfg,T,bias,sample", [(LAYER, 40, 1.5, (0, 13, 27, 39)),
                                               (LAYER, 2, None, (0, 1)),
                                               (SMALL, 33, 0.7, tuple(range(33)))])
def test_layer_grouped_multi_token(cfg, T, bias, sample):
    """T > 1 on the CUDA-core grouped path (tensor-core threshold 0: each
    expert read once for all of its tokens, tokens in passes of 4, ragged last
    pass); sampled tokens against the oracle, and the same step split into
    single-token calls."""
    L = make_layer(cfg, seed=4, bias_std=bias)
    x = synth.tokens(T, cfg.H, seed=14, device=DEV)
    ctx = ctx_for(cfg, T)
    moeq4.moe_set_mma_min_tokens(ctx, 0)
    lay = moeq4.Layer.from_dict(L)
    y = torch.empty((T, cfg.H), device=DEV)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    moeq4.moe_layer_decode(ctx, lay, x, T, y, idx)
    torch.cuda.synchronize()
    Ln = np_layer(L)
    xn = np_of(x)
    for t in sample:
        ref = _oracle_layer(cfg, Ln, xn[t])
        assert idx[t].cpu().tolist() == ref["idx"].tolist()
        assert_y_close(y[t].cpu().numpy(), ref["y"], f"token {t}")
    y1 = torch.empty((1, cfg.H), device=DEV)
    for t in sample[:2]:
        moeq4.moe_layer_decode(ctx, lay, x[t:t + 1], 1, y1)
        torch.cuda.synchronize()
        assert_y_close(y1[0].cpu().numpy(), y[t].cpu().numpy().astype(np.float64), f"single {t}")


def test_layer_prenorm_rmsnorm_exact_and_residual():
    cfg = SMALL
    T = 4
    L = make_layer(cfg, seed=2, bias_std=1.0)
    h = (synth.tokens(T, cfg.H, seed=9, device=DEV).float() * 3).half()
    h[1, :5] = torch.tensor([60000.0, 6e-8, -6e-8, 0.0, 1e-3], dtype=torch.float16)
    h0 = np_of(h).copy()
    ctx = ctx_for(cfg, T)
    y = torch.empty((T, cfg.H), device=DEV)
    xn = torch.empty((T, cfg.H), dtype=torch.float16, device=DEV)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    moeq4.moe_layer_decode(ctx, moeq4.Layer.from_dict(L), h, T, y, idx, x_norm=xn,
                           flags=moeq4.MOE_PRENORM)
    torch.cuda.synchronize()
    Ln = np_layer(L)
    for t in range(T):
        x_ref = oracle.rmsnorm(h0[t], cfg.rms_eps)
        np.testing.assert_array_equal(np_of(xn)[t], x_ref)
        ref = _oracle_layer(cfg, Ln, x_ref)
        assert idx[t].cpu().tolist() == ref["idx"].tolist()
        assert_y_close(y[t].cpu().numpy(), ref["y"])
        href = oracle.residual_add(h0[t], ref["y"])
        assert_half_close(np_of(h)[t], href)


# ------------------------------------------------------------------- stack ----

def _stack_layers(cfg, n_layers, seed, bias_std=1.5):
    return [make_layer(cfg, seed=seed, layer=l, bias_std=bias_std) for l in range(n_layers)]


def test_stack_graph_equals_layer_by_layer_and_oracle_forced():
    cfg = TINY
    n_layers, T = 4, 6
    Ls = _stack_layers(cfg, n_layers, seed=11)
    h0 = synth.tokens(T, cfg.H, seed=12, device=DEV)
    ctx = ctx_for(cfg, 1)
    # (a) graph-replayed stack
    h_stack = h0.clone()
    y_last = torch.empty((T, cfg.H), device=DEV)
    layers = [moeq4.Layer.from_dict(L) for L in Ls]
    moeq4.moe_stack_decode(ctx, layers, h_stack, T, y_last)
    # (b) the same decode as individual layer calls
    h_ref = h0.clone()
    y = torch.empty((1, cfg.H), device=DEV)
    for t in range(T):
        for lay in layers:
            moeq4.moe_layer_decode(ctx, lay, h_ref[t:t + 1], 1, y, flags=moeq4.MOE_PRENORM)
    torch.cuda.synchronize()
    assert torch.equal(h_stack, h_ref)
    assert torch.equal(y_last[T - 1], y[0])
    # (c) oracle-forced: each layer on the oracle's own residual stream
    Lns = [np_layer(L) for L in Ls]
    hy = torch.empty((1, cfg.H), device=DEV)
    xn = torch.empty((1, cfg.H), dtype=torch.float16, device=DEV)
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    for t in range(2):
        h_or = np_of(h0)[t].copy()
        for l in range(n_layers):
            x_or = oracle.rmsnorm(h_or, cfg.rms_eps)
            ref = _oracle_layer(cfg, Lns[l], x_or)
            hg = torch.from_numpy(h_or.view(np.int16).copy()).view(torch.float16).to(DEV)[None]
            moeq4.moe_layer_decode(ctx, layers[l], hg, 1, hy, idx, x_norm=xn,
                                   flags=moeq4.MOE_PRENORM)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(np_of(xn)[0], x_or)
            assert idx[0].cpu().tolist() == ref["idx"].tolist()
            assert_y_close(hy[0].cpu().numpy(), ref["y"], f"token {t} layer {l}")
            h_or = oracle.residual_add(h_or, ref["y"])


# --------------------------------------------------------------- streaming ----

def _streaming_setup(cfg, Ls):
    host_stores, slots, tables = [], [], []
    nb = synth.blob_bytes(cfg.H, cfg.I)
    for L in Ls:
        hs = torch.empty((cfg.E, nb), dtype=torch.uint8, pin_memory=True)
        hs.copy_(L["experts"].cpu())
        host_stores.append(hs)
        slots.append(torch.zeros((cfg.S, nb), dtype=torch.uint8, device=DEV))
        tables.append(moeq4.new_lfu_table())
    return host_stores, slots, tables


def test_streaming_matches_resident_bitwise_and_oracle_cache():
    cfg = TINY.with_(S=4)                  # small cache: many evictions
    n_layers, T = 3, 24
    Ls = _stack_layers(cfg, n_layers, seed=21)
    hs, slots, tables = _streaming_setup(cfg, Ls)
    ctx = ctx_for(cfg, 1)
    copy_stream = torch.cuda.Stream()
    st_layers = []
    for l, L in enumerate(Ls):
        moeq4.moe_lfu_init(ctx, tables[l], cfg.S)
        st_layers.append(moeq4.Layer(L["router_w"], L["router_scale"], L["router_bias"],
                                     L["shared"], None, hs[l], slots[l], tables[l]))
    res_layers = [moeq4.Layer.from_dict(L) for L in Ls]
    h0 = synth.tokens(T, cfg.H, seed=22, device=DEV)
    h_st, h_rs = h0.clone(), h0.clone()
    y_st = torch.empty((1, cfg.H), device=DEV)
    y_rs = torch.empty((1, cfg.H), device=DEV)
    so = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    for t in range(T):
        for l in range(n_layers):
            moeq4.moe_layer_decode(ctx, st_layers[l], h_st[t:t + 1], 1, y_st, slot_of=so,
                                   flags=moeq4.MOE_PRENORM, copy_stream=copy_stream)
            moeq4.moe_layer_decode(ctx, res_layers[l], h_rs[t:t + 1], 1, y_rs,
                                   flags=moeq4.MOE_PRENORM)
            torch.cuda.synchronize()
            assert torch.equal(y_st, y_rs), (t, l)
    assert torch.equal(h_st, h_rs)
    # oracle-forced replay: the oracle's own stream drives routing, and its
    # LFU model must predict the GPU cache exactly.
    Lns = [np_layer(L) for L in Ls]
    for l in range(n_layers):
        moeq4.moe_lfu_init(ctx, tables[l], cfg.S)
    caches = [oracle.LfuCache(cfg.S) for _ in range(n_layers)]
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    for t in range(T):
        h_or = np_of(h0)[t].copy()
        for l in range(n_layers):
            x_or = oracle.rmsnorm(h_or, cfg.rms_eps)
            ref = oracle.moe_layer(cfg, Lns[l], x_or)
            so_ref, _ = caches[l].token(ref["idx"])
            hg = torch.from_numpy(h_or.view(np.int16).copy()).view(torch.float16).to(DEV)[None]
            moeq4.moe_layer_decode(ctx, st_layers[l], hg, 1, y_st, idx, slot_of=so,
                                   flags=moeq4.MOE_PRENORM, copy_stream=copy_stream)
            torch.cuda.synchronize()
            assert idx[0].cpu().tolist() == ref["idx"].tolist()
            assert so[0].cpu().tolist() == so_ref.tolist()
            assert_y_close(y_st[0].cpu().numpy(), ref["y"])
            h_or = oracle.residual_add(h_or, ref["y"])
    for l in range(n_layers):
        tb = moeq4.read_lfu_table(tables[l])
        assert (tb.hits, tb.misses) == (int(caches[l].hits[0]), int(caches[l].misses[0]))
        assert list(tb.expert)[:cfg.S] == caches[l].expert.tolist()


def test_streaming_copy_failure_invalidates_table(monkeypatch):
    cfg = TINY
    Ls = _stack_layers(cfg, 1, seed=31)
    hs, slots, tables = _streaming_setup(cfg, Ls)
    monkeypatch.setenv("MOEQ4_FAIL_COPY_AT", "1")       # the second blob copy fails
    ctx = ctx_for(cfg, 1)
    moeq4.moe_lfu_init(ctx, tables[0], cfg.S)
    L = Ls[0]
    lay = moeq4.Layer(L["router_w"], L["router_scale"], None, L["shared"], None, hs[0],
                      slots[0], tables[0])
    x = synth.tokens(1, cfg.H, seed=1, device=DEV)
    y = torch.empty((1, cfg.H), device=DEV)
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_layer_decode(ctx, lay, x, 1, y, copy_stream=torch.cuda.Stream())
    assert ei.value.code == moeq4.MOE_ERR_CACHE_STATE
    torch.cuda.synchronize()
    assert moeq4.read_lfu_table(tables[0]).valid == 0
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_layer_decode(ctx, lay, x, 1, y, copy_stream=torch.cuda.Stream())
    assert ei.value.code == moeq4.MOE_ERR_CACHE_STATE


# -------------------------------------------------------------- validation ----

def test_argument_checks():
    cfg = TINY
    L = make_layer(cfg, seed=0)
    ctx = ctx_for(cfg, 2)
    x = synth.tokens(2, cfg.H, seed=0, device=DEV)
    y = torch.empty((2, cfg.H), device=DEV)
    lay = moeq4.Layer.from_dict(L)
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_layer_decode(ctx, lay, x, 3, y)
    assert ei.value.code == moeq4.MOE_ERR_UNSUPPORTED_SHAPE
    raw = torch.empty(cfg.H * 2 + 8, dtype=torch.uint8, device=DEV)
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_layer_decode(ctx, lay, raw[2:].data_ptr(), 1, y)
    assert ei.value.code == moeq4.MOE_ERR_ALIGNMENT
    st = moeq4.Layer(L["router_w"], L["router_scale"], None, L["shared"], None, None, None, None)
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_layer_decode(ctx, st, x, 1, y)
    assert ei.value.code == moeq4.MOE_ERR_INVALID_ARG


def test_smaller_context_keeps_larger_context_working():
    """Kernel shared-memory limits belong to the process: creating a context
    for a small shape after a large one must not shrink them under the large
    context (router, grouped kernels and the fused kernel all take more
    shared memory at the layer shape)."""
    big = ctx_for(LAYER, 4)
    small = ctx_for(TINY, 4)
    L = make_layer(LAYER, seed=12, bias_std=1.5)
    lay = moeq4.Layer.from_dict(L)
    Ln = np_layer(L)
    for T in (3, 1):
        x = synth.tokens(T, LAYER.H, seed=13 + T, device=DEV)
        y = torch.empty((T, LAYER.H), device=DEV)
        idx = torch.empty((T, LAYER.k), dtype=torch.int32, device=DEV)
        moeq4.moe_layer_decode(big, lay, x, T, y, idx)
        moeq4.moe_ctx_check(big)
        for t in range(T):
            ref = _oracle_layer(LAYER, Ln, np_of(x)[t])
            assert idx[t].cpu().tolist() == ref["idx"].tolist()
            assert_y_close(y[t].cpu().numpy(), ref["y"], f"T={T} token {t}")
    small.close()
    big.close()


def test_bounded_wait_gives_up_and_context_recovers(monkeypatch):
    """Failure detection without a GPU fault.  A streaming layer runs as three
    launches (router; shared expert; routed experts with the down rows), and
    the last waits for every gate/up item of the step, the shared launch's
    included.  The host withholds the shared launch (MOEQ4_WITHHOLD_SHARED_AT),
    so that wait cannot be met: with a 1 ms bound the kernel gives up,
    records MOE_ERR_TIMEOUT and leaves.  moe_ctx_check reports it and resets
    the counters; the next resident and streaming calls on the same context
    match the oracle."""
    cfg = TINY
    Ls = _stack_layers(cfg, 1, seed=41)
    hs, slots, tables = _streaming_setup(cfg, Ls)
    monkeypatch.setenv("MOEQ4_WITHHOLD_SHARED_AT", "0")
    ctx = ctx_for(cfg, 1)
    moeq4.moe_set_wait_ns(ctx, 1_000_000)
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_set_wait_ns(ctx, 10)
    assert ei.value.code == moeq4.MOE_ERR_INVALID_ARG
    moeq4.moe_lfu_init(ctx, tables[0], cfg.S)
    L = Ls[0]
    st = moeq4.Layer(L["router_w"], L["router_scale"], L["router_bias"], L["shared"], None, hs[0],
                     slots[0], tables[0])
    rs = moeq4.Layer.from_dict(L)
    cs = torch.cuda.Stream()
    x = synth.tokens(3, cfg.H, seed=42, device=DEV)
    y = torch.empty((1, cfg.H), device=DEV)
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    moeq4.moe_layer_decode(ctx, st, x[0:1], 1, y, copy_stream=cs)
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_ctx_check(ctx)
    assert ei.value.code == moeq4.MOE_ERR_TIMEOUT
    moeq4.moe_ctx_check(ctx)                          # cleared
    Ln = np_layer(L)
    for t, lay in ((1, rs), (2, st)):
        moeq4.moe_layer_decode(ctx, lay, x[t:t + 1], 1, y, idx, copy_stream=cs)
        moeq4.moe_ctx_check(ctx)
        ref = _oracle_layer(cfg, Ln, np_of(x)[t])
        assert idx[0].cpu().tolist() == ref["idx"].tolist()
        assert_y_close(y[0].cpu().numpy(), ref["y"], f"after recovery, token {t}")
    ctx.close()
