"""GPU parity of the single-token fused layer kernel (the decode hot path).

T = 1 resident calls of moe_layer_decode and moe_stack_decode run the fused
kernel; these tests cover its template variants, ragged router items, the
in-kernel RMSNorm and residual update, bounded-wait status reporting, and the
30-layer stack in the configuration the benchmark times, checked layer by
layer against the oracle on the oracle's own residual stream.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER, TINY, MoeConfig
from gpu_util import assert_half_close, assert_y_close, make_layer, np_layer, np_of

pytestmark = pytest.mark.gpu
DEV = "cuda"

RAGGED = MoeConfig(H=448, E=37, k=3, I=320, Is=192, S=7)        # E % 8 != 0
WIDE = MoeConfig(H=3072, E=64, k=8, I=1024, Is=1024, S=16)      # 2 down chunks per lane


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moeq4.load()
    yield
    torch.cuda.synchronize()


def to_dev16(h16_np):
    return torch.from_numpy(h16_np.view(np.int16).copy()).view(torch.float16).to(DEV)


@pytest.mark.parametrize("cfg,bias", [(TINY, None), (RAGGED, 1.0), (WIDE, 0.5), (LAYER, 1.5)])
def test_fused_layer_parity(cfg, bias):
    L = make_layer(cfg, seed=5, bias_std=bias)
    ctx = moeq4.Context(cfg, 1)
    lay = moeq4.Layer.from_dict(L)
    Ln = np_layer(L)
    y = torch.empty((1, cfg.H), device=DEV)
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((1, cfg.k), device=DEV)
    for s in range(3):
        x = synth.tokens(1, cfg.H, seed=40 + s, device=DEV)
        moeq4.moe_layer_decode(ctx, lay, x, 1, y, idx, w)
        moeq4.moe_ctx_check(ctx)
        ref = oracle.moe_layer(cfg, Ln, np_of(x)[0])
        assert idx[0].cpu().tolist() == ref["idx"].tolist()
        np.testing.assert_allclose(w[0].cpu().numpy(), ref["w"], rtol=2e-6, atol=1e-7)
        assert_y_close(y[0].cpu().numpy(), ref["y"], f"{cfg} token {s}")


@pytest.mark.parametrize("cfg,boundary_tie", [(RAGGED, False), (WIDE, False), (LAYER, True)])
def test_fused_router_ties_and_near_ties(cfg, boundary_tie):
    """Crafted router rows: an exact tie among the picks, two logits that
    differ only far below the top-k's coarse key (the larger one has the
    higher index; with k = 3 they compete for the last place), and, when
    boundary_tie, an exact tie across the k-th place."""
    L = make_layer(cfg, seed=9)
    x = synth.tokens(1, cfg.H, seed=10, device=DEV)
    sgn = torch.sign(x[0].float()).to(torch.int8)
    xa = x[0].float().abs()
    c_small = int(torch.where(xa > 0, xa, torch.full_like(xa, 1e9)).argmin())
    Wr = L["router_w"].clone()
    sc = L["router_scale"].clone()
    rows_a = [3, 11]                                   # exact tie, value 100
    rows_d = [5, 9]                                    # near tie, value 80 (row 9 larger)
    n_b = max(0, cfg.k - 4 + (1 if boundary_tie else 0))
    rows_b = list(range(12, 12 + n_b))                 # exact tie, value 50
    for r in rows_a:
        Wr[r] = sgn * 100
    for r in rows_d:
        Wr[r] = sgn * 80
    Wr[9, c_small] = sgn[c_small] * 81
    for r in rows_b:
        Wr[r] = sgn * 50
    for r in rows_a + rows_d + rows_b:
        sc[r] = sc[0]
    L2 = dict(L, router_w=Wr, router_scale=sc)
    ctx = moeq4.Context(cfg, 1)
    lay = moeq4.Layer.from_dict(L2)
    y = torch.empty((1, cfg.H), device=DEV)
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((1, cfg.k), device=DEV)
    moeq4.moe_layer_decode(ctx, lay, x, 1, y, idx, w)
    moeq4.moe_ctx_check(ctx)
    ref = oracle.moe_layer(cfg, np_layer(L2), np_of(x)[0])
    expect = (rows_a + [9, 5] + rows_b)[:cfg.k]
    assert ref["idx"].tolist() == expect
    assert idx[0].cpu().tolist() == expect
    np.testing.assert_allclose(w[0].cpu().numpy(), ref["w"], rtol=2e-6, atol=1e-7)
    assert_y_close(y[0].cpu().numpy(), ref["y"], f"{cfg} ties")


def test_fused_prenorm_single_token():
    cfg = LAYER
    L = make_layer(cfg, seed=6, bias_std=1.5)
    ctx = moeq4.Context(cfg, 1)
    lay = moeq4.Layer.from_dict(L)
    Ln = np_layer(L)
    h = (synth.tokens(1, cfg.H, seed=7, device=DEV).float() * 2.5).half()
    h[0, :4] = torch.tensor([300.0, 6e-8, -1e-4, 0.0], dtype=torch.float16)
    h0 = np_of(h)[0].copy()
    y = torch.empty((1, cfg.H), device=DEV)
    xn = torch.empty((1, cfg.H), dtype=torch.float16, device=DEV)
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    moeq4.moe_layer_decode(ctx, lay, h, 1, y, idx, x_norm=xn, flags=moeq4.MOE_PRENORM)
    moeq4.moe_ctx_check(ctx)
    x_ref = oracle.rmsnorm(h0, cfg.rms_eps)
    np.testing.assert_array_equal(np_of(xn)[0], x_ref)
    ref = oracle.moe_layer(cfg, Ln, x_ref)
    assert idx[0].cpu().tolist() == ref["idx"].tolist()
    assert_y_close(y[0].cpu().numpy(), ref["y"])
    assert_half_close(np_of(h)[0], oracle.residual_add(h0, ref["y"]))


def test_fused_repeatable_bitwise():
    """Same input, many launches (alternating counters, epochs): identical bits."""
    cfg = LAYER
    L = make_layer(cfg, seed=8)
    ctx = moeq4.Context(cfg, 1)
    lay = moeq4.Layer.from_dict(L)
    x = synth.tokens(1, cfg.H, seed=9, device=DEV)
    y0 = torch.empty((1, cfg.H), device=DEV)
    y = torch.empty((1, cfg.H), device=DEV)
    moeq4.moe_layer_decode(ctx, lay, x, 1, y0)
    for _ in range(25):
        moeq4.moe_layer_decode(ctx, lay, x, 1, y)
    moeq4.moe_ctx_check(ctx)
    assert torch.equal(y, y0)


def _oracle_layer_sparse(cfg, Ld, x16):
    """Oracle layer that copies only the experts the oracle itself selects
    (the full stack does not fit comfortably in host memory)."""
    Wr = np_of(Ld["router_w"]); sc = np_of(Ld["router_scale"])
    rb = None if Ld["router_bias"] is None else np_of(Ld["router_bias"])
    lg = oracle.router_logits(Wr, sc, rb, x16, cfg.E, cfg.H)
    idx = oracle.topk(lg, cfg.k)
    w = oracle.topk_weights(oracle.softmax(lg), idx, cfg.renorm)
    xd = x16.view(np.float16).astype(np.float64)
    ys, _ = oracle.expert_ffn(np_of(Ld["shared"]), cfg.H, cfg.Is, xd, cfg.gelu)
    yr = np.stack([oracle.expert_ffn(np_of(Ld["experts"][int(e)]), cfg.H, cfg.I, xd, cfg.gelu)[0]
                   for e in idx])
    return idx, oracle.combine(ys, yr, w)


def test_stack_full_size_in_bench_configuration():
    """30 Gemma-like layers (13 GB), decoded as the benchmark does; the graph
    equals layer-by-layer calls bit for bit, and every layer matches the
    oracle on the oracle's own residual stream (sampled tokens)."""
    cfg = LAYER
    n_layers, T = 30, 3
    layers = [synth.layer_weights(cfg, 0, l, DEV, bias_std=1.5) for l in range(n_layers)]
    objs = [moeq4.Layer.from_dict(d) for d in layers]
    h0 = synth.tokens(T, cfg.H, seed=1, device=DEV)
    ctx = moeq4.Context(cfg, 1)
    h_stack = h0.clone()
    y_last = torch.empty((T, cfg.H), device=DEV)
    moeq4.moe_stack_decode(ctx, objs, h_stack, T, y_last)
    moeq4.moe_ctx_check(ctx)
    h_ref = h0.clone()
    y = torch.empty((1, cfg.H), device=DEV)
    for t in range(T):
        for lay in objs:
            moeq4.moe_layer_decode(ctx, lay, h_ref[t:t + 1], 1, y, flags=moeq4.MOE_PRENORM)
    moeq4.moe_ctx_check(ctx)
    assert torch.equal(h_stack, h_ref)
    assert torch.equal(y_last[T - 1], y[0])
    # oracle-forced, token 0: every layer on the oracle's own stream
    xn = torch.empty((1, cfg.H), dtype=torch.float16, device=DEV)
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device=DEV)
    h_or = np_of(h0)[0].copy()
    for l in range(n_layers):
        x_or = oracle.rmsnorm(h_or, cfg.rms_eps)
        ridx, ry = _oracle_layer_sparse(cfg, layers[l], x_or)
        hg = to_dev16(h_or)[None]
        moeq4.moe_layer_decode(ctx, objs[l], hg, 1, y, idx, x_norm=xn, flags=moeq4.MOE_PRENORM)
        moeq4.moe_ctx_check(ctx)
        np.testing.assert_array_equal(np_of(xn)[0], x_or)
        assert idx[0].cpu().tolist() == ridx.tolist(), l
        assert_y_close(y[0].cpu().numpy(), ry, f"layer {l}")
        h_or = oracle.residual_add(h_or, ry)
