"""moe_router_topk_noalloc: the router entry point for callers that cannot
allocate device memory (its scratch is a static device array).

Collected last on purpose: it must pass alone in a fresh process and after
every other test.  Its outputs are checked against moe_router_topk, the
context-based entry point, on two calls in a row (the static scratch keeps
the previous call's contents): indices bit for bit, weights within the
tolerance of the other GPU tests.
"""
import numpy as np
import pytest
import torch

from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER, MoeConfig
from gpu_util import assert_y_close

RAGGED = MoeConfig(H=448, E=37, k=3, I=320, Is=192, S=7)


def _bad_shape(**kw):
    args = dict(n_experts=128, hidden=2816, top_k=8, renorm=1, T=1)
    args.update(kw)
    fake = 1 << 20                      # aligned, never dereferenced: the call must fail first
    with pytest.raises(moeq4.MoeError) as ei:
        moeq4.moe_router_topk_noalloc(args["n_experts"], args["hidden"], args["top_k"],
                                      args["renorm"], fake, fake, None, fake, args["T"],
                                      fake, fake, stream=0)
    return ei.value


@pytest.mark.parametrize("kw", [dict(T=65), dict(T=257, n_experts=8, top_k=2),
                                dict(hidden=6208), dict(T=0)])
def test_noalloc_rejects_sizes_beyond_the_static_scratch(kw):
    build.build()
    err = _bad_shape(**kw)
    assert err.code == moeq4.MOE_ERR_UNSUPPORTED_SHAPE
    if kw.get("T", 1) > 0:
        assert ("static scratch" in str(err)) == ("T" in kw)


def _router_inputs(cfg, T, seed, bias):
    d = synth.layer_weights(cfg, seed, 0, "cuda", bias_std=bias, experts=False)
    x = synth.tokens(T, cfg.H, seed=seed + 1, device="cuda")
    return d, x


def _both(cfg, ctx, d, x, T):
    idx_n = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
    w_n = torch.full((T, cfg.k), -1.0, dtype=torch.float32, device="cuda")
    moeq4.moe_router_topk_noalloc(cfg.E, cfg.H, cfg.k, cfg.renorm, d["router_w"],
                                  d["router_scale"], d["router_bias"], x, T, idx_n, w_n)
    idx_c = torch.empty_like(idx_n)
    w_c = torch.empty_like(w_n)
    moeq4.moe_router_topk(ctx, d["router_w"], d["router_scale"], d["router_bias"], x, T,
                          idx_c, w_c)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx_n.cpu().numpy(), idx_c.cpu().numpy())
    assert_y_close(w_n.cpu().numpy(), w_c.cpu().numpy().astype(np.float64), "topk_w")


@pytest.mark.gpu
@pytest.mark.parametrize("cfg,calls", [
    (LAYER, [(64, 11, 1.5), (3, 12, None)]),      # first call at the size limit T * E = 8192
    (RAGGED, [(9, 21, None), (5, 22, 0.7)]),
])
def test_noalloc_matches_router_on_two_calls_in_a_row(cfg, calls):
    build.build()
    moeq4.load()
    assert torch.cuda.is_available()
    ctx = moeq4.Context(cfg, max(T for T, _, _ in calls))
    for T, seed, bias in calls:
        d, x = _router_inputs(cfg, T, seed, bias)
        _both(cfg, ctx, d, x, T)
    ctx.close()
