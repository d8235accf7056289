"""moe_router_topk_noalloc: the router entry point for callers that cannot
allocate device memory (its scratch is a static device array).

Collected last on purpose: it must pass alone in a fresh process and after
every other test.  Its outputs are checked on two calls in a row (the static
scratch keeps the previous call's contents) against moe_router_topk, the
context-based entry point (indices and weights bit for bit: both run the same
exact integer dot and fixed-order epilogue), and against the CPU oracle
(indices bit for bit, weights within the tolerance the router parity tests
use).  Two more cases cover the kernel's shared-memory limit: a call at the
layer shape after a small-shape context was created, and a call at the
largest accepted hidden size with no context at all.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER, TINY, MoeConfig
from gpu_util import np_of

RAGGED = MoeConfig(H=448, E=37, k=3, I=320, Is=192, S=7)
WIDEST = MoeConfig(H=6144, E=16, k=2, I=64, Is=64, S=4)     # hidden at the entry point's limit


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
    d = synth.layer_weights(cfg, seed, 0, "cpu", bias_std=bias, experts=False)
    d = {k: (None if v is None else v.to("cuda")) for k, v in d.items()}
    x = synth.tokens(T, cfg.H, seed=seed + 1, device="cuda")
    return d, x


def _noalloc(cfg, d, x, T):
    idx = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, cfg.k), -1.0, dtype=torch.float32, device="cuda")
    moeq4.moe_router_topk_noalloc(cfg.E, cfg.H, cfg.k, cfg.renorm, d["router_w"],
                                  d["router_scale"], d["router_bias"], x, T, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


def _against_oracle(cfg, d, x, idx, w):
    Wr, sc = np_of(d["router_w"]), np_of(d["router_scale"])
    rb = np_of(d["router_bias"])
    xn = np_of(x)
    for t in range(xn.shape[0]):
        lg = oracle.router_logits(Wr, sc, rb, xn[t], cfg.E, cfg.H)
        ridx = oracle.topk(lg, cfg.k)
        assert idx[t].tolist() == ridx.tolist(), f"token {t}"
        rw = oracle.topk_weights(oracle.softmax(lg), ridx, cfg.renorm)
        np.testing.assert_allclose(w[t], rw, rtol=2e-6, atol=1e-7)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg,calls", [
    (LAYER, [(64, 11, 1.5), (3, 12, None)]),      # first call at the size limit T * E = 8192
    (RAGGED, [(9, 21, None), (5, 22, 0.7)]),
])
def test_noalloc_matches_router_and_oracle_on_two_calls_in_a_row(cfg, calls):
    build.build()
    moeq4.load()
    assert torch.cuda.is_available()
    ctx = moeq4.Context(cfg, max(T for T, _, _ in calls))
    for T, seed, bias in calls:
        d, x = _router_inputs(cfg, T, seed, bias)
        idx_n, w_n = _noalloc(cfg, d, x, T)
        idx_c = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
        w_c = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
        moeq4.moe_router_topk(ctx, d["router_w"], d["router_scale"], d["router_bias"], x, T,
                              idx_c, w_c)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx_n, idx_c.cpu().numpy())
        np.testing.assert_array_equal(w_n, w_c.cpu().numpy())
        _against_oracle(cfg, d, x, idx_n, w_n)
    ctx.close()


@pytest.mark.gpu
def test_noalloc_layer_shape_after_a_small_context():
    """A context of a small shape must not leave the router kernel unable to
    take the layer shape's shared memory in the entry point without one."""
    build.build()
    moeq4.load()
    small = moeq4.Context(TINY, 1)
    d, x = _router_inputs(LAYER, 2, 31, 1.5)
    idx, w = _noalloc(LAYER, d, x, 2)
    _against_oracle(LAYER, d, x, idx, w)
    small.close()


@pytest.mark.gpu
def test_noalloc_widest_hidden_without_a_context():
    build.build()
    moeq4.load()
    d, x = _router_inputs(WIDEST, 3, 41, 0.5)
    idx, w = _noalloc(WIDEST, d, x, 3)
    _against_oracle(WIDEST, d, x, idx, w)
