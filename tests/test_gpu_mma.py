"""Tensor-core (tcgen05) buckets of the multi-token path against the oracle.

Multi-token steps group the (token, expert) pairs by expert; in a step of two
or more tokens a bucket of at least the configured size (and the shared
expert once T reaches it) runs on the tensor cores.  These tests force every
bucket of such steps onto that path (threshold 1, buckets of one pair up),
concentrate whole steps on eight experts (buckets of 130 pairs: tiles of 64,
64 and a ragged 2), and compare each token with the oracle and with the
CUDA-core path (threshold 0).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_expert_int8_b200 import build, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER, TINY, MoeConfig
from gpu_util import assert_y_close, make_layer, np_layer, np_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moeq4.load()
    assert torch.cuda.is_available()
    yield
    torch.cuda.synchronize()


def _run(cfg, L, x, T, tau):
    ctx = moeq4.Context(cfg, T)
    moeq4.moe_set_mma_min_tokens(ctx, tau)
    y = torch.empty((T, cfg.H), device=DEV)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    moeq4.moe_layer_decode(ctx, moeq4.Layer.from_dict(L), x, T, y, idx)
    moeq4.moe_ctx_check(ctx)
    return y.cpu().numpy(), idx.cpu().numpy()


def _check_tokens(cfg, L, x, y, idx, tokens):
    Ln = np_layer(L)
    xn = np_of(x)
    for t in tokens:
        ref = oracle.moe_layer(cfg, Ln, xn[t])
        assert idx[t].tolist() == ref["idx"].tolist(), f"token {t}"
        assert_y_close(y[t], ref["y"], f"token {t}")


def test_mma_threshold_setting():
    ctx = moeq4.Context(LAYER, 4)
    with pytest.raises(moeq4.MoeError) as e:
        moeq4.moe_set_mma_min_tokens(ctx, -1)
    assert e.value.code == moeq4.MOE_ERR_INVALID_ARG
    moeq4.moe_set_mma_min_tokens(ctx, 1)
    moeq4.moe_set_mma_min_tokens(ctx, 0)
    # hidden 320 is not a multiple of the 128-row tile: CUDA cores only
    small = MoeConfig(H=320, E=40, k=5, I=192, Is=128, S=11)
    ctx2 = moeq4.Context(small, 4)
    with pytest.raises(moeq4.MoeError) as e:
        moeq4.moe_set_mma_min_tokens(ctx2, 32)
    assert e.value.code == moeq4.MOE_ERR_UNSUPPORTED_SHAPE
    moeq4.moe_set_mma_min_tokens(ctx2, 0)


def test_mma_every_bucket_tiny():
    """Threshold 1: every routed bucket (1 to a few dozen pairs) and the shared
    expert (70 tokens: a full tile and a ragged 6) on the tensor cores."""
    cfg, T = TINY, 70
    L = make_layer(cfg, seed=21, bias_std=1.5)
    x = synth.tokens(T, cfg.H, seed=22, device=DEV)
    y_tc, idx_tc = _run(cfg, L, x, T, 1)
    y_cc, idx_cc = _run(cfg, L, x, T, 0)
    np.testing.assert_array_equal(idx_tc, idx_cc)
    _check_tokens(cfg, L, x, y_tc, idx_tc, range(T))
    for t in range(T):
        assert_y_close(y_tc[t], y_cc[t].astype(np.float64), f"tensor vs CUDA cores, token {t}")


@pytest.mark.parametrize("cfg,T", [(LAYER, 2), (LAYER, 3), (TINY, 2), (TINY, 5)])
def test_mma_smallest_steps_match_oracle_and_cuda_cores(cfg, T):
    """The smallest multi-token steps on the tensor cores: one-pair buckets
    (16-row tiles holding one or two tokens) and a shared expert of T tokens;
    every token against the oracle and against the CUDA-core path."""
    L = make_layer(cfg, seed=27 + T, bias_std=1.5)
    x = synth.tokens(T, cfg.H, seed=28 + T, device=DEV)
    y_tc, idx_tc = _run(cfg, L, x, T, 1)
    y_cc, idx_cc = _run(cfg, L, x, T, 0)
    np.testing.assert_array_equal(idx_tc, idx_cc)
    _check_tokens(cfg, L, x, y_tc, idx_tc, range(T))
    for t in range(T):
        assert_y_close(y_tc[t], y_cc[t].astype(np.float64), f"tensor vs CUDA cores, token {t}")


@pytest.mark.parametrize("T,sample", [(8, tuple(range(8))), (200, (0, 63, 64, 130, 199))])
def test_mma_layer_small_buckets(T, sample):
    """Layer shape, threshold 1: T = 8 (buckets of one or two pairs, each a
    16-row tile, and the shared expert's 8 tokens on the tensor cores) and
    T = 200 (every bucket, about a dozen pairs each, on the tensor cores; the
    shared expert in tiles of 64, 64, 64 and 8)."""
    cfg = LAYER
    L = make_layer(cfg, seed=23, bias_std=1.5)
    x = synth.tokens(T, cfg.H, seed=24, device=DEV)
    y, idx = _run(cfg, L, x, T, 1)
    _check_tokens(cfg, L, x, y, idx, sample)


def test_mma_layer_concentrated_buckets():
    """Layer shape, default threshold, T = 130, a router bias that sends every
    token to experts 0..7: eight routed buckets of 130 pairs and the shared
    expert, each as tiles of 64, 64 and 2 tokens."""
    cfg, T = LAYER, 130
    L = make_layer(cfg, seed=25, bias_std=None)
    bias = torch.zeros(cfg.E, dtype=torch.float32)
    bias[:cfg.k] = 1.0e4
    L["router_bias"] = bias.to(DEV)
    x = synth.tokens(T, cfg.H, seed=26, device=DEV)
    y, idx = _run(cfg, L, x, T, 32)
    assert (np.sort(idx, axis=1) == np.arange(cfg.k)).all()
    _check_tokens(cfg, L, x, y, idx, (0, 1, 63, 64, 127, 128, 129))
