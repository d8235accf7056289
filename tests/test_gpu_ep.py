"""Expert-parallel device steps on the GPU against the oracle.

One GPU here, so several ranks are emulated by one process: each rank's
device steps run in turn and the host moves the rows between them exactly as
the all-to-alls of `ep_layer` would (no kernel waits on another).  The
collective path itself runs over an NCCL group of one rank, and over gloo
with two and four ranks in the CPU suite.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from bit_quantized_expert_int8_b200 import build, ep, moeq4, synth
from bit_quantized_expert_int8_b200.config import LAYER
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


def _backend(ctx, cfg, L, rank, world):
    epr = cfg.E // world
    return ep.CudaEpBackend(ctx, cfg, L["router_w"], L["router_scale"], L["router_bias"], L["shared"],
                            L["experts"][rank * epr:(rank + 1) * epr], DEV)


@pytest.mark.parametrize("n_ranks", [1, 2, 4, 8])
def test_ep_dispatch_matches_stable_sort(n_ranks):
    cfg, T = LAYER, 40
    ctx = moeq4.Context(cfg, T)
    g = torch.Generator().manual_seed(7 + n_ranks)
    idx = torch.randint(0, cfg.E, (T, cfg.k), generator=g, dtype=torch.int32).to(DEV)
    x = synth.tokens(T, cfg.H, seed=9, device=DEV)
    P = T * cfg.k
    send_x = torch.empty((P, cfg.H), dtype=torch.float16, device=DEV)
    send_e = torch.empty(P, dtype=torch.int32, device=DEV)
    order = torch.empty(P, dtype=torch.int32, device=DEV)
    counts = torch.empty(n_ranks, dtype=torch.int32, device=DEV)
    moeq4.moe_ep_dispatch(ctx, idx, T, n_ranks, x, send_x, send_e, order, counts)
    moeq4.moe_ctx_check(ctx)
    flat = idx.cpu().numpy().reshape(-1)
    epr = cfg.E // n_ranks
    ref_order = np.concatenate([np.nonzero(flat // epr == d)[0] for d in range(n_ranks)])
    assert counts.cpu().tolist() == [int((flat // epr == d).sum()) for d in range(n_ranks)]
    assert np.array_equal(order.cpu().numpy(), ref_order)
    assert np.array_equal(send_e.cpu().numpy(), flat[ref_order] % epr)
    assert torch.equal(send_x, x[torch.from_numpy(ref_order // cfg.k).to(DEV)])
    # and back: rows in send order return to pair order
    y_sorted = torch.randn((P, cfg.H), device=DEV)
    y_pairs = torch.empty_like(y_sorted)
    moeq4.moe_ep_unpermute(ctx, y_sorted, order, P, y_pairs)
    assert torch.equal(y_pairs[order.long()], y_sorted)


def test_ep_dispatch_rejects_bad_shapes():
    ctx = moeq4.Context(LAYER, 4)
    t = torch.zeros(64, dtype=torch.int32, device=DEV)
    x = torch.zeros((4, LAYER.H), dtype=torch.float16, device=DEV)
    with pytest.raises(moeq4.MoeError) as e:
        moeq4.moe_ep_dispatch(ctx, t, 4, 3, x, x, t, t, t)        # 3 does not divide 128
    assert e.value.code == moeq4.MOE_ERR_UNSUPPORTED_SHAPE
    # more rows than the context holds: max_tokens 4 holds 4 * 9 / 2 = 18
    with pytest.raises(moeq4.MoeError) as e:
        moeq4.moe_ffn_rows(ctx, x, 4, t, 19, x, x)
    assert e.value.code == moeq4.MOE_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("R,tau", [(20, 0), (20, 1), (100, 1)])
def test_ffn_rows_matches_oracle(R, tau):
    """Rows on the CUDA-core grouped kernels (tensor-core threshold 0) and on
    tcgen05 (threshold 1); 16 local experts with uneven row counts (some
    none).  A context of ceil(2 R / (k + 1)) tokens is the smallest that holds
    R rows."""
    cfg = LAYER
    L = make_layer(cfg, seed=51)
    ctx = moeq4.Context(cfg, -(-2 * R // (cfg.k + 1)))
    moeq4.moe_set_mma_min_tokens(ctx, tau)
    n_local = 16
    g = torch.Generator().manual_seed(R)
    rows_e = torch.randint(0, n_local - 3, (R,), generator=g, dtype=torch.int32).to(DEV)
    x = synth.tokens(R, cfg.H, seed=52, device=DEV)
    y = torch.empty((R, cfg.H), device=DEV)
    local = L["experts"][32:32 + n_local]
    moeq4.moe_ffn_rows(ctx, local, n_local, rows_e, R, x, y)
    moeq4.moe_ctx_check(ctx)
    xs = np_of(x).view(np.float16).astype(np.float64)
    ln = np_of(local)
    yc = y.cpu().numpy()
    for r in range(R):
        ref = oracle.expert_ffn(ln[int(rows_e[r])], cfg.H, cfg.I, xs[r], cfg.gelu)[0]
        assert_y_close(yc[r], ref, f"row {r}")


@pytest.mark.parametrize("T", [1, 2, 37])
def test_shared_ffn_matches_oracle(T):
    """moe_shared_ffn: T = 1 on the CUDA-core grouped kernels, T = 2 and 37 on
    tcgen05 (tiles of 16 and 64 rows), every row against the oracle."""
    cfg = LAYER
    L = make_layer(cfg, seed=56)
    ctx = moeq4.Context(cfg, T)
    x = synth.tokens(T, cfg.H, seed=57 + T, device=DEV)
    y = torch.empty((T, cfg.H), device=DEV)
    moeq4.moe_shared_ffn(ctx, L["shared"], x, T, y)
    moeq4.moe_ctx_check(ctx)
    xs = np_of(x).view(np.float16).astype(np.float64)
    sh = np_of(L["shared"])
    yc = y.cpu().numpy()
    for t in range(T):
        ref = oracle.expert_ffn(sh, cfg.H, cfg.Is, xs[t], cfg.gelu)[0]
        assert_y_close(yc[t], ref, f"row {t}")


def test_ep_layer_emulated_four_ranks():
    """Four ranks of 32 experts each on one GPU, 40, 8, 64 and 1 tokens: every
    rank's device steps in turn, rows moved between them on the host in the
    order of the all-to-alls."""
    cfg = LAYER
    L = make_layer(cfg, seed=53, bias_std=1.5)
    Ts = (40, 8, 64, 1)
    world = len(Ts)
    ctxs = [moeq4.Context(cfg, 2 * sum(Ts)) for _ in range(world)]   # any routing fits
    bes = [_backend(ctxs[r], cfg, L, r, world) for r in range(world)]
    xs = [synth.tokens(T, cfg.H, seed=60 + r, device=DEV) for r, T in enumerate(Ts)]
    st = []
    for r in range(world):
        idx, w = bes[r].route(xs[r], Ts[r])
        send_x, send_e, order, counts = bes[r].dispatch(xs[r], idx, Ts[r], world)
        st.append(dict(idx=idx, w=w, send_x=send_x, send_e=send_e, order=order, counts=counts,
                       starts=np.concatenate([[0], np.cumsum(counts)])))
    # rows for rank d: from every source rank s, in rank order
    y_out = [None] * world
    back = [dict() for _ in range(world)]
    for d in range(world):
        parts_x = [st[s]["send_x"][st[s]["starts"][d]:st[s]["starts"][d + 1]] for s in range(world)]
        parts_e = [st[s]["send_e"][st[s]["starts"][d]:st[s]["starts"][d + 1]] for s in range(world)]
        recv_x = torch.cat(parts_x).contiguous()
        recv_e = torch.cat(parts_e).contiguous()
        R = recv_x.shape[0]
        y = bes[d].ffn_rows(recv_e, recv_x, R)
        o = 0
        for s in range(world):
            n = parts_x[s].shape[0]
            back[s][d] = y[o:o + n]
            o += n
    for s in range(world):
        y_back = torch.cat([back[s][d] for d in range(world)]).contiguous()
        P = Ts[s] * cfg.k
        y_pairs = bes[s].unpermute(y_back, st[s]["order"], P)
        y_sh = bes[s].shared(xs[s], Ts[s])
        y_out[s] = bes[s].combine(y_pairs, y_sh, st[s]["w"], Ts[s]).cpu().numpy()
    for c in ctxs:
        moeq4.moe_ctx_check(c)
    Ln = np_layer(L)
    for s in range(world):
        x16 = np_of(xs[s])
        for t in sorted({0, Ts[s] // 2, Ts[s] - 1}):
            ref = oracle.moe_layer(cfg, Ln, x16[t])
            assert st[s]["idx"][t].cpu().tolist() == ref["idx"].tolist(), f"rank {s} token {t}"
            assert_y_close(y_out[s][t], ref["y"], f"rank {s} token {t}")


def _nccl_worker(port, out):
    """Child process: `ep_layer` over an NCCL group of one rank."""
    try:
        torch.cuda.set_device(0)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
        try:
            moeq4.load()
            cfg, T = LAYER, 36
            L = make_layer(cfg, seed=54)
            ctx = moeq4.Context(cfg, 2 * T)          # the T * k received rows fit
            x = synth.tokens(T, cfg.H, seed=55, device=DEV)
            y, idx = ep.ep_layer(_backend(ctx, cfg, L, 0, 1), x, T)
            torch.cuda.synchronize()
            moeq4.moe_ctx_check(ctx)
            Ln = np_layer(L)
            x16 = np_of(x)
            yc = y.cpu().numpy()
            for t in (0, 17, 35):
                ref = oracle.moe_layer(cfg, Ln, x16[t])
                assert idx[t].cpu().tolist() == ref["idx"].tolist(), f"token {t}: routing"
                assert_y_close(yc[t], ref["y"], f"token {t}")
            out["result"] = "ok"
        finally:
            dist.barrier()
            dist.destroy_process_group()
    except Exception as e:                            # reported to the parent
        out["result"] = repr(e)


def test_ep_layer_nccl_one_rank():
    """`ep_layer` with its collectives over an NCCL group of one rank (in a
    child process, which owns the process group from start to end)."""
    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        p = ctx.Process(target=_nccl_worker, args=(port, out))
        p.start()
        p.join(timeout=600)
        if p.is_alive():
            p.kill()
        res = dict(out)
    assert res.get("result") == "ok", (res, p.exitcode)
