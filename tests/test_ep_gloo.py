"""Expert-parallel layer over two and four ranks (gloo, CPU).

`ep_layer` moves rows between the device steps of each rank with
all-to-alls; here every device step is done by the oracle (a test-only
backend), so the test checks the exchange itself: split sizes, send order,
return order, uneven token counts per rank, a rank that receives nothing.
Each token's output must equal the oracle's whole layer for that token.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bit_quantized_expert_int8_b200 import ep, synth
from bit_quantized_expert_int8_b200.config import TINY
from gpu_util import np_layer


class OracleBackend:
    """The device steps of one rank, computed by the oracle on the CPU."""

    device = torch.device("cpu")

    def __init__(self, cfg, L, rank, world):
        self.cfg, self.L = cfg, L
        self.H, self.k = cfg.H, cfg.k
        self.epr = cfg.E // world
        self.local = L["experts"][rank * self.epr:(rank + 1) * self.epr]

    def route(self, x, T):
        c = self.cfg
        x16 = x.view(torch.int16).numpy().view(np.uint16)
        idx = np.zeros((T, c.k), np.int32)
        w = np.zeros((T, c.k), np.float64)
        for t in range(T):
            lg = oracle.router_logits(self.L["router_w"], self.L["router_scale"], self.L["router_bias"],
                                      x16[t], c.E, c.H)
            idx[t] = oracle.topk(lg, c.k)
            w[t] = oracle.topk_weights(oracle.softmax(lg), idx[t], c.renorm)
        return torch.from_numpy(idx), torch.from_numpy(w)

    def dispatch(self, x, idx, T, world):
        flat = idx.numpy().reshape(-1)
        dest = flat // self.epr
        order = np.concatenate([np.nonzero(dest == d)[0] for d in range(world)]).astype(np.int32)
        counts = [int((dest == d).sum()) for d in range(world)]
        send_x = x[torch.from_numpy((order // self.k).astype(np.int64))].contiguous()
        send_e = torch.from_numpy((flat[order] % self.epr).astype(np.int32))
        return send_x, send_e, torch.from_numpy(order), counts

    def ffn_rows(self, recv_e, recv_x, R):
        c = self.cfg
        xs = recv_x.float().numpy().astype(np.float64)
        y = np.zeros((R, c.H), np.float64)
        for r in range(R):
            y[r] = oracle.expert_ffn(self.local[int(recv_e[r])], c.H, c.I, xs[r], c.gelu)[0]
        return torch.from_numpy(y)

    def unpermute(self, y_back, order, P):
        out = torch.empty_like(y_back)
        out[order.long()] = y_back
        return out

    def shared(self, x, T):
        c = self.cfg
        xs = x.float().numpy().astype(np.float64)
        return torch.from_numpy(np.stack([oracle.expert_ffn(self.L["shared"], c.H, c.Is, xs[t], c.gelu)[0]
                                          for t in range(T)]))

    def combine(self, y_pairs, y_sh, w, T):
        k = self.k
        yp, ys, wn = y_pairs.numpy(), y_sh.numpy(), w.numpy()
        return torch.from_numpy(np.stack([oracle.combine(ys[t], yp[t * k:(t + 1) * k], wn[t])
                                          for t in range(T)]))


def _layer(cfg, rank0_only):
    d = synth.layer_weights(cfg, 41, 0, "cpu", bias_std=1.5)
    if rank0_only:
        bias = torch.zeros(cfg.E, dtype=torch.float32)
        bias[:cfg.k] = 1.0e4                          # every pair to experts 0..k-1 (rank 0)
        d["router_bias"] = bias
    return np_layer(d)


def _worker(rank, world, port, Ts, rank0_only, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        cfg = TINY
        L = _layer(cfg, rank0_only)
        T = Ts[rank]
        x = synth.tokens(T, cfg.H, seed=300 + rank)
        y, idx = ep.ep_layer(OracleBackend(cfg, L, rank, world), x, T)
        x16 = x.view(torch.int16).numpy().view(np.uint16)
        worst = 0.0
        for t in range(T):
            ref = oracle.moe_layer(cfg, L, x16[t])
            assert idx[t].tolist() == ref["idx"].tolist(), f"rank {rank} token {t}: routing"
            worst = max(worst, float(np.abs(y[t].numpy() - ref["y"]).max()))
        out[rank] = ("ok", worst)
    except Exception as e:                            # reported to the parent
        out[rank] = ("fail", repr(e))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(world, Ts, rank0_only=False):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, Ts, rank0_only, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        for p in procs:
            if p.is_alive():
                p.kill()
        res = dict(out)
    assert sorted(res) == list(range(world)), res
    for r, (status, val) in res.items():
        assert status == "ok", f"rank {r}: {val}"
        assert val < 1e-12, f"rank {r}: max |y - oracle| = {val}"


def test_ep_two_ranks_uneven_tokens():
    """Rank 0 holds 3 tokens, rank 1 holds 5; experts 0..7 on rank 0, 8..15 on
    rank 1 (TINY: 16 experts, top-2)."""
    _run(2, (3, 5))


def test_ep_one_rank_receives_nothing():
    """Every pair goes to rank 0's experts: rank 1 sends all of its pairs and
    receives no rows."""
    _run(2, (4, 2), rank0_only=True)


def test_ep_four_ranks():
    """Four ranks of 4 experts each, 1 to 4 tokens per rank."""
    _run(4, (2, 3, 1, 4))
