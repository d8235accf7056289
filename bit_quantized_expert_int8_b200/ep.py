"""Expert-parallel MoE layer over the ranks of a process group.

The experts of a layer are partitioned over the N ranks (rank r owns experts
r * E / N .. (r + 1) * E / N - 1); the router, the shared expert and the
combine are replicated, and every rank routes its own tokens.  One layer of a
rank's T tokens:

1. route: top-k of the exact router logits (``moe_router_topk``);
2. dispatch: the T * k (token, expert) pairs sorted by the rank that owns the
   expert, their x rows packed in that order (``moe_ep_dispatch``);
3. all-to-all of the pair counts, then of the x rows and expert indices;
4. each rank applies its experts to the rows it received (``moe_ffn_rows``:
   the grouped / tensor-core kernels, one expert read once for all its rows);
5. all-to-all of the output rows back to the ranks they came from;
6. rows back in pair order (``moe_ep_unpermute``), the shared expert
   (``moe_shared_ffn``) and the fixed-order combine (``moe_combine``).

The pages run one process on one machine (the per-expert FFN of their
pipeline, step 2-3 of section 04 of "Gemma 4 26B : Comment faire tourner un
LLM en 2 Go de RAM"); this is the scale-out reading of that step for GPUs
joined by NVLink, with the exchanges on torch.distributed (NCCL on GPUs).
Each device step is a call of the C ABI (``CudaEpBackend``); the module only
moves tensors between the calls and the collectives.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import moeq4


def _a2a_rows(out, inp, out_counts, in_counts, group=None):
    """All-to-all of row blocks: inp holds in_counts[r] rows for rank r in rank
    order; out receives out_counts[r] rows from rank r.  fp16 rows (an even
    number of columns) travel as int32 pairs: the same bits, in a type every
    backend moves."""
    if out.dtype == torch.float16:
        out, inp = out.view(torch.int32), inp.view(torch.int32)
    dist.all_to_all_single(out, inp, output_split_sizes=list(out_counts),
                           input_split_sizes=list(in_counts), group=group)


def ep_layer(backend, x, T: int, group=None):
    """One expert-parallel MoE layer of this rank's T tokens (x [T, H] fp16 on
    the backend's device).  Every rank of the group calls it (with its own T).
    Returns (y [T, H] fp32, topk_idx [T, k])."""
    world = dist.get_world_size(group)
    H, k, dev = backend.H, backend.k, backend.device
    idx, w = backend.route(x, T)
    send_x, send_e, order, counts = backend.dispatch(x, idx, T, world)
    cnt = torch.tensor(counts, dtype=torch.int64, device=dev)
    rcnt = torch.empty_like(cnt)
    dist.all_to_all_single(rcnt, cnt, group=group)
    rcounts = [int(v) for v in rcnt.tolist()]
    R = sum(rcounts)
    recv_x = torch.empty((R, H), dtype=send_x.dtype, device=dev)
    recv_e = torch.empty((R,), dtype=send_e.dtype, device=dev)
    _a2a_rows(recv_x, send_x, rcounts, counts, group)
    _a2a_rows(recv_e, send_e, rcounts, counts, group)
    y_recv = backend.ffn_rows(recv_e, recv_x, R)
    P = T * k
    y_back = torch.empty((P, H), dtype=y_recv.dtype, device=dev)
    _a2a_rows(y_back, y_recv, counts, rcounts, group)
    y_pairs = backend.unpermute(y_back, order, P)
    y_sh = backend.shared(x, T)
    return backend.combine(y_pairs, y_sh, w, T), idx


class CudaEpBackend:
    """Device steps of one rank through the C ABI.

    ctx: a ``moeq4.Context`` whose max_tokens covers the rows this rank can
    receive: ``moe_ffn_rows`` takes up to max_tokens * (k + 1) / 2 rows, so
    2 * N * T when every pair of N ranks of T tokens may come here.
    local_experts: uint8 [E / N, blob] on the device, the experts this rank
    owns; router and shared weights are the full layer's."""

    def __init__(self, ctx, cfg, router_w, router_scale, router_bias, shared, local_experts,
                 device="cuda"):
        self.ctx, self.cfg = ctx, cfg
        self.H, self.k, self.device = cfg.H, cfg.k, torch.device(device)
        self.router_w, self.router_scale, self.router_bias = router_w, router_scale, router_bias
        self.shared_blob = shared
        self.local_experts = local_experts.contiguous()
        self.n_local = self.local_experts.shape[0]

    def route(self, x, T):
        idx = torch.empty((T, self.k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=self.device)
        moeq4.moe_router_topk(self.ctx, self.router_w, self.router_scale, self.router_bias, x, T,
                              idx, w)
        return idx, w

    def dispatch(self, x, idx, T, world):
        P = T * self.k
        send_x = torch.empty((P, self.H), dtype=torch.float16, device=self.device)
        send_e = torch.empty((P,), dtype=torch.int32, device=self.device)
        order = torch.empty((P,), dtype=torch.int32, device=self.device)
        counts = torch.empty((world,), dtype=torch.int32, device=self.device)
        moeq4.moe_ep_dispatch(self.ctx, idx, T, world, x, send_x, send_e, order, counts)
        return send_x, send_e, order, [int(v) for v in counts.tolist()]

    def ffn_rows(self, recv_e, recv_x, R):
        y = torch.empty((R, self.H), dtype=torch.float32, device=self.device)
        if R:
            moeq4.moe_ffn_rows(self.ctx, self.local_experts, self.n_local, recv_e, R, recv_x, y)
        return y

    def unpermute(self, y_back, order, P):
        y_pairs = torch.empty((P, self.H), dtype=torch.float32, device=self.device)
        moeq4.moe_ep_unpermute(self.ctx, y_back, order, P, y_pairs)
        return y_pairs

    def shared(self, x, T):
        y = torch.empty((T, self.H), dtype=torch.float32, device=self.device)
        moeq4.moe_shared_ffn(self.ctx, self.shared_blob, x, T, y)
        return y

    def combine(self, y_pairs, y_sh, w, T):
        y = torch.empty((T, self.H), dtype=torch.float32, device=self.device)
        moeq4.moe_combine(self.ctx, y_pairs, y_sh, w, T, y)
        return y
