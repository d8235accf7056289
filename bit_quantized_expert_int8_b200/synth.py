"""Seeded synthetic inputs for the MoE decode hot path.

This module is the one place that produces input bytes.  The CUDA library and
the CPU oracle both consume its output and neither calls the other; the
module holds none of the hot path's arithmetic (no dequantisation, routing,
FFN, cache or combine).  What it does hold is the data recipe:

* pre-quantisation weights ~ N(0, 0.02) for router, shared and routed experts;
* 4-bit affine group quantiser used only to *produce* test weights: per group
  of 64, scale = fp16((max - min) / 15), bias = fp16(min),
  code = clamp(round_half_even((w - bias) / scale), 0, 15) (scale 0 -> code 0),
  eight codes per uint32, lowest column in the lowest nibble;
* int8 router quantiser: scale = fp16(max|w| / 127),
  code = clamp(round_half_even(w / scale), -127, 127);
* activations ~ N(0, 1) rounded to fp16;
* per-expert router bias ~ N(0, 1.5) in fp32 for the skewed-popularity stack.

Every tensor is drawn from its own ``torch.Generator`` seeded by a hash of
(seed, layer, role, expert), so any expert can be regenerated alone.  The
generator runs on the device it is asked for; CPU and CUDA streams differ, so
a test that needs the same bytes on both sides generates once and copies.
"""
from __future__ import annotations

import torch

from .config import GROUP, WEIGHT_STD, MoeConfig

_MASK64 = (1 << 64) - 1


def seed_for(*keys: int) -> int:
    """63-bit seed from integer keys (splitmix64 finaliser over a fold)."""
    z = 0x9E3779B97F4A7C15
    for key in keys:
        z = (z ^ (int(key) & _MASK64)) & _MASK64
        z = (z + 0x9E3779B97F4A7C15) & _MASK64
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        z = z ^ (z >> 31)
    return z & ((1 << 63) - 1)


ROLE_ROUTER, ROLE_BIAS, ROLE_SHARED, ROLE_EXPERT, ROLE_TOKENS = 1, 2, 3, 4, 5


def randn(shape, seed: int, device="cpu", std: float = 1.0) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device,
                       dtype=torch.float32) * std


def quantize_q4(w: torch.Tensor):
    """Group-64 affine 4-bit quantiser (test-data producer).

    w float32 [R, K] -> (codes int32 [R, K/8] holding uint32 bit patterns,
    scale fp16 [R, K/64], bias fp16 [R, K/64]).
    """
    R, K = w.shape
    assert K % GROUP == 0
    g = w.reshape(R, K // GROUP, GROUP)
    mn = g.amin(-1)
    mx = g.amax(-1)
    s16 = ((mx - mn) / 15.0).to(torch.float16)
    b16 = mn.to(torch.float16)
    s = s16.float()[..., None]
    b = b16.float()[..., None]
    safe = torch.where(s > 0, s, torch.ones_like(s))
    q = torch.round((g - b) / safe)
    q = torch.where(s > 0, q, torch.zeros_like(q)).clamp_(0, 15).to(torch.int64)
    q = q.reshape(R, K // 8, 8)
    shifts = torch.arange(8, device=w.device, dtype=torch.int64) * 4
    word = (q << shifts).sum(-1)                      # < 2^32
    word = torch.where(word >= 2**31, word - 2**32, word).to(torch.int32)
    return word, s16, b16


def quantize_router(w: torch.Tensor):
    """int8 router quantiser (test-data producer): w [E, H] -> (int8, fp16)."""
    s16 = (w.abs().amax(-1) / 127.0).to(torch.float16)
    s = s16.float()[:, None]
    safe = torch.where(s > 0, s, torch.ones_like(s))
    q = torch.round(w / safe)
    q = torch.where(s > 0, q, torch.zeros_like(q)).clamp_(-127, 127)
    return q.to(torch.int8), s16


def blob_bytes(H: int, I: int) -> int:
    """Size of one tiled expert blob: I/16 gate/up tiles of 18 H bytes and
    H/16 down tiles of 9 I bytes."""
    return (I // 16) * 18 * H + (H // 16) * 9 * I


def _row_bytes(t: torch.Tensor) -> torch.Tensor:
    """[R, ...] tensor -> its bytes as uint8 [R, bytes per row]."""
    return t.contiguous().view(torch.uint8).reshape(t.shape[0], -1)


def pack_blob(qg, sg, bg, qd, sd, bd, H: int, I: int) -> torch.Tensor:
    """Tiled expert blob from the quantised gate/up matrix ([2I] rows: gate
    0..I-1, up I..2I-1) and down matrix ([H] rows).

    Gate/up tile t (intermediate indices 16t..16t+15), 18 H bytes: gate
    codes of the 16 rows, up codes of the 16 rows, gate scales, up scales,
    gate biases, up biases.  Down tile t (output rows 16t..16t+15), 9 I
    bytes: codes, scales, biases of the 16 rows.  Gate/up tiles first."""
    def gu(t):
        b = _row_bytes(t)                                   # [2I, n]
        return b.reshape(2, I // 16, 16, -1).permute(1, 0, 2, 3).reshape(I // 16, -1)

    def dn(t):
        return _row_bytes(t).reshape(H // 16, -1)
    tiles_gu = torch.cat([gu(qg), gu(sg), gu(bg)], dim=1)   # [I/16, 18 H]
    tiles_dn = torch.cat([dn(qd), dn(sd), dn(bd)], dim=1)   # [H/16, 9 I]
    return torch.cat([tiles_gu.reshape(-1), tiles_dn.reshape(-1)])


def expert_blob(H: int, I: int, seed: int, device="cpu",
                std: float = WEIGHT_STD, out: torch.Tensor | None = None):
    """One expert (gate, up, down) drawn N(0, std) and quantised into a blob."""
    w_gu = randn((2 * I, H), seed_for(seed, 0), device, std)
    w_dn = randn((H, I), seed_for(seed, 1), device, std)
    qg, sg, bg = quantize_q4(w_gu)
    qd, sd, bd = quantize_q4(w_dn)
    blob = pack_blob(qg, sg, bg, qd, sd, bd, H, I)
    assert blob.numel() == blob_bytes(H, I)
    if out is None:
        return blob
    out.copy_(blob)
    return out


def layer_weights(cfg: MoeConfig, seed: int, layer: int = 0, device="cpu",
                  bias_std: float | None = None, experts: bool = True):
    """All weights of one MoE layer.

    Returns dict: router_w int8 [E,H], router_scale fp16 [E],
    router_bias fp32 [E] or None, shared uint8 [blob(Is)],
    experts uint8 [E, blob(I)] (omitted when experts=False).
    """
    H, E = cfg.H, cfg.E
    wr = randn((E, H), seed_for(seed, layer, ROLE_ROUTER), device, WEIGHT_STD)
    rq, rs = quantize_router(wr)
    d = dict(router_w=rq, router_scale=rs, router_bias=None)
    if bias_std is not None:
        d["router_bias"] = randn((E,), seed_for(seed, layer, ROLE_BIAS),
                                 device, bias_std)
    d["shared"] = expert_blob(H, cfg.Is, seed_for(seed, layer, ROLE_SHARED),
                              device)
    if experts:
        nb = blob_bytes(H, cfg.I)
        ex = torch.empty((E, nb), dtype=torch.uint8, device=device)
        for e in range(E):
            expert_blob(H, cfg.I, seed_for(seed, layer, ROLE_EXPERT, e),
                        device, out=ex[e])
        d["experts"] = ex
    return d


def routed_expert(cfg: MoeConfig, seed: int, layer: int, e: int, device="cpu"):
    """Regenerate routed expert e of a layer alone (same bytes as in
    ``layer_weights`` on the same device)."""
    return expert_blob(cfg.H, cfg.I, seed_for(seed, layer, ROLE_EXPERT, e),
                       device)


def tokens(T: int, H: int, seed: int, device="cpu", stream: int = 0):
    """T activation rows ~ N(0, 1) rounded to fp16."""
    return randn((T, H), seed_for(seed, ROLE_TOKENS, stream), device,
                 1.0).to(torch.float16)


def routing_sequence(T: int, E: int, k: int, seed: int, zipf: float = 1.1):
    """Synthetic top-k routings for cache tests: T rows of k distinct experts
    drawn without replacement with Zipf-like popularity (rank r has weight
    r^-zipf over a seeded permutation of the experts)."""
    g = torch.Generator()
    g.manual_seed(seed_for(seed, 77))
    perm = torch.randperm(E, generator=g)
    rank_w = torch.arange(1, E + 1, dtype=torch.float64) ** (-zipf)
    w = torch.empty(E, dtype=torch.float64)
    w[perm] = rank_w
    rows = torch.multinomial(w.expand(T, E), k, replacement=False,
                             generator=g)
    return rows.to(torch.int32)


# ------------------------------------------------------- hard activations --
# Token rows for edge-case parity tests: magnitudes and shapes that the N(0, 1)
# workload never produces.  Like everything here they are plain seeded data.

def outlier_tokens(T: int, H: int, seed: int, device="cpu", factor: float = 1000.0,
                   every: int = 4, offset: int = 17):
    """N(0, 1) rows in which channel `offset` of every `every`-th 64-column
    group is `factor` times larger: groups whose one channel dwarfs the other
    63 (outlier channels), rounded to fp16."""
    x = randn((T, H), seed_for(seed, ROLE_TOKENS, 101), device, 1.0)
    ch = torch.arange(offset, H, GROUP * every, device=device)
    x[:, ch] *= factor
    return x.clamp(-65504.0, 65504.0).to(torch.float16)


def student_t_tokens(T: int, H: int, seed: int, device="cpu", df: int = 3):
    """Heavy-tailed rows: Student-t with `df` degrees of freedom,
    z / sqrt(chi2_df / df) from seeded normals, rounded to fp16."""
    z = randn((T, H), seed_for(seed, ROLE_TOKENS, 102), device, 1.0)
    c = randn((df, T, H), seed_for(seed, ROLE_TOKENS, 103), device, 1.0)
    t = z / torch.sqrt((c * c).sum(0) / df)
    return t.clamp(-65504.0, 65504.0).to(torch.float16)


def extreme_tokens(T: int, H: int, seed: int, device="cpu"):
    """N(0, 1) rows with, at seeded positions of every row, the fp16 extremes:
    +-65504, the smallest subnormal (+-2^-24), the largest subnormal
    (1023 * 2^-24), a mid subnormal, and zeros (including -0)."""
    x = randn((T, H), seed_for(seed, ROLE_TOKENS, 104), device, 1.0).to(torch.float16)
    specials = torch.tensor([65504.0, -65504.0, 2.0 ** -24, -(2.0 ** -24), 1023 * 2.0 ** -24,
                             -(517 * 2.0 ** -24), 0.0, -0.0], dtype=torch.float16)
    g = torch.Generator(device="cpu")
    g.manual_seed(seed_for(seed, ROLE_TOKENS, 105))
    for t in range(T):
        pos = torch.randperm(H, generator=g)[:3 * specials.numel()]
        x[t, pos.to(device)] = specials.repeat(3).to(device)
    return x
