"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks one oracle function against something it does not compute
itself: hand-built groups with known values, exact rational arithmetic,
textbook constants, library routines for special cases, closed forms and
brute force on tiny shapes.  A dropped term, a swapped operand, a wrong
nibble order or index fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_expert_int8_b200 import synth
from bit_quantized_expert_int8_b200.config import TINY, MoeConfig

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def h16(v):
    return np.array(v, dtype=np.float16).view(np.uint16)


# ---------------------------------------------------------------- fp16 -----

def test_half_to_double_matches_numpy_on_all_finite_halves():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    fin = np.isfinite(ref)
    got = np.array([oracle.half_to_double(int(b)) for b in bits[fin][::7]])
    np.testing.assert_array_equal(got, ref[fin][::7])


def test_double_to_half_round_to_nearest_even():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(2000) * 10.0 ** rng.integers(-9, 5, 2000),
        [0.0, -0.0, 65504.0, 65519.999, 65520.0, -65520.0, 2.0 ** -24,
         2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14 - 2.0 ** -26, 1.0 + 2.0 ** -11,
         1.0 + 3 * 2.0 ** -11, 2047.5, 2048.0 + 1.0, 1e-9],
    ])
    for v in vals:
        with np.errstate(over="ignore"):
            ref = int(np.array(v, dtype=np.float64).astype(np.float16).view(np.uint16))
        assert oracle.double_to_half(float(v)) == ref, v
    # ties go to even: 1 + 2^-11 lies halfway between 1 and 1 + 2^-10
    assert oracle.double_to_half(1.0 + 2.0 ** -11) == 0x3C00
    assert oracle.double_to_half(1.0 + 3 * 2.0 ** -11) == 0x3C02


# -------------------------------------------------------------- dequant ----

def _group(scale, bias, words):
    q = np.array(words, dtype=np.uint32)
    return q, h16([scale]), h16([bias])


def test_nibble_order_low_nibble_first():
    # 0x76543210 holds codes 0..7 from the lowest nibble up
    q = np.array([0x76543210] + [0] * 7, dtype=np.uint32)
    s, b = h16([1.0]), h16([0.0])
    got = [oracle.dequant(q, s, b, 64, 0, c) for c in range(8)]
    assert got == [0.0, 1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0]
    q = np.array([0xFEDCBA98] + [0] * 7, dtype=np.uint32)
    got = [oracle.dequant(q, s, b, 64, 0, c) for c in range(8)]
    assert got == [8.0, 9.0, 10.0, 11.0, 12.0, 13.0, 14.0, 15.0]


def test_affine_identity_scale_half_bias_minus_four():
    words = [0x76543210, 0xFEDCBA98] * 4
    q = np.array(words, dtype=np.uint32)
    s, b = h16([0.5]), h16([-4.0])
    for c in range(64):
        code = (c % 8) + 8 * ((c // 8) % 2)
        assert oracle.dequant(q, s, b, 64, 0, c) == -4.0 + 0.5 * code


def test_group_and_row_indexing():
    # 2 rows x 128 columns: 2 groups per row with distinct scale/bias
    K = 128
    q = np.full((2, K // 8), 0x11111111, dtype=np.uint32)      # every code 1
    s = h16([[1.0, 2.0], [4.0, 8.0]])
    b = h16([[0.0, 0.5], [0.25, -1.0]])
    want = {(0, 0): 1.0, (0, 63): 1.0, (0, 64): 2.5, (0, 127): 2.5,
            (1, 0): 4.25, (1, 64): 7.0, (1, 127): 7.0}
    for (r, c), v in want.items():
        assert oracle.dequant(q.ravel(), s.ravel(), b.ravel(), K, r, c) == v


# ----------------------------------------------------------------- GELU ----

def test_gelu_textbook_values_and_limits():
    # erf form equals g * Phi(g); Phi(1) = 0.841344746068543
    assert oracle.gelu(1.0, 1) == pytest.approx(0.8413447460685429, abs=1e-15)
    assert oracle.gelu(-1.0, 1) == pytest.approx(-0.15865525393145707, abs=1e-15)
    # tanh form at 1: 0.5 (1 + tanh(sqrt(2/pi) * 1.044715))
    assert oracle.gelu(1.0, 0) == pytest.approx(0.8411919906082768, abs=1e-15)
    for v in (0, 1):
        assert oracle.gelu(0.0, v) == 0.0
        assert oracle.gelu(30.0, v) == pytest.approx(30.0, rel=1e-15)
        assert abs(oracle.gelu(-30.0, v)) < 1e-12
    # the two forms agree to within the known 5e-4 bound on a grid
    for g in np.linspace(-6, 6, 241):
        assert abs(oracle.gelu(g, 0) - oracle.gelu(g, 1)) < 5e-4


# ------------------------------------------------------------------ FFN ----

def _dense(q, s, b, rows, K):
    """Brute force dequantisation of a whole q4 matrix with numpy."""
    q = q.reshape(rows, K // 8).astype(np.uint64)
    codes = (q[:, :, None] >> (np.arange(8, dtype=np.uint64) * 4)) & 0xF
    codes = codes.reshape(rows, K).astype(np.float64)
    sc = np.repeat(s.view(np.float16).reshape(rows, K // 64).astype(np.float64), 64, 1)
    bi = np.repeat(b.view(np.float16).reshape(rows, K // 64).astype(np.float64), 64, 1)
    return sc * codes + bi


def _tiled_rows(blob, H, I):
    """This test's own reading of the tiled expert blob: I/16 gate/up tiles of
    18 H bytes (gate codes, up codes, gate scales, up scales, gate biases, up
    biases, 16 rows each), then H/16 down tiles of 9 I bytes (codes, scales,
    biases of 16 rows).  Returns row-major byte arrays: gate/up codes,
    scales, biases ([2I] rows, gate first), down codes, scales, biases."""
    nt = I // 16
    gu = blob[: nt * 18 * H].reshape(nt, 18 * H)

    def rows(a, n):
        return np.ascontiguousarray(a.reshape(nt, 2, 16, n).transpose(1, 0, 2, 3).reshape(2 * I, n))
    q = rows(gu[:, : 16 * H], H // 2)
    sc = rows(gu[:, 16 * H: 17 * H], H // 32)
    bi = rows(gu[:, 17 * H:], H // 32)
    dn = blob[nt * 18 * H:].reshape(H // 16, 9 * I)
    dq = np.ascontiguousarray(dn[:, : 8 * I]).reshape(H, I // 2)
    ds = np.ascontiguousarray(dn[:, 8 * I: 8 * I + I // 2]).reshape(H, I // 32)
    db = np.ascontiguousarray(dn[:, 8 * I + I // 2:]).reshape(H, I // 32)
    return q, sc, bi, dq, ds, db


def _blob_parts(blob, H, I):
    q, sc, bi, dq, ds, db = _tiled_rows(blob, H, I)
    Wgu = _dense(q.view(np.uint32), sc.view(np.uint16), bi.view(np.uint16), 2 * I, H)
    Wd = _dense(dq.view(np.uint32), ds.view(np.uint16), db.view(np.uint16), H, I)
    return Wgu[:I], Wgu[I:], Wd


def _gelu_np(g, variant):
    if variant == 1:
        from scipy.special import erf
        return 0.5 * g * (1 + erf(g / math.sqrt(2)))
    return 0.5 * g * (1 + np.tanh(math.sqrt(2 / math.pi) * (g + 0.044715 * g ** 3)))


@pytest.mark.parametrize("H,I,variant", [(64, 64, 0), (256, 128, 0), (128, 192, 1)])
def test_expert_ffn_against_dense_brute_force(H, I, variant):
    blob = synth.expert_blob(H, I, seed=H * 7 + I).numpy()
    x = np.random.default_rng(H + I).standard_normal(H)
    y, h = oracle.expert_ffn(blob, H, I, x, variant)
    Wg, Wu, Wd = _blob_parts(blob, H, I)
    h_ref = _gelu_np(Wg @ x, variant) * (Wu @ x)
    y_ref = Wd @ h_ref
    np.testing.assert_allclose(h, h_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-14)


def test_expert_ffn_closed_forms():
    H, I = 64, 64
    blob = np.zeros(synth.blob_bytes(H, I), np.uint8)
    x = np.random.default_rng(3).standard_normal(H)
    # all-zero weights (scale 0, bias 0) -> h = 0, y = 0
    y, h = oracle.expert_ffn(blob, H, I, x)
    assert not y.any() and not h.any()
    # every weight equal: gate = up = w0 * sum(x); down weights all w1
    w0, w1 = 0.25, -0.5
    nt = I // 16
    gu = blob[: nt * 18 * H].reshape(nt, 18 * H)
    gu[:, : 16 * H] = 0x33                    # every code 3
    gu[:, 16 * H:] = np.tile(h16([0.0625]).view(np.uint8), H)   # scales and biases 1/16
    # down: code 0 everywhere, bias w1
    dn = blob[nt * 18 * H:].reshape(H // 16, 9 * I)
    dn[:, 8 * I + I // 2:] = np.tile(h16([w1]).view(np.uint8), I // 4)
    y, h = oracle.expert_ffn(blob, H, I, x)
    g = w0 * x.sum()
    assert np.allclose(h, oracle.gelu(g, 0) * g, rtol=1e-13)
    assert np.allclose(y, w1 * I * oracle.gelu(g, 0) * g, rtol=1e-12)


# --------------------------------------------------------------- router ----

def test_router_logits_equal_exact_rational_result():
    rng = np.random.default_rng(5)
    E, H = 8, 320
    W = rng.integers(-127, 128, (E, H)).astype(np.int8)
    x = (rng.standard_normal(H) * 10.0 ** rng.integers(-6, 4, H)).astype(np.float16)
    x[:5] = [65504, -65504, 6e-8, -6e-8, 0]
    scale = (rng.random(E) * 0.01).astype(np.float16)
    bias = rng.standard_normal(E).astype(np.float32)
    got = oracle.router_logits(W, scale.view(np.uint16), bias, x.view(np.uint16), E, H)
    for e in range(E):
        exact = sum(Fraction(int(W[e, c])) * Fraction(float(x[c])) for c in range(H))
        ref = float(exact) * float(scale[e])          # one rounding each
        ref = ref + float(bias[e])
        assert got[e] == ref


def test_router_zero_weights_give_uniform_first_k():
    E, H, k = 16, 64, 4
    W = np.zeros((E, H), np.int8)
    x = h16(np.random.default_rng(0).standard_normal(H))
    lg = oracle.router_logits(W, h16(np.ones(E)), None, x, E, H)
    assert not lg.any()
    idx = oracle.topk(lg, k)
    assert idx.tolist() == [0, 1, 2, 3]
    w = oracle.topk_weights(oracle.softmax(lg), idx, 1)
    np.testing.assert_allclose(w, 0.25, rtol=1e-15)


def test_topk_matches_sorted_brute_force_with_ties():
    rng = np.random.default_rng(11)
    for trial in range(300):
        E = int(rng.integers(2, 140))
        k = int(rng.integers(1, min(E, 9) + 1))
        lg = np.round(rng.standard_normal(E), int(rng.integers(0, 3)))  # many ties
        ref = sorted(range(E), key=lambda e: (-lg[e], e))[:k]
        assert oracle.topk(lg, k).tolist() == ref


def test_softmax_sums_to_one_and_matches_scipy():
    from scipy.special import softmax as sp_softmax
    rng = np.random.default_rng(2)
    for _ in range(50):
        lg = rng.standard_normal(128) * 4
        p = oracle.softmax(lg)
        assert abs(p.sum() - 1.0) <= 1e-12
        np.testing.assert_allclose(p, sp_softmax(lg), rtol=1e-13)
    np.testing.assert_allclose(oracle.softmax(np.full(10, 3.7)), 0.1, rtol=1e-15)
    # renormalised top-k weights equal the softmax of the selected logits
    lg = rng.standard_normal(128)
    idx = oracle.topk(lg, 8)
    w = oracle.topk_weights(oracle.softmax(lg), idx, 1)
    np.testing.assert_allclose(w, sp_softmax(lg[idx]), rtol=1e-13)
    assert abs(w.sum() - 1) < 1e-15 * 8
    raw = oracle.topk_weights(oracle.softmax(lg), idx, 0)
    np.testing.assert_allclose(raw, sp_softmax(lg)[idx], rtol=1e-13)


# -------------------------------------------------------------- combine ----

def test_combine_special_cases():
    rng = np.random.default_rng(8)
    H, k = 96, 4
    ys, yr = rng.standard_normal(H), rng.standard_normal((k, H))
    np.testing.assert_array_equal(oracle.combine(ys, yr, np.zeros(k)), ys)
    for j in range(k):
        e = np.zeros(k); e[j] = 1.0
        np.testing.assert_array_equal(oracle.combine(ys, yr, e), ys + yr[j])
    w = rng.random(k)
    np.testing.assert_allclose(oracle.combine(ys, yr, w), ys + w @ yr, rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------ MoE layer ----

def _tiny_layer(cfg, seed=0, bias_std=None):
    d = synth.layer_weights(cfg, seed, 0, "cpu", bias_std=bias_std)
    return {k: (None if v is None else
                (v.view(torch.uint16) if v.dtype == torch.float16 else v).numpy())
            for k, v in d.items()}


def test_layer_against_dense_brute_force():
    cfg = TINY
    L = _tiny_layer(cfg, seed=0, bias_std=1.0)
    x = synth.tokens(1, cfg.H, 0)[0].view(torch.uint16).numpy()
    out = oracle.moe_layer(cfg, L, x)
    xd = x.view(np.float16).astype(np.float64)
    # router in exact rational arithmetic, full sort, scipy softmax
    from scipy.special import softmax as sp_softmax
    W = L["router_w"].astype(np.int64)
    sc = L["router_scale"].view(np.float16).astype(np.float64)
    lg = np.array([float(sum(Fraction(int(W[e, c])) * Fraction(float(xd[c]))
                             for c in range(cfg.H))) * sc[e] + float(L["router_bias"][e])
                   for e in range(cfg.E)])
    np.testing.assert_array_equal(out["logits"], lg)
    idx = sorted(range(cfg.E), key=lambda e: (-lg[e], e))[:cfg.k]
    assert out["idx"].tolist() == idx
    w = sp_softmax(lg[idx])
    np.testing.assert_allclose(out["w"], w, rtol=1e-13)
    Wg, Wu, Wd = _blob_parts(L["shared"], cfg.H, cfg.Is)
    y = Wd @ (_gelu_np(Wg @ xd, 0) * (Wu @ xd))
    for j, e in enumerate(idx):
        Wg, Wu, Wd = _blob_parts(L["experts"][e], cfg.H, cfg.I)
        y = y + w[j] * (Wd @ (_gelu_np(Wg @ xd, 0) * (Wu @ xd)))
    np.testing.assert_allclose(out["y"], y, rtol=1e-11, atol=1e-13)


# -------------------------------------------------------------- RMSNorm ----

def test_rmsnorm_closed_forms():
    H = 256
    # constant input c: mean(h^2) = c^2, output rounds to 1.0
    for c in (0.5, 3.0, -7.25):
        x = oracle.rmsnorm(h16(np.full(H, c)), 1e-6)
        assert (x == h16([math.copysign(1.0, c)])).all()
    # one non-zero element a: output sqrt(H) there (eps = 0), zeros elsewhere
    h = np.zeros(H, np.float16); h[17] = 5.0
    x = oracle.rmsnorm(h.view(np.uint16), 0.0)
    assert x[17] == h16([16.0])[0] and not np.delete(x, 17).any()
    # scale by 2 and sign flip are exact symmetries when eps = 0
    h = h16(np.random.default_rng(4).standard_normal(H))
    x1 = oracle.rmsnorm(h, 0.0)
    h2 = h16(h.view(np.float16).astype(np.float64) * 2)
    np.testing.assert_array_equal(oracle.rmsnorm(h2, 0.0), x1)
    hn = h16(-h.view(np.float16).astype(np.float64))
    np.testing.assert_array_equal(oracle.rmsnorm(hn, 0.0), h16(-x1.view(np.float16).astype(np.float64)))


def test_rmsnorm_sum_of_squares_is_exact():
    # values spanning 2^-24 .. 6e4: a fp64 running sum would drop the tiny
    # squares; the oracle must equal the exact big-integer result.
    H = 64
    vals = np.array([60000.0, 2.0 ** -24, 3 * 2.0 ** -24, 1.5] * 16, np.float16)
    vals[::5] *= -1
    x = oracle.rmsnorm(vals.view(np.uint16), 1e-6)
    ss = sum(int(float(v) * 2 ** 24) ** 2 for v in vals)     # exact integer
    ms = (float(ss) * 2.0 ** -48) / H
    r = 1.0 / math.sqrt(ms + 1e-6)
    ref = np.array([float(v) * r for v in vals]).astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(x, ref)


def test_residual_add_rounds_once_to_half():
    h = h16([1.0, 2048.0, -0.5])
    out = oracle.residual_add(h, [2.0 ** -11, 1.0, 0.25])
    # 1 + 2^-11 ties to even -> 1; 2049 ties to even -> 2048
    np.testing.assert_array_equal(out, h16([1.0, 2048.0, -0.25]))


# ------------------------------------------------------------------ LFU ----

def _read_trace(path):
    steps = []
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            req, slots = line.split("|")
            req = [int(v) for v in req.split()]
            st = []
            for tok in slots.split():
                if tok == "-":
                    st.append(None)
                else:
                    e, c, s = (int(v) for v in tok.split("."))
                    st.append((e, c, s))
            steps.append((req, st))
    return steps


def test_lfu_hand_trace_golden():
    steps = _read_trace(os.path.join(GOLDEN, "lfu_trace_s4_k2.txt"))
    c = oracle.LfuCache(4)
    for req, want in steps:
        c.token(req)
        got = [None if c.expert[s] < 0 else
               (int(c.expert[s]), int(c.count[s]), int(c.seq[s])) for s in range(4)]
        assert got == want, (req, got, want)
    assert int(c.hits[0]) == 2 and int(c.misses[0]) == 6


class NaiveLfu:
    """Second, independently written LFU model: a list of dict entries,
    eviction chosen by sorting candidates on (count, insertion order)."""

    def __init__(self, S):
        self.S = S
        self.entries = [None] * S
        self.t = 0
        self.hits = self.misses = 0

    def token(self, idx):
        where = {}
        resident = {en["e"]: s for s, en in enumerate(self.entries) if en}
        for e in sorted(idx):
            if e in resident:
                s = resident[e]
                self.entries[s]["n"] += 1
                where[e] = s
                self.hits += 1
        for e in sorted(idx):
            if e in where:
                continue
            empty = [s for s in range(self.S) if self.entries[s] is None]
            if empty:
                s = empty[0]
            else:
                cand = [s for s in range(self.S) if s not in where.values()]
                s = min(cand, key=lambda s: (self.entries[s]["n"], self.entries[s]["t"]))
            self.t += 1
            self.entries[s] = {"e": e, "n": 1, "t": self.t}
            where[e] = s
            self.misses += 1
        return [where[e] for e in idx]


def test_lfu_matches_naive_model_on_random_sequences():
    rng = np.random.default_rng(9)
    for trial in range(40):
        k = int(rng.integers(1, 9))
        S = int(rng.integers(k + 1, 17))
        E = int(rng.integers(S, 48))
        c, n = oracle.LfuCache(S), NaiveLfu(S)
        for t in range(250):
            idx = rng.choice(E, size=k, replace=False).astype(np.int32)
            slot_of, miss = c.token(idx)
            assert slot_of.tolist() == n.token(idx.tolist())
        assert (int(c.hits[0]), int(c.misses[0])) == (n.hits, n.misses)


def test_lfu_zipf_routing_hit_rate_is_sane():
    seq = synth.routing_sequence(512, 128, 8, seed=0).numpy()
    c, n = oracle.LfuCache(16), NaiveLfu(16)
    for row in seq:
        assert c.token(row)[0].tolist() == n.token(row.tolist())
    hits, misses = int(c.hits[0]), int(c.misses[0])
    assert hits + misses == 512 * 8
    assert 0.05 < hits / (hits + misses) < 0.95


def test_lfu_rejects_impossible_requests():
    c = oracle.LfuCache(2)
    with pytest.raises(ValueError):
        c.token([1, 2, 3])             # S <= k: no victim can exist
    c = oracle.LfuCache(8)
    with pytest.raises(ValueError):
        c.token([4, 4])


# ------------------------------------------------------ LFU over chunks --
def _read_chunk_trace(path):
    """[(chunk rows, n_batch, [(batch, expert, slot)], slot states)] from the
    golden chunk trace."""
    out = []
    rows = None
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            if line.startswith("chunk"):
                rows = [[int(v) for v in tok.split()] for tok in line[len("chunk"):].split(";")]
            else:
                head, miss, slots = line.split("|")
                nb = int(head.split()[1])
                ms = []
                for tok in miss.split():
                    b, rest = tok.split(":")
                    e, sl = rest.split(">")
                    ms.append((int(b), int(e), int(sl)))
                st = [None if tok == "-" else tuple(int(v) for v in tok.split("."))
                      for tok in slots.split()]
                out.append((rows, nb, ms, st))
    return out


def _state(c):
    return [None if c.expert[s] < 0 else (int(c.expert[s]), int(c.count[s]), int(c.seq[s]))
            for s in range(c.S)]


def test_lfu_chunk_hand_trace_golden():
    """The chunk rule against the hand-derived trace: batches, misses in
    insertion order and the slot contents after every chunk."""
    c = oracle.LfuCache(4)
    for rows, nb, ms, st in _read_chunk_trace(os.path.join(GOLDEN, "lfu_chunk_trace_s4_k2.txt")):
        slot_of, batch_of, miss, n_batch = c.chunk(np.array(rows, np.int32))
        assert (n_batch, miss, _state(c)) == (nb, ms, st), rows
    assert int(c.hits[0]) == 5 and int(c.misses[0]) == 12


class NaiveChunkLfu(NaiveLfu):
    """Independent model of the chunk rule: distinct experts with their uses,
    pinned slots as a Python set, a new batch when no slot is free."""

    def chunk(self, rows):
        uses = {}
        for r in rows:
            for e in r:
                uses[e] = uses.get(e, 0) + 1
        where, batch_e = {}, {}
        resident = {en["e"]: s for s, en in enumerate(self.entries) if en}
        pinned = set()
        for e in sorted(uses):
            if e in resident:
                s = resident[e]
                self.entries[s]["n"] += uses[e]
                where[e], batch_e[e] = s, 0
                pinned.add(s)
                self.hits += 1
        batch, misses = 0, []
        for e in sorted(uses):
            if e in where:
                continue
            empty = [s for s in range(self.S) if self.entries[s] is None]
            cand = [s for s in range(self.S) if s not in pinned]
            if not empty and not cand:
                batch += 1
                pinned = set()
                cand = list(range(self.S))
            s = empty[0] if empty else min(cand, key=lambda s: (self.entries[s]["n"], self.entries[s]["t"]))
            self.t += 1
            self.entries[s] = {"e": e, "n": uses[e], "t": self.t}
            where[e], batch_e[e] = s, batch
            pinned.add(s)
            misses.append((batch, e, s))
            self.misses += 1
        return ([[where[e] for e in r] for r in rows], [[batch_e[e] for e in r] for r in rows],
                misses, batch + 1)


def test_lfu_chunk_matches_naive_model():
    rng = np.random.default_rng(21)
    for trial in range(30):
        k = int(rng.integers(1, 9))
        S = int(rng.integers(k + 1, 33))
        E = int(rng.integers(S, 96))
        c, n = oracle.LfuCache(S), NaiveChunkLfu(S)
        for step in range(12):
            T = int(rng.integers(1, 40))
            p = 1.0 / (1.0 + np.arange(E)) ** 1.2          # skewed choices
            p /= p.sum()
            rows = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
            slot_of, batch_of, miss, nb = c.chunk(rows)
            n_slot, n_batch_of, n_miss, n_nb = n.chunk(rows.tolist())
            assert slot_of.tolist() == n_slot and batch_of.tolist() == n_batch_of
            assert miss == n_miss and nb == n_nb
            # every expert of the chunk is copied at most once, and a batch
            # never holds more experts than slots
            assert len({e for _, e, _ in miss}) == len(miss)
            for b in range(nb):
                assert len({int(e) for e in rows[batch_of == b]}) <= S
        assert (int(c.hits[0]), int(c.misses[0])) == (n.hits, n.misses)


def test_lfu_one_token_chunks_are_the_token_rule():
    """A chunk of one token is the per-token rule exactly (one batch; same
    slots, counts, insertion numbers and totals)."""
    rng = np.random.default_rng(5)
    a, b = oracle.LfuCache(16), oracle.LfuCache(16)
    for t in range(400):
        idx = rng.choice(128, size=8, replace=False).astype(np.int32)
        sa, ma = a.token(idx)
        sb, bb, mb, nb = b.chunk(idx[None, :])
        assert sa.tolist() == sb[0].tolist() and nb == 1
        assert ma == [(e, s) for _, e, s in mb]
    assert _state(a) == _state(b)
    assert (int(a.hits[0]), int(a.misses[0])) == (int(b.hits[0]), int(b.misses[0]))


def test_lfu_chunk_rejects_bad_requests():
    with pytest.raises(ValueError):
        oracle.LfuCache(2).chunk(np.array([[1, 2]], np.int32))      # S <= k
    with pytest.raises(ValueError):
        oracle.LfuCache(8).chunk(np.array([[7, 7]], np.int32))
