"""Helpers shared by the GPU parity tests (no arithmetic of the method)."""
import numpy as np
import torch

from bit_quantized_expert_int8_b200 import synth

# Tolerance on fp32/fp64 layer outputs against the fp64 oracle.
REL_L2 = 1e-3
MAX_ABS = 2e-3


def np_of(t):
    if t is None:
        return None
    t = t.detach().cpu()
    if t.dtype == torch.float16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def np_layer(d):
    return {k: np_of(v) for k, v in d.items()}


def to_dev(d, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in d.items()}


def assert_y_close(y_gpu, y_ref, what=""):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    d = y_gpu - y_ref
    rel = np.linalg.norm(d) / max(np.linalg.norm(y_ref), 1e-30)
    mx = np.abs(d).max() if d.size else 0.0
    assert rel <= REL_L2 and mx <= MAX_ABS, f"{what}: rel L2 {rel:.3e}, max abs {mx:.3e}"
    return rel, mx


def half_ulp_diff(a16, b16):
    """Distance in fp16 units in the last place between two uint16 arrays."""
    a = a16.astype(np.int32)
    b = b16.astype(np.int32)
    a = np.where(a & 0x8000, -(a & 0x7FFF), a)
    b = np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(a - b)


def assert_half_close(h_gpu16, h_ref16, what=""):
    """fp16 residual check: |gpu - ref| <= 1 ulp of ref + the y tolerance
    (h + y can cancel, where ulps of a tiny result say nothing)."""
    g = np.asarray(h_gpu16).view(np.float16).astype(np.float64)
    r = np.asarray(h_ref16).view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(r).astype(np.float16)).astype(np.float64)
    bad = np.abs(g - r) > ulp + MAX_ABS
    assert not bad.any(), f"{what}: {bad.sum()} residual entries off, worst {np.abs(g - r).max():.3e}"


def make_layer(cfg, seed, layer=0, device="cuda", bias_std=None):
    """Generate on the CPU for small shapes, on the GPU for large ones; the
    oracle always receives a CPU copy of the very same bytes."""
    gen_dev = "cpu" if cfg.H * cfg.I * cfg.E <= 2 ** 24 else device
    d = synth.layer_weights(cfg, seed, layer, gen_dev, bias_std=bias_std)
    return to_dev(d, device)


def assert_y_close_scaled(y_gpu, y_ref, what=""):
    """Tolerance for outputs far above unit size (inputs near the fp16 range
    fed to the FFN without a norm): rel L2 <= 1e-3 as always, and max abs
    <= 2e-3 * max(1, max |y_ref|).  An fp32 result of size M carries rounding
    error of order M * 2^-24 * sqrt(terms), so no fp32 arithmetic meets a
    fixed absolute bound once M is in the thousands; for M <= 1 this is the
    plain bound."""
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    d = y_gpu - y_ref
    rel = np.linalg.norm(d) / max(np.linalg.norm(y_ref), 1e-30)
    scale = max(1.0, float(np.abs(y_ref).max()) if y_ref.size else 1.0)
    mx = np.abs(d).max() if d.size else 0.0
    assert rel <= REL_L2 and mx <= MAX_ABS * scale, \
        f"{what}: rel L2 {rel:.3e}, max abs {mx:.3e} (scale {scale:.3e})"
    return rel, mx
