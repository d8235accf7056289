"""Host logic of the batched bench: which kernel serves each expert."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_bucket_split_rules():
    b = _bench()
    counts = [0, 1, 3, 4, 5, 40, 0, 2]
    # a step of one token never reaches these kernels (the fused kernel serves it);
    # from two tokens every used bucket runs on tcgen05
    assert b.bucket_split(counts, T=1) == (0, 6)
    assert b.bucket_split(counts, T=8) == (6, 0)
    # large step: by default every used bucket on tcgen05
    assert b.bucket_split(counts, T=32) == (6, 0)
    # a threshold of 4 pairs leaves the smaller buckets on the grouped kernels
    assert b.bucket_split(counts, T=32, min_tokens=4) == (3, 3)
    assert b.bucket_split(counts, T=256, min_tokens=1) == (6, 0)
    assert b.bucket_split(counts, T=256, min_tokens=0) == (0, 6)
    assert b.bucket_split([0] * 16, T=64) == (0, 0)
