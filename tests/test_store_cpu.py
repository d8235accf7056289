"""The storage tier's reader on the CPU: an expert file in the store's
format (blobs padded to 4 KiB, layer-major) read back with parallel pread
through the library's C ABI (moe_store_*), byte for byte; the error paths
(missing or short file, out-of-range layer or expert)."""
import os

import numpy as np
import pytest

from bit_quantized_expert_int8_b200 import build, moeq4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moeq4.load()


def _file(tmp_path, n_layers, n_experts, blob, seed=0):
    rng = np.random.default_rng(seed)
    layers = [rng.integers(0, 256, size=(n_experts, blob), dtype=np.uint8) for _ in range(n_layers)]
    path = tmp_path / "experts.bin"
    moeq4.write_expert_file(path, layers, blob)
    return path, layers


def test_stride_is_blob_padded_to_4k():
    assert moeq4.store_stride(4096) == 4096
    assert moeq4.store_stride(10000) == 12288
    assert moeq4.store_stride(3345408) == 3346432          # the layer shape's routed blob


def test_store_reads_blobs_byte_for_byte(tmp_path):
    blob = 10000
    path, layers = _file(tmp_path, 3, 7, blob)
    assert os.path.getsize(path) == 3 * 7 * moeq4.store_stride(blob)
    st = moeq4.Store(path, 3, 7, blob, n_threads=3, n_staging=2)
    rng = np.random.default_rng(1)
    total = 0
    for trial in range(20):
        layer = int(rng.integers(0, 3))
        n = int(rng.integers(0, 6))                       # more blobs than staging buffers too
        ex = rng.choice(7, size=n, replace=False).astype(np.int32)
        dst = [np.zeros(blob, np.uint8) for _ in range(n)]
        st.read(layer, ex, dst)
        for e, d in zip(ex, dst):
            np.testing.assert_array_equal(d, layers[layer][e])
        total += n
    b, secs, direct = st.stats()
    assert b == total * blob and secs >= 0.0
    st.close()


def test_store_refuses_bad_files_and_requests(tmp_path):
    blob = 4096
    path, _ = _file(tmp_path, 1, 4, blob)
    with pytest.raises(moeq4.MoeError):
        moeq4.Store(tmp_path / "missing.bin", 1, 4, blob)
    with pytest.raises(moeq4.MoeError):
        moeq4.Store(path, 2, 4, blob)                     # file shorter than 2 layers
    with pytest.raises(moeq4.MoeError):
        moeq4.Store(path, 1, 4, 1000)                     # blob size not a multiple of 16
    st = moeq4.Store(path, 1, 4, blob, n_threads=2, n_staging=4)
    buf = [np.zeros(blob, np.uint8)]
    with pytest.raises(moeq4.MoeError):
        st.read(0, [4], buf)                              # expert out of range
    with pytest.raises(moeq4.MoeError):
        st.read(1, [0], buf)                              # layer out of range
    st.read(0, [3], buf)                                  # still usable afterwards
    st.close()
