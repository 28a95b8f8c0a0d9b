"""Argument checks of the GPU encoder's C ABI that are decided on the host,
before any CUDA call (so they run without a GPU): the codebook must give
every exponent present in the histogram a code, the histogram must count n
weights, the destination must hold the blob, and large inputs need a
workspace."""
import ctypes

import numpy as np
import pytest

import ecf8_synth as synth

FAKE = 1 << 20  # 16-byte-aligned, never dereferenced


@pytest.fixture(scope="module")
def L():
    import lossless_fp8_weight_b200 as lib
    return lib


def _call(L, n, hist, cb, cap, ws=FAKE, ws_bytes=1 << 30, x=FAKE, blob=FAKE, C=32, T=32):
    got = ctypes.c_size_t(0)
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    return L._lib.ecf8_encode_device(x, n, h.ctypes.data, ctypes.byref(cb), C, T, blob, cap, ctypes.byref(got), ws,
                                     ws_bytes, 0)


def _setup(L, n=100_000):
    x = synth.alpha_sweep_point(1.7, 448.0).tensors[0].generate(count=n)
    h = L.histogram(x)
    cb = L.build_codebook(h)
    size = ctypes.c_size_t(0)
    assert L._lib.ecf8_encoded_size(h.ctypes.data, n, ctypes.byref(cb), 32, 32, ctypes.byref(size)) == 0
    return h, cb, size.value


def test_capacity_and_workspace(L):
    h, cb, size = _setup(L)
    assert _call(L, 100_000, h, cb, size - 1) == -3  # CAPACITY
    assert _call(L, 100_000, h, cb, size, ws=0) == -8  # WORKSPACE
    need = L._lib.ecf8_encode_device_workspace_size(100_000)
    assert _call(L, 100_000, h, cb, size, ws_bytes=need - 1) == -8


def test_codebook_must_cover_the_histogram(L):
    h, cb, size = _setup(L)
    present = int(np.flatnonzero(h)[0])
    bad = L.Codebook.from_buffer_copy(cb)
    bad.len[present] = 0
    assert _call(L, 100_000, h, bad, size) == -4  # CODEBOOK (also no longer canonical)


def test_histogram_must_count_n(L):
    h, cb, size = _setup(L)
    assert _call(L, 100_001, h, cb, size) == -1


def test_alignment(L):
    h, cb, size = _setup(L)
    assert _call(L, 100_000, h, cb, size, x=FAKE + 1) == -5
    assert _call(L, 100_000, h, cb, size, blob=FAKE + 8) == -5
    d_hist = FAKE + 4
    assert L._lib.ecf8_histogram_device(FAKE, 10, d_hist, 0) == -5
