"""Argument errors of the FP8 decode entry points, on CPU: every one is
decided before the library touches the device, so these calls never reach
CUDA.  Device pointers are fake 16-byte-aligned addresses that are never
dereferenced."""
import ctypes

import numpy as np
import pytest

import ecf8_synth as synth

FAKE = 1 << 20


@pytest.fixture(scope="module")
def L():
    import lossless_fp8_weight_b200 as lib
    return lib


@pytest.fixture(scope="module")
def info(L):
    return L.blob_info(L.encode(synth.single_normal_1k().tensors[0].generate(count=50_000)))


def _decode(L, info, blob=FAKE, blob_size=None, out=FAKE, n=None):
    size = info.blob_bytes if blob_size is None else blob_size
    return L._lib.ecf8_decode(ctypes.byref(info), blob, size, out, info.n if n is None else n, 0, 0)


def test_decode_refuses_a_short_blob_buffer(L, info):
    assert _decode(L, info, blob_size=info.blob_bytes - 1) == -1
    assert _decode(L, info, blob_size=0) == -1


def test_decode_refuses_n_that_is_not_the_blobs(L, info):
    assert _decode(L, info, n=info.n - 1) == -1
    assert _decode(L, info, n=info.n + 1) == -1


def test_decode_refuses_null_and_misaligned_pointers(L, info):
    assert _decode(L, info, blob=0) == -1
    assert _decode(L, info, out=0) == -1
    assert _decode(L, info, blob=FAKE + 8) == -5
    assert _decode(L, info, out=FAKE + 4) == -5
    assert L._lib.ecf8_decode(None, FAKE, 1 << 20, FAKE, 0, 0, 0) == -1


def test_decode_refuses_a_damaged_info(L, info):
    bad = L.Info.from_buffer_copy(info)
    bad.blob_bytes += 16  # no longer the layout of (n, code_bits, C, T)
    assert _decode(L, bad, blob_size=bad.blob_bytes) == -2
    bad = L.Info.from_buffer_copy(info)
    bad.len[15] = 1  # Kraft sum above 1
    assert _decode(L, bad) == -4
    bad = L.Info.from_buffer_copy(info)
    bad.chunk_bytes, bad.group_chunks = 16, 64  # a layout the kernels do not implement
    assert _decode(L, bad) in (-2, -6)


def _batch(L, info, count, blob_size=None):
    arr = (L.Tensor * count)()
    for i in range(count):
        arr[i].info = ctypes.pointer(info)
        arr[i].d_blob = FAKE
        arr[i].blob_size = info.blob_bytes if blob_size is None else blob_size
        arr[i].d_out = FAKE
    return arr


def test_batched_refuses_a_short_blob_buffer(L, info):
    arr = _batch(L, info, 3)
    arr[1].blob_size = info.blob_bytes - 16
    assert L._lib.ecf8_decode_batched(arr, 3, 0, 0, 0, 0) == -1
    assert L._lib.ecf8_decode_batched_noalloc(arr, 3, 0, 0) == -1
    assert L._lib.ecf8_decode_batched_ctas(arr, 3, 0, 0, 0, 0, 4) == -1
    # beyond the inline limit, with a workspace: still refused before any copy
    big = _batch(L, info, L.BATCH_INLINE_MAX + 5)
    big[L.BATCH_INLINE_MAX + 2].blob_size = 1
    ws = L.batched_workspace_size(L.BATCH_INLINE_MAX + 5)
    assert L._lib.ecf8_decode_batched(big, L.BATCH_INLINE_MAX + 5, FAKE, ws, 0, 0) == -1


def test_batched_counts_and_workspace(L, info):
    assert L._lib.ecf8_decode_batched(None, 1, 0, 0, 0, 0) == -1
    assert L._lib.ecf8_decode_batched(None, -1, 0, 0, 0, 0) == -1
    assert L._lib.ecf8_decode_batched(None, 0, 0, 0, 0, 0) == 0  # nothing to do
    big = _batch(L, info, L.BATCH_INLINE_MAX + 1)
    assert L._lib.ecf8_decode_batched(big, L.BATCH_INLINE_MAX + 1, 0, 0, 0, 0) == -8
    ws = L.batched_workspace_size(L.BATCH_INLINE_MAX + 1)
    assert L._lib.ecf8_decode_batched(big, L.BATCH_INLINE_MAX + 1, FAKE, ws - 1, 0, 0) == -8
    assert L._lib.ecf8_decode_batched(big, L.BATCH_INLINE_MAX + 1, FAKE + 8, ws, 0, 0) == -5
    over = _batch(L, info, L.NOALLOC_MAX_TENSORS + 1)
    assert L._lib.ecf8_decode_batched_noalloc(over, L.NOALLOC_MAX_TENSORS + 1, 0, 0) == -9


def test_empty_tensors_need_no_pointers(L):
    info = L.blob_info(L.encode(np.zeros(0, np.uint8)))
    arr = (L.Tensor * 1)()
    arr[0].info = ctypes.pointer(info)
    assert L._lib.ecf8_decode_batched(arr, 1, 0, 0, 0, 0) == 0
    assert L._lib.ecf8_decode(ctypes.byref(info), 0, 0, 0, 0, 0, 0) == 0
