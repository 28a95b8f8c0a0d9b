"""Argument checks of the decode-on-use pipeline (ecf8_pipeline_create) on
CPU: every one of them is decided before any CUDA call, so no GPU is needed.
The pool rules follow the ECF8 walkthrough §3.2.2 (a pool sized for the
largest layer, reused cyclically) and the DFloat11 article §4 (decode ahead
while the current layer computes): a slot must hold its layer's outputs, and
the slot decoded ahead must never be the one in use (n_slots >= depth + 1)."""
import ctypes

import numpy as np
import pytest

import ecf8_synth as synth


@pytest.fixture(scope="module")
def L():
    import lossless_fp8_weight_b200 as lib
    return lib


def _infos(L, sizes):
    spec = synth.alpha_sweep_point(1.7, 448.0).tensors[0]
    return [L.blob_info(L.encode(spec.generate(count=n))) for n in sizes]


FAKE = 1 << 20  # a 16-byte-aligned address that is never dereferenced


def _create(L, layers, slots, slot_bytes, depth, workspace=0, ws_bytes=0):
    n = len(layers)
    larr = (L.Layer * n)()
    keep = []
    for l, tensors in enumerate(layers):
        tarr = (L.LayerTensor * max(1, len(tensors)))()
        for i, (info, off) in enumerate(tensors):
            keep.append(info)
            tarr[i].info = ctypes.pointer(info)
            tarr[i].d_blob = FAKE
            tarr[i].blob_size = info.blob_bytes
            tarr[i].out_offset = off
        keep.append(tarr)
        larr[l].tensors = tarr
        larr[l].count = len(tensors)
    sarr = (ctypes.c_void_p * len(slots))(*slots)
    h = ctypes.c_void_p()
    rc = L._lib.ecf8_pipeline_create(larr, n, sarr, len(slots), slot_bytes, depth, 0, workspace, ws_bytes, 0, 0,
                                     ctypes.byref(h))
    return rc, h


def test_pool_must_outnumber_the_lookahead(L):
    infos = _infos(L, [1000])
    layer = [(infos[0], 0)]
    rc, h = _create(L, [layer, layer], [FAKE], 4096, depth=1)
    assert rc == -1 and not h.value  # ARG: 1 slot, 1 layer ahead
    rc, _ = _create(L, [layer], [FAKE, FAKE], 4096, depth=2)
    assert rc == -1
    rc, _ = _create(L, [layer], [FAKE], 4096, depth=-1)
    assert rc == -1


def test_slot_must_hold_every_tensor_of_every_layer(L):
    a, b = _infos(L, [1000, 3000])
    rc, _ = _create(L, [[(a, 0), (b, 1008)]], [FAKE, FAKE], 1008 + 3000 - 1, depth=1)
    assert rc == -1
    rc, _ = _create(L, [[(a, 0)], [(b, 0)]], [FAKE, FAKE], 2999, depth=1)
    assert rc == -1


def test_alignment_of_offsets_and_slots(L):
    (a,) = _infos(L, [1000])
    rc, _ = _create(L, [[(a, 8)]], [FAKE, FAKE], 4096, depth=1)
    assert rc == -5  # ALIGN
    rc, _ = _create(L, [[(a, 0)]], [FAKE, FAKE + 8], 4096, depth=1)
    assert rc == -5
    rc, _ = _create(L, [[(a, 0)]], [FAKE, 0], 4096, depth=1)
    assert rc == -1


def test_large_layers_need_a_workspace(L):
    (a,) = _infos(L, [100])
    layer = [(a, 0)] * (L.BATCH_INLINE_MAX + 1)
    rc, _ = _create(L, [layer], [FAKE, FAKE], 4096, depth=1)
    assert rc == -8  # WORKSPACE
    need = L.batched_workspace_size(L.BATCH_INLINE_MAX + 1)
    rc, _ = _create(L, [layer], [FAKE, FAKE], 4096, depth=1, workspace=FAKE, ws_bytes=need - 1)
    assert rc == -8
    rc, _ = _create(L, [layer], [FAKE, FAKE], 4096, depth=1, workspace=FAKE + 4, ws_bytes=need)
    assert rc == -5


def test_null_and_empty_arguments(L):
    h = ctypes.c_void_p()
    assert L._lib.ecf8_pipeline_create(None, 1, None, 1, 0, 0, 0, 0, 0, 0, 0, ctypes.byref(h)) == -1
    assert L._lib.ecf8_pipeline_create(None, 0, None, 0, 0, 0, 0, 0, 0, 0, 0, None) == -1
    assert L._lib.ecf8_pipeline_acquire(None, 0, 0, ctypes.byref(ctypes.c_void_p())) == -1
    assert L._lib.ecf8_pipeline_release(None, 0, 0) == -1
    L._lib.ecf8_pipeline_destroy(None)  # a no-op


def test_blob_buffers_must_hold_their_blobs(L):
    (a,) = _infos(L, [1000])
    n = 1
    larr = (L.Layer * n)()
    tarr = (L.LayerTensor * 1)()
    tarr[0].info = ctypes.pointer(a)
    tarr[0].d_blob = FAKE
    tarr[0].blob_size = a.blob_bytes - 1
    tarr[0].out_offset = 0
    larr[0].tensors = tarr
    larr[0].count = 1
    sarr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    h = ctypes.c_void_p()
    assert L._lib.ecf8_pipeline_create(larr, n, sarr, 2, 4096, 1, 0, 0, 0, 0, 0, ctypes.byref(h)) == -1
    assert not h.value
