"""The bounds-checked build (libecf8_checked.so, -DECF8_CHECKED) on GPU: every
kernel store and table read tests its index against its buffer and sets
ECF8_STATUS_BOUNDS instead of going out of range.  compute-sanitizer is not
available here, so this build stands in for it: valid blobs must decode
bit-exactly with status 0, and damaged blobs (gap, offset and stream damage,
the walkthrough's §5.3 failure mode) may report decode errors but must never
trip a bounds check."""
import ctypes
import os

import numpy as np
import pytest

import ecf8_synth as synth
import oracle

pytestmark = pytest.mark.gpu

BOUNDS = 8


@pytest.fixture(scope="module")
def env(gpu_available):
    import torch
    import lossless_fp8_weight_b200 as L
    from lossless_fp8_weight_b200 import _build
    so = ctypes.CDLL(_build.build(checked=True))
    so.ecf8_decode_batched.argtypes = [ctypes.POINTER(L.Tensor), ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p, ctypes.c_void_p]
    return L, torch, so


def _decode(env, blobs):
    L, torch, so = env
    infos = [L.blob_info(b) for b in blobs]
    d_blobs = [torch.from_numpy(b).cuda() for b in blobs]
    # guard bytes around each output catch writes outside it
    outs = [torch.full((i.n + 64,), 0xC3, dtype=torch.uint8, device="cuda") for i in infos]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    items = [L.BatchItem(i, b, o[32:32 + i.n]) for i, b, o in zip(infos, d_blobs, outs)]
    arr, _keep = L.make_batch(items)
    ws = torch.empty(max(16, L.batched_workspace_size(len(items))), dtype=torch.uint8, device="cuda")
    rc = so.ecf8_decode_batched(arr, len(items), ws.data_ptr(), ws.numel(), status.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    got = [o.cpu().numpy() for o in outs]
    intact = all((g[:32] == 0xC3).all() and (g[-32:] == 0xC3).all() for g in got)
    return [g[32:-32] for g in got], int(status.item()), intact


SPECS = [synth.alpha_sweep_point(1.7, 448.0).tensors[0], synth.alpha_sweep_point(1.5, 448.0).tensors[0],
         synth.single_normal_1k().tensors[0]]


@pytest.mark.parametrize("n", [1, 17, 33, 4097, 300_007, 2_000_003])
def test_valid_blobs_pass_every_check(env, n):
    xs = [s.generate(begin=5, count=n) for s in SPECS]
    got, status, intact = _decode(env, [oracle.encode(x) for x in xs])
    assert status == 0 and intact
    for g, x in zip(got, xs):
        assert np.array_equal(g, x)


def test_a_mixed_batch_of_layer_tensors_passes_every_check(env):
    xs = [t.generate(count=1_000_000) for t in synth.llama3_8b_layer().tensors]
    L = env[0]
    got, status, intact = _decode(env, [L.encode(x) for x in xs])
    assert status == 0 and intact
    for g, x in zip(got, xs):
        assert np.array_equal(g, x)


@pytest.mark.parametrize("seed", range(6))
def test_damaged_blobs_never_trip_a_bounds_check(env, seed):
    r = np.random.default_rng(seed)
    x = SPECS[seed % len(SPECS)].generate(begin=1000 * seed, count=500_000 + seed)
    blob = oracle.encode(x)
    hd = oracle.blob_header(blob)
    damaged = []
    b = blob.copy()  # stream bytes
    pos = hd["stream_off"] + r.integers(0, max(1, hd["code_bits"] // 8), size=200)
    b[pos] ^= r.integers(1, 256, size=pos.size).astype(np.uint8)
    damaged.append(b)
    b = blob.copy()  # gap nibbles
    pos = hd["gaps_off"] + r.integers(0, max(1, hd["groups_off"] - hd["gaps_off"]), size=50)
    b[pos] = r.integers(0, 256, size=pos.size).astype(np.uint8)
    damaged.append(b)
    b = blob.copy()  # group offsets: small and huge changes
    g = r.integers(0, max(1, hd["n_groups"]), size=4)
    for k in g:
        b[hd["groups_off"] + 8 * int(k) + int(r.integers(0, 8))] ^= np.uint8(1 << int(r.integers(0, 8)))
    damaged.append(b)
    for bad in damaged:
        _, status, intact = _decode(env, [bad])
        assert intact
        assert not status & BOUNDS, status


# ---- the BF16 decoder in the checked build ----

def _bf16_decode_checked(env, blob, layout, guard=32):
    L, torch, so = env
    so.ecf8_bf16_decode_layout.argtypes = [ctypes.POINTER(L.Bf16Info), ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_int]
    info = L.bf16_blob_info(blob)
    d_blob = torch.from_numpy(blob).cuda()
    d_table = torch.from_numpy(L.bf16_table(info)).cuda()
    buf = torch.full((info.n + 2 * guard,), 0x3C3C, dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = so.ecf8_bf16_decode_layout(ctypes.byref(info), d_blob.data_ptr(), d_table.data_ptr(),
                                    buf.data_ptr() + 2 * guard, info.n, status.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream, L.BF16_LAYOUTS[layout])
    assert rc == 0
    torch.cuda.synchronize()
    got = buf.cpu().numpy().view(np.uint16)
    intact = (got[:guard] == 0x3C3C).all() and (got[-guard:] == 0x3C3C).all()
    return got[guard:-guard], int(status.item()), intact


def _bf16_layouts(L, blob):
    info = L.bf16_blob_info(blob)
    lens = info.lengths
    if lens[lens > 0].min() == 1:
        return ["wide"]
    return ["wide", "narrow"] + (["narrow_lane", "byte"] if L.bf16_table_nodes(info) + 1 <= 32 else [])


def _bf16_inputs():
    r = np.random.default_rng(17)
    spec = synth.llama3_8b_layer_bf16().tensors[0]
    return [spec.generate_bf16(begin=11, count=250_003),                       # byte / narrow_lane / narrow / wide
            r.integers(0, 1 << 16, 120_001).astype(np.uint16),                # 255 nodes: narrow / wide
            np.where(r.random(90_001) < 0.95, 0x3F80, 0xC000).astype(np.uint16),  # 1-bit codes: wide
            spec.generate_bf16(begin=5, count=17)]


@pytest.mark.parametrize("k", range(4))
def test_bf16_valid_blobs_pass_every_check(env, k):
    L = env[0]
    x = _bf16_inputs()[k]
    blob = oracle.bf16_encode(x)
    for layout in _bf16_layouts(L, blob):
        got, status, intact = _bf16_decode_checked(env, blob, layout)
        assert status == 0 and intact, layout
        assert np.array_equal(got, x), layout


@pytest.mark.parametrize("seed", range(3))
def test_bf16_damaged_blobs_never_trip_a_bounds_check(env, seed):
    L = env[0]
    r = np.random.default_rng(100 + seed)
    x = _bf16_inputs()[0]
    blob = oracle.bf16_encode(x)
    hd = oracle.bf16_blob_header(blob)
    damaged = []
    b = blob.copy()
    pos = hd["stream_off"] + r.integers(0, hd["code_bits"] // 8, size=150)
    b[pos] ^= r.integers(1, 256, size=pos.size).astype(np.uint8)
    damaged.append(b)
    b = blob.copy()
    pos = hd["gaps_off"] + r.integers(0, hd["groups_off"] - hd["gaps_off"], size=40)
    b[pos] = r.integers(0, 256, size=pos.size).astype(np.uint8)
    damaged.append(b)
    b = blob.copy()
    for g in r.integers(1, hd["n_groups"], size=3):
        b[hd["groups_off"] + 8 * int(g) + int(r.integers(0, 8))] ^= np.uint8(1 << int(r.integers(0, 8)))
    damaged.append(b)
    for bad in damaged:
        for layout in _bf16_layouts(L, blob):
            _, status, intact = _bf16_decode_checked(env, bad, layout)
            assert intact, layout
            assert not status & BOUNDS, (layout, status)
