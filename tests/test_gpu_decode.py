"""GPU decode parity: the sm_100a kernels, called through the C ABI, must give
back exactly the bytes the CPU oracle decodes (and therefore the original
tensor: ECF8 is lossless, walkthrough §1, arXiv 2510.02676 abstract).

All comparisons are bit-exact: decoding is integer work.
"""
import numpy as np
import pytest

import ecf8_synth as synth
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(gpu_available):
    import torch
    from lossless_fp8_weight_b200 import _build
    _build.build()
    import lossless_fp8_weight_b200 as L
    torch.cuda.init()
    return L, torch


def _to_dev(torch, a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_decode(env, blob: np.ndarray, guard: int = 64):
    """Decode on the GPU into a buffer with guard bytes on both sides; returns
    (output, status, guards-intact)."""
    L, torch = env
    info = L.blob_info(blob)
    d_blob = _to_dev(torch, blob)
    buf = torch.full((info.n + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    out = buf[guard:guard + info.n]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.decode(info, d_blob, out if info.n else buf, status=status)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    intact = bool((b[:guard] == 0xA5).all() and (b[guard + info.n:] == 0xA5).all())
    return b[guard:guard + info.n], int(status.item()), intact


def check_parity(env, x: np.ndarray):
    blob = oracle.encode(x)  # the oracle's blob: the GPU must parse it
    want = oracle.decode(blob, x.size)
    got, status, intact = gpu_decode(env, blob)
    assert status == 0 and intact
    assert np.array_equal(got, want)
    assert np.array_equal(got, x)


# ------------------------------------------------------------------ small and ragged

SIZES = [1, 2, 3, 7, 8, 31, 32, 33, 63, 64, 65, 255, 4095, 4096, 4097, 32767, 32768, 32769,
         131071, 131072 * 3 + 17, 1 << 20]


@pytest.mark.parametrize("n", SIZES)
def test_gaussian_sizes(env, n):
    check_parity(env, synth.single_normal_1k().tensors[0].generate(count=min(n, 1 << 20)))


def test_single_normal_1k_workload(env):
    """1024x1024, w ~ N(0,1)*16 (the small single-tensor workload)."""
    check_parity(env, synth.single_normal_1k().tensors[0].generate())


def test_every_byte_value_and_specials(env):
    r = np.random.default_rng(5)
    base = np.arange(256, dtype=np.uint8)
    x = np.concatenate([base, r.permutation(np.repeat(base, 997)), np.array([0x7F, 0xFF, 0x00, 0x80] * 999, np.uint8)])
    check_parity(env, x)


def test_uniform_random_bytes(env):
    check_parity(env, np.random.default_rng(6).integers(0, 256, size=2_000_003).astype(np.uint8))


def test_single_symbol_tensor(env):
    check_parity(env, np.full(1_000_001, 0x38, np.uint8))
    check_parity(env, np.full(33, 0xFF, np.uint8))


def test_two_symbols(env):
    r = np.random.default_rng(7)
    check_parity(env, np.where(r.random(500_000) < 0.01, 0x40, 0x00).astype(np.uint8))


def test_deepest_code_takes_the_long_path(env):
    """Fibonacci exponent counts: codes of up to 15 bits, which span two or
    three stream bytes; the byte state machine carries them across byte steps
    through its tree nodes like any shorter code."""
    fib = [1, 1]
    while len(fib) < 16:
        fib.append(fib[-1] + fib[-2])
    reps = 200
    e = np.repeat(np.arange(16, dtype=np.uint8), np.array(fib) * reps)
    e = np.random.default_rng(8).permutation(e)
    x = (e << 3) | np.random.default_rng(9).integers(0, 8, e.size).astype(np.uint8)
    assert oracle.blob_header(oracle.encode(x))["max_len"] == 15
    check_parity(env, x)


@pytest.mark.parametrize("alpha,max_abs", [(1.5, 28.0), (1.5, 448.0), (2.0, 448.0), (1.7, 112.0)])
def test_alpha_stable_prefix(env, alpha, max_abs):
    spec = synth.alpha_sweep_point(alpha, max_abs).tensors[0]
    check_parity(env, spec.generate(count=3_000_001))


def test_group_starts_inside_8_weight_blocks(env):
    """Format 3 orders the codes of each whole 8-weight block 0 4 1 5 2 6 3 7,
    so a group that starts or ends inside a block owns a scattered subset of
    the block's weights.  This tensor's group starts fall on every position
    within a block (checked from the blob's offsets), and the decode must
    still equal the oracle's byte for byte, ending in a partial last block."""
    for alpha, max_abs in [(1.7, 448.0), (1.5, 28.0)]:
        x = synth.alpha_sweep_point(alpha, max_abs).tensors[0].generate(begin=777, count=2_000_003)
        blob = oracle.encode(x)
        hd = oracle.blob_header(blob)
        offs = blob[hd["groups_off"]:hd["groups_off"] + 8 * (hd["n_groups"] + 1)].view("<u8")
        assert set(int(o) % 8 for o in offs[1:-1]) == set(range(8))
        got, status, intact = gpu_decode(env, blob)
        assert status == 0 and intact
        assert np.array_equal(got, oracle.decode(blob, x.size))
        assert np.array_equal(got, x)


def test_library_blob_decodes_too(env):
    L, _ = env
    x = synth.llama3_8b_layer().tensors[1].generate()
    blob = L.encode(x)
    got, status, intact = gpu_decode(env, blob)
    assert status == 0 and intact and np.array_equal(got, oracle.decode(blob, x.size))


def test_empty_tensor_is_a_no_op(env):
    L, torch = env
    blob = oracle.encode(np.zeros(0, np.uint8))
    info = L.blob_info(blob)
    d = _to_dev(torch, blob)
    out = torch.empty(16, dtype=torch.uint8, device="cuda")
    before = L.launch_count()
    L.decode(info, d, out)
    assert L.launch_count() == before


# ------------------------------------------------------------------ argument errors

def test_argument_errors(env):
    L, torch = env
    x = synth.single_normal_1k().tensors[0].generate(count=10_000)
    blob = L.encode(x)
    info = L.blob_info(blob)
    d = _to_dev(torch, np.concatenate([np.zeros(16, np.uint8), blob]))
    out = torch.empty(x.size + 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(L.Ecf8Error) as e:
        L.decode(info, int(d.data_ptr()) + 1, out)
    assert e.value.code == -5
    with pytest.raises(L.Ecf8Error) as e:
        L.decode(info, int(d.data_ptr()) + 16, int(out.data_ptr()) + 8)
    assert e.value.code == -5
    odd = L.encode(x, chunk_bytes=16, group_chunks=64)
    with pytest.raises(L.Ecf8Error) as e:
        L.decode(L.blob_info(odd), _to_dev(torch, odd), out)
    assert e.value.code == -6
    with pytest.raises(L.Ecf8Error) as e:  # a device buffer shorter than the blob
        L.decode(info, d[16:16 + info.blob_bytes - 1], out)
    assert e.value.code == -1


# ------------------------------------------------------------------ corrupt blobs

def _corrupt_and_decode(env, blob, where, flip):
    bad = blob.copy()
    bad[where] ^= flip
    return gpu_decode(env, bad)


def test_corrupt_gap_is_reported_and_contained(env):
    """A wrong gap desynchronises a thread (walkthrough §5.3): the kernel must
    say so and must not write outside the output."""
    x = synth.single_normal_1k().tensors[0].generate()
    blob = oracle.encode(x)
    hd = oracle.blob_header(blob)
    _, status, intact = _corrupt_and_decode(env, blob, hd["gaps_off"] + 40, 0x30)
    assert intact and status & 3  # the group's code count no longer matches its offsets, or no code



def test_corrupt_offsets_are_reported_and_contained(env):
    x = synth.single_normal_1k().tensors[0].generate()
    blob = oracle.encode(x)
    hd = oracle.blob_header(blob)
    _, status, intact = _corrupt_and_decode(env, blob, hd["groups_off"] + 8 * 5 + 7, 0x40)  # huge offset
    assert intact and status & 4
    _, status, intact = _corrupt_and_decode(env, blob, hd["groups_off"] + 8 * 5, 0x01)
    assert intact and status & 1


def test_corrupt_stream_is_reported_and_contained(env):
    x = synth.single_normal_1k().tensors[0].generate()
    blob = oracle.encode(x)
    hd = oracle.blob_header(blob)
    r = np.random.default_rng(4)
    bad = blob.copy()
    pos = hd["stream_off"] + r.integers(0, hd["code_bits"] // 8, size=50)
    bad[pos] ^= 0x5A
    _, status, intact = gpu_decode(env, bad)
    assert intact and status != 0


def test_single_symbol_book_seeing_a_one_bit(env):
    x = np.full(100_000, 0x38, np.uint8)
    blob = oracle.encode(x)
    hd = oracle.blob_header(blob)
    _, status, intact = _corrupt_and_decode(env, blob, hd["stream_off"] + 1000, 0x80)
    assert intact and status & 2


# ------------------------------------------------------------------ batched

def _batched(env, blobs, workspace=True):
    L, torch = env
    infos = [L.blob_info(b) for b in blobs]
    d_blobs = [_to_dev(torch, b) for b in blobs]
    outs = [torch.full((i.n,), 0xA5, dtype=torch.uint8, device="cuda") for i in infos]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws_bytes = L.batched_workspace_size(len(blobs))
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda") if workspace else None
    items = [L.BatchItem(i, b, o) for i, b, o in zip(infos, d_blobs, outs)]
    L.decode_batched(items, workspace=ws, status=status)
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in outs], int(status.item())


def test_batched_mixed_tensors_inline(env):
    r = np.random.default_rng(10)
    xs = [synth.single_normal_1k().tensors[0].generate(count=n) for n in (1, 33, 4097, 1 << 20, 77777)]
    xs += [r.integers(0, 256, size=123_457).astype(np.uint8), np.full(5, 0x38, np.uint8)]
    blobs = [oracle.encode(x) for x in xs]
    outs, status = _batched(env, blobs)
    assert status == 0
    for x, b, o in zip(xs, blobs, outs):
        assert np.array_equal(o, oracle.decode(b, x.size)) and np.array_equal(o, x)


def test_batched_many_tensors_uses_workspace(env):
    L, _ = env
    r = np.random.default_rng(11)
    xs = [synth.alpha_sweep_point(1.7, 448.0).tensors[0].generate(begin=int(r.integers(0, 1 << 24)),
                                                                  count=int(r.integers(1, 60_000)))
          for _ in range(150)]
    blobs = [L.encode(x) for x in xs]
    assert L.batched_workspace_size(len(blobs)) > 0
    outs, status = _batched(env, blobs)
    assert status == 0
    for x, b, o in zip(xs, blobs, outs):
        assert np.array_equal(o, oracle.decode(b, x.size))


def test_batched_without_workspace_fails_loudly(env):
    L, _ = env
    blobs = [L.encode(np.full(100, 0x38, np.uint8)) for _ in range(70)]
    with pytest.raises(L.Ecf8Error) as e:
        _batched(env, blobs, workspace=False)
    assert e.value.code == -8


def test_batched_decode_in_a_captured_graph(env):
    """A batch that travels in the launch's parameters (up to 64 tensors)
    copies nothing from the host, so it records into a CUDA graph and replays
    to the same bytes; a larger batch copies its descriptors from a host
    array and refuses capture (ECF8_ERR_CAPTURE) without enqueueing."""
    L, torch = env
    xs = [synth.single_normal_1k().tensors[0].generate(begin=7 * k, count=20_000 + 1000 * k) for k in range(5)]
    blobs = [L.encode(x) for x in xs]
    infos = [L.blob_info(b) for b in blobs]
    d_blobs = [_to_dev(torch, b) for b in blobs]
    outs = [torch.zeros(i.n, dtype=torch.uint8, device="cuda") for i in infos]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    batch = L.make_batch([L.BatchItem(i, b, o) for i, b, o in zip(infos, d_blobs, outs)])
    side = torch.cuda.Stream()
    L.decode_batched(batch, status=status, stream=side)  # first call outside capture: kernel attributes
    torch.cuda.synchronize()
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        L.decode_batched(batch, status=status, stream=side)
    g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for x, o in zip(xs, outs):
        assert np.array_equal(o.cpu().numpy(), x)

    big = [L.encode(np.full(100, 0x38, np.uint8)) for _ in range(L.BATCH_INLINE_MAX + 1)]
    big_infos = [L.blob_info(b) for b in big]
    big_dev = [_to_dev(torch, b) for b in big]
    big_out = [torch.empty(100, dtype=torch.uint8, device="cuda") for _ in big]
    ws = torch.empty(L.batched_workspace_size(len(big)), dtype=torch.uint8, device="cuda")
    big_batch = L.make_batch([L.BatchItem(i, b, o) for i, b, o in zip(big_infos, big_dev, big_out)])
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=side):
        with pytest.raises(L.Ecf8Error) as e:
            L.decode_batched(big_batch, workspace=ws, status=status, stream=side)
    assert e.value.code == -10
    L.decode_batched(big_batch, workspace=ws, status=status)  # outside capture it runs
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and all((o.cpu().numpy() == 0x38).all() for o in big_out)


def test_back_to_back_decodes_into_one_buffer_keep_stream_order(env):
    """Decodes launched back to back may start early (dependent launch) but
    must not write before the previous grid ends: alternate two tensors into
    one buffer with no synchronisation, reading a copy after each."""
    L, torch = env
    specs = [synth.alpha_sweep_point(1.7, 448.0).tensors[0], synth.alpha_sweep_point(1.5, 448.0).tensors[0]]
    xs = [s.generate(begin=99, count=3_000_017) for s in specs]
    infos, blobs = [], []
    for x in xs:
        b = L.encode(x)
        infos.append(L.blob_info(b))
        blobs.append(torch.from_numpy(b).cuda())
    out = torch.empty(xs[0].size, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    copies = []
    for k in range(12):
        j = k % 2
        L.decode(infos[j], blobs[j], out, status=status)
        copies.append((j, out.clone()))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for j, c in copies:
        assert np.array_equal(c.cpu().numpy(), xs[j])
