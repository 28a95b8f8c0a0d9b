"""GPU decoder of the BF16 variant (DFloat11 article §2-§3) against the
oracle: bit-exact BF16 output on seeded inputs spanning many groups and a
ragged tail, the full Llama-3-8B decoder layer in BF16 (sampled against the
oracle, and whole against the input the oracle round-trips), the decoded
tensor used as torch.bfloat16, edge cases, argument errors, and damaged
streams that must be reported without writing outside the output."""
import numpy as np
import pytest

import ecf8_synth as synth
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(gpu_available):
    import torch
    import lossless_fp8_weight_b200 as L
    return L, torch


def _decode(env, blob, guard=64, layout="auto"):
    L, torch = env
    info = L.bf16_blob_info(blob)
    d_blob = torch.from_numpy(blob).cuda()
    d_table = torch.from_numpy(L.bf16_table(info)).cuda()
    buf = torch.full((info.n + 2 * guard,), 0x5A5A, dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    launches = L.launch_count()
    L.bf16_decode(info, d_blob, d_table, buf[guard:guard + info.n], status, layout=layout)
    torch.cuda.synchronize()
    if info.n:
        assert L.launch_count() == launches + 1
    got = buf.cpu().numpy().view(np.uint16)
    intact = (got[:guard] == 0x5A5A).all() and (got[guard + info.n:] == 0x5A5A).all()
    return got[guard:guard + info.n], int(status.item()), bool(intact)


def _bf16_bits(f32) -> np.ndarray:
    u = np.asarray(f32, dtype=np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _cases():
    r = np.random.default_rng(5)
    spec = synth.llama3_8b_layer_bf16().tensors[0]
    return {
        "normal_multi_group": spec.generate_bf16(begin=123, count=300_007),
        "random_bits": r.integers(0, 1 << 16, 200_003).astype(np.uint16),
        "single_symbol": np.full(70_001, 0x4049, dtype=np.uint16),
        "two_symbols": np.where(r.random(100_000) < 0.97, 0x3F80, 0xC000).astype(np.uint16),
        "skewed_16bit_codes": (((np.minimum(r.geometric(0.5, 150_000), 230) + 10) << 7)
                               | r.integers(0, 256, 150_000) & 0x807F).astype(np.uint16),
        "specials": np.tile(np.array([0x7F80, 0xFF80, 0x7FC0, 0x0000, 0x8000, 0x0001, 0x807F, 0x3F80],
                                     dtype=np.uint16), 4001),
        "wide_dynamic_range": _bf16_bits(r.standard_normal(123_457) * np.exp(r.uniform(-60, 60, 123_457))),
    }


CASES = _cases()


@pytest.mark.parametrize("name", list(CASES))
def test_decode_matches_the_oracle(env, name):
    x = CASES[name]
    blob = oracle.bf16_encode(x)
    want = oracle.bf16_decode(blob, x.size)
    got, status, intact = _decode(env, blob)
    assert status == 0 and intact
    assert np.array_equal(got, want)
    assert np.array_equal(got, x)


def _layouts(L, blob):
    """Every table layout that can hold the blob's code."""
    info = L.bf16_blob_info(blob)
    lens = info.lengths
    if lens[lens > 0].min() == 1:
        return ["wide"]
    small = L.bf16_table_nodes(info) + 1 <= 32
    return ["wide", "narrow"] + (["narrow_lane", "byte"] if small else [])


@pytest.mark.parametrize("name", list(CASES))
def test_every_table_layout_gives_the_same_output(env, name):
    L, torch = env
    x = CASES[name]
    blob = oracle.bf16_encode(x)
    want = oracle.bf16_decode(blob, x.size)
    for layout in _layouts(L, blob):
        got, status, intact = _decode(env, blob, layout=layout)
        assert status == 0 and intact, layout
        assert np.array_equal(got, want), layout


def test_a_layout_that_cannot_hold_the_code_is_refused(env):
    L, torch = env
    blob = oracle.bf16_encode(CASES["two_symbols"])  # 1-bit codes: wide only
    info = L.bf16_blob_info(blob)
    d_blob = torch.from_numpy(blob).cuda()
    d_table = torch.from_numpy(L.bf16_table(info)).cuda()
    out = torch.empty(info.n, dtype=torch.int16, device="cuda")
    for layout in ("narrow", "narrow_lane", "byte"):
        with pytest.raises(L.Ecf8Error) as e:
            L.bf16_decode(info, d_blob, d_table, out, layout=layout)
        assert e.value.code == -6
    blob = oracle.bf16_encode(CASES["random_bits"])  # 255 nodes: no lane-private or byte table
    info = L.bf16_blob_info(blob)
    for layout in ("narrow_lane", "byte"):
        with pytest.raises(L.Ecf8Error) as e:
            L.bf16_decode(info, torch.from_numpy(blob).cuda(), torch.from_numpy(L.bf16_table(info)).cuda(),
                          torch.empty(info.n, dtype=torch.int16, device="cuda"), layout=layout)
        assert e.value.code == -6


@pytest.mark.parametrize("n", [1, 2, 15, 16, 17, 31, 33, 1000, 4095, 8191, 8192, 8193, 65_537])
def test_small_and_ragged_sizes(env, n):
    L, torch = env
    x = synth.llama3_8b_layer_bf16().tensors[2].generate_bf16(begin=n, count=n)
    blob = oracle.bf16_encode(x)
    want = oracle.bf16_decode(blob, n)
    for layout in _layouts(L, blob):
        got, status, intact = _decode(env, blob, layout=layout)
        assert status == 0 and intact, layout
        assert np.array_equal(got, want), layout


@pytest.mark.parametrize("cap", [8, 12])
def test_length_capped_codes(env, cap):
    x = CASES["wide_dynamic_range"]
    ln = oracle.bf16_code_lengths(np.bincount((x >> 7) & 0xFF, minlength=256).astype(np.uint64), cap)
    blob = oracle.bf16_encode(x, lengths=ln)
    got, status, intact = _decode(env, blob)
    assert status == 0 and intact and np.array_equal(got, x)


def test_single_exponent_with_a_long_code(env):
    x = np.full(40_000, 0xC0A0, dtype=np.uint16) ^ (np.arange(40_000) & 0x7F).astype(np.uint16)
    ln = np.zeros(256, np.uint8)
    ln[(0xC0A0 >> 7) & 0xFF] = 5
    blob = oracle.bf16_encode(x, lengths=ln)
    got, status, intact = _decode(env, blob)
    assert status == 0 and intact and np.array_equal(got, x)


def test_full_llama3_8b_layer(env):
    """Every projection of the layer at full size.  The two 4M-weight ones
    against the oracle's decode of the same blob element by element; the
    others (where the oracle's bit-serial decode takes tens of seconds) whole
    against the input, which the oracle's round trip reproduces (lossless:
    DFloat11 article §3)."""
    L, torch = env
    for spec in synth.llama3_8b_layer_bf16().tensors:
        x = spec.generate_bf16()
        blob = L.bf16_encode(x)
        got, status, intact = _decode(env, blob)
        assert status == 0 and intact
        if x.size <= 4 * 1024 * 1024:
            assert np.array_equal(got, oracle.bf16_decode(blob, x.size))
        assert np.array_equal(got, x)


def _batched(env, blobs, guard=64):
    L, torch = env
    infos = [L.bf16_blob_info(b) for b in blobs]
    keep, items, bufs = [], [], []
    for info, blob in zip(infos, blobs):
        d_blob = torch.from_numpy(blob).cuda()
        d_table = torch.from_numpy(L.bf16_table(info)).cuda()
        buf = torch.full((info.n + 2 * guard,), 0x5A5A, dtype=torch.int16, device="cuda")
        keep += [d_blob, d_table]
        bufs.append(buf)
        items.append((info, d_blob, d_table, buf[guard:guard + info.n]))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    launches = L.launch_count()
    L.bf16_decode_batched(items, status)
    torch.cuda.synchronize()
    outs = []
    for info, buf in zip(infos, bufs):
        got = buf.cpu().numpy().view(np.uint16)
        assert (got[:guard] == 0x5A5A).all() and (got[guard + info.n:] == 0x5A5A).all()
        outs.append(got[guard:guard + info.n])
    return outs, int(status.item()), L.launch_count() - launches


def test_batched_mixed_layouts_and_an_empty_tensor(env):
    L = env[0]
    xs = list(CASES.values()) + [np.zeros(0, np.uint16)]
    blobs = [oracle.bf16_encode(x) for x in xs]
    outs, status, launches = _batched(env, blobs)
    assert status == 0
    assert launches == len({L.bf16_auto_layout(L.bf16_blob_info(b)) for b in blobs if x_size(b)})
    for got, x, blob in zip(outs, xs, blobs):
        assert np.array_equal(got, oracle.bf16_decode(blob, x.size))


def x_size(blob):
    return int(oracle.bf16_blob_header(blob)["n"])


def test_batched_more_tensors_than_one_launch_carries(env):
    L = env[0]
    spec = synth.llama3_8b_layer_bf16().tensors[1]
    xs = [spec.generate_bf16(begin=7919 * k, count=3000 + 977 * k) for k in range(L.BF16_BATCH_MAX + 9)]
    blobs = [oracle.bf16_encode(x) for x in xs]
    outs, status, launches = _batched(env, blobs)
    assert status == 0 and launches == 2
    for got, x in zip(outs, xs):
        assert np.array_equal(got, x)


def test_batched_full_llama3_8b_layer(env):
    L = env[0]
    xs = [t.generate_bf16() for t in synth.llama3_8b_layer_bf16().tensors]
    blobs = [L.bf16_encode(x) for x in xs]
    outs, status, launches = _batched(env, blobs)
    assert status == 0 and launches == 1
    for got, x in zip(outs, xs):
        assert np.array_equal(got, x)


def test_output_is_a_usable_bfloat16_tensor(env):
    L, torch = env
    w = torch.randn(4096, 1024, dtype=torch.float32).to(torch.bfloat16)
    blob = L.bf16_encode(w)
    info = L.bf16_blob_info(blob)
    out = torch.empty_like(w, device="cuda")
    L.bf16_decode(info, torch.from_numpy(blob).cuda(), torch.from_numpy(L.bf16_table(info)).cuda(), out)
    assert torch.equal(out.cpu(), w)
    v = torch.randn(1024, dtype=torch.bfloat16, device="cuda")
    assert torch.equal(out @ v, w.cuda() @ v)


def test_empty_and_argument_errors(env):
    L, torch = env
    blob = oracle.bf16_encode(np.zeros(0, np.uint16))
    info = L.bf16_blob_info(blob)
    L.bf16_decode(info, 0, 0, 0)  # n = 0: nothing launched, nothing touched
    x = CASES["normal_multi_group"][:5000]
    blob = oracle.bf16_encode(x)
    info = L.bf16_blob_info(blob)
    d_blob = torch.from_numpy(blob).cuda()
    d_table = torch.from_numpy(L.bf16_table(info)).cuda()
    out = torch.empty(5008, dtype=torch.int16, device="cuda")
    with pytest.raises(L.Ecf8Error) as e:
        L.bf16_decode(info, d_blob, d_table, out[1:])
    assert e.value.code == -5
    with pytest.raises(L.Ecf8Error) as e:
        L.bf16_decode(info, 0, d_table, out)
    assert e.value.code == -1
    other = L.bf16_blob_info(oracle.bf16_encode(x, chunk_bytes=16, group_chunks=8))
    with pytest.raises(L.Ecf8Error) as e:
        L.bf16_decode(other, d_blob, d_table, out)
    assert e.value.code == -6


@pytest.mark.parametrize("seed", range(4))
def test_damaged_streams_are_reported_and_stay_in_bounds(env, seed):
    r = np.random.default_rng(seed)
    x = CASES["normal_multi_group"]
    blob = oracle.bf16_encode(x)
    hd = oracle.bf16_blob_header(blob)
    kinds = []
    b = blob.copy()
    pos = hd["stream_off"] + r.integers(0, hd["code_bits"] // 8, size=100)
    b[pos] ^= r.integers(1, 256, size=pos.size).astype(np.uint8)
    kinds.append(b)
    b = blob.copy()
    pos = hd["gaps_off"] + r.integers(0, hd["groups_off"] - hd["gaps_off"], size=40)
    b[pos] = r.integers(0, 256, size=pos.size).astype(np.uint8)
    kinds.append(b)
    b = blob.copy()
    k = int(r.integers(1, hd["n_groups"]))
    b[hd["groups_off"] + 8 * k:hd["groups_off"] + 8 * k + 8] = np.frombuffer(
        np.uint64(int(r.integers(0, 1 << 40))).tobytes(), np.uint8)
    kinds.append(b)
    L = env[0]
    for bad in kinds:
        for layout in _layouts(L, blob):
            got, status, intact = _decode(env, bad, layout=layout)
            assert intact, layout
            assert status != 0 or np.array_equal(got, x), layout
