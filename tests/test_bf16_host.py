"""Host side of the BF16 variant (DFloat11 article §2-§3) in libecf8: the
library encoder writes the oracle's bytes, the header parser agrees with the
oracle's, the nibble-state decode table walks every stream back to its
exponents, and an emulation of the GPU kernel's per-lane partition (gap, bit
budget, zero-padding codes, warp scan, stage placement) reproduces the input
(ECF8 walkthrough §3.2.1 for the gap / group-offset plan the kernel shares)."""
import numpy as np
import pytest

import oracle
import lossless_fp8_weight_b200 as L


def _bf16_bits(f32) -> np.ndarray:
    u = np.asarray(f32, dtype=np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _cases():
    r = np.random.default_rng(11)
    return {
        "normal": _bf16_bits(r.standard_normal(40_003) * 0.02),
        "random_bits": r.integers(0, 1 << 16, 30_001).astype(np.uint16),
        "single_symbol": np.full(5000, 0x4049, dtype=np.uint16),
        "two_symbols": np.where(r.random(7777) < 0.9, 0x3F80, 0x4000).astype(np.uint16),
        "skewed_capped": (((np.minimum(r.geometric(0.5, 20_000), 200) + 20) << 7)
                          | r.integers(0, 128, 20_000)).astype(np.uint16),
        "one": np.array([0xBF80], dtype=np.uint16),
        "empty": np.zeros(0, dtype=np.uint16),
    }


CASES = _cases()


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("C,T", [(32, 32), (4, 1), (8, 3)])
def test_library_encoder_writes_the_oracle_bytes(name, C, T):
    x = CASES[name]
    a = L.bf16_encode(x, chunk_bytes=C, group_chunks=T)
    b = oracle.bf16_encode(x, chunk_bytes=C, group_chunks=T)
    assert np.array_equal(a, b)
    assert np.array_equal(L.bf16_code_lengths(x), oracle.bf16_blob_header(b)["lengths"])


def test_given_lengths_and_a_length_cap():
    x = CASES["skewed_capped"]
    for cap in (9, 12, 16):
        ln = L.bf16_code_lengths(x, cap)
        assert ln.max() <= cap
        assert np.array_equal(L.bf16_encode(x, lengths=ln), oracle.bf16_encode(x, lengths=ln))
    # a non-optimal but complete code: every present exponent at length 8
    ln = np.zeros(256, np.uint8)
    ln[:] = 8
    assert np.array_equal(L.bf16_encode(x, lengths=ln), oracle.bf16_encode(x, lengths=ln))


@pytest.mark.parametrize("name", list(CASES))
def test_blob_info_matches_the_header(name):
    x = CASES[name]
    blob = oracle.bf16_encode(x)
    hd = oracle.bf16_blob_header(blob)
    i = L.bf16_blob_info(blob)
    assert i.n == x.size and i.code_bits == hd["code_bits"] and i.n_groups == hd["n_groups"]
    assert i.max_len == hd["max_len"] and i.blob_bytes == blob.size
    assert (i.stream_off, i.kept_off, i.gaps_off, i.groups_off) == (hd["stream_off"], hd["kept_off"],
                                                                     hd["gaps_off"], hd["groups_off"])
    assert np.array_equal(i.lengths, hd["lengths"])


def test_blob_info_rejects_damaged_headers():
    blob = oracle.bf16_encode(CASES["normal"])
    for off, val in [(0, 0x00), (4, 2), (40, 7), (80, 1)]:
        b = blob.copy()
        b[off] ^= val if val else 0xFF
        with pytest.raises(L.Ecf8Error):
            L.bf16_blob_info(b)
    b = blob.copy()
    hd = oracle.bf16_blob_header(blob)
    b[hd["lens_off"] + int(np.argmax(hd["lengths"]))] += 1  # breaks the Kraft sum
    with pytest.raises(L.Ecf8Error):
        L.bf16_blob_info(b)
    with pytest.raises(L.Ecf8Error):
        L.bf16_blob_info(blob[:100])


def _table(info):
    """(exponents, count, next node) per entry, and the error node."""
    t = L.bf16_table(info).view(np.uint32).reshape(256 * 16, 2).astype(np.int64)
    return t[:, 0], (t[:, 1] >> 16) // 8, (t[:, 1] >> 7) & 0xFF, L.bf16_table_nodes(info)


def _stream_bits(blob, hd):
    words = blob[hd["stream_off"]:hd["stream_off"] + 4 * ((hd["code_bits"] + 31) // 32)].view("<u4")
    return np.unpackbits(words.astype(">u4").view(np.uint8))[:hd["code_bits"]]


@pytest.mark.parametrize("name", [n for n in CASES if n != "empty"])
def test_table_walk_decodes_the_whole_stream(name):
    """Walk the table over the stream a nibble at a time from the root."""
    x = CASES[name]
    blob = oracle.bf16_encode(x)
    hd = oracle.bf16_blob_header(blob)
    syms, cnt, nxt, err = _table(L.bf16_blob_info(blob))
    bits = _stream_bits(blob, hd)
    bits = np.concatenate([bits, np.zeros((-bits.size) % 4, np.uint8)])
    nibs = bits.reshape(-1, 4) @ np.array([8, 4, 2, 1])
    node, out = 0, []
    for v in nibs:
        e = node * 16 + int(v)
        out += [(int(syms[e]) >> (8 * j)) & 0xFF for j in range(int(cnt[e]))]
        node = int(nxt[e])
        assert node != err
    lmin = int(hd["lengths"][hd["lengths"] > 0].min())
    pad = (-hd["code_bits"]) % 4  # zero bits after the stream decode as the all-zeros code
    extra = pad // lmin
    assert len(out) == x.size + extra
    assert np.array_equal(np.array(out[:x.size], dtype=np.uint16), (x >> 7) & 0xFF)


def test_table_node_count_is_the_internal_nodes():
    """A complete code over k exponents has k - 1 internal nodes."""
    for name in ("normal", "random_bits", "two_symbols", "skewed_capped"):
        info = L.bf16_blob_info(oracle.bf16_encode(CASES[name]))
        assert L.bf16_table_nodes(info) == int((info.lengths > 0).sum()) - 1


def test_table_error_node_and_invalid_bits():
    x = CASES["single_symbol"]
    info = L.bf16_blob_info(oracle.bf16_encode(x))
    syms, cnt, nxt, err = _table(info)
    assert err == 1  # the root is the only node
    assert cnt[0] == 4 and syms[0] == 0x80808080 and nxt[0] == 0  # four 1-bit codes 0 of exponent 128
    for v in range(1, 16):
        assert nxt[v] == err and cnt[v] == 0  # a 1 bit is no code
    for s_ in range(err, 256):
        assert (nxt[16 * s_:16 * s_ + 16] == err).all()  # the error node (and the unused ones) absorb
    # a single exponent with a 3-bit code: one exponent per three zero bits
    ln = np.zeros(256, np.uint8)
    ln[128] = 3
    blob = oracle.bf16_encode(x, lengths=ln)
    assert np.array_equal(oracle.bf16_decode(blob, x.size), x)
    syms, cnt, nxt, err = _table(L.bf16_blob_info(blob))
    assert err == 3
    node, got = 0, 0
    for _ in range(6):  # 24 zero bits = 8 codes
        e = node * 16
        got += int(cnt[e])
        node = int(nxt[e])
    assert got == 8 and node == 0


def _emulate_kernel(blob, x_size):
    """The GPU kernel's per-lane plan in numpy (C = T = 32): lane bits from its
    gap to the next chunk's gap, 68-nibble walk over zero-padded bits, padding
    codes removed by count, warp scan, byte placement relative to the group's
    16-aligned base, then join with the kept bytes."""
    hd = oracle.bf16_blob_header(blob)
    info = L.bf16_blob_info(blob)
    syms, cnt_t, nxt, err = _table(info)
    lens = hd["lengths"]
    lmin = int(lens[lens > 0].min())
    gaps_b = blob[hd["gaps_off"]:hd["groups_off"]]
    groups = blob[hd["groups_off"]:hd["groups_off"] + 8 * (hd["n_groups"] + 1)].view("<u8")
    sbytes = blob[hd["stream_off"]:hd["kept_off"]]
    kept = blob[hd["kept_off"]:hd["kept_off"] + x_size]
    out = np.full(x_size, 0xDEAD, dtype=np.uint32)
    nchunks = hd["n_groups"] * 32

    def gap_of(c):
        return (int(gaps_b[c // 2]) >> (4 * (c % 2))) & 15 if c < nchunks else 0

    for g in range(hd["n_groups"]):
        off0, off1 = int(groups[g]), int(groups[g + 1])
        assert off1 - off0 <= 8192
        counts, lane_syms = [], []
        for lane in range(32):
            c = g * 32 + lane
            gap = gap_of(c)
            gap_next = gap_of(c + 1) if (lane < 31 or g + 1 < hd["n_groups"]) else 0
            bit0 = c * 256
            left = max(hd["code_bits"] - bit0, 0)
            stop = min(left, 256 + gap_next)
            E = max(stop - gap, 0)
            assert E <= 271
            w = sbytes[32 * c:32 * c + 36]  # 9 words: the chunk and one more (inside the 16-byte tail)
            assert w.size == 36
            bits = np.unpackbits(w.view("<u4").astype(">u4").view(np.uint8))[gap:gap + 272].copy()
            bits = np.concatenate([bits, np.zeros(272 - bits.size, np.uint8)])
            bits[E:] = 0
            node, got = 0, []
            for j in range(68):
                v = int(bits[4 * j:4 * j + 4] @ np.array([8, 4, 2, 1]))
                e = node * 16 + v
                got += [(int(syms[e]) >> (8 * q)) & 0xFF for q in range(int(cnt_t[e]))]
                node = int(nxt[e])
            assert node != err and len(got) <= 4 * 69
            extra = (272 - E) // lmin
            assert len(got) >= extra
            cnt = len(got) - extra
            counts.append(cnt)
            lane_syms.append(got[:cnt])
        assert sum(counts) == off1 - off0
        stage = np.zeros(8192 + 32, np.uint8)
        start = 0
        for lane in range(32):
            q = (off0 & 15) + start
            stage[q:q + counts[lane]] = lane_syms[lane]
            start += counts[lane]
        base = off0 & ~15
        for p in range(off0, off1):
            e = int(stage[p - base])
            k = int(kept[p])
            out[p] = ((k >> 7) << 15) | (e << 7) | (k & 0x7F)
    return out.astype(np.uint16)


@pytest.mark.parametrize("name", ["normal", "random_bits", "single_symbol", "two_symbols", "skewed_capped", "one"])
def test_kernel_plan_emulation_reproduces_the_input(name):
    x = CASES[name][:12_000]
    blob = oracle.bf16_encode(x)
    assert np.array_equal(_emulate_kernel(blob, x.size), x)


def _layout(info):
    """The decoder's table layout for a code: wide when a 1-bit code exists,
    else byte steps when the tree has at most 31 nodes, else narrow."""
    lens = info.lengths
    want = "wide" if lens[lens > 0].min() == 1 else "byte" if L.bf16_table_nodes(info) + 1 <= 32 else "narrow"
    assert L.bf16_auto_layout(info) == want
    return want


@pytest.mark.parametrize("name", ["normal", "random_bits", "skewed_capped", "two_symbols"])
def test_narrow_entries_hold_at_most_two_exponents(name):
    """With no 1-bit code a nibble ends at most two codes, so the narrow
    32-bit entry (16 bits of exponents, node, 8 x count <= 16) loses nothing."""
    info = L.bf16_blob_info(oracle.bf16_encode(CASES[name]))
    syms, cnt, nxt, err = _table(info)
    live = slice(0, 16 * (err + 1))
    if _layout(info) == "wide":
        assert cnt[live].max() <= 4
    else:
        assert cnt[live].max() <= 2 and (syms[live] >> 16 == 0).all() and nxt[live].max() <= err


def test_gpu_cases_cover_every_table_layout():
    r = np.random.default_rng(5)
    seen = {
        _layout(L.bf16_blob_info(oracle.bf16_encode(x)))
        for x in (CASES["normal"], CASES["random_bits"], CASES["two_symbols"], CASES["skewed_capped"],
                  _bf16_bits(r.standard_normal(50_000) * np.exp(r.uniform(-60, 60, 50_000))))
    }
    assert seen == {"wide", "narrow", "byte"}


@pytest.mark.parametrize("name", ["normal", "two_symbols", "skewed_capped"])
def test_byte_steps_compose_two_nibble_steps(name):
    """The byte-step entry the device builds for (node, byte) is the nibble
    walk of the byte's high then low nibble: at most 4 exponents when no code
    has 1 bit (a byte then ends at most 1 + 3 // 2 + ... codes)."""
    info = L.bf16_blob_info(oracle.bf16_encode(CASES[name]))
    syms, cnt, nxt, err = _table(info)
    lens = info.lengths
    for node in range(err + 1):
        for byte in range(256):
            e1 = node * 16 + (byte >> 4)
            e2 = int(nxt[e1]) * 16 + (byte & 15)
            k = int(cnt[e1]) + int(cnt[e2])
            if lens[lens > 0].min() >= 2:
                assert k <= 4
            got = (int(syms[e1]) | (int(syms[e2]) << (8 * int(cnt[e1])))) & ((1 << 32) - 1)
            assert got >> (8 * k) == 0 or k == 4


def test_encoder_refuses_lengths_that_are_not_a_complete_code():
    x = CASES["two_symbols"]
    e = (x >> 7) & 0xFF
    for bad in ({127: 1, 128: 2}, {127: 2, 128: 2}, {127: 17, 128: 1}, {127: 1}):
        ln = np.zeros(256, np.uint8)
        for k, v in bad.items():
            ln[k] = v
        with pytest.raises(L.Ecf8Error):
            L.bf16_encode(x, lengths=ln)
    ln = np.zeros(256, np.uint8)
    ln[np.unique(e)] = 1  # complete: two 1-bit codes
    assert np.array_equal(oracle.bf16_decode(L.bf16_encode(x, lengths=ln), x.size), x)
    one = np.full(100, 0x3F80, np.uint16)
    ln = np.zeros(256, np.uint8)
    ln[127] = 4  # a single value may take any length
    assert np.array_equal(L.bf16_encode(one, lengths=ln), oracle.bf16_encode(one, lengths=ln))


@pytest.mark.parametrize("C,T", [(32, 32), (4, 1), (12, 5)])
def test_threaded_encoder_matches_the_serial_oracle(C, T):
    """Over 1M weights a thread the library packs ranges concurrently (shared
    boundary words OR-ed, gaps and offsets per range); the bytes must not
    depend on that split."""
    import ecf8_synth as synth
    x = synth.llama3_8b_layer_bf16().tensors[1].generate_bf16(begin=99, count=3_300_017)
    x[::4099] ^= 0x4000  # a wider exponent spread
    ln = L.bf16_code_lengths(x)
    assert np.array_equal(ln, oracle.bf16_blob_header(oracle.bf16_encode(x[:1000], lengths=ln))["lengths"])
    assert np.array_equal(L.bf16_encode(x, lengths=ln, chunk_bytes=C, group_chunks=T),
                          oracle.bf16_encode(x, lengths=ln, chunk_bytes=C, group_chunks=T))


FAKE = 1 << 20  # a 16-byte-aligned address that is never dereferenced


def test_argument_errors_are_returned_before_any_device_work():
    """Every error path of the BF16 entry points returns before a CUDA call,
    so it can be exercised without a GPU."""
    import ctypes
    lib = L._lib
    ARG, CODEBOOK, CAPACITY, ALIGN, UNSUPPORTED = -1, -4, -3, -5, -6
    x = CASES["normal"]
    ln = L.bf16_code_lengths(x)
    size = ctypes.c_size_t(0)
    assert lib.ecf8_bf16_code_lengths(x.ctypes.data, x.size, 16, None) == ARG
    assert lib.ecf8_bf16_code_lengths(x.ctypes.data, x.size, 0, ln.ctypes.data) == ARG
    assert lib.ecf8_bf16_code_lengths(x.ctypes.data, x.size, 17, ln.ctypes.data) == ARG
    assert lib.ecf8_bf16_encoded_size(x.ctypes.data, x.size, ln.ctypes.data, 6, 32, ctypes.byref(size)) == ARG
    assert lib.ecf8_bf16_encoded_size(x.ctypes.data, x.size, ln.ctypes.data, 32, 0, ctypes.byref(size)) == ARG
    assert lib.ecf8_bf16_encoded_size(x.ctypes.data, x.size, ln.ctypes.data, 32, 32, None) == ARG
    assert lib.ecf8_bf16_encoded_size(x.ctypes.data, x.size, ln.ctypes.data, 32, 32, ctypes.byref(size)) == 0
    small = np.zeros(size.value - 1, np.uint8)
    got = ctypes.c_size_t(0)
    assert lib.ecf8_bf16_encode(x.ctypes.data, x.size, ln.ctypes.data, 32, 32, small.ctypes.data, small.size,
                                ctypes.byref(got)) == CAPACITY
    assert lib.ecf8_bf16_blob_info(None, 0, None) == ARG
    assert lib.ecf8_bf16_build_table(None, FAKE) == ARG
    assert lib.ecf8_bf16_table_nodes(None) == 0
    assert lib.ecf8_bf16_auto_layout(None) == ARG

    blob = L.bf16_encode(x)
    info = L.bf16_blob_info(blob)
    dec = lib.ecf8_bf16_decode_layout
    ref = ctypes.byref(info)
    assert dec(ref, FAKE, FAKE, FAKE, info.n + 1, None, None, -1) == ARG          # n differs from the header
    assert dec(ref, FAKE, FAKE, FAKE, info.n, None, None, 7) == ARG               # no such layout
    assert dec(ref, None, FAKE, FAKE, info.n, None, None, -1) == ARG              # null blob
    assert dec(ref, FAKE + 4, FAKE, FAKE, info.n, None, None, -1) == ALIGN        # unaligned blob
    assert dec(ref, FAKE, FAKE, FAKE + 2, info.n, None, None, -1) == ALIGN        # unaligned output
    wide_only = L.bf16_blob_info(L.bf16_encode(CASES["two_symbols"]))
    assert dec(ctypes.byref(wide_only), FAKE, FAKE, FAKE, wide_only.n, None, None, 3) == UNSUPPORTED
    other = L.bf16_blob_info(L.bf16_encode(x, chunk_bytes=16, group_chunks=8))
    assert dec(ctypes.byref(other), FAKE, FAKE, FAKE, other.n, None, None, -1) == UNSUPPORTED
    empty = L.bf16_blob_info(L.bf16_encode(np.zeros(0, np.uint16)))
    assert dec(ctypes.byref(empty), None, None, None, 0, None, None, -1) == 0    # nothing to do

    T = L.Bf16Tensor
    assert lib.ecf8_bf16_decode_batched(None, -1, None, None) == ARG
    assert lib.ecf8_bf16_decode_batched(None, 0, None, None) == 0
    arr = (T * 2)(T(ctypes.pointer(info), FAKE, FAKE, FAKE), T(ctypes.pointer(other), FAKE, FAKE, FAKE))
    assert lib.ecf8_bf16_decode_batched(arr, 2, None, None) == UNSUPPORTED    # checked before anything runs
    arr = (T * 1)(T(None, FAKE, FAKE, FAKE))
    assert lib.ecf8_bf16_decode_batched(arr, 1, None, None) == ARG
