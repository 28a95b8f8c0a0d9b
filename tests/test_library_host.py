"""Host side of libecf8 on CPU: the C ABI loads and exports what include/ecf8.h
declares, the encoder writes exactly the oracle's bytes, and the blob parser
rejects damaged headers.  No GPU call is made here."""
import ctypes
import os
import re

import numpy as np
import pytest

import ecf8_synth as synth
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from lossless_fp8_weight_b200 import _build
    _build.build()
    import lossless_fp8_weight_b200 as lib
    return lib


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "ecf8.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ecf8_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function(L):
    names = _declared_functions()
    assert "ecf8_decode" in names and "ecf8_decode_batched" in names and "ecf8_encode" in names
    so = ctypes.CDLL(L.library_path())
    for nm in names:
        assert hasattr(so, nm), nm


def test_abi_version_and_strerror(L):
    so = ctypes.CDLL(L.library_path())
    assert so.ecf8_abi_version() == 2
    so.ecf8_strerror.restype = ctypes.c_char_p
    assert so.ecf8_strerror(0) == b"ok"
    assert so.ecf8_strerror(-5).startswith(b"device pointer")


@pytest.mark.parametrize("n", [0, 1, 2, 3, 7, 31, 32, 33, 4095, 4096, 4097, 65537])
@pytest.mark.parametrize("layout", [(32, 32), (32, 128), (4, 1), (16, 3), (8, 5), (64, 64)])
def test_encoder_bytes_equal_oracle(L, n, layout):
    x = synth.single_normal_1k().tensors[0].generate(count=n) if n else np.zeros(0, np.uint8)
    C, T = layout
    assert np.array_equal(L.encode(x, chunk_bytes=C, group_chunks=T), oracle.encode(x, chunk_bytes=C, group_chunks=T))


def test_encoder_bytes_equal_oracle_on_hard_inputs(L):
    r = np.random.default_rng(3)
    fib = [1, 1]
    while len(fib) < 16:
        fib.append(fib[-1] + fib[-2])
    cases = [
        r.integers(0, 256, size=200_003).astype(np.uint8),           # all 16 exponents, incompressible
        np.full(70_001, 0x7F, np.uint8),                                # one symbol (NaN pattern)
        np.repeat(np.arange(16, dtype=np.uint8) << 3, fib),           # depth-15 code
        np.concatenate([np.zeros(5000, np.uint8), np.full(5000, 0x80, np.uint8)]),  # +-0
        synth.alpha_sweep_point(1.5, 28.0).tensors[0].generate(count=3_000_000),   # mostly 1-bit codes
        # three encoder thread ranges whose even splits (1,000,001 and 2,000,003)
        # fall inside 8-weight blocks, and a last block of 5 weights
        synth.single_normal_1k().tensors[0].generate(count=3_000_005),
    ]
    for x in cases:
        assert np.array_equal(L.encode(x), oracle.encode(x))


@pytest.mark.parametrize("max_len", [4, 5, 7, 9, 12, 16])
def test_codebook_equals_oracle(L, max_len):
    r = np.random.default_rng(max_len)
    for _ in range(200):
        k = int(r.integers(1, 17))
        h = np.zeros(16, np.uint64)
        h[r.choice(16, k, replace=False)] = r.integers(1, 10 ** int(r.integers(1, 9)), size=k)
        if (1 << max_len) < k:
            continue
        cb = L.build_codebook(h, max_len)
        want = oracle.code_lengths(h, max_len)
        assert np.array_equal(cb.lengths, want)
        codes = oracle.canonical_codes(want)
        assert [cb.code[s] for s in range(16) if want[s]] == [int(codes[s]) for s in range(16) if want[s]]


def test_histogram_equals_oracle(L):
    x = np.random.default_rng(1).integers(0, 256, size=3_000_001).astype(np.uint8)
    assert np.array_equal(L.histogram(x), oracle.histogram(x))


def test_blob_info_reads_header(L):
    x = synth.single_normal_1k().tensors[0].generate()
    blob = L.encode(x)
    info = L.blob_info(blob)
    hd = oracle.blob_header(blob)
    assert info.n == x.size and info.code_bits == hd["code_bits"] and info.n_groups == hd["n_groups"]
    assert info.blob_bytes == blob.size and info.stream_off == hd["stream_off"]
    assert np.array_equal(info.lengths, hd["lengths"])


def test_blob_info_rejects_damage(L):
    x = synth.single_normal_1k().tensors[0].generate(count=100_000)
    blob = L.encode(x)
    for off, bit in [(0, 1), (4, 1), (8, 1), (18, 1), (24, 4), (32, 1), (36, 1), (56, 1), (88, 1)]:
        bad = blob.copy()
        bad[off] ^= bit
        with pytest.raises(L.Ecf8Error):
            L.blob_info(bad)
    bad = blob.copy()
    bad[36] = 12  # the version-1 table field: version 2 reserves it as 0
    with pytest.raises(L.Ecf8Error):
        L.blob_info(bad)
    bad = blob.copy()
    bad[96 + 9] = 1  # lengths no longer satisfy Kraft
    with pytest.raises(L.Ecf8Error):
        L.blob_info(bad)
    with pytest.raises(L.Ecf8Error):
        L.blob_info(blob[: blob.size - 1])


def test_encode_rejects_bad_codebooks(L):
    x = synth.single_normal_1k().tensors[0].generate(count=10_000)
    cb = L.build_codebook(L.histogram(x[:10]))  # lacks exponents present later
    with pytest.raises(L.Ecf8Error) as e:
        L.encode(x, codebook=cb)
    assert e.value.code == -4
    with pytest.raises(L.Ecf8Error):
        L.build_codebook(np.ones(16, np.uint64), max_len=3)


def test_layout_support_and_workspace_sizes(L):
    assert L.layout_supported(32, 32)
    assert not L.layout_supported(32, 128)
    assert not L.layout_supported(4, 1)
    assert L.batched_workspace_size(1) == 0 and L.batched_workspace_size(64) == 0
    assert L.batched_workspace_size(65) == 65 * 96


def test_encoded_size_bound_covers_every_input(L):
    """The histogram-free bound holds for the worst inputs of every layout: the
    16-bit-code tensor of a skewed 16-value code, uniform random bytes, and
    sizes around the chunk and group boundaries."""
    fib = [1, 1]
    while len(fib) < 16:
        fib.append(fib[-1] + fib[-2])
    deep = np.repeat(np.arange(16, dtype=np.uint8) << 3, fib)
    r = np.random.default_rng(17)
    for C, T in [(32, 32), (4, 1), (16, 3), (64, 64)]:
        for x in [deep, r.integers(0, 256, size=100_001).astype(np.uint8), np.zeros(1, np.uint8)]:
            assert L.encode(x, chunk_bytes=C, group_chunks=T).size <= L.encoded_size_bound(x.size, C, T)
        # all 16-bit codes: the largest stream any code allows
        x = np.zeros(4097, np.uint8)
        h = np.zeros(16, np.uint64)
        h[0] = x.size
        cb = L.Codebook()
        cb.len[0] = 16
        cb.code[0] = 0
        size = ctypes.c_size_t(0)
        assert L._lib.ecf8_encoded_size(h.ctypes.data, x.size, ctypes.byref(cb), C, T, ctypes.byref(size)) == 0
        assert size.value == L.encoded_size_bound(x.size, C, T)
    assert L.encoded_size_bound(10, 3, 1) == 0  # chunk bytes not a multiple of 4


def test_compression_of_pages_like_weights(L):
    """Gaussian-like FP8 weights: exponent entropy ~2.6 bits, so ECF8 stores
    about 6.7 of 8 bits (the pages report up to 26.9% savings)."""
    x = synth.llama3_8b_layer().tensors[1].generate()
    info = L.blob_info(L.encode(x))
    assert 1.15 < info.ratio < 1.4
