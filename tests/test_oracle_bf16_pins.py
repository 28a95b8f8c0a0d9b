"""Pins of the BF16-variant oracle (oracle/bf16_oracle.c) against things other
than itself: the BF16 bit layout as torch stores it, brute-force optimal
prefix codes on small alphabets (with and without a length limit), prefix
freedom and canonical order, Kraft equality, a hand-derived worked blob,
gaps and offsets recomputed with numpy from the code lengths, and round
trips over edge cases.  (DFloat11 article §2: the exponent field is entropy
coded, sign and mantissa kept; ECF8 walkthrough §3.1.1-§3.2.1 for the code,
stream, gap and offset layout shared with the ECF8 blob.)"""
import itertools

import numpy as np
import pytest

import oracle


def _bf16_bits(f32: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even float32 -> BF16 bit patterns (test input helper)."""
    u = f32.astype(np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_split_matches_the_bf16_layout_torch_uses():
    torch = pytest.importorskip("torch")
    r = np.random.default_rng(1)
    f = (r.standard_normal(5000) * np.exp(r.uniform(-20, 20, 5000))).astype(np.float32)
    t = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for x in t[:500]:
        x = int(x)
        sign = x >> 15
        e = oracle.bf16_exponent(x)
        kept = oracle.bf16_kept(x)
        assert e == (x >> 7) & 0xFF
        assert kept >> 7 == sign and kept & 0x7F == x & 0x7F
        assert oracle.bf16_join(e, kept) == x
        # the exponent field is the float32 exponent of the bf16 value itself
        f32 = np.array([x << 16], dtype=np.uint32).view(np.float32)[0]
        assert e == (np.array([f32], dtype=np.float32).view(np.uint32)[0] >> 23) & 0xFF


def _cost(w, lengths):
    return sum(int(a) * int(b) for a, b in zip(w, lengths))


def _best_cost(w, max_len):
    """Minimum sum w*l over length vectors with Kraft sum <= 1, by enumeration."""
    k = len(w)
    best = None
    for ls in itertools.product(range(1, max_len + 1), repeat=k):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            c = _cost(w, ls)
            best = c if best is None or c < best else best
    return best


@pytest.mark.parametrize("seed", range(12))
def test_huffman_is_optimal_on_small_alphabets(seed):
    r = np.random.default_rng(seed)
    k = int(r.integers(2, 7))
    syms = r.choice(256, size=k, replace=False)
    w = r.integers(1, 1000, size=k)
    h = np.zeros(256, dtype=np.uint64)
    h[syms] = w
    ln = oracle.bf16_huffman_lengths(h)
    assert _cost(w, ln[syms]) == _best_cost(w, k - 1)
    assert (ln[np.setdiff1d(np.arange(256), syms)] == 0).all()


@pytest.mark.parametrize("seed", range(10))
def test_package_merge_is_optimal_under_the_limit(seed):
    r = np.random.default_rng(100 + seed)
    k = int(r.integers(3, 7))
    syms = r.choice(256, size=k, replace=False)
    w = (2 ** r.integers(0, 12, size=k)).astype(np.int64) + r.integers(0, 3, size=k)
    limit = int(r.integers(int(np.ceil(np.log2(k))), k))
    h = np.zeros(256, dtype=np.uint64)
    h[syms] = w
    ln = oracle.bf16_package_merge_lengths(h, limit)
    assert ln[syms].max() <= limit
    assert sum(2.0 ** -int(l) for l in ln[syms]) <= 1.0
    assert _cost(w, ln[syms]) == _best_cost(w, limit)


def test_skewed_256_symbol_code_is_capped_complete_and_ordered():
    h = np.array([2 ** (40 - min(i, 40)) + 1 for i in range(256)], dtype=np.uint64)  # forces depth > 16
    assert oracle.bf16_huffman_lengths(h).max() > 16
    ln = oracle.bf16_code_lengths(h, 16)
    assert ln.max() == 16 and ln.min() >= 1
    assert sum(2.0 ** -int(l) for l in ln) == 1.0
    order = np.argsort(-h.astype(np.float64), kind="stable")
    assert all(ln[order[i]] <= ln[order[i + 1]] for i in range(255))  # heavier never longer


def test_canonical_codes_are_prefix_free_and_ordered():
    r = np.random.default_rng(7)
    h = np.zeros(256, dtype=np.uint64)
    syms = r.choice(256, size=40, replace=False)
    h[syms] = r.integers(1, 10 ** 6, size=40)
    ln = oracle.bf16_code_lengths(h, 16)
    code = oracle.bf16_canonical_codes(ln)
    words = [(int(ln[s]), int(code[s]), int(s)) for s in syms]
    for (la, ca, _), (lb, cb, _) in itertools.permutations(words, 2):
        if la <= lb:
            assert (cb >> (lb - la)) != ca  # no code is a prefix of another
    ranked = sorted(words, key=lambda t: (t[0], t[2]))
    vals = [c << (16 - l) for l, c, _ in ranked]  # left-aligned: canonical codes ascend
    assert vals == sorted(vals) and len(set(vals)) == len(vals)


def test_worked_example_by_hand():
    """Exponents 127, 127, 128, 126 (weights 127:2, 126:1, 128:1): 126 and 128
    merge first (weight 1, lower ids), then 127 with that node, so 127 gets 1
    bit and 126, 128 get 2; canonical codes 127 = 0, 126 = 10, 128 = 11.  The
    stream is 0 0 11 10, MSB first in a little-endian word: 0x38000000."""
    vals = [(0, 127, 0x11), (1, 127, 0x05), (0, 128, 0x7F), (1, 126, 0x00)]
    x = np.array([(s << 15) | (e << 7) | m for s, e, m in vals], dtype=np.uint16)
    blob = oracle.bf16_encode(x, chunk_bytes=4, group_chunks=1)
    hd = oracle.bf16_blob_header(blob)
    assert hd["magic"] == 0x31314644 and hd["code_bits"] == 6 and hd["n_groups"] == 1 and hd["max_len"] == 2
    assert hd["lengths"][127] == 1 and hd["lengths"][126] == 2 and hd["lengths"][128] == 2
    assert hd["lengths"].sum() == 5
    assert blob[hd["stream_off"]:hd["stream_off"] + 4].tolist() == [0x00, 0x00, 0x00, 0x38]
    assert blob[hd["kept_off"]:hd["kept_off"] + 4].tolist() == [0x11, 0x85, 0x7F, 0x80]
    assert blob[hd["groups_off"]:hd["groups_off"] + 16].view("<u8").tolist() == [0, 4]
    assert blob[hd["gaps_off"]] == 0
    assert np.array_equal(oracle.bf16_decode(blob, 4), x)


@pytest.mark.parametrize("C,T", [(32, 32), (4, 1), (8, 3)])
def test_gaps_and_offsets_recomputed_from_lengths(C, T):
    r = np.random.default_rng(C * 10 + T)
    x = _bf16_bits(r.standard_normal(20_001) * 0.05)
    blob = oracle.bf16_encode(x, chunk_bytes=C, group_chunks=T)
    hd = oracle.bf16_blob_header(blob)
    ln = hd["lengths"].astype(np.int64)
    l = ln[(x >> 7) & 0xFF]
    starts = np.concatenate([[0], np.cumsum(l)])  # last entry: the stream end
    chunk_bits = 8 * C
    chunks = hd["n_groups"] * T
    gaps = blob[hd["gaps_off"]:hd["gaps_off"] + 4 * ((chunks + 7) // 8)].view("<u4")
    offs = blob[hd["groups_off"]:hd["groups_off"] + 8 * (hd["n_groups"] + 1)].view("<u8")
    for c in range(chunks):
        i = int(np.searchsorted(starts, c * chunk_bits, side="left"))
        want_gap = int(starts[i] - c * chunk_bits) if i < starts.size else 0
        assert (int(gaps[c // 8]) >> (4 * (c % 8))) & 15 == want_gap, c
        if c % T == 0:
            assert int(offs[c // T]) == min(i, x.size), c
    assert int(offs[-1]) == x.size


@pytest.mark.parametrize("case", ["empty", "one", "two", "single_symbol", "all_256", "random_bits", "specials"])
def test_round_trip_edge_cases(case):
    r = np.random.default_rng(3)
    x = {
        "empty": np.zeros(0, dtype=np.uint16),
        "one": np.array([0x3F80], dtype=np.uint16),
        "two": np.array([0x3F80, 0xBF80], dtype=np.uint16),
        "single_symbol": np.full(1000, 0x4049, dtype=np.uint16),
        "all_256": r.permutation(np.repeat((np.arange(256, dtype=np.uint16) << 7), 9)) | r.integers(0, 128, 2304).astype(np.uint16),
        "random_bits": r.integers(0, 1 << 16, 50_001).astype(np.uint16),
        "specials": np.array([0x7F80, 0xFF80, 0x7FC0, 0x0000, 0x8000, 0x0001, 0x807F] * 300, dtype=np.uint16),
    }[case]
    blob = oracle.bf16_encode(x)
    assert np.array_equal(oracle.bf16_decode(blob, x.size), x)


def _read_bf16_golden():
    """Key/value lines of tests/golden/bf16_worked_example.txt (comments skipped)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "bf16_worked_example.txt")
    g = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, *v = line.split()
                g[k] = v
    return g


def test_hand_derived_golden_blob():
    """The oracle reproduces a blob worked out on paper (the fixture's header
    gives the derivation): lengths, canonical codes, a code straddling the
    chunk boundary (gap 1), group offsets, stream words and kept bytes."""
    g = _read_bf16_golden()
    x = np.array([int(v, 16) for v in g["weights"]], dtype=np.uint16)
    C, T = int(g["chunk_bytes"][0]), int(g["group_chunks"][0])
    blob = oracle.bf16_encode(x, chunk_bytes=C, group_chunks=T)
    hd = oracle.bf16_blob_header(blob)
    want_len = np.zeros(256, np.uint8)
    for kv in g["lengths"]:
        k, v = kv.split(":")
        want_len[int(k)] = int(v)
    assert np.array_equal(hd["lengths"], want_len)
    codes = oracle.bf16_canonical_codes(want_len)
    for kv in g["codes"]:
        k, v = kv.split(":")
        assert int(codes[int(k)]) == int(v)
    assert hd["code_bits"] == int(g["code_bits"][0]) and hd["n_groups"] == int(g["n_groups"][0])
    words = [int(v, 16) for v in g["stream_words"]]
    assert blob[hd["stream_off"]:hd["stream_off"] + 4 * len(words)].view("<u4").tolist() == words
    gaps = [int(v, 16) for v in g["gap_words"]]
    assert blob[hd["gaps_off"]:hd["gaps_off"] + 4 * len(gaps)].view("<u4").tolist() == gaps
    offs = [int(v) for v in g["group_offsets"]]
    assert blob[hd["groups_off"]:hd["groups_off"] + 8 * len(offs)].view("<u8").tolist() == offs
    kept = [int(v, 16) for v in g["kept_bytes"]]
    assert blob[hd["kept_off"]:hd["kept_off"] + len(kept)].tolist() == kept
    assert np.array_equal(oracle.bf16_decode(blob, x.size), x)
