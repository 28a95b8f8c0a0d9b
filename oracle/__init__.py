"""ECF8 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Python access to the plain bit-serial C oracle in ``ecf8_oracle.c``.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package; the library under ``lossless_fp8_weight_b200/`` never does.

The oracle fixes what the GPU path must compute: ``decode(encode(x)) == x`` byte
for byte (ECF8 walkthrough p1 §1; arXiv 2510.02676 abstract), with the blob
layout and the code construction spelled out step by step in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ecf8_oracle.c")
_SO = os.path.join(_HERE, "libecf8_oracle.so")

NSYM = 16


_BF16_SRC = os.path.join(_HERE, "bf16_oracle.c")
_BF16_SO = os.path.join(_HERE, "libbf16_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracles (ECF8 and its BF16 variant) with gcc into this directory."""
    for src, so in ((_SRC, _SO), (_BF16_SRC, _BF16_SO)):
        if force or not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
            subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", so, src])
    return _SO


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p, u64, u32, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int
        lib.oracle_histogram.argtypes = [p, u64, p]
        lib.oracle_huffman_lengths.argtypes = [p, p]
        lib.oracle_package_merge_lengths.argtypes = [p, i32, p]
        lib.oracle_code_lengths.argtypes = [p, i32, p]
        lib.oracle_canonical_codes.argtypes = [p, p]
        lib.oracle_encoded_size.argtypes = [p, u64, p, u32, u32]
        lib.oracle_encoded_size.restype = u64
        lib.oracle_encode.argtypes = [p, u64, p, u32, u32, p, u64, ctypes.POINTER(u64)]
        lib.oracle_decode.argtypes = [p, u64, p, u64]
        lib.oracle_check_index.argtypes = [p, u64]
        for f in ("oracle_exponent", "oracle_nibble"):
            getattr(lib, f).argtypes = [ctypes.c_uint8]
        lib.oracle_join.argtypes = [i32, i32]
        lib.oracle_join.restype = ctypes.c_uint8
        _lib = lib
    return _lib


def _u8(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.uint8).reshape(-1))
    return a


def exponent(b: int) -> int:
    return int(_load().oracle_exponent(b))


def nibble(b: int) -> int:
    return int(_load().oracle_nibble(b))


def join(e: int, nib: int) -> int:
    return int(_load().oracle_join(e, nib))


def histogram(x) -> np.ndarray:
    x = _u8(x)
    h = np.zeros(NSYM, dtype=np.uint64)
    _load().oracle_histogram(x.ctypes.data, x.size, h.ctypes.data)
    return h


def _hist(h) -> np.ndarray:
    h = np.ascontiguousarray(np.asarray(h, dtype=np.uint64).reshape(-1))
    assert h.size == NSYM
    return h


def huffman_lengths(hist) -> np.ndarray:
    h = _hist(hist)
    out = np.zeros(NSYM, dtype=np.uint8)
    if _load().oracle_huffman_lengths(h.ctypes.data, out.ctypes.data) != 0:
        raise ValueError("huffman failed")
    return out


def package_merge_lengths(hist, max_len: int) -> np.ndarray:
    h = _hist(hist)
    out = np.zeros(NSYM, dtype=np.uint8)
    if _load().oracle_package_merge_lengths(h.ctypes.data, max_len, out.ctypes.data) != 0:
        raise ValueError("no code fits max_len")
    return out


def code_lengths(hist, max_len: int = 16) -> np.ndarray:
    h = _hist(hist)
    out = np.zeros(NSYM, dtype=np.uint8)
    if _load().oracle_code_lengths(h.ctypes.data, max_len, out.ctypes.data) != 0:
        raise ValueError("no code fits max_len")
    return out


def canonical_codes(lengths) -> np.ndarray:
    ln = _u8(lengths)
    out = np.zeros(NSYM, dtype=np.uint32)
    if _load().oracle_canonical_codes(ln.ctypes.data, out.ctypes.data) != 0:
        raise ValueError("bad lengths")
    return out


def encode(x, lengths=None, chunk_bytes: int = 32, group_chunks: int = 32, max_len: int = 16) -> np.ndarray:
    """Blob for ``x`` (uint8 E4M3 bytes).  Lengths default to the code built
    from ``x``'s own exponent histogram."""
    x = _u8(x)
    ln = code_lengths(histogram(x), max_len) if lengths is None else _u8(lengths)
    lib = _load()
    size = lib.oracle_encoded_size(x.ctypes.data, x.size, ln.ctypes.data, chunk_bytes, group_chunks)
    if size == 0:
        raise ValueError("bad layout parameters")
    blob = np.empty(size, dtype=np.uint8)
    got = ctypes.c_uint64(0)
    rc = lib.oracle_encode(x.ctypes.data, x.size, ln.ctypes.data, chunk_bytes, group_chunks,
                           blob.ctypes.data, size, ctypes.byref(got))
    if rc != 0:
        raise ValueError(f"oracle_encode failed ({rc})")
    assert got.value == size
    return blob


def decode(blob, n: int) -> np.ndarray:
    b = _u8(blob)
    out = np.empty(n, dtype=np.uint8)
    rc = _load().oracle_decode(b.ctypes.data, b.size, out.ctypes.data, n)
    if rc != 0:
        raise ValueError(f"oracle_decode failed ({rc})")
    return out


def decode_into(blob, out: np.ndarray) -> int:
    """Decode into a preallocated uint8 array; returns the C status."""
    b = _u8(blob)
    return int(_load().oracle_decode(b.ctypes.data, b.size, out.ctypes.data, out.size))


def check_index(blob) -> int:
    """0 when the blob's gaps and group offsets equal the ones the serial walk
    recomputes; 2 gap, 3 offset, 4 stream, -1 header."""
    b = _u8(blob)
    return int(_load().oracle_check_index(b.ctypes.data, b.size))


def blob_header(blob) -> dict:
    """Header fields, read with numpy from the fixed little-endian layout."""
    b = _u8(blob)
    u32 = lambda o: int(b[o:o + 4].view("<u4")[0])  # noqa: E731
    u64 = lambda o: int(b[o:o + 8].view("<u8")[0])  # noqa: E731
    return {
        "magic": u32(0), "version": u32(4), "n": u64(8), "code_bits": u64(16),
        "chunk_bytes": u32(24), "group_chunks": u32(28), "n_groups": u32(32), "reserved": u32(36),
        "max_len": u32(40), "header_bytes": u32(44), "reserved48": u64(48), "gaps_off": u64(56),
        "groups_off": u64(64), "stream_off": u64(72), "nibbles_off": u64(80), "total": u64(88),
        "lengths": b[96:112].copy(),
    }


# ---------------------------------------------------------------- BF16 variant (bf16_oracle.c)

_bf16 = None


def _load_bf16():
    global _bf16
    if _bf16 is None:
        build()
        lib = ctypes.CDLL(_BF16_SO)
        p, u64, u32, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int
        lib.bf16_histogram.argtypes = [p, u64, p]
        lib.bf16_huffman_lengths.argtypes = [p, p]
        lib.bf16_package_merge_lengths.argtypes = [p, i32, p]
        lib.bf16_code_lengths.argtypes = [p, i32, p]
        lib.bf16_canonical_codes.argtypes = [p, p]
        lib.bf16_encoded_size.argtypes = [p, u64, p, u32, u32]
        lib.bf16_encoded_size.restype = u64
        lib.bf16_encode.argtypes = [p, u64, p, u32, u32, p, u64, ctypes.POINTER(u64)]
        lib.bf16_decode.argtypes = [p, u64, p, u64]
        lib.bf16_exponent.argtypes = [ctypes.c_uint16]
        lib.bf16_kept.argtypes = [ctypes.c_uint16]
        lib.bf16_join.argtypes = [i32, i32]
        lib.bf16_join.restype = ctypes.c_uint16
        _bf16 = lib
    return _bf16


def _u16(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x).reshape(-1).view(np.uint16) if np.asarray(x).dtype != np.uint16
                                else np.asarray(x).reshape(-1))


def bf16_exponent(x: int) -> int:
    return int(_load_bf16().bf16_exponent(x))


def bf16_kept(x: int) -> int:
    return int(_load_bf16().bf16_kept(x))


def bf16_join(e: int, kept: int) -> int:
    return int(_load_bf16().bf16_join(e, kept))


def bf16_histogram(x) -> np.ndarray:
    a = _u16(x)
    h = np.zeros(256, dtype=np.uint64)
    _load_bf16().bf16_histogram(a.ctypes.data, a.size, h.ctypes.data)
    return h


def _hist256(h) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(h, dtype=np.uint64))
    assert a.size == 256
    return a


def bf16_huffman_lengths(hist) -> np.ndarray:
    h = _hist256(hist)
    out = np.zeros(256, dtype=np.uint8)
    _load_bf16().bf16_huffman_lengths(h.ctypes.data, out.ctypes.data)
    return out


def bf16_package_merge_lengths(hist, max_len: int) -> np.ndarray:
    h = _hist256(hist)
    out = np.zeros(256, dtype=np.uint8)
    if _load_bf16().bf16_package_merge_lengths(h.ctypes.data, max_len, out.ctypes.data) != 0:
        raise ValueError("no code of that length limit")
    return out


def bf16_code_lengths(hist, max_len: int = 16) -> np.ndarray:
    h = _hist256(hist)
    out = np.zeros(256, dtype=np.uint8)
    if _load_bf16().bf16_code_lengths(h.ctypes.data, max_len, out.ctypes.data) != 0:
        raise ValueError("no code of that length limit")
    return out


def bf16_canonical_codes(lengths) -> np.ndarray:
    ln = np.ascontiguousarray(np.asarray(lengths, dtype=np.uint8))
    out = np.zeros(256, dtype=np.uint32)
    if _load_bf16().bf16_canonical_codes(ln.ctypes.data, out.ctypes.data) != 0:
        raise ValueError("lengths above 16")
    return out


def bf16_encode(x, lengths=None, chunk_bytes: int = 32, group_chunks: int = 32, max_len: int = 16) -> np.ndarray:
    """BF16 values (uint16 bit patterns) -> blob, by the plain serial encoder."""
    a = _u16(x)
    ln = bf16_code_lengths(bf16_histogram(a), max_len) if lengths is None else \
        np.ascontiguousarray(np.asarray(lengths, dtype=np.uint8))
    lib = _load_bf16()
    size = int(lib.bf16_encoded_size(a.ctypes.data, a.size, ln.ctypes.data, chunk_bytes, group_chunks))
    blob = np.zeros(max(size, 256), dtype=np.uint8)
    got = ctypes.c_uint64(0)
    rc = lib.bf16_encode(a.ctypes.data, a.size, ln.ctypes.data, chunk_bytes, group_chunks, blob.ctypes.data,
                         blob.size, ctypes.byref(got))
    if rc != 0:
        raise ValueError(f"bf16_encode failed ({rc})")
    return blob[:got.value].copy()


def bf16_decode(blob, n: int) -> np.ndarray:
    b = _u8(blob)
    out = np.zeros(n, dtype=np.uint16)
    rc = _load_bf16().bf16_decode(b.ctypes.data, b.size, out.ctypes.data, n)
    if rc != 0:
        raise ValueError(f"bf16_decode failed ({rc})")
    return out


def bf16_blob_header(blob) -> dict:
    b = _u8(blob)
    u32 = lambda o: int(b[o:o + 4].view("<u4")[0])  # noqa: E731
    u64 = lambda o: int(b[o:o + 8].view("<u8")[0])  # noqa: E731
    h = {"magic": u32(0), "version": u32(4), "n": u64(8), "code_bits": u64(16), "chunk_bytes": u32(24),
         "group_chunks": u32(28), "n_groups": u32(32), "max_len": u32(36), "lens_off": u64(40),
         "gaps_off": u64(48), "groups_off": u64(56), "stream_off": u64(64), "kept_off": u64(72), "total": u64(80)}
    h["lengths"] = b[h["lens_off"]:h["lens_off"] + 256].copy()
    return h
