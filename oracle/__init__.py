"""ECF8 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Python access to the plain bit-serial C oracle in ``ecf8_oracle.c``.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package; the library under ``lossless_fp8_weight_b200/`` never does.

The oracle fixes what the GPU path must compute: ``decode(encode(x)) == x`` byte
for byte (ECF8 walkthrough p1 §1; arXiv 2510.02676 abstract), with the blob
layout, code construction and decode table spelled out step by step in the C
source.
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
LUT_BITS = 12
LUT_MAX_SYMS = 6


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into this directory."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", _SO, _SRC])
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
        lib.oracle_lut_entry.argtypes = [p, u32]
        lib.oracle_lut_entry.restype = u32
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


def lut_entry(lengths, pattern: int) -> int:
    ln = _u8(lengths)
    return int(_load().oracle_lut_entry(ln.ctypes.data, pattern))


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
    """0 when the blob's gaps, group offsets and decode table equal the ones the
    serial walk recomputes; 1 table, 2 gap, 3 offset, 4 stream, -1 header."""
    b = _u8(blob)
    return int(_load().oracle_check_index(b.ctypes.data, b.size))


def blob_header(blob) -> dict:
    """Header fields, read with numpy from the fixed little-endian layout."""
    b = _u8(blob)
    u32 = lambda o: int(b[o:o + 4].view("<u4")[0])  # noqa: E731
    u64 = lambda o: int(b[o:o + 8].view("<u8")[0])  # noqa: E731
    return {
        "magic": u32(0), "version": u32(4), "n": u64(8), "code_bits": u64(16),
        "chunk_bytes": u32(24), "group_chunks": u32(28), "n_groups": u32(32), "lut_bits": u32(36),
        "max_len": u32(40), "header_bytes": u32(44), "lut_off": u64(48), "gaps_off": u64(56),
        "groups_off": u64(64), "stream_off": u64(72), "nibbles_off": u64(80), "total": u64(88),
        "lengths": b[96:112].copy(),
    }
