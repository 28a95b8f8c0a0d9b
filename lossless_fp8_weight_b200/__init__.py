"""ECF8 lossless FP8 E4M3 weight codec: Python binding of libecf8.

Thin ctypes layer over the C ABI in ``include/ecf8.h``: it marshals arguments
and nothing else.  Encoding runs in the library's host code; every step of
decoding runs in its sm_100a kernels.  PyTorch is used only to hand over
device pointers and the current CUDA stream.  There is no CPU fallback: if
``libecf8.so`` is missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libecf8.so")



def _ensure_built() -> None:
    """Compile libecf8.so in place when it is missing or older than its
    sources (the build script is loaded by path, so this package's own import
    does not recurse)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("_ecf8_build", os.path.join(_HERE, "_build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    if mod.stale():
        try:
            mod.build()
        except Exception as e:  # no toolchain: the decoder has no CPU fallback
            raise ImportError(f"{_SO} is missing or stale and could not be built: {e}") from e


_ensure_built()
_lib = ctypes.CDLL(_SO)

OK = 0
ERRORS = {-1: "ARG", -2: "FORMAT", -3: "CAPACITY", -4: "CODEBOOK", -5: "ALIGN", -6: "UNSUPPORTED", -7: "CUDA",
          -8: "WORKSPACE", -9: "TOO_MANY", -10: "CAPTURE"}
STATUS_COUNT_MISMATCH = 1
STATUS_BAD_CODE = 2
STATUS_BAD_OFFSETS = 4
BATCH_INLINE_MAX = 64
NOALLOC_MAX_TENSORS = 1024
DEFAULT_CHUNK_BYTES = 32
DEFAULT_GROUP_CHUNKS = 32


class Codebook(ctypes.Structure):
    _fields_ = [("len", ctypes.c_uint8 * 16), ("code", ctypes.c_uint16 * 16), ("max_len", ctypes.c_uint32),
                ("n_symbols", ctypes.c_uint32)]

    @property
    def lengths(self) -> np.ndarray:
        return np.frombuffer(bytes(self.len), dtype=np.uint8).copy()


class Info(ctypes.Structure):
    _fields_ = [("n", ctypes.c_uint64), ("code_bits", ctypes.c_uint64), ("blob_bytes", ctypes.c_uint64),
                ("gaps_off", ctypes.c_uint64), ("groups_off", ctypes.c_uint64),
                ("stream_off", ctypes.c_uint64), ("nibbles_off", ctypes.c_uint64),
                ("chunk_bytes", ctypes.c_uint32), ("group_chunks", ctypes.c_uint32), ("n_groups", ctypes.c_uint32),
                ("max_len", ctypes.c_uint32), ("len", ctypes.c_uint8 * 16)]

    @property
    def lengths(self) -> np.ndarray:
        return np.frombuffer(bytes(self.len), dtype=np.uint8).copy()

    @property
    def ratio(self) -> float:
        return self.n / self.blob_bytes if self.blob_bytes else 0.0


class Tensor(ctypes.Structure):
    _fields_ = [("info", ctypes.POINTER(Info)), ("d_blob", ctypes.c_void_p), ("blob_size", ctypes.c_size_t),
                ("d_out", ctypes.c_void_p)]


_p, _sz, _u32, _i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_int
_lib.ecf8_histogram.argtypes = [_p, _sz, _p]
_lib.ecf8_build_codebook.argtypes = [_p, _u32, ctypes.POINTER(Codebook)]
_lib.ecf8_encoded_size.argtypes = [_p, _sz, ctypes.POINTER(Codebook), _u32, _u32, ctypes.POINTER(_sz)]
_lib.ecf8_encoded_size_bound.argtypes = [_sz, _u32, _u32]
_lib.ecf8_encoded_size_bound.restype = _sz
_lib.ecf8_encode.argtypes = [_p, _sz, ctypes.POINTER(Codebook), _u32, _u32, _p, _sz, ctypes.POINTER(_sz)]
_lib.ecf8_blob_info.argtypes = [_p, _sz, ctypes.POINTER(Info)]
_lib.ecf8_layout_supported.argtypes = [_u32, _u32]
_lib.ecf8_decode.argtypes = [ctypes.POINTER(Info), _p, _sz, _p, _sz, _p, _p]
_lib.ecf8_batched_workspace_size.argtypes = [_i32]
_lib.ecf8_batched_workspace_size.restype = _sz
_lib.ecf8_decode_batched.argtypes = [ctypes.POINTER(Tensor), _i32, _p, _sz, _p, _p]
_lib.ecf8_decode_batched_noalloc.argtypes = [ctypes.POINTER(Tensor), _i32, _p, _p]
_lib.ecf8_decode_batched_ctas.argtypes = [ctypes.POINTER(Tensor), _i32, _p, _sz, _p, _p, _u32]
_lib.ecf8_histogram_device.argtypes = [_p, _sz, _p, _p]
_lib.ecf8_encode_device_workspace_size.argtypes = [_sz]
_lib.ecf8_encode_device_workspace_size.restype = _sz
_lib.ecf8_encode_device.argtypes = [_p, _sz, _p, ctypes.POINTER(Codebook), _u32, _u32, _p, _sz, ctypes.POINTER(_sz),
                                    _p, _sz, _p]


class Bf16Info(ctypes.Structure):
    _fields_ = [("n", ctypes.c_uint64), ("code_bits", ctypes.c_uint64), ("blob_bytes", ctypes.c_uint64),
                ("lens_off", ctypes.c_uint64), ("gaps_off", ctypes.c_uint64), ("groups_off", ctypes.c_uint64),
                ("stream_off", ctypes.c_uint64), ("kept_off", ctypes.c_uint64),
                ("chunk_bytes", ctypes.c_uint32), ("group_chunks", ctypes.c_uint32), ("n_groups", ctypes.c_uint32),
                ("max_len", ctypes.c_uint32), ("len", ctypes.c_uint8 * 256)]

    @property
    def lengths(self) -> np.ndarray:
        return np.frombuffer(bytes(self.len), dtype=np.uint8).copy()

    @property
    def ratio(self) -> float:
        return 2 * self.n / self.blob_bytes if self.blob_bytes else 0.0


_lib.ecf8_bf16_code_lengths.argtypes = [_p, _sz, _u32, _p]
_lib.ecf8_bf16_encoded_size.argtypes = [_p, _sz, _p, _u32, _u32, ctypes.POINTER(_sz)]
_lib.ecf8_bf16_encode.argtypes = [_p, _sz, _p, _u32, _u32, _p, _sz, ctypes.POINTER(_sz)]
_lib.ecf8_bf16_blob_info.argtypes = [_p, _sz, ctypes.POINTER(Bf16Info)]
_lib.ecf8_bf16_table_bytes.restype = _sz
_lib.ecf8_bf16_build_table.argtypes = [ctypes.POINTER(Bf16Info), _p]
_lib.ecf8_bf16_table_nodes.argtypes = [ctypes.POINTER(Bf16Info)]
_lib.ecf8_bf16_table_nodes.restype = _u32
_lib.ecf8_bf16_decode.argtypes = [ctypes.POINTER(Bf16Info), _p, _p, _p, _sz, _p, _p]
_lib.ecf8_bf16_decode_layout.argtypes = [ctypes.POINTER(Bf16Info), _p, _p, _p, _sz, _p, _p, _i32]
_lib.ecf8_bf16_auto_layout.argtypes = [ctypes.POINTER(Bf16Info)]
BF16_LAYOUTS = {"auto": -1, "wide": 0, "narrow": 1, "narrow_lane": 2, "byte": 3}
BF16_BATCH_MAX = 32


class Bf16Tensor(ctypes.Structure):
    _fields_ = [("info", ctypes.POINTER(Bf16Info)), ("d_blob", ctypes.c_void_p), ("d_table", ctypes.c_void_p),
                ("d_out", ctypes.c_void_p)]


_lib.ecf8_bf16_decode_batched.argtypes = [ctypes.POINTER(Bf16Tensor), _i32, _p, _p]


class LayerTensor(ctypes.Structure):
    _fields_ = [("info", ctypes.POINTER(Info)), ("d_blob", ctypes.c_void_p), ("blob_size", ctypes.c_size_t),
                ("out_offset", ctypes.c_size_t)]


class Layer(ctypes.Structure):
    _fields_ = [("tensors", ctypes.POINTER(LayerTensor)), ("count", ctypes.c_int)]


_lib.ecf8_pipeline_create.argtypes = [ctypes.POINTER(Layer), _i32, ctypes.POINTER(ctypes.c_void_p), _i32, _sz, _i32,
                                      _u32, _p, _sz, _p, _p, ctypes.POINTER(ctypes.c_void_p)]
_lib.ecf8_pipeline_acquire.argtypes = [_p, _i32, _p, ctypes.POINTER(ctypes.c_void_p)]
_lib.ecf8_pipeline_release.argtypes = [_p, _i32, _p]
_lib.ecf8_pipeline_destroy.argtypes = [_p]
_lib.ecf8_pipeline_destroy.restype = None
_lib.ecf8_launch_count.restype = ctypes.c_uint64
_lib.ecf8_strerror.restype = ctypes.c_char_p
_lib.ecf8_strerror.argtypes = [_i32]


class Ecf8Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {_lib.ecf8_strerror(code).decode()} ({ERRORS.get(code, code)})")
        self.code = code


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise Ecf8Error(rc, what)


def library_path() -> str:
    return _SO


def launch_count() -> int:
    """Decode kernels launched by this process so far."""
    return int(_lib.ecf8_launch_count())


def _host_u8(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a CPU torch tensor
        x = x.detach().contiguous().view(-1).numpy()
    a = np.ascontiguousarray(np.asarray(x).reshape(-1))
    if a.dtype != np.uint8:
        a = a.view(np.uint8)
    return a


def histogram(fp8) -> np.ndarray:
    x = _host_u8(fp8)
    h = np.zeros(16, dtype=np.uint64)
    _check(_lib.ecf8_histogram(x.ctypes.data, x.size, h.ctypes.data), "ecf8_histogram")
    return h


def build_codebook(hist, max_len: int = 16) -> Codebook:
    h = np.ascontiguousarray(np.asarray(hist, dtype=np.uint64))
    cb = Codebook()
    _check(_lib.ecf8_build_codebook(h.ctypes.data, max_len, ctypes.byref(cb)), "ecf8_build_codebook")
    return cb


def encode(fp8, codebook: Optional[Codebook] = None, chunk_bytes: int = DEFAULT_CHUNK_BYTES,
           group_chunks: int = DEFAULT_GROUP_CHUNKS, max_len: int = 16) -> np.ndarray:
    """Compress E4M3 bytes (numpy uint8 / float8 view, or CPU tensor) into a blob."""
    x = _host_u8(fp8)
    h = histogram(x)
    cb = codebook if codebook is not None else build_codebook(h, max_len)
    size = ctypes.c_size_t(0)
    _check(_lib.ecf8_encoded_size(h.ctypes.data, x.size, ctypes.byref(cb), chunk_bytes, group_chunks,
                                  ctypes.byref(size)), "ecf8_encoded_size")
    blob = np.empty(size.value, dtype=np.uint8)
    got = ctypes.c_size_t(0)
    _check(_lib.ecf8_encode(x.ctypes.data, x.size, ctypes.byref(cb), chunk_bytes, group_chunks, blob.ctypes.data,
                            blob.size, ctypes.byref(got)), "ecf8_encode")
    assert got.value == blob.size
    return blob


def histogram_device(d_fp8, stream=None) -> np.ndarray:
    """Exponent histogram of a CUDA uint8 tensor, computed on the GPU (the
    call waits for it and returns a host array)."""
    import torch
    n = d_fp8.numel()
    d_hist = torch.empty(16, dtype=torch.int64, device=d_fp8.device)
    _check(_lib.ecf8_histogram_device(_ptr(d_fp8), n, _ptr(d_hist), _stream(stream)), "ecf8_histogram_device")
    return d_hist.cpu().numpy().astype(np.uint64)


def encode_device(d_fp8, codebook: Optional[Codebook] = None, chunk_bytes: int = DEFAULT_CHUNK_BYTES,
                  group_chunks: int = DEFAULT_GROUP_CHUNKS, max_len: int = 16, stream=None, hist=None):
    """Compress a CUDA uint8 tensor of E4M3 bytes on the GPU; returns the blob
    as a CUDA uint8 tensor (the same bytes as ``encode`` of the same input)."""
    import torch
    x = d_fp8.reshape(-1)
    if x.dtype != torch.uint8:
        x = x.view(torch.uint8)
    n = x.numel()
    h = histogram_device(x, stream) if hist is None else np.ascontiguousarray(np.asarray(hist, dtype=np.uint64))
    cb = codebook if codebook is not None else build_codebook(h, max_len)
    size = ctypes.c_size_t(0)
    _check(_lib.ecf8_encoded_size(h.ctypes.data, n, ctypes.byref(cb), chunk_bytes, group_chunks, ctypes.byref(size)),
           "ecf8_encoded_size")
    blob = torch.empty(size.value, dtype=torch.uint8, device=x.device)
    ws = torch.empty(max(16, _lib.ecf8_encode_device_workspace_size(n)), dtype=torch.uint8, device=x.device)
    got = ctypes.c_size_t(0)
    _check(_lib.ecf8_encode_device(_ptr(x), n, h.ctypes.data, ctypes.byref(cb), chunk_bytes, group_chunks, _ptr(blob),
                                   blob.numel(), ctypes.byref(got), _ptr(ws), ws.numel(), _stream(stream)),
           "ecf8_encode_device")
    assert got.value == blob.numel()
    return blob


def encoded_size_bound(n: int, chunk_bytes: int = DEFAULT_CHUNK_BYTES, group_chunks: int = DEFAULT_GROUP_CHUNKS) -> int:
    """Blob bytes that suffice for any n weights in this layout (no histogram needed)."""
    return int(_lib.ecf8_encoded_size_bound(n, chunk_bytes, group_chunks))


def blob_info(blob) -> Info:
    b = _host_u8(blob)
    info = Info()
    _check(_lib.ecf8_blob_info(b.ctypes.data, b.size, ctypes.byref(info)), "ecf8_blob_info")
    return info


def blob_info_device(d_blob) -> Info:
    """blob_info of a blob held in device memory (a CUDA uint8 tensor): only
    its 128-byte header is copied to the host, which is all the parser reads."""
    hdr = np.ascontiguousarray(d_blob[:128].cpu().numpy())
    if hdr.size < 128:
        raise Ecf8Error(-2, "ecf8_blob_info")
    info = Info()
    _check(_lib.ecf8_blob_info(hdr.ctypes.data, int(d_blob.numel() * d_blob.element_size()), ctypes.byref(info)),
           "ecf8_blob_info")
    return info


def layout_supported(chunk_bytes: int, group_chunks: int) -> bool:
    return bool(_lib.ecf8_layout_supported(chunk_bytes, group_chunks))


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


def _nbytes(t, default: int) -> int:
    """Bytes of a torch tensor argument; a raw pointer is taken to hold `default`."""
    if t is None or isinstance(t, int):
        return int(default)
    return int(t.numel() * t.element_size())


def _stream(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def decode(info: Info, d_blob, d_out, status=None, stream=None, blob_size: Optional[int] = None) -> None:
    """Asynchronously decode one blob already in device memory into d_out
    (torch uint8 CUDA tensors or raw device pointers) on ``stream``.  The
    bytes readable at d_blob are the tensor's size, or ``blob_size`` (which a
    raw pointer needs; it defaults to the blob's own size)."""
    size = _nbytes(d_blob, info.blob_bytes) if blob_size is None else int(blob_size)
    _check(_lib.ecf8_decode(ctypes.byref(info), _ptr(d_blob), size, _ptr(d_out), info.n, _ptr(status),
                            _stream(stream)), "ecf8_decode")


def batched_workspace_size(count: int) -> int:
    return int(_lib.ecf8_batched_workspace_size(count))


@dataclass
class BatchItem:
    info: Info
    d_blob: object
    d_out: object


def make_batch(items: Sequence[BatchItem]):
    """The ctypes array a batched decode takes; keep it alive while reused."""
    arr = (Tensor * len(items))()
    keep = []
    for i, it in enumerate(items):
        keep.append(it.info)
        arr[i].info = ctypes.pointer(it.info)
        arr[i].d_blob = _ptr(it.d_blob)
        arr[i].blob_size = _nbytes(it.d_blob, it.info.blob_bytes)
        arr[i].d_out = _ptr(it.d_out)
    return arr, keep


def decode_batched(items, workspace=None, status=None, stream=None, max_ctas: int = 0) -> None:
    """Decode several blobs in one kernel launch.  ``items`` is a list of
    BatchItem or the pair returned by make_batch.  ``max_ctas`` > 0 caps the
    persistent grid (one CTA per SM otherwise), leaving SMs to other kernels."""
    if isinstance(items, tuple):
        arr = items[0]
    else:
        arr, _keep = make_batch(items)
    ws = _ptr(workspace)
    ws_bytes = int(workspace.numel() * workspace.element_size()) if workspace is not None and not isinstance(
        workspace, int) else 0
    if max_ctas:
        _check(_lib.ecf8_decode_batched_ctas(arr, len(arr), ws, ws_bytes, _ptr(status), _stream(stream),
                                             int(max_ctas)), "ecf8_decode_batched_ctas")
    else:
        _check(_lib.ecf8_decode_batched(arr, len(arr), ws, ws_bytes, _ptr(status), _stream(stream)),
               "ecf8_decode_batched")


def decode_batched_noalloc(items, status=None, stream=None) -> None:
    """Like decode_batched, but with no workspace: the descriptor table lives
    in device memory the library holds (ECF8_NOALLOC_MAX_TENSORS entries), for
    callers that cannot allocate device memory while they decode.  Calls that
    can overlap on the GPU share that table and race; order them on one
    stream."""
    if isinstance(items, tuple):
        arr = items[0]
    else:
        arr, _keep = make_batch(items)
    _check(_lib.ecf8_decode_batched_noalloc(arr, len(arr), _ptr(status), _stream(stream)),
           "ecf8_decode_batched_noalloc")


@dataclass
class PipelineTensor:
    """One tensor of a pipeline layer: its blob info, device blob, and the
    byte offset of its FP8 output inside a slot (multiple of 16)."""
    info: Info
    d_blob: object
    out_offset: int


class Pipeline:
    """Decode-on-use over a fixed pool of slots (ecf8_pipeline_* in the C
    ABI): layer m is decoded into slot m % len(slots) on ``decode_stream``,
    ``depth`` layers ahead; ``acquire(l, stream)`` makes ``stream`` wait for
    layer l and returns its slot, ``release(l, stream)`` lets the slot be
    reused once the work already on ``stream`` is done."""

    def __init__(self, layers, slots, slot_bytes: int, depth: int = 1, max_ctas: int = 0, workspace=None,
                 status=None, decode_stream=None):
        self._slots = list(slots)
        self._keep = []
        n = len(layers)
        larr = (Layer * n)()
        for l, tensors in enumerate(layers):
            tarr = (LayerTensor * max(1, len(tensors)))()
            for i, t in enumerate(tensors):
                self._keep.append(t.info)
                tarr[i].info = ctypes.pointer(t.info)
                tarr[i].d_blob = _ptr(t.d_blob)
                tarr[i].blob_size = _nbytes(t.d_blob, t.info.blob_bytes)
                tarr[i].out_offset = int(t.out_offset)
            self._keep.append(tarr)
            larr[l].tensors = tarr
            larr[l].count = len(tensors)
        sarr = (ctypes.c_void_p * len(self._slots))(*[_ptr(x) for x in self._slots])
        ws = _ptr(workspace)
        ws_bytes = int(workspace.numel() * workspace.element_size()) if workspace is not None else 0
        self._decode_stream = decode_stream
        h = ctypes.c_void_p()
        _check(_lib.ecf8_pipeline_create(larr, n, sarr, len(self._slots), int(slot_bytes), int(depth),
                                         int(max_ctas), ws, ws_bytes, _ptr(status), _stream(decode_stream),
                                         ctypes.byref(h)), "ecf8_pipeline_create")
        self._h = h

    def acquire(self, layer: int, stream=None) -> int:
        """Device address of layer's slot; ``stream`` waits for its decode."""
        w = ctypes.c_void_p()
        _check(_lib.ecf8_pipeline_acquire(self._h, int(layer), _stream(stream), ctypes.byref(w)),
               "ecf8_pipeline_acquire")
        return int(w.value or 0)

    def release(self, layer: int, stream=None) -> None:
        _check(_lib.ecf8_pipeline_release(self._h, int(layer), _stream(stream)), "ecf8_pipeline_release")

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.ecf8_pipeline_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()


# ---- BF16 variant: 8-bit exponent field coded, sign + mantissa byte kept ----

def _host_u16(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a CPU torch tensor (bfloat16 or int16)
        import torch
        t = x.detach().contiguous().view(-1)
        if t.dtype != torch.int16:
            t = t.view(torch.int16)
        x = t.numpy()
    a = np.ascontiguousarray(np.asarray(x).reshape(-1))
    if a.dtype != np.uint16:
        a = a.view(np.uint16)
    return a


def bf16_code_lengths(x, max_len: int = 16) -> np.ndarray:
    """Code lengths (256 entries) for the exponent fields of BF16 bit patterns."""
    a = _host_u16(x)
    ln = np.zeros(256, dtype=np.uint8)
    _check(_lib.ecf8_bf16_code_lengths(a.ctypes.data, a.size, max_len, ln.ctypes.data), "ecf8_bf16_code_lengths")
    return ln


def bf16_encode(x, lengths=None, chunk_bytes: int = DEFAULT_CHUNK_BYTES, group_chunks: int = DEFAULT_GROUP_CHUNKS,
                max_len: int = 16) -> np.ndarray:
    """Compress BF16 weights (bit patterns as uint16, or a CPU bfloat16 tensor) into a blob."""
    a = _host_u16(x)
    ln = bf16_code_lengths(a, max_len) if lengths is None else np.ascontiguousarray(np.asarray(lengths, np.uint8))
    size = ctypes.c_size_t(0)
    _check(_lib.ecf8_bf16_encoded_size(a.ctypes.data, a.size, ln.ctypes.data, chunk_bytes, group_chunks,
                                       ctypes.byref(size)), "ecf8_bf16_encoded_size")
    blob = np.empty(size.value, dtype=np.uint8)
    got = ctypes.c_size_t(0)
    _check(_lib.ecf8_bf16_encode(a.ctypes.data, a.size, ln.ctypes.data, chunk_bytes, group_chunks, blob.ctypes.data,
                                 blob.size, ctypes.byref(got)), "ecf8_bf16_encode")
    assert got.value == blob.size
    return blob


def bf16_blob_info(blob) -> Bf16Info:
    b = _host_u8(blob)
    info = Bf16Info()
    _check(_lib.ecf8_bf16_blob_info(b.ctypes.data, b.size, ctypes.byref(info)), "ecf8_bf16_blob_info")
    return info


def bf16_table(info: Bf16Info) -> np.ndarray:
    """The decode table of info's code (host uint8 array; copy it to the device once)."""
    t = np.zeros(int(_lib.ecf8_bf16_table_bytes()), dtype=np.uint8)
    _check(_lib.ecf8_bf16_build_table(ctypes.byref(info), t.ctypes.data), "ecf8_bf16_build_table")
    return t


def bf16_table_nodes(info: Bf16Info) -> int:
    """Tree nodes of info's code; the node with this index is the table's error node."""
    return int(_lib.ecf8_bf16_table_nodes(ctypes.byref(info)))


def bf16_auto_layout(info: Bf16Info) -> str:
    """The table layout ``bf16_decode`` picks for info's code."""
    rc = _lib.ecf8_bf16_auto_layout(ctypes.byref(info))
    if rc < 0:
        raise Ecf8Error(rc, "ecf8_bf16_auto_layout")
    return {v: k for k, v in BF16_LAYOUTS.items()}[rc]


def bf16_decode(info: Bf16Info, d_blob, d_table, d_out, status=None, stream=None, layout: str = "auto") -> None:
    """Asynchronously decode one BF16 blob in device memory into d_out (n
    uint16/bfloat16 elements) with the device copy of ``bf16_table(info)``;
    ``layout`` forces one of the decoder's table layouts (same output)."""
    _check(_lib.ecf8_bf16_decode_layout(ctypes.byref(info), _ptr(d_blob), _ptr(d_table), _ptr(d_out), info.n,
                                        _ptr(status), _stream(stream), BF16_LAYOUTS[layout]), "ecf8_bf16_decode")


def bf16_decode_batched(items, status=None, stream=None) -> None:
    """Asynchronously decode several BF16 blobs: ``items`` is a sequence of
    (info, d_blob, d_table, d_out); one launch per table layout present."""
    infos = [it[0] for it in items]
    arr = (Bf16Tensor * max(1, len(items)))()
    for k, (info, d_blob, d_table, d_out) in enumerate(items):
        arr[k] = Bf16Tensor(ctypes.pointer(infos[k]), _ptr(d_blob), _ptr(d_table), _ptr(d_out))
    _check(_lib.ecf8_bf16_decode_batched(arr, len(items), _ptr(status), _stream(stream)), "ecf8_bf16_decode_batched")
