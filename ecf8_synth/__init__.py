"""Seeded synthetic FP8 E4M3 weight tensors and the workloads built from them.

This module draws inputs only; it contains none of the codec.  Both the CPU
oracle's tests and the GPU decoder's tests and benchmark take their tensors
from here, so the two sides see the same bytes.

Distributions follow the ECF8 walkthrough ("ECF8 浮点数压缩技术", p1 §2.1):
weights of trained networks are modelled as symmetric alpha-stable with alpha
in [1.5, 2]; alpha = 2 is the Gaussian.  Values are scaled in float64 and cast
to E4M3 with round-to-nearest-even, saturating at +-448.

Seeds: tensor ``t`` of workload ``c`` uses ``20251002 + 1000 * c + t``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_SO = os.path.join(_HERE, "libecf8_synth.so")

SEED_BASE = 20251002


def build(force: bool = False) -> str:
    """Compile the generator with gcc (OpenMP) into this directory."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", _SO, _SRC, "-lm"])
    return _SO


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, dbl, p = ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
        lib.synth_splitmix64.restype = u64
        lib.synth_splitmix64.argtypes = [u64, u64]
        lib.synth_uniform.restype = dbl
        lib.synth_uniform.argtypes = [u64, u64]
        lib.synth_e4m3.restype = ctypes.c_uint8
        lib.synth_e4m3.argtypes = [dbl]
        lib.synth_gaussian.restype = None
        lib.synth_gaussian.argtypes = [u64, u64, u64, dbl, p]
        lib.synth_bf16.restype = ctypes.c_uint16
        lib.synth_bf16.argtypes = [dbl]
        lib.synth_gaussian_bf16.restype = None
        lib.synth_gaussian_bf16.argtypes = [u64, u64, u64, dbl, p]
        lib.synth_sas_max_abs.restype = dbl
        lib.synth_sas_max_abs.argtypes = [u64, u64, dbl]
        lib.synth_sas.restype = None
        lib.synth_sas.argtypes = [u64, u64, u64, dbl, dbl, p]
        lib.synth_normal_raw.restype = None
        lib.synth_normal_raw.argtypes = [u64, u64, u64, p]
        lib.synth_sas_raw.restype = None
        lib.synth_sas_raw.argtypes = [u64, u64, u64, dbl, p]
        lib.synth_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def splitmix64(seed: int, counter: int) -> int:
    return int(_load().synth_splitmix64(seed, counter))


def uniform(seed: int, counter: int) -> float:
    return float(_load().synth_uniform(seed, counter))


def e4m3(x: float) -> int:
    """RNE cast of one double to an E4M3FN byte, saturating at +-448."""
    return int(_load().synth_e4m3(float(x)))


def bf16(x: float) -> int:
    """BF16 bit pattern of one double (through float32, nearest even)."""
    return int(_load().synth_bf16(float(x)))


def normal_raw(seed: int, n: int, begin: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_normal_raw(seed, begin, n, out.ctypes.data)
    return out


def sas_raw(seed: int, n: int, alpha: float, begin: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_sas_raw(seed, begin, n, alpha, out.ctypes.data)
    return out


def max_threads() -> int:
    return int(_load().synth_max_threads())


@dataclass(frozen=True)
class TensorSpec:
    """One synthetic FP8 weight tensor: shape, law and seed."""

    name: str
    rows: int
    cols: int
    seed: int
    dist: str  # "normal" or "sas"
    alpha: float = 2.0
    sigma: float = 1.0  # normal: values are sigma * N(0, 1)
    max_abs: float = 448.0  # sas: scale so that max |w| equals this

    @property
    def n(self) -> int:
        return self.rows * self.cols

    def scale(self) -> float:
        if self.dist != "sas":
            return self.sigma
        m = _load().synth_sas_max_abs(self.seed, self.n, self.alpha)
        return self.max_abs / m

    def generate(self, begin: int = 0, count: Optional[int] = None, scale: Optional[float] = None,
                 out: Optional[np.ndarray] = None) -> np.ndarray:
        """Bytes [begin, begin + count) of the tensor, row-major, as uint8."""
        count = self.n - begin if count is None else count
        if out is None:
            out = np.empty(count, dtype=np.uint8)
        assert out.dtype == np.uint8 and out.size >= count and out.flags.c_contiguous
        lib = _load()
        if self.dist == "normal":
            lib.synth_gaussian(self.seed, begin, count, self.sigma, out.ctypes.data)
        elif self.dist == "sas":
            s = self.scale() if scale is None else scale
            lib.synth_sas(self.seed, begin, count, self.alpha, s, out.ctypes.data)
        else:
            raise ValueError(self.dist)
        return out[:count]

    def generate_bf16(self, begin: int = 0, count: Optional[int] = None) -> np.ndarray:
        """Elements [begin, begin + count) as BF16 bit patterns (uint16):
        sigma * N(0, 1) rounded to BF16 (normal tensors only)."""
        if self.dist != "normal":
            raise ValueError("BF16 tensors are drawn from the normal law")
        count = self.n - begin if count is None else count
        out = np.empty(count, dtype=np.uint16)
        _load().synth_gaussian_bf16(self.seed, begin, count, self.sigma, out.ctypes.data)
        return out


@dataclass
class Workload:
    """A named set of tensors decoded together."""

    name: str
    description: str
    tensors: List[TensorSpec] = field(default_factory=list)

    @property
    def n_total(self) -> int:
        return sum(t.n for t in self.tensors)


def _seed(cfg: int, t: int) -> int:
    return SEED_BASE + 1000 * cfg + t


def single_normal_1k() -> Workload:
    """One 1024x1024 tensor, N(0,1)*16."""
    return Workload("single_1024x1024_normal16", "1024x1024 E4M3, w ~ N(0,1)*16",
                    [TensorSpec("w", 1024, 1024, _seed(1, 0), "normal", sigma=16.0)])


LLAMA3_8B_LAYER = [("q_proj", 4096, 4096), ("k_proj", 1024, 4096), ("v_proj", 1024, 4096),
                   ("o_proj", 4096, 4096), ("gate_proj", 14336, 4096), ("up_proj", 14336, 4096),
                   ("down_proj", 4096, 14336)]


def llama3_8b_layer(alpha: float = 1.8, max_abs: float = 448.0) -> Workload:
    """Seven projections of one Llama-3-8B decoder layer, SaS alpha=1.8, max|w|=448."""
    return Workload("llama3_8b_layer_sas1.8", "Llama-3-8B decoder layer (7 tensors), SaS a=1.8, max|w|=448",
                    [TensorSpec(nm, r, c, _seed(2, i), "sas", alpha=alpha, max_abs=max_abs)
                     for i, (nm, r, c) in enumerate(LLAMA3_8B_LAYER)])


def llama3_8b_layer_bf16(sigma: float = 0.02) -> Workload:
    """The seven Llama-3-8B decoder-layer projections in BF16, w ~ N(0, sigma^2)
    (the BF16 variant's workload: a BF16 checkpoint layer)."""
    return Workload("llama3_8b_layer_bf16_normal", f"Llama-3-8B decoder layer (7 tensors) BF16, w ~ N(0,1)*{sigma}",
                    [TensorSpec(nm, r, c, _seed(6, i), "normal", sigma=sigma)
                     for i, (nm, r, c) in enumerate(LLAMA3_8B_LAYER)])


SWEEP_ALPHAS = (1.5, 1.7, 1.9, 2.0)
SWEEP_MAXES = (448.0, 112.0, 28.0)


def alpha_sweep_point(alpha: float, max_abs: float) -> Workload:
    """One 14336x4096 tensor at (alpha, max|w|)."""
    idx = SWEEP_ALPHAS.index(alpha) * len(SWEEP_MAXES) + SWEEP_MAXES.index(max_abs)
    return Workload(f"ffn_14336x4096_sas{alpha}_max{int(max_abs)}",
                    f"14336x4096 E4M3, SaS a={alpha}, max|w|={max_abs}",
                    [TensorSpec("w", 14336, 4096, _seed(3, idx), "sas", alpha=alpha, max_abs=max_abs)])


def moe_experts(n_experts: int = 256, alpha: float = 1.7) -> Workload:
    """256 experts x {gate, up 2048x7168; down 7168x2048}, SaS alpha=1.7, per-expert scale."""
    ts = []
    for e in range(n_experts):
        for j, (nm, r, c) in enumerate((("gate", 2048, 7168), ("up", 2048, 7168), ("down", 7168, 2048))):
            ts.append(TensorSpec(f"expert{e}.{nm}", r, c, _seed(4, 3 * e + j), "sas", alpha=alpha, max_abs=448.0))
    return Workload(f"moe_{n_experts}x3_sas{alpha}", f"{n_experts} experts x 3 tensors, SaS a={alpha}", ts)


LLAMA3_70B_LAYER = [("q_proj", 8192, 8192), ("k_proj", 1024, 8192), ("v_proj", 1024, 8192),
                    ("o_proj", 8192, 8192), ("gate_proj", 28672, 8192), ("up_proj", 28672, 8192),
                    ("down_proj", 8192, 28672)]


def llama3_70b_layer(layer: int, alpha: float = 1.8) -> Workload:
    """One of the 80 Llama-3-70B decoder layers (7 tensors), SaS alpha=1.8, max|w|=448."""
    return Workload(f"llama3_70b_layer{layer}", f"Llama-3-70B layer {layer}",
                    [TensorSpec(nm, r, c, _seed(5, 7 * layer + i), "sas", alpha=alpha, max_abs=448.0)
                     for i, (nm, r, c) in enumerate(LLAMA3_70B_LAYER)])
