"""Seeded synthetic inputs for the MC-Sparse hot path.

This package makes inputs only: bf16 Q/K/V tensors in the [B, N, H, d] layout,
shaped like the workloads the MC-Sparse pages measure on (Wan2.1 480p/720p video
latents, a MiniMax-H3 768p clip, a voxel-latent 3D asset) plus a tiny low-rank
case. It holds none of the method's arithmetic; the CPU oracle and the CUDA path
both consume what it writes. The random draws are counter based (see
``synth.c``), so one head of one step can be regenerated on its own.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

TENSORS = {"q": 0, "k": 1, "v": 2}


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so beside it (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_fill.restype = ctypes.c_int
        lib.synth_fill.argtypes = [
            ctypes.c_int, ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
            ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
        ]
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, density, schedule and value model."""

    name: str
    H: int
    N: int
    d: int
    density: float
    grid: tuple = ()          # (T, Y, X) token grid, empty for the low-rank model
    model: int = 1            # 0 = low-rank peaky, 1 = smooth 3D field
    gamma: float = 0.6
    drift: float = 0.05
    heavy_k: bool = False
    seed: int = 1000
    B: int = 1
    group: int = 128
    anchors: tuple = (0,)
    steps: int = 2
    layers: int = 1
    extra_density: tuple = field(default=())

    @property
    def topk(self) -> int:
        return topk_for(self.N, self.density)

    @property
    def G(self) -> int:
        return (self.N + self.group - 1) // self.group


def topk_for(N: int, density: float) -> int:
    """K = floor(s*N + 0.5): the nominal density s counted in KV tokens."""
    return int(math.floor(density * N + 0.5))


# The five workloads. Seeds are 1000 + workload number.
WORKLOADS = {
    "tiny": Workload("tiny", H=2, N=4096, d=64, density=0.25, model=0, seed=1001, steps=3, anchors=(0,)),
    "wan13b_480p": Workload("wan13b_480p", H=12, N=32760, d=128, density=0.25, grid=(21, 30, 52),
                            seed=1002, steps=5, anchors=(0,)),
    "wan14b_720p": Workload("wan14b_720p", H=40, N=75600, d=128, density=0.20, grid=(21, 45, 80),
                            seed=1003, steps=2, anchors=(0,)),
    "h3_768p": Workload("h3_768p", H=24, N=87696, d=128, density=0.15, grid=(87, 24, 42), heavy_k=True,
                        drift=0.03, seed=1004, steps=30, anchors=(0, 10, 20), extra_density=(0.25,)),
    "asset3d": Workload("asset3d", H=16, N=65536, d=64, density=0.15, grid=(64, 32, 32), seed=1005,
                        steps=12, anchors=(1,), layers=8),
}


def generate(w: Workload, tensor: str, step: int = 0, layer: int = 0, heads=None,
             nthreads: int | None = None) -> np.ndarray:
    """Return bf16 bit patterns (uint16) shaped [B, N, Hs, d] for heads ``heads``.

    ``heads`` defaults to all heads; a ``range`` selects a contiguous subset so a
    single head can be regenerated alone. Batch entries b > 0 use seed + 7919*b.
    """
    lib = _load()
    if heads is None:
        heads = range(w.H)
    h0, h1 = heads.start, heads.stop
    T, Y, X = w.grid if w.grid else (0, 0, 0)
    nthreads = nthreads or os.cpu_count() or 1
    out = np.empty((w.B, w.N, h1 - h0, w.d), dtype=np.uint16)
    for b in range(w.B):
        dst = np.ascontiguousarray(out[b])
        rc = lib.synth_fill(w.model, w.seed + 7919 * b, TENSORS[tensor], step, layer, w.H, h0, h1, w.N, w.d,
                            T, Y, X, w.gamma, w.drift, int(w.heavy_k), nthreads,
                            dst.ctypes.data_as(ctypes.c_void_p))
        if rc != 0:
            raise RuntimeError(f"synth_fill failed with code {rc}")
        out[b] = dst
    return out


def small(N: int, H: int = 1, d: int = 64, density: float = 0.25, seed: int = 7, B: int = 1,
          model: int = 0, grid: tuple = ()) -> Workload:
    """A ragged or tiny low-rank workload for parity and edge-case tests."""
    return Workload(f"small_N{N}_H{H}_d{d}", H=H, N=N, d=d, density=density, model=model, grid=grid,
                    seed=seed, B=B)


def to_torch_bf16(bits: np.ndarray):
    """View uint16 bf16 bit patterns as a torch.bfloat16 CPU tensor (no copy)."""
    import torch

    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
