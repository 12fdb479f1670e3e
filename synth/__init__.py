"""Seeded synthetic inputs shared by the tests, the bench and the oracle.

The workloads stand in for Wan2.2 activations and weights, which are not
available here: spatiotemporally correlated activation fields with dynamic
outlier channels (DeltaQuant page, key design 1 and background section) and
Gaussian weights with outlier input columns.  This module draws numbers and
shapes them; it contains none of the method's arithmetic.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile libsynth.so in place (gcc, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        U = ctypes.c_uint64
        L = ctypes.c_longlong
        lib.synth_activations.argtypes = [P, I, I, I, I, I, I, I, I, D, D, U, U]
        lib.synth_weight.argtypes = [P, I, I, D, D, U]
        lib.synth_normal_bf16.argtypes = [P, L, D, U, U]
        lib.synth_uniform_f32.argtypes = [P, L, D, D, U, U]
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Workload:
    """One layer shape with its input recipe."""
    name: str
    T: int
    H: int
    W: int
    Ci: int
    Co: int
    rank: int
    cube: tuple
    grid: tuple
    x_outliers: tuple          # (fraction of channels, factor)
    w_outliers: tuple          # (fraction of input columns, factor); (0, 1) = none
    gelu: bool = False
    sweep: tuple = field(default_factory=tuple)   # extra cube shapes swept on this layer

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    def with_cube(self, cube):
        return Workload(self.name, self.T, self.H, self.W, self.Ci, self.Co, self.rank, tuple(cube),
                        self.grid, self.x_outliers, self.w_outliers, self.gelu, self.sweep)


def _coarse(T, H, W):
    # a grid 1 x 4 x 4 coarser than the token lattice (t, h, w)
    return (T, math.ceil(H / 4), math.ceil(W / 4))


WORKLOADS = {
    "tiny": Workload("tiny", 4, 8, 8, 256, 256, 16, (1, 2, 2), (2, 2, 2), (0.02, 40.0), (0.01, 20.0)),
    "wan480p_proj": Workload("wan480p_proj", 21, 30, 52, 5120, 5120, 32, (1, 2, 2), _coarse(21, 30, 52),
                             (0.01, 50.0), (0.01, 20.0)),
    "wan720p_ffn_up": Workload("wan720p_ffn_up", 21, 45, 80, 5120, 13824, 32, (2, 2, 2), _coarse(21, 45, 80),
                               (0.01, 50.0), (0.01, 20.0)),
    "wan720p_ffn_down": Workload("wan720p_ffn_down", 21, 45, 80, 13824, 5120, 32, (1, 2, 2), _coarse(21, 45, 80),
                                 (0.005, 80.0), (0.0, 1.0), gelu=True),
    "wan480p_cube_sweep": Workload("wan480p_cube_sweep", 21, 30, 52, 5120, 5120, 32, (1, 2, 2), _coarse(21, 30, 52),
                                   (0.01, 50.0), (0.01, 20.0),
                                   sweep=((1, 1, 1), (1, 2, 2), (2, 2, 2), (2, 4, 4), (21, 30, 52))),
}

# base seeds per workload (any fixed value works; recorded for reproducibility)
SEEDS = {"tiny": 0xD17A0000, "wan480p_proj": 0xD17A0001, "wan720p_ffn_up": 0xD17A0002,
         "wan720p_ffn_down": 0xD17A0003, "wan480p_cube_sweep": 0xD17A0004}


def activations(wl: Workload, seed: int | None = None, tau: int = 0) -> np.ndarray:
    """X as uint16 BF16 bits, shape (N, Ci), rows in (t, h, w) row-major order."""
    lib = _load()
    seed = SEEDS.get(wl.name, 1) if seed is None else seed
    X = np.empty((wl.N, wl.Ci), dtype=np.uint16)
    gT, gH, gW = wl.grid
    rc = lib.synth_activations(X.ctypes.data, wl.T, wl.H, wl.W, wl.Ci, gT, gH, gW, int(wl.gelu),
                               float(wl.x_outliers[0]), float(wl.x_outliers[1]), seed & (2**64 - 1),
                               tau)
    if rc != 0:
        raise RuntimeError(f"synth_activations failed ({rc})")
    return X


def weight(wl: Workload, seed: int | None = None) -> np.ndarray:
    """W as uint16 BF16 bits, shape (Co, Ci); the layer computes y = x W^T."""
    lib = _load()
    seed = (SEEDS.get(wl.name, 1) if seed is None else seed) ^ 0x5EED
    Wt = np.empty((wl.Co, wl.Ci), dtype=np.uint16)
    rc = lib.synth_weight(Wt.ctypes.data, wl.Co, wl.Ci, float(wl.w_outliers[0]), float(wl.w_outliers[1]),
                          seed & (2**64 - 1))
    if rc != 0:
        raise RuntimeError(f"synth_weight failed ({rc})")
    return Wt


def normal_bf16(shape, sd: float = 1.0, seed: int = 1, stream: int = 0) -> np.ndarray:
    lib = _load()
    out = np.empty(shape, dtype=np.uint16)
    lib.synth_normal_bf16(out.ctypes.data, out.size, float(sd), seed & (2**64 - 1), stream)
    return out


def uniform_f32(shape, lo: float, hi: float, seed: int = 1, stream: int = 0) -> np.ndarray:
    lib = _load()
    out = np.empty(shape, dtype=np.float32)
    lib.synth_uniform_f32(out.ctypes.data, out.size, float(lo), float(hi), seed & (2**64 - 1), stream)
    return out

