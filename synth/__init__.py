"""Seeded synthetic inputs for the fused W4A4 + low-rank linear layer.

This package draws the activations X and the weight factors R, L1, L2 as BF16
bit patterns (numpy uint16) with the shapes and value distributions of the
workloads below. It contains no quantizer and no matmul: the oracle and the
CUDA path both take their inputs from here and share nothing else.

The generator itself (splitmix64 counter streams, Box-Muller normals,
Marsaglia-Tsang gamma variates, Student-t, BF16 round-to-nearest-even) is
defined in ``synth.c``.

Workloads (TwinQuant, "Learnable Subspace Decomposition for 4-Bit LLM
Quantization": shapes of the LLaMA3-8B attention projections and the LLaMA3 /
Qwen3 MLP projections that its kernel profile, Tables 6-7, covers; group size
128 and rank 128/256 from Section 5.1 and Table 2). Outlier channels are the
first round(p*m) entries of a seeded Fisher-Yates permutation of X's columns,
multiplied by the stated factor after drawing.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

NORMAL = 0
STUDENT_T = 1

# tensor ids of the stream keys
ID_X, ID_R, ID_L1, ID_L2, ID_XPERM = 0, 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _get_lib():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_fill_bf16.restype = ctypes.c_int
        lib.synth_fill_bf16.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
            ctypes.c_double, ctypes.c_double, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_int]
        lib.synth_permutation.restype = ctypes.c_int
        lib.synth_permutation.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                          ctypes.c_int]
        lib.synth_element_uniforms.restype = ctypes.c_int
        lib.synth_element_uniforms.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64,
                                               ctypes.c_int, ctypes.c_uint64]
        lib.synth_mix64.restype = ctypes.c_uint64
        lib.synth_mix64.argtypes = [ctypes.c_uint64]
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def fill(rows: int, cols: int, dist: int, p1: float, p2: float, seed: int, tensor_id: int,
         colmul: np.ndarray | None = None, with_values: bool = False):
    """Draw a rows x cols BF16 tensor (uint16 bits). Optionally also the float64 draws."""
    lib = _get_lib()
    out = np.empty((rows, cols), dtype=np.uint16)
    vals = np.empty((rows, cols), dtype=np.float64) if with_values else None
    cm = None
    if colmul is not None:
        cm = np.ascontiguousarray(colmul, dtype=np.float64)
        assert cm.shape == (cols,)
    rc = lib.synth_fill_bf16(out.ctypes.data, vals.ctypes.data if vals is not None else None,
                             rows, cols, dist, p1, p2, seed, tensor_id,
                             cm.ctypes.data if cm is not None else None, _threads())
    if rc != 0:
        raise ValueError("synth_fill_bf16 failed with code %d" % rc)
    return (out, vals) if with_values else out


def permutation(n: int, seed: int, tensor_id: int) -> np.ndarray:
    lib = _get_lib()
    p = np.empty(n, dtype=np.int32)
    lib.synth_permutation(p.ctypes.data, n, seed, tensor_id)
    return p


def element_uniforms(count: int, seed: int, tensor_id: int, e: int) -> np.ndarray:
    lib = _get_lib()
    u = np.empty(count, dtype=np.float64)
    lib.synth_element_uniforms(u.ctypes.data, count, seed, tensor_id, e)
    return u


def mix64(z: int) -> int:
    return int(_get_lib().synth_mix64(z & 0xFFFFFFFFFFFFFFFF))


@dataclass(frozen=True)
class Workload:
    name: str
    b: int
    m: int
    n: int
    r: int
    x_dist: tuple      # (dist, p1, p2)
    x_outlier: tuple   # (fraction of channels, factor)
    r_dist: tuple
    l_dist: tuple      # used for both L1 and L2


WORKLOADS = {
    # Tiny case: 16 x 512 x 512, rank 32.
    "tiny": Workload("tiny", 16, 512, 512, 32, (NORMAL, 0.0, 1.0), (0.02, 20.0),
                     (STUDENT_T, 3.0, 0.02), (NORMAL, 0.0, 0.05)),
    # Decode q/o projection of a LLaMA3-8B-like layer: b in {1, 4, 16}.
    "decode": Workload("decode", 16, 4096, 4096, 128, (NORMAL, 0.0, 1.0), (0.01, 30.0),
                       (STUDENT_T, 3.0, 0.02), (NORMAL, 0.0, 0.03)),
    # Prefill gate/up projection.
    "gateup": Workload("gateup", 2048, 4096, 14336, 128, (NORMAL, 0.0, 1.0), (0.01, 30.0),
                       (STUDENT_T, 3.0, 0.02), (NORMAL, 0.0, 0.03)),
    # Prefill down projection: heavy-tailed activations (Student-t nu=2.5).
    "down": Workload("down", 4096, 14336, 4096, 256, (STUDENT_T, 2.5, 1.0), (0.005, 50.0),
                     (STUDENT_T, 3.0, 0.015), (NORMAL, 0.0, 0.02)),
    # Large MLP of a Qwen3-32B-like layer.
    "large": Workload("large", 8192, 5120, 25600, 256, (NORMAL, 0.0, 1.0), (0.01, 30.0),
                      (STUDENT_T, 3.0, 0.02), (NORMAL, 0.0, 0.03)),
}

DECODE_BATCHES = (1, 4, 16)


def outlier_channels(m: int, frac: float, seed: int) -> np.ndarray:
    count = int(np.floor(frac * m + 0.5))
    return np.sort(permutation(m, seed, ID_XPERM)[:count])


def make_x(wl: Workload, b: int | None = None, seed: int = 0) -> np.ndarray:
    b = wl.b if b is None else b
    colmul = np.ones(wl.m, dtype=np.float64)
    colmul[outlier_channels(wl.m, wl.x_outlier[0], seed)] = wl.x_outlier[1]
    d = wl.x_dist
    return fill(b, wl.m, d[0], d[1], d[2], seed, ID_X, colmul)


def make_weights(wl: Workload, seed: int = 0, m: int | None = None, n: int | None = None,
                 r: int | None = None):
    """R (m x n), L1 (m x r), L2 (r x n) as BF16 bits, row-major."""
    m = wl.m if m is None else m
    n = wl.n if n is None else n
    r = wl.r if r is None else r
    R = fill(m, n, wl.r_dist[0], wl.r_dist[1], wl.r_dist[2], seed, ID_R)
    L1 = fill(m, r, wl.l_dist[0], wl.l_dist[1], wl.l_dist[2], seed, ID_L1)
    L2 = fill(r, n, wl.l_dist[0], wl.l_dist[1], wl.l_dist[2], seed, ID_L2)
    return R, L1, L2


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of BF16 bit patterns to float32 (a bit shift, no rounding)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bits with round-to-nearest-even (NaN -> 0x7FC0)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = (u & 0x7F800000) == 0x7F800000
    nan &= (u & 0x007FFFFF) != 0
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def sample_rows(b: int, count: int, seed: int) -> np.ndarray:
    """A seeded, sorted subset of row indices (always includes the first and last row)."""
    if count >= b:
        return np.arange(b)
    p = permutation(b, seed, 7)
    pick = set(int(v) for v in p[:max(0, count - 2)])
    pick.update({0, b - 1})
    return np.array(sorted(pick), dtype=np.int64)
