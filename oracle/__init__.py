"""TEST INFRASTRUCTURE ONLY: the CPU oracle of the fused W4A4 + low-rank layer.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never links, loads or calls it.

This module is argument marshalling around ``twq_oracle.cpp`` (plain
single-threaded C++, fp64 accumulation); see that file for the definition and
the passages of TwinQuant it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "twq_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

FUSED, W4A4_ONLY, LOWRANK_ONLY = 0, 1, 2
GROUP = 128


# IEEE float semantics: no fast-math, no contraction, SSE2 floats
CXX = ["g++", "-std=c++17", "-O2", "-fno-fast-math", "-ffp-contract=off", "-msse2",
       "-mfpmath=sse", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with IEEE float semantics (no fast-math, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(CXX + ["-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int64


def _load(path):
    """The oracle's C library at `path`, with its argument types declared."""
    lib = ctypes.CDLL(path)
    for name, args in {
        "twq_ref_quant_group_f32": [_P, ctypes.c_int, _P, _P],
        "twq_ref_quant_group_f32_a8": [_P, ctypes.c_int, _P, _P],
        "twq_ref_quantize_rows_q": [_P, _I, _I, _I, ctypes.c_int, _P, _P],
        "twq_ref_quantize_rows": [_P, _I, _I, _I, _P, _P],
        "twq_ref_quantize_cols": [_P, _I, _I, _P, _P],
        "twq_ref_pack_nibbles": [_P, _I, _P],
        "twq_ref_unpack_nibbles": [_P, _I, _P],
        "twq_ref_quantize_act": [_P, _I, _I, _I, _P, _P],
        "twq_ref_pack_weights": [_P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P],
        "twq_ref_linear": [_P, _P, _I, _I, _P, _P, _I, _P, _P, _I, _P, ctypes.c_int, _P, _I,
                           _P, _P, _P, _P],
        "twq_ref_dequant_matmul": [_P, _P, _I, _I, _P, _P, _I, _P, _P, _I, _P, ctypes.c_int,
                                   _P],
    }.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.twq_ref_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.twq_ref_f32_to_bf16.restype = ctypes.c_uint16
    lib.twq_ref_qmax.restype = ctypes.c_int
    lib.twq_ref_qmax_a8.restype = ctypes.c_int
    return lib


def _get():
    global _lib
    if _lib is None:
        _lib = _load(build())
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def _check(rc, what):
    if rc != 0:
        raise ValueError("%s failed (code %d)" % (what, rc))


def qmax() -> int:
    return _get().twq_ref_qmax()


def qmax_a8() -> int:
    """q_max of the W4A8 activations (Eq. (1) with k = 8)."""
    return _get().twq_ref_qmax_a8()


def quant_group_f32(v, a8=False):
    v = _c(v, np.float32)
    q = np.empty(v.size, np.int8)
    s = np.empty(1, np.float32)
    fn = _get().twq_ref_quant_group_f32_a8 if a8 else _get().twq_ref_quant_group_f32
    _check(fn(_ptr(v), v.size, _ptr(q), _ptr(s)), "quant_group")
    return q, float(s[0])


def quantize_rows(x_bits, a8=False):
    """X (rows x m BF16 bits) -> codes (rows x m int8), scales (rows x m/128 fp32);
    q_max = 7, or 127 for the W4A8 activations (a8)."""
    x = _c(x_bits, np.uint16)
    rows, m = x.shape
    q = np.empty((rows, m), np.int8)
    s = np.empty((rows, m // GROUP), np.float32)
    _check(_get().twq_ref_quantize_rows_q(_ptr(x), rows, m, m, qmax_a8() if a8 else qmax(),
                                          _ptr(q), _ptr(s)), "quantize_rows")
    return q, s


def quantize_cols(w_bits):
    """W (m x cols BF16 bits) -> codes (cols x m int8), scales (m/128 x cols fp32)."""
    w = _c(w_bits, np.uint16)
    m, cols = w.shape
    q = np.empty((cols, m), np.int8)
    s = np.empty((m // GROUP, cols), np.float32)
    _check(_get().twq_ref_quantize_cols(_ptr(w), m, cols, _ptr(q), _ptr(s)), "quantize_cols")
    return q, s


def pack_nibbles(q):
    q = _c(q, np.int8)
    out = np.empty(q.shape[:-1] + (q.shape[-1] // 2,), np.uint8)
    _check(_get().twq_ref_pack_nibbles(_ptr(q), q.size, _ptr(out)), "pack_nibbles")
    return out


def unpack_nibbles(p):
    p = _c(p, np.uint8)
    q = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.int8)
    _check(_get().twq_ref_unpack_nibbles(_ptr(p), q.size, _ptr(q)), "unpack_nibbles")
    return q


def quantize_act(x_bits):
    """The library's activation format: xq (rows x m/2 uint8), sx (rows x m/128 fp32)."""
    x = _c(x_bits, np.uint16)
    rows, m = x.shape
    xq = np.empty((rows, m // 2), np.uint8)
    sx = np.empty((rows, m // GROUP), np.float32)
    _check(_get().twq_ref_quantize_act(_ptr(x), rows, m, m, _ptr(xq), _ptr(sx)), "quantize_act")
    return xq, sx


def pack_weights(R, L1, L2):
    """The library's weight format: dict rq, sr, l1q, sl1, l2t."""
    R = _c(R, np.uint16)
    m, n = R.shape
    r = 0 if L1 is None else L1.shape[1]
    L1c = _c(L1, np.uint16) if r else None
    L2c = _c(L2, np.uint16) if r else None
    out = dict(rq=np.empty((n, m // 2), np.uint8), sr=np.empty((m // GROUP, n), np.float32),
               l1q=np.empty((r, m // 2), np.uint8), sl1=np.empty((m // GROUP, r), np.float32),
               l2t=np.empty((n, r), np.uint16))
    _check(_get().twq_ref_pack_weights(_ptr(R), _ptr(L1c), _ptr(L2c), m, n, r, _ptr(out["rq"]),
                                       _ptr(out["sr"]), _ptr(out["l1q"]), _ptr(out["sl1"]),
                                       _ptr(out["l2t"])), "pack_weights")
    return out


def linear(qx, sx, qr, sr, ql1, sl1, L2, mode=FUSED, rows=None, want=("y",)):
    """Y for the listed rows from unpacked codes. Returns dict of the wanted outputs
    among y (BF16 bits), y64 (float64), h64 (float64), hb (BF16 bits)."""
    qx = _c(qx, np.int8)
    sx = _c(sx, np.float32)
    b, m = qx.shape
    n = qr.shape[0] if qr is not None else L2.shape[1]
    r = 0 if ql1 is None else ql1.shape[0]
    rows_a = None if rows is None else _c(rows, np.int64)
    nr = b if rows_a is None else rows_a.size
    out = {}
    if "y" in want:
        out["y"] = np.empty((nr, n), np.uint16)
    if "y64" in want:
        out["y64"] = np.empty((nr, n), np.float64)
    if "h64" in want:
        out["h64"] = np.empty((nr, max(r, 1)), np.float64)
    if "hb" in want:
        out["hb"] = np.empty((nr, max(r, 1)), np.uint16)
    qr_c = None if qr is None else _c(qr, np.int8)
    sr_c = None if sr is None else _c(sr, np.float32)
    ql1_c = None if ql1 is None else _c(ql1, np.int8)
    sl1_c = None if sl1 is None else _c(sl1, np.float32)
    l2_c = None if L2 is None else _c(L2, np.uint16)
    _check(_get().twq_ref_linear(_ptr(qx), _ptr(sx), b, m, _ptr(qr_c), _ptr(sr_c), n,
                                 _ptr(ql1_c), _ptr(sl1_c), r, _ptr(l2_c), mode, _ptr(rows_a), nr,
                                 _ptr(out.get("y")), _ptr(out.get("y64")), _ptr(out.get("h64")),
                                 _ptr(out.get("hb"))), "linear")
    return out


def dequant_matmul(qx, sx, qr, sr, ql1, sl1, L2, mode=FUSED):
    qx = _c(qx, np.int8)
    sx = _c(sx, np.float32)
    b, m = qx.shape
    n = qr.shape[0] if qr is not None else L2.shape[1]
    r = 0 if ql1 is None else ql1.shape[0]
    y = np.empty((b, n), np.float64)
    _check(_get().twq_ref_dequant_matmul(
        _ptr(qx), _ptr(sx), b, m, _ptr(None if qr is None else _c(qr, np.int8)),
        _ptr(None if sr is None else _c(sr, np.float32)), n,
        _ptr(None if ql1 is None else _c(ql1, np.int8)),
        _ptr(None if sl1 is None else _c(sl1, np.float32)), r,
        _ptr(None if L2 is None else _c(L2, np.uint16)), mode, _ptr(y)), "dequant_matmul")
    return y


def f32_to_bf16(f: float) -> int:
    return int(_get().twq_ref_f32_to_bf16(f))


def layer(x_bits, R, L1, L2, mode=FUSED, rows=None, want=("y",), a8=False):
    """End to end from BF16 inputs: quantize X (rows x m), R, L1, then the layer.
    a8: W4A8, the activations quantized with q_max = 127 (8-bit codes)."""
    qx, sx = quantize_rows(x_bits, a8=a8)
    qr, sr = quantize_cols(R)
    if L1 is not None and L1.shape[1] > 0:
        ql1, sl1 = quantize_cols(L1)
    else:
        ql1 = sl1 = None
        L2 = None
    return linear(qx, sx, qr, sr, ql1, sl1, L2, mode=mode, rows=rows, want=want)


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _f64_to_bf16(f):
    """fp64 -> fp32 (RNE) -> BF16 (RNE) bit patterns, finite inputs."""
    u = np.asarray(f, np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def fold_transforms(Q, G, U, V, R, rounded=True):
    """Offline fold of TwinQuant §4.1 (Eq. (6) and the factors after it):
    U' = Q^-1 U G, V' = G^-1 V, R' = Q^-1 R, with Q orthogonal (§4.2: Q^T Q = I,
    read as Q^-1 = Q^T) and G invertible (G^-1 by numpy's LU inverse).

    Q: m x m fp32, G: r x r fp32; U (m x r), V (r x n), R (m x n): BF16 bits.
    Returns BF16 bits of (U', V', R') in fp64 arithmetic, or the fp64 values
    themselves if not `rounded`."""
    q = np.asarray(Q, np.float32).astype(np.float64)
    g = np.asarray(G, np.float32).astype(np.float64)
    u, v, r = _bf16_to_f64(U), _bf16_to_f64(V), _bf16_to_f64(R)
    l1 = q.T @ (u @ g)
    l2 = np.linalg.inv(g) @ v
    rr = q.T @ r
    if not rounded:
        return l1, l2, rr
    return _f64_to_bf16(l1), _f64_to_bf16(l2), _f64_to_bf16(rr)


def layer_s2q(x_bits, R, L1, L2, rows=None, want=("y",)):
    """The layer with the pages' INT4 stage 2 (TwinQuant §4.3: H is requantized to
    4 bits on chip and multiplied by the 4-bit V). Readings: H is first rounded to
    BF16 (as in the BF16 stage 2); Q_H is Eq. (1) on it per token in groups of 128
    along r; V = L2 is quantized per output column in groups of 128 along r; both
    with q_max = 7. Then, per group g of r (Eq. (2) applied group by group):

        Y_lr[i, j] = sum_g sH[i, g] * sV[g, j] * sum_{k in g} qH[i, k] * qV[j, k]
        Y          = bf16(float(Y_res + Y_lr))

    Needs r % 128 == 0. Returns a dict of the wanted outputs among y (BF16 bits),
    y64 (float64), hb (BF16 bits of H), qh, sh (codes and scales of H)."""
    qx, sx = quantize_rows(x_bits)
    qr, sr = quantize_cols(R)
    ql1, sl1 = quantize_cols(L1)
    r = ql1.shape[0]
    if r % GROUP:
        raise ValueError("the INT4 stage 2 needs r % 128 == 0")
    res = linear(qx, sx, qr, sr, None, None, None, mode=W4A4_ONLY, rows=rows, want=("y64",))["y64"]
    hb = linear(qx, sx, None, None, ql1, sl1, L2, mode=LOWRANK_ONLY, rows=rows, want=("hb",))["hb"]
    qh, sh = quantize_rows(hb)          # Eq. (1) on bf16(H), per token, groups of 128 along r
    qv, sv = quantize_cols(L2)          # Eq. (1) on L2 (r x n), per column, groups along r
    # the grouped integer GEMM of Eq. (2), with qH as the activations and qV as the weights
    ylr = linear(qh, sh, qv, sv, None, None, None, mode=W4A4_ONLY, want=("y64",))["y64"]
    total = res + ylr
    out = {"y": _f64_to_bf16(total), "y64": total, "hb": hb, "qh": qh, "sh": sh}
    return {k: out[k] for k in want}
