"""Python binding of libtwq.so (include/twq.h): argument marshalling only.

Each function has the name of the C entry point without the ``twq_`` prefix.
Tensors are torch CUDA tensors; the binding allocates outputs as the caller
(the library itself never allocates) and passes the current CUDA stream.
Every step of the layer runs in the library's kernels; there is no fallback:
if the library is missing or a tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtwq.so")

OK = 0
STATUS_NAMES = {0: "TWQ_OK", 1: "TWQ_ERR_INVALID_ARG", 2: "TWQ_ERR_UNSUPPORTED",
                3: "TWQ_ERR_MISALIGNED", 4: "TWQ_ERR_CUDA", 5: "TWQ_ERR_NOT_IMPLEMENTED",
                6: "TWQ_ERR_DEVICE"}

# Every extern "C" symbol that include/twq.h declares.
EXPORTS = ("twq_version", "twq_status_string", "twq_weights_sizes", "twq_act_sizes",
           "twq_quantize_act", "twq_pack_weights", "twq_fused_linear", "twq_w4a4_only",
           "twq_lowrank_only", "twq_unfused_workspace_bytes", "twq_unfused_linear",
           "twq_device_status", "twq_launches_per_call", "twq_unfused_linear_noalloc",
           "twq_fused_linear_x", "twq_fold_workspace_bytes", "twq_fold_transforms",
           "twq_fused_linear_x_host", "twq_quantize_act_a8", "twq_fused_linear_a8",
           "twq_fused_linear_x_a8", "twq_pack_l2_int4", "twq_fused_linear_s2q",
           "twq_linear_host", "twq_release_cache", "twq_selftest_wait_timeout",
           "twq_quantize_act_i8", "twq_fused_linear_i8")


class TwqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (what, STATUS_NAMES.get(status, "?"), status))


class _Weights(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int64), ("n", ctypes.c_int64), ("r", ctypes.c_int64),
                ("rq", ctypes.c_void_p), ("sr", ctypes.c_void_p), ("l1q", ctypes.c_void_p),
                ("sl1", ctypes.c_void_p), ("l2t", ctypes.c_void_p)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libtwq.so not found at %s: build it with __graft_entry__.build() "
                           "or `python rank_residual_w4a4_b200/_build.py`" % path)
    lib = ctypes.CDLL(path)
    P, I, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "twq_version": ([], ctypes.c_int),
        "twq_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "twq_weights_sizes": ([I, I, I, P], ctypes.c_int),
        "twq_act_sizes": ([I, I, P], ctypes.c_int),
        "twq_quantize_act": ([P, I, I, I, P, P, P], ctypes.c_int),
        "twq_pack_weights": ([P, P, P, P, P], ctypes.c_int),
        "twq_fused_linear": ([P, P, I, P, P, P], ctypes.c_int),
        "twq_w4a4_only": ([P, P, I, P, P, P], ctypes.c_int),
        "twq_lowrank_only": ([P, P, I, P, P, P], ctypes.c_int),
        "twq_unfused_workspace_bytes": ([I, I, I], S),
        "twq_unfused_linear": ([P, P, I, P, P, P, S, P], ctypes.c_int),
        "twq_device_status": ([P], ctypes.c_int),
        "twq_launches_per_call": ([ctypes.c_char_p], ctypes.c_int),
        "twq_unfused_linear_noalloc": ([P, P, I, P, P, P], ctypes.c_int),
        "twq_fused_linear_x": ([P, I, I, P, P, P], ctypes.c_int),
        "twq_fused_linear_x_host": ([P, I, P, P, P, P, P], ctypes.c_int),
        "twq_quantize_act_a8": ([P, I, I, I, P, P, P], ctypes.c_int),
        "twq_fused_linear_a8": ([P, P, I, P, P, P], ctypes.c_int),
        "twq_fused_linear_x_a8": ([P, I, I, P, P, P], ctypes.c_int),
        "twq_pack_l2_int4": ([P, I, I, P, P, P], ctypes.c_int),
        "twq_fused_linear_s2q": ([P, P, I, P, P, P, P, P], ctypes.c_int),
        "twq_fold_workspace_bytes": ([I, I, I], S),
        "twq_fold_transforms": ([P, P, P, P, P, I, I, I, P, P, P, P, S, P], ctypes.c_int),
        "twq_linear_host": ([P, I, P, P, P, P, P, P, P], ctypes.c_int),
        "twq_release_cache": ([], None),
        "twq_selftest_wait_timeout": ([P, P, I, P, P, I, P], ctypes.c_int),
        "twq_quantize_act_i8": ([P, I, I, I, P, P, P], ctypes.c_int),
        "twq_fused_linear_i8": ([P, P, I, P, P, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != OK:
        raise TwqError(status, what)


def _dev(t: torch.Tensor, name: str, dtype) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be on a CUDA device (the library has no CPU path)" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def version() -> int:
    return load().twq_version()


def weights_sizes(m: int, n: int, r: int):
    arr = (ctypes.c_size_t * 5)()
    _check(load().twq_weights_sizes(m, n, r, arr), "twq_weights_sizes")
    return tuple(int(v) for v in arr)


def act_sizes(b: int, m: int):
    arr = (ctypes.c_size_t * 2)()
    _check(load().twq_act_sizes(b, m, arr), "twq_act_sizes")
    return tuple(int(v) for v in arr)


@dataclass
class Weights:
    """Packed weights of one layer (device tensors) in the library's format."""
    m: int
    n: int
    r: int
    rq: torch.Tensor    # n x m/2 uint8
    sr: torch.Tensor    # m/128 x n float32
    l1q: torch.Tensor   # r x m/2 uint8
    sl1: torch.Tensor   # m/128 x r float32
    l2t: torch.Tensor   # n x r bfloat16

    def __setattr__(self, name, value):
        object.__setattr__(self, name, value)
        if name != "_c":
            object.__setattr__(self, "_c", None)  # a field changed: rebuild the C view

    def c_struct(self) -> _Weights:
        """The C-ABI view (built once; the library only reads it during a call). It
        follows field reassignment, not a tensor re-pointed in place (Tensor.set_)."""
        c = getattr(self, "_c", None)
        if c is None:
            nz = lambda t: t.data_ptr() if t.numel() else None
            c = _Weights(self.m, self.n, self.r, self.rq.data_ptr(), self.sr.data_ptr(),
                         nz(self.l1q), nz(self.sl1), nz(self.l2t))
            object.__setattr__(self, "_c", c)
        return c

    @staticmethod
    def empty(m: int, n: int, r: int, device) -> "Weights":
        return Weights(m, n, r,
                       torch.empty((n, m // 2), dtype=torch.uint8, device=device),
                       torch.empty((m // 128, n), dtype=torch.float32, device=device),
                       torch.empty((r, m // 2), dtype=torch.uint8, device=device),
                       torch.empty((m // 128, r), dtype=torch.float32, device=device),
                       torch.empty((n, r), dtype=torch.bfloat16, device=device))


def quantize_act(x: torch.Tensor, xq: torch.Tensor | None = None, sx: torch.Tensor | None = None,
                 stream=None):
    """BF16 X (b x m) -> packed codes (b x m/2 uint8) and scales (b x m/128 fp32)."""
    b, m = x.shape
    if xq is None:
        xq = torch.empty((b, m // 2), dtype=torch.uint8, device=x.device)
    if sx is None:
        sx = torch.empty((b, max(m // 128, 1)), dtype=torch.float32, device=x.device)
    _check(load().twq_quantize_act(_dev(x, "x", torch.bfloat16), b, m, m,
                                   _dev(xq, "xq", torch.uint8), _dev(sx, "sx", torch.float32),
                                   _stream(stream)), "twq_quantize_act")
    return xq, sx


def pack_weights(R: torch.Tensor, L1: torch.Tensor | None, L2: torch.Tensor | None,
                 out: Weights | None = None, stream=None) -> Weights:
    """BF16 R (m x n), L1 (m x r), L2 (r x n) -> packed Weights."""
    m, n = R.shape
    r = 0 if L1 is None else L1.shape[1]
    w = Weights.empty(m, n, r, R.device) if out is None else out
    cw = w.c_struct()
    _check(load().twq_pack_weights(
        _dev(R, "R", torch.bfloat16),
        _dev(L1, "L1", torch.bfloat16) if r else None,
        _dev(L2, "L2", torch.bfloat16) if r else None,
        ctypes.byref(cw), _stream(stream)), "twq_pack_weights")
    return w


def _layer(fn: str, xq, sx, w: Weights, y, stream):
    b = xq.shape[0]
    if y is None:
        y = torch.empty((b, w.n), dtype=torch.bfloat16, device=xq.device)
    cw = w.c_struct()
    _check(getattr(load(), fn)(_dev(xq, "xq", torch.uint8), _dev(sx, "sx", torch.float32), b,
                               ctypes.byref(cw), _dev(y, "y", torch.bfloat16), _stream(stream)), fn)
    return y


def fused_linear(xq, sx, w: Weights, y=None, stream=None):
    return _layer("twq_fused_linear", xq, sx, w, y, stream)


def quantize_act_a8(x: torch.Tensor, xq8: torch.Tensor | None = None,
                    sx: torch.Tensor | None = None, stream=None):
    """W4A8 activations: BF16 X (b x m) -> int8 codes (b x m, q_max = 127) and scales
    (b x m/128 fp32)."""
    b, m = x.shape
    if xq8 is None:
        xq8 = torch.empty((b, m), dtype=torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty((b, max(m // 128, 1)), dtype=torch.float32, device=x.device)
    _check(load().twq_quantize_act_a8(_dev(x, "x", torch.bfloat16), b, m, m,
                                      _dev(xq8, "xq8", torch.int8), _dev(sx, "sx", torch.float32),
                                      _stream(stream)), "twq_quantize_act_a8")
    return xq8, sx


def quantize_act_i8(x: torch.Tensor, xq8: torch.Tensor | None = None,
                    sx: torch.Tensor | None = None, stream=None):
    """BF16 X (b x m) -> the 4-bit codes of quantize_act stored one per byte (b x m int8,
    values in [-7, 7]) and the same scales (b x m/128 fp32)."""
    b, m = x.shape
    if xq8 is None:
        xq8 = torch.empty((b, m), dtype=torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty((b, max(m // 128, 1)), dtype=torch.float32, device=x.device)
    _check(load().twq_quantize_act_i8(_dev(x, "x", torch.bfloat16), b, m, m,
                                      _dev(xq8, "xq8", torch.int8), _dev(sx, "sx", torch.float32),
                                      _stream(stream)), "twq_quantize_act_i8")
    return xq8, sx


def fused_linear_i8(xq8, sx, w: Weights, y=None, stream=None):
    """The fused layer on activation codes stored one per byte (quantize_act_i8)."""
    b = xq8.shape[0]
    if y is None:
        y = torch.empty((b, w.n), dtype=torch.bfloat16, device=xq8.device)
    cw = w.c_struct()
    _check(load().twq_fused_linear_i8(_dev(xq8, "xq8", torch.int8), _dev(sx, "sx", torch.float32),
                                      b, ctypes.byref(cw), _dev(y, "y", torch.bfloat16),
                                      _stream(stream)), "twq_fused_linear_i8")
    return y


def fused_linear_a8(xq8, sx, w: Weights, y=None, stream=None):
    """The fused W4A8 layer on codes from quantize_act_a8 (decode batches, b <= 16)."""
    b = xq8.shape[0]
    if y is None:
        y = torch.empty((b, w.n), dtype=torch.bfloat16, device=xq8.device)
    cw = w.c_struct()
    _check(load().twq_fused_linear_a8(_dev(xq8, "xq8", torch.int8), _dev(sx, "sx", torch.float32),
                                      b, ctypes.byref(cw), _dev(y, "y", torch.bfloat16),
                                      _stream(stream)), "twq_fused_linear_a8")
    return y


def pack_l2_int4(L2: torch.Tensor, stream=None):
    """The INT4 stage 2's V: BF16 L2 (r x n) -> 4-bit codes (n x r/2 uint8) and scales
    ((r/128) x n fp32), groups of 128 along r per output column."""
    r, n = L2.shape
    l2q = torch.empty((n, r // 2), dtype=torch.uint8, device=L2.device)
    sl2q = torch.empty((max(r // 128, 1), n), dtype=torch.float32, device=L2.device)
    _check(load().twq_pack_l2_int4(_dev(L2, "L2", torch.bfloat16), r, n,
                                   _dev(l2q, "l2q", torch.uint8), _dev(sl2q, "sl2q", torch.float32),
                                   _stream(stream)), "twq_pack_l2_int4")
    return l2q, sl2q


def fused_linear_s2q(xq, sx, w: Weights, l2q, sl2q, y=None, stream=None):
    """The fused layer with the INT4 stage 2 (H requantized on chip, 4-bit L2)."""
    b = xq.shape[0]
    if y is None:
        y = torch.empty((b, w.n), dtype=torch.bfloat16, device=xq.device)
    cw = w.c_struct()
    _check(load().twq_fused_linear_s2q(_dev(xq, "xq", torch.uint8), _dev(sx, "sx", torch.float32),
                                       b, ctypes.byref(cw), _dev(l2q, "l2q", torch.uint8),
                                       _dev(sl2q, "sl2q", torch.float32),
                                       _dev(y, "y", torch.bfloat16), _stream(stream)),
           "twq_fused_linear_s2q")
    return y


def fused_linear_x(x: torch.Tensor, w: Weights, y=None, stream=None, a8: bool = False):
    """BF16 X (b x m, rows may be strided) -> Y in one launch, quantizing X inside
    the layer kernel (decode batches, b <= 16). a8: W4A8 (8-bit activation codes)."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise TypeError("x must be a 2-D torch tensor")
    if not x.is_cuda:
        raise ValueError("x must be on a CUDA device (the library has no CPU path)")
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be torch.bfloat16, got %s" % x.dtype)
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along m")
    b = x.shape[0]
    ldx = x.stride(0) if b > 1 else x.shape[1]
    if y is None:
        y = torch.empty((b, w.n), dtype=torch.bfloat16, device=x.device)
    cw = w.c_struct()
    fn = "twq_fused_linear_x_a8" if a8 else "twq_fused_linear_x"
    _check(getattr(load(), fn)(x.data_ptr(), ldx, b, ctypes.byref(cw),
                               _dev(y, "y", torch.bfloat16), _stream(stream)), fn)
    return y


def fused_linear_x_host(x_host: torch.Tensor, w: Weights, x_dev: torch.Tensor,
                        y_dev: torch.Tensor, y_host: torch.Tensor, stream=None):
    """One decode step from host memory to host memory on `stream`: copy x_host into
    x_dev, run fused_linear_x, copy y_dev into y_host. Nothing is synchronized; y_host
    holds Y once the stream reaches the end of the step. Host tensors should be pinned."""
    for t, name in ((x_host, "x_host"), (y_host, "y_host")):
        if not isinstance(t, torch.Tensor) or t.is_cuda:
            raise TypeError("%s must be a host (CPU) torch tensor" % name)
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise TypeError("%s must be a contiguous torch.bfloat16 tensor" % name)
    b = x_host.shape[0]
    if x_host.shape != (b, w.m) or y_host.shape != (b, w.n):
        raise ValueError("x_host must be (b, m) and y_host (b, n)")
    if x_dev.shape != (b, w.m) or y_dev.shape != (b, w.n):
        raise ValueError("x_dev must be (b, m) and y_dev (b, n)")
    cw = w.c_struct()
    _check(load().twq_fused_linear_x_host(x_host.data_ptr(), b, ctypes.byref(cw),
                                          _dev(x_dev, "x_dev", torch.bfloat16),
                                          _dev(y_dev, "y_dev", torch.bfloat16),
                                          y_host.data_ptr(), _stream(stream)),
           "twq_fused_linear_x_host")
    return y_host


class DecodeStep:
    """A prepared twq_fused_linear_x_host call for a serving loop. The device
    buffers, the pinned host output and the stream are checked once; each call
    passes a host X of the same shape and the layer's weights (their C view is
    cached on the Weights object), so a step costs one C call."""

    def __init__(self, x_dev: torch.Tensor, y_dev: torch.Tensor, y_host: torch.Tensor, stream=None):
        self._b, self._m = x_dev.shape
        if y_dev.shape[0] != self._b or y_host.shape != y_dev.shape:
            raise ValueError("x_dev (b, m), y_dev and y_host (b, n) must agree")
        if not isinstance(y_host, torch.Tensor) or y_host.is_cuda:
            raise TypeError("y_host must be a host (CPU) torch tensor")
        if y_host.dtype != torch.bfloat16 or not y_host.is_contiguous():
            raise TypeError("y_host must be a contiguous torch.bfloat16 tensor")
        self._n = y_dev.shape[1]
        self._xd = _dev(x_dev, "x_dev", torch.bfloat16)
        self._yd = _dev(y_dev, "y_dev", torch.bfloat16)
        self._yh = y_host.data_ptr()
        self._keep = (x_dev, y_dev, y_host)  # the buffers outlive the prepared call
        self._st = _stream(stream)
        self._fn = load().twq_fused_linear_x_host
        self.y_host = y_host

    def __call__(self, x_host: torch.Tensor, w: Weights) -> torch.Tensor:
        if x_host.is_cuda or x_host.dtype != torch.bfloat16 or not x_host.is_contiguous():
            raise TypeError("x_host must be a contiguous host torch.bfloat16 tensor")
        if x_host.shape[0] != self._b or x_host.shape[1] != self._m or w.m != self._m or w.n != self._n:
            raise ValueError("x_host and w must match the prepared shapes")
        _check(self._fn(x_host.data_ptr(), self._b, ctypes.byref(w.c_struct()), self._xd, self._yd,
                        self._yh, self._st), "twq_fused_linear_x_host")
        return self.y_host


class LinearHostStep:
    """A prepared twq_linear_host call: one layer call for any batch from host memory
    to host memory (H2D copy of X, the quantizer and the fused layer, or the one-launch
    layer for decode batches, D2H copy of Y), all enqueued on one stream by one C call.
    The device buffers (X, codes, scales, Y), the pinned host output and the stream are
    checked once."""

    def __init__(self, b: int, m: int, n: int, device, stream=None, y_host: torch.Tensor | None = None):
        self._b, self._m, self._n = b, m, n
        self.x_dev = torch.empty((b, m), dtype=torch.bfloat16, device=device)
        self.xq = torch.empty((b, m), dtype=torch.int8, device=device)  # codes, one per byte
        self.sx = torch.empty((b, max(m // 128, 1)), dtype=torch.float32, device=device)
        self.y_dev = torch.empty((b, n), dtype=torch.bfloat16, device=device)
        if y_host is None:
            y_host = torch.empty((b, n), dtype=torch.bfloat16).pin_memory()
        if y_host.is_cuda or y_host.dtype != torch.bfloat16 or not y_host.is_contiguous() \
                or tuple(y_host.shape) != (b, n):
            raise TypeError("y_host must be a contiguous host torch.bfloat16 tensor of shape (b, n)")
        self.y_host = y_host
        self._ptrs = (self.x_dev.data_ptr(), self.xq.data_ptr(), self.sx.data_ptr(),
                      self.y_dev.data_ptr(), y_host.data_ptr())
        self._st = _stream(stream)
        self._fn = load().twq_linear_host

    def __call__(self, x_host: torch.Tensor, w: Weights) -> torch.Tensor:
        if x_host.is_cuda or x_host.dtype != torch.bfloat16 or not x_host.is_contiguous():
            raise TypeError("x_host must be a contiguous host torch.bfloat16 tensor")
        if tuple(x_host.shape) != (self._b, self._m) or w.m != self._m or w.n != self._n:
            raise ValueError("x_host and w must match the prepared shapes")
        xd, xq, sx, yd, yh = self._ptrs
        _check(self._fn(x_host.data_ptr(), self._b, ctypes.byref(w.c_struct()), xd, xq, sx, yd,
                        yh, self._st), "twq_linear_host")
        return self.y_host


def selftest_wait_timeout(xq, sx, w: Weights, y=None, wait_limit_ns: int = 100000, stream=None):
    """Run the prefill kernel with its X copies withheld and short bounded waits (see
    twq_selftest_wait_timeout); returns y (unspecified). Read device_status() after it."""
    return _layer_extra("twq_selftest_wait_timeout", xq, sx, w, y, stream, int(wait_limit_ns))


def _layer_extra(fn: str, xq, sx, w: Weights, y, stream, extra):
    b = xq.shape[0]
    if y is None:
        y = torch.empty((b, w.n), dtype=torch.bfloat16, device=xq.device)
    cw = w.c_struct()
    _check(getattr(load(), fn)(_dev(xq, "xq", torch.uint8), _dev(sx, "sx", torch.float32), b,
                               ctypes.byref(cw), _dev(y, "y", torch.bfloat16), extra,
                               _stream(stream)), fn)
    return y


def release_cache() -> None:
    """Drop the library's host-side caches (call after a cudaDeviceReset)."""
    load().twq_release_cache()


def fold_workspace_bytes(m: int, n: int, r: int) -> int:
    return int(load().twq_fold_workspace_bytes(m, n, r))


def fold_transforms(Q, G, U, V, R, workspace=None, stream=None):
    """Offline fold U' = Q^T U G, V' = G^-1 V, R' = Q^T R (BF16 outputs); synchronizes."""
    m, r = U.shape
    n = V.shape[1]
    dev = U.device
    out = (torch.empty((m, r), dtype=torch.bfloat16, device=dev),
           torch.empty((r, n), dtype=torch.bfloat16, device=dev),
           torch.empty((m, n), dtype=torch.bfloat16, device=dev))
    nbytes = fold_workspace_bytes(m, n, r)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(load().twq_fold_transforms(
        _dev(Q, "Q", torch.float32), _dev(G, "G", torch.float32), _dev(U, "U", torch.bfloat16),
        _dev(V, "V", torch.bfloat16), _dev(R, "R", torch.bfloat16), m, n, r,
        _dev(out[0], "L1_out", torch.bfloat16), _dev(out[1], "L2_out", torch.bfloat16),
        _dev(out[2], "R_out", torch.bfloat16), _dev(workspace, "workspace", torch.uint8),
        workspace.numel(), _stream(stream)), "twq_fold_transforms")
    return out


def w4a4_only(xq, sx, w: Weights, y=None, stream=None):
    return _layer("twq_w4a4_only", xq, sx, w, y, stream)


def lowrank_only(xq, sx, w: Weights, y=None, stream=None):
    return _layer("twq_lowrank_only", xq, sx, w, y, stream)


def unfused_workspace_bytes(b: int, n: int, r: int) -> int:
    return int(load().twq_unfused_workspace_bytes(b, n, r))


def unfused_linear(xq, sx, w: Weights, y=None, workspace=None, stream=None):
    b = xq.shape[0]
    if y is None:
        y = torch.empty((b, w.n), dtype=torch.bfloat16, device=xq.device)
    nbytes = unfused_workspace_bytes(b, w.n, w.r)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=xq.device)
    cw = w.c_struct()
    _check(load().twq_unfused_linear(_dev(xq, "xq", torch.uint8), _dev(sx, "sx", torch.float32), b,
                                     ctypes.byref(cw), _dev(y, "y", torch.bfloat16),
                                     _dev(workspace, "workspace", torch.uint8),
                                     workspace.numel(), _stream(stream)), "twq_unfused_linear")
    return y


def unfused_linear_noalloc(xq, sx, w: Weights, y=None, stream=None):
    """twq_unfused_linear with the library's own fixed scratch (no workspace argument);
    for callers that may not allocate device memory. Calls that overlap on the GPU race
    on the shared scratch."""
    return _layer("twq_unfused_linear_noalloc", xq, sx, w, y, stream)


def device_status() -> int:
    """Synchronizes; returns 0 or the site code of a kernel wait that ran out."""
    code = ctypes.c_int(0)
    st = load().twq_device_status(ctypes.byref(code))
    if st not in (OK, 6):
        raise TwqError(st, "twq_device_status")
    return code.value


def launches_per_call(entry_point: str) -> int:
    return int(load().twq_launches_per_call(entry_point.encode()))
