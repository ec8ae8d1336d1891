"""The C ABI on the host: the library loads, exports what include/twq.h declares,
and rejects bad arguments with status codes before touching the GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from rank_residual_w4a4_b200 import _build, twq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "twq.h")


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return twq.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(twq_[a-z0-9_]+)\s*\(", text)))


def test_header_lists_the_five_entry_points():
    names = declared_functions()
    for ep in ("twq_quantize_act", "twq_pack_weights", "twq_fused_linear", "twq_lowrank_only",
               "twq_w4a4_only"):
        assert ep in names


def test_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", twq.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    declared = declared_functions()
    missing = [n for n in declared if n not in exported]
    assert not missing, missing
    assert set(declared) == set(twq.EXPORTS)
    # nothing else leaks out of the library except the declared C ABI
    leaked = [s for s in exported if s.startswith("twq") and s not in declared]
    assert not leaked, leaked


def test_version_and_strings(lib):
    assert lib.twq_version() >= 100
    assert lib.twq_status_string(0) == b"ok"
    assert lib.twq_status_string(3).startswith(b"misaligned")


def test_weight_sizes_closed_form(lib):
    # Observation 2 (TwinQuant §3) on a 4096 x 4096 projection: the low-rank part here is
    # 4-bit L1 (+ per-group fp32 scales) and BF16 L2.
    m = n = 4096
    for r in (0, 32, 128, 256):
        rq, sr, l1q, sl1, l2t = twq.weights_sizes(m, n, r)
        assert rq == n * m // 2 and sr == (m // 128) * n * 4
        assert l1q == r * m // 2 and sl1 == (m // 128) * r * 4 and l2t == n * r * 2
    assert twq.act_sizes(16, 4096) == (16 * 2048, 16 * 32 * 4)


@pytest.mark.parametrize("b,m,want", [(-1, 128, 1), (1, 100, 1), (1, 0, 1), (1, (1 << 24) + 128, 2),
                                      ((1 << 30) + 1, 128, 2)])
def test_act_sizes_rejects_bad_shapes(lib, b, m, want):
    arr = (ctypes.c_size_t * 2)()
    assert lib.twq_act_sizes(b, m, arr) == want


@pytest.mark.parametrize("m,n,r,want", [(100, 128, 16, 1), (128, 100, 16, 1), (128, 128, 8, 1),
                                        (128, 128, 272, 2), (0, 128, 0, 1), (128, 128, -16, 1)])
def test_weight_sizes_rejects_bad_shapes(lib, m, n, r, want):
    arr = (ctypes.c_size_t * 5)()
    assert lib.twq_weights_sizes(m, n, r, arr) == want


def _w(m=512, n=512, r=32, p=0x100000):
    return twq._Weights(m, n, r, p, p, p if r else None, p if r else None, p if r else None)


A = 0x100000  # 16-byte aligned fake device address (never dereferenced on these paths)


def test_quantize_act_validation(lib):
    q = lib.twq_quantize_act
    assert q(None, 4, 512, 512, A, A, None) == 1
    assert q(A, 4, 500, 512, A, A, None) == 1
    assert q(A, 4, 512, 256, A, A, None) == 1
    assert q(A + 2, 4, 512, 512, A, A, None) == 3
    assert q(A, 4, 512, 516, A, A, None) == 3
    assert q(A, -1, 512, 512, A, A, None) == 1
    assert q(None, 0, 512, 512, None, None, None) == 0  # b == 0: nothing to do


@pytest.mark.parametrize("fn", ["twq_fused_linear", "twq_w4a4_only", "twq_lowrank_only"])
def test_layer_validation(lib, fn):
    f = getattr(lib, fn)
    w = _w()
    assert f(None, A, 4, ctypes.byref(w), A, None) == 1
    assert f(A, A, 4, None, A, None) == 1
    assert f(A + 8, A, 4, ctypes.byref(w), A, None) == 3
    assert f(A, A, 4, ctypes.byref(w), A + 4, None) == 3
    bad = _w(m=500)
    assert f(A, A, 4, ctypes.byref(bad), A, None) == 1
    big = _w(r=272)
    assert f(A, A, 4, ctypes.byref(big), A, None) == 2
    assert f(A, A, 0, ctypes.byref(w), None, None) == 0
    misw = _w()
    misw.l2t = A + 2
    expect = 0 if fn == "twq_w4a4_only" else 3
    if expect:
        assert f(A, A, 4, ctypes.byref(misw), A, None) == 3


def test_fused_linear_x_validation(lib):
    f = lib.twq_fused_linear_x
    w = _w()
    assert f(None, 512, 4, ctypes.byref(w), A, None) == 1
    assert f(A, 512, 4, None, A, None) == 1
    assert f(A, 256, 4, ctypes.byref(w), A, None) == 1       # ldx < m
    assert f(A, 512, -1, ctypes.byref(w), A, None) == 1
    assert f(A + 2, 512, 4, ctypes.byref(w), A, None) == 3
    assert f(A, 516, 4, ctypes.byref(w), A, None) == 3       # row stride breaks 16 bytes
    assert f(A, 512, 4, ctypes.byref(w), A + 4, None) == 3
    assert f(A, 512, 0, ctypes.byref(w), None, None) == 0    # b == 0: nothing to do
    # outside the in-kernel quantizer's limits: rejected, nothing launched
    assert f(A, 512, 17, ctypes.byref(w), A, None) == 2      # b > 16
    assert f(A, 512, 4, ctypes.byref(_w(r=144)), A, None) == 2
    assert f(A, 8320, 4, ctypes.byref(_w(m=8320)), A, None) == 2  # m/128 > 64
    big = _w(r=272)
    assert f(A, 512, 4, ctypes.byref(big), A, None) == 2


def test_fused_linear_x_host_validation(lib):
    # every rejection happens before anything is enqueued, so these run without a GPU
    f = lib.twq_fused_linear_x_host
    w = _w()
    assert f(A, 4, None, A, A, A, None) == 1
    assert f(None, 4, ctypes.byref(w), A, A, A, None) == 1   # no host X
    assert f(A, 4, ctypes.byref(w), A, A, None, None) == 1   # no host Y
    assert f(A, 4, ctypes.byref(w), None, A, A, None) == 1   # no device X
    assert f(A, -1, ctypes.byref(w), A, A, A, None) == 1
    assert f(A, 4, ctypes.byref(w), A + 2, A, A, None) == 3
    assert f(A, 4, ctypes.byref(w), A, A + 4, A, None) == 3
    assert f(None, 0, ctypes.byref(w), None, None, None, None) == 0   # b == 0: nothing to do
    assert f(A, 17, ctypes.byref(w), A, A, A, None) == 2     # b > 16
    assert f(A, 4, ctypes.byref(_w(r=144)), A, A, A, None) == 2


def test_w4a8_validation(lib):
    # every rejection happens before anything is launched
    q = lib.twq_quantize_act_a8
    assert q(None, 4, 512, 512, A, A, None) == 1
    assert q(A, 4, 500, 512, A, A, None) == 1            # m % 128
    assert q(A, 4, 512, 256, A, A, None) == 1            # ldx < m
    assert q(A, 4, 512, 516, A, A, None) == 3            # row stride breaks 16 bytes
    assert q(A, 4, 512, 512, A + 8, A, None) == 3
    assert q(None, 0, 512, 512, None, None, None) == 0   # b == 0: nothing to do
    f = lib.twq_fused_linear_a8
    w = _w()
    assert f(None, A, 4, ctypes.byref(w), A, None) == 1
    assert f(A, A, 4, None, A, None) == 1
    assert f(A + 4, A, 4, ctypes.byref(w), A, None) == 3
    assert f(A, A, 0, ctypes.byref(w), None, None) == 0
    fx = lib.twq_fused_linear_x_a8
    assert fx(None, 512, 4, ctypes.byref(w), A, None) == 1
    assert fx(A, 256, 4, ctypes.byref(w), A, None) == 1
    assert fx(A, 516, 4, ctypes.byref(w), A, None) == 3
    assert fx(A, 512, 17, ctypes.byref(w), A, None) == 2
    assert fx(A, 512, 0, ctypes.byref(w), None, None) == 0


def test_s2q_validation(lib):
    # every rejection happens before anything is launched
    pk = lib.twq_pack_l2_int4
    assert pk(None, 128, 256, A, A, None) == 1
    assert pk(A, 96, 256, A, A, None) == 1      # r % 128
    assert pk(A, 128, 200, A, A, None) == 1     # n % 128
    assert pk(A, 384, 256, A, A, None) == 2     # r > 256
    assert pk(A + 2, 128, 256, A, A, None) == 3
    f = lib.twq_fused_linear_s2q
    w = _w(r=128)
    assert f(A, A, 4, None, A, A, A, None) == 1
    assert f(A, A, 4, ctypes.byref(_w(r=0)), A, A, A, None) == 1
    assert f(A, A, 4, ctypes.byref(_w(r=64)), A, A, A, None) == 2
    assert f(A, A, 4, ctypes.byref(w), None, A, A, None) == 1
    assert f(A, A, 4, ctypes.byref(w), A + 4, A, A, None) == 3
    assert f(A, A, 0, ctypes.byref(w), A, A, None, None) == 0


def test_fold_validation(lib):
    f = lib.twq_fold_transforms
    ws = lib.twq_fold_workspace_bytes(256, 128, 32)
    assert ws >= 2 * 32 * 32 * 8 + 32 * 32 * 4 + 256 * 32 * 4
    args = lambda **kw: [kw.get(k, d) for k, d in (
        ("Q", A), ("G", A), ("U", A), ("V", A), ("R", A), ("m", 256), ("n", 128), ("r", 32),
        ("L1", A), ("L2", A), ("Ro", A), ("ws", A), ("wsb", ws), ("st", None))]
    assert f(*args(Q=None)) == 1
    assert f(*args(m=0)) == 1
    assert f(*args(r=1025)) == 2
    assert f(*args(ws=A + 16)) == 3          # workspace must be 256-byte aligned
    assert f(*args(wsb=ws - 1)) == 1
    assert lib.twq_fold_workspace_bytes(0, 1, 1) == 0


def test_lowrank_needs_rank(lib):
    w = _w(r=0)
    assert lib.twq_lowrank_only(A, A, 4, ctypes.byref(w), A, None) == 1


def test_unfused_workspace(lib):
    assert lib.twq_unfused_workspace_bytes(16, 512, 32) >= 16 * 512 * 8 + 16 * 32 * 2
    w = _w()
    assert lib.twq_unfused_linear(A, A, 4, ctypes.byref(w), A, None, 1 << 20, None) == 1
    assert lib.twq_unfused_linear(A, A, 4, ctypes.byref(w), A, A, 16, None) == 1


def test_pack_validation(lib):
    w = _w()
    assert lib.twq_pack_weights(None, A, A, ctypes.byref(w), None) == 1
    assert lib.twq_pack_weights(A, None, A, ctypes.byref(w), None) == 1
    assert lib.twq_pack_weights(A + 2, A, A, ctypes.byref(w), None) == 3
    w0 = _w(r=0)
    # r == 0: L1 and L2 may be NULL (would launch, so only the rejection paths run here)
    assert lib.twq_pack_weights(None, None, None, ctypes.byref(w0), None) == 1


def test_launch_accounting(lib):
    assert twq.launches_per_call("twq_fused_linear") == 1
    assert twq.launches_per_call("twq_unfused_linear") == 4
    assert twq.launches_per_call("twq_unfused_linear_noalloc") == 4
    assert twq.launches_per_call("twq_fused_linear_x") == 1
    assert twq.launches_per_call("twq_fused_linear_x_host") == 1
    for ep in ("twq_quantize_act_a8", "twq_fused_linear_a8", "twq_fused_linear_x_a8",
               "twq_pack_l2_int4", "twq_fused_linear_s2q"):
        assert twq.launches_per_call(ep) == 1
    assert twq.launches_per_call("twq_fold_transforms") == 5
    assert twq.launches_per_call("nope") == -1


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(4, 512, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        twq.quantize_act(x, torch.zeros(4, 256, dtype=torch.uint8),
                         torch.zeros(4, 4, dtype=torch.float32))


def test_byte_code_entry_points_validation(lib):
    # the prefill form: the 4-bit codes one per byte; every rejection before any launch
    q = lib.twq_quantize_act_i8
    assert q(None, 40, 512, 512, A, A, None) == 1
    assert q(A, 40, 500, 512, A, A, None) == 1            # m % 128
    assert q(A, 40, 512, 256, A, A, None) == 1            # ldx < m
    assert q(A, 40, 512, 516, A, A, None) == 3            # row stride breaks 16 bytes
    assert q(A, 40, 512, 512, A + 8, A, None) == 3
    assert q(A, -1, 512, 512, A, A, None) == 1
    assert q(None, 0, 512, 512, None, None, None) == 0    # b == 0: nothing to do
    f = lib.twq_fused_linear_i8
    w = _w()
    assert f(None, A, 40, ctypes.byref(w), A, None) == 1
    assert f(A, A, 40, None, A, None) == 1
    assert f(A + 8, A, 40, ctypes.byref(w), A, None) == 3
    assert f(A, A, 40, ctypes.byref(w), A + 4, None) == 3
    assert f(A, A, 40, ctypes.byref(_w(m=500)), A, None) == 1
    assert f(A, A, 40, ctypes.byref(_w(r=272)), A, None) == 2
    assert f(A, A, 0, ctypes.byref(w), None, None) == 0


def test_linear_host_validation(lib):
    # (x_host, b, w, x_dev, xq, sx, y_dev, y_host, stream): rejections before any copy
    f = lib.twq_linear_host
    w = _w()
    assert f(A, 40, None, A, A, A, A, A, None) == 1          # no weights
    assert f(None, 40, ctypes.byref(w), A, A, A, A, A, None) == 1   # no host X
    assert f(A, 40, ctypes.byref(w), A, A, A, A, None, None) == 1   # no host Y
    assert f(A, 40, ctypes.byref(w), None, A, A, A, A, None) == 1   # no device X
    assert f(A, 40, ctypes.byref(w), A, A, A, None, A, None) == 1   # no device Y
    assert f(A, -1, ctypes.byref(w), A, A, A, A, A, None) == 1
    assert f(None, 0, ctypes.byref(w), None, None, None, None, None, None) == 0
    assert f(A, 40, ctypes.byref(w), A + 2, A, A, A, A, None) == 3  # misaligned device X
    # a prefill batch needs the code and scale buffers, aligned
    assert f(A, 40, ctypes.byref(w), A, None, A, A, A, None) == 1
    assert f(A, 40, ctypes.byref(w), A, A, None, A, A, None) == 1
    assert f(A, 40, ctypes.byref(w), A, A + 8, A, A, A, None) == 3
    assert f(A, 40, ctypes.byref(w), A, A, A, A + 4, A, None) == 3
    assert f(A, 40, ctypes.byref(_w(m=500)), A, A, A, A, A, None) == 1
    assert f(A, 40, ctypes.byref(_w(r=272)), A, A, A, A, A, None) == 2


def test_wait_selftest_validation(lib):
    f = lib.twq_selftest_wait_timeout
    w = _w(r=0)
    assert f(None, A, 300, ctypes.byref(w), A, 100000, None) == 1
    assert f(A + 8, A, 300, ctypes.byref(w), A, 100000, None) == 3
    assert f(A, A, 300, ctypes.byref(w), A, 999, None) == 1            # below 1 us
    assert f(A, A, 300, ctypes.byref(w), A, 2000000000, None) == 1     # above 1 s
    # shapes the prefill kernel does not take are refused, nothing launched
    assert f(A, A, 4, ctypes.byref(w), A, 100000, None) == 2           # b <= 16
    assert f(A, A, 300, ctypes.byref(_w(n=384, r=0)), A, 100000, None) == 2  # n % 256


def test_release_cache_is_host_only(lib):
    # no GPU here: the call only clears host-side tables
    lib.twq_release_cache()
    lib.twq_release_cache()
