"""twq_unfused_linear_noalloc: the unfused comparator for callers that may not allocate
device memory (it uses a fixed scratch array inside the library instead of a workspace).

Called through the C ABI and checked against the existing twq_unfused_linear (which
takes a caller-allocated workspace), within the tests' Y tolerance, on two calls in a
row with different shapes so the second call runs over the scratch the first one left.
This file is collected last so that a failure here stops a -x run only after every
other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from helpers import assert_y_close, bits_of, to_dev

pytestmark = pytest.mark.gpu

UNSUPPORTED = 2


@pytest.fixture(scope="module")
def lib(device):
    from rank_residual_w4a4_b200 import _build, twq
    _build.build()
    return twq.load()


def _case(device, b, m, n, r, seed):
    from rank_residual_w4a4_b200 import twq
    wl = synth.WORKLOADS["tiny"]
    x = synth.fill(b, m, wl.x_dist[0], wl.x_dist[1], wl.x_dist[2], seed, synth.ID_X)
    R, L1, L2 = synth.make_weights(wl, seed=seed, m=m, n=n, r=r)
    w = twq.pack_weights(to_dev(R, device), to_dev(L1, device), to_dev(L2, device))
    xq, sx = twq.quantize_act(to_dev(x, device))
    return w, xq, sx


def _call_noalloc(lib, w, xq, sx):
    y = torch.empty((xq.shape[0], w.n), dtype=torch.bfloat16, device=xq.device)
    cw = w.c_struct()
    st = lib.twq_unfused_linear_noalloc(xq.data_ptr(), sx.data_ptr(), xq.shape[0], ctypes.byref(cw),
                                        y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, "twq_unfused_linear_noalloc returned %d" % st
    return y


def test_noalloc_matches_workspace_version_twice(lib, device):
    """Same kernels and arithmetic as twq_unfused_linear, so the results are bitwise
    equal (which is within the tests' Y tolerance too)."""
    from rank_residual_w4a4_b200 import twq
    for shape, seed in (((200, 512, 384, 144), 21), ((33, 256, 256, 32), 22)):
        w, xq, sx = _case(device, *shape, seed=seed)
        y_ref = twq.unfused_linear(xq, sx, w)
        y = _call_noalloc(lib, w, xq, sx)
        torch.cuda.synchronize()
        assert np.array_equal(bits_of(y), bits_of(y_ref)), "noalloc %s" % (shape,)
        assert_y_close(bits_of(y), bits_of(y_ref), "noalloc %s" % (shape,))
    assert twq.device_status() == 0


def test_noalloc_without_low_rank_has_no_size_limit(lib, device):
    """r == 0: the comparator is the W4A4 kernel alone, which uses no scratch, so a batch
    whose fp32 intermediates would not fit in the fixed array still runs."""
    from rank_residual_w4a4_b200 import twq
    w, xq, sx = _case(device, 4096, 256, 1024, 0, seed=23)  # 4096 x 1024 x 8 B = 32 MiB
    y = _call_noalloc(lib, w, xq, sx)
    y_ref = twq.unfused_linear(xq, sx, w)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y), bits_of(y_ref))
    assert twq.device_status() == 0


def test_noalloc_after_release_cache(lib, device):
    """twq_release_cache() forgets the resolved scratch address; the next call resolves it
    again and gives the same result."""
    from rank_residual_w4a4_b200 import twq
    w, xq, sx = _case(device, 64, 256, 256, 32, seed=24)
    y0 = _call_noalloc(lib, w, xq, sx)
    lib.twq_release_cache()
    y1 = _call_noalloc(lib, w, xq, sx)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y0), bits_of(y1))
    assert twq.device_status() == 0


def test_noalloc_rejects_beyond_the_fixed_scratch(lib, device):
    from rank_residual_w4a4_b200 import twq
    # b x n fp32 twice plus b x r BF16 must fit in 16 MiB; 2048 x 1024 x 8 bytes does not.
    w = twq.Weights.empty(128, 1024, 16, device)
    cw = w.c_struct()
    b = 2048
    xq = torch.zeros((b, 64), dtype=torch.uint8, device=device)
    sx = torch.zeros((b, 1), dtype=torch.float32, device=device)
    y = torch.empty((b, 1024), dtype=torch.bfloat16, device=device)
    st = lib.twq_unfused_linear_noalloc(xq.data_ptr(), sx.data_ptr(), b, ctypes.byref(cw),
                                        y.data_ptr(), None)
    assert st == UNSUPPORTED
