"""twq_linear_host: one layer call from host memory to host memory for any batch (the call
a user with host activations makes). Its Y must be bitwise the device path's: the same
kernels on the same inputs, with the copies around them."""
import numpy as np
import pytest
import torch

import synth
from helpers import bits_of, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def twq(device):
    from rank_residual_w4a4_b200 import _build, twq as binding
    _build.build()
    binding.load()
    return binding


@pytest.mark.parametrize("b,m,n,r", [(200, 512, 384, 144), (4, 1024, 256, 128), (1, 256, 128, 0),
                                     (300, 256, 256, 256), (16, 512, 256, 256)])
def test_linear_host_matches_the_device_path(twq, device, b, m, n, r):
    wl = synth.WORKLOADS["tiny"]
    x = synth.fill(b, m, *wl.x_dist, 31, synth.ID_X)
    R, L1, L2 = synth.make_weights(wl, seed=31, m=m, n=n, r=r)
    w = twq.pack_weights(to_dev(R, device), to_dev(L1, device) if r else None,
                         to_dev(L2, device) if r else None)
    xq, sx = twq.quantize_act(to_dev(x, device))
    y_dev = bits_of(twq.fused_linear(xq, sx, w))
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    s = torch.cuda.Stream(device)
    step = twq.LinearHostStep(b, m, n, device, stream=s)
    for _ in range(2):  # twice: the second call reuses the buffers the first one left
        yh = step(xh, w)
        s.synchronize()
        assert np.array_equal(yh.view(torch.int16).numpy().view(np.uint16), y_dev)
    assert twq.device_status() == 0


def test_linear_host_rejects_bad_arguments(twq, device):
    import ctypes
    lib = twq.load()
    w = twq.Weights.empty(256, 128, 16, device)
    xh = torch.zeros((4, 256), dtype=torch.bfloat16)
    yh = torch.zeros((4, 128), dtype=torch.bfloat16)
    xd = torch.zeros((4, 256), dtype=torch.bfloat16, device=device)
    yd = torch.zeros((4, 128), dtype=torch.bfloat16, device=device)
    cw = w.c_struct()
    # a null host buffer: rejected before anything is enqueued
    assert lib.twq_linear_host(None, 4, ctypes.byref(cw), xd.data_ptr(), None, None, yd.data_ptr(),
                               yh.data_ptr(), None) == 1  # TWQ_ERR_INVALID_ARG
    assert lib.twq_linear_host(xh.data_ptr(), -1, ctypes.byref(cw), xd.data_ptr(), None, None,
                               yd.data_ptr(), yh.data_ptr(), None) == 1
