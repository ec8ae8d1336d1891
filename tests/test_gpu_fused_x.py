"""GPU parity of twq_fused_linear_x: the decode layer kernel that quantizes X
itself (TwinQuant §4.3: the activation is quantized once, on chip, for both
GEMMs that read it).

Its arithmetic is the standalone quantizer's, so its Y must be bitwise equal to
twq_quantize_act followed by twq_fused_linear on every input, and within the
oracle tolerance of the CPU oracle."""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_y_close, bits_of, to_dev
from test_gpu_parity import every_absmax, tie_sweep

pytestmark = pytest.mark.gpu

SHAPES = [  # b, m, n, r: clusters of 4 and of 8, ragged splits, a CTA with no groups, r = 0
    (1, 4096, 512, 128), (7, 4096, 256, 128), (16, 8192, 256, 128), (16, 5120, 256, 64),
    (5, 1024, 384, 48), (16, 128, 128, 16), (2, 640, 128, 32), (16, 4096, 128, 0),
    (3, 2048, 256, 0),
]


@pytest.fixture(scope="module")
def twq(device):
    from rank_residual_w4a4_b200 import _build, twq as binding
    _build.build()
    binding.load()
    return binding


def _operands(b, m, n, r, seed):
    w = synth.WORKLOADS["tiny"]
    x = synth.fill(b, m, w.x_dist[0], w.x_dist[1], w.x_dist[2], seed, synth.ID_X)
    R, L1, L2 = synth.make_weights(w, seed=seed, m=m, n=n, r=r)
    return x, R, (L1 if r else None), (L2 if r else None)


def _pack(twq, dev, R, L1, L2):
    r = 0 if L1 is None else L1.shape[1]
    return twq.pack_weights(to_dev(R, dev), to_dev(L1, dev) if r else None,
                            to_dev(L2, dev) if r else None)


def _two_call(twq, xd, w):
    return bits_of(twq.fused_linear(*twq.quantize_act(xd), w))


def _status_clean(twq):
    assert twq.device_status() == 0, "a kernel's bounded wait ran out"


@pytest.mark.parametrize("b,m,n,r", SHAPES)
def test_fused_x_matches_two_call_path_and_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=21)
    w = _pack(twq, device, R, L1, L2)
    xd = to_dev(x, device)
    y = bits_of(twq.fused_linear_x(xd, w))
    assert np.array_equal(y, _two_call(twq, xd, w)), "fused_x != quantize + fused %s" % ((b, m, n, r),)
    mode = oracle.FUSED if r else oracle.W4A4_ONLY
    ref = oracle.layer(x, R, L1, L2, mode=mode)["y"]
    assert_y_close(y, ref, "fused_x %s" % ((b, m, n, r),))
    _status_clean(twq)


def test_fused_x_strided_rows(twq, device):
    import torch
    b, m, n, r = 9, 1024, 256, 32
    x, R, L1, L2 = _operands(b, m, n, r, seed=22)
    w = _pack(twq, device, R, L1, L2)
    wide = torch.zeros((b, m + 136), dtype=torch.bfloat16, device=device)
    wide.fill_(float("nan"))  # columns outside the view must never be read
    wide[:, 64:64 + m] = to_dev(x, device)
    view = wide[:, 64:64 + m]
    assert view.stride(0) == m + 136
    y = bits_of(twq.fused_linear_x(view, w))
    assert np.array_equal(y, _two_call(twq, to_dev(x, device), w))
    _status_clean(twq)


def _adversarial_x(case, b, m):
    rng = np.random.default_rng(31)
    if case == "ties":  # absmax 7 then x.5 values: every code is a rounding tie
        g = np.concatenate([[7.0], np.tile(np.arange(-7, 7) + 0.5, 10)[:127]]).astype(np.float32)
        f = np.tile(g, (b, m // 128))
    elif case == "zero_groups":  # alternate groups all zero
        f = rng.uniform(-2, 2, (b, m)).astype(np.float32)
        f.reshape(b, m // 128, 128)[:, ::2] = 0.0
    elif case == "subnormal":
        f = np.tile((np.arange(128) + 1) * np.float32(2.0 ** -133), (b, m // 128))
    elif case == "absmax_lanes":  # +-absmax at every one of the 128 positions
        f = rng.uniform(-1, 1, (b, m)).astype(np.float32).reshape(b, m // 128, 128)
        for t in range(b):
            for g in range(m // 128):
                pos = (t * 7 + g * 13) % 128
                f[t, g, pos] = (3.0 if (t + g) % 2 else -3.0)
        f = f.reshape(b, m)
    elif case.startswith("tie_sweep"):  # every near-tie quotient (see tie_sweep)
        part = int(case[-1])
        f = tie_sweep(72, m)[16 * part:16 * part + b]
    elif case == "huge":  # scales above 2^125: the exact-division path
        f = np.tile(np.linspace(-1.5, 1.5, m, dtype=np.float32) * np.float32(2.0 ** 126), (b, 1))
    else:  # outliers: a few channels 50x larger, as in the activation recipe
        f = rng.standard_normal((b, m)).astype(np.float32)
        f[:, synth.outlier_channels(m, 0.01, seed=3)] *= 50.0
    return synth.f32_to_bf16(f.astype(np.float32))


@pytest.mark.parametrize("case", ["ties", "zero_groups", "subnormal", "absmax_lanes", "outliers",
                                  "huge", "tie_sweep0", "tie_sweep1", "tie_sweep2", "tie_sweep3"])
def test_fused_x_adversarial_inputs(twq, device, case):
    b, m, n, r = 16, 2048, 256, 64
    _, R, L1, L2 = _operands(b, m, n, r, seed=23)
    w = _pack(twq, device, R, L1, L2)
    x = _adversarial_x(case, b, m)
    xd = to_dev(x, device)
    y = bits_of(twq.fused_linear_x(xd, w))
    assert np.array_equal(y, _two_call(twq, xd, w)), case
    _status_clean(twq)


def test_fused_x_every_absmax(twq, device):
    # every BF16 absmax through the in-kernel quantizer: 16 tokens x 64 groups per call
    b, m, n, r = 16, 8192, 128, 16
    _, R, L1, L2 = _operands(b, m, n, r, seed=26)
    w = _pack(twq, device, R, L1, L2)
    allx = synth.f32_to_bf16(every_absmax(16 * 32, m))
    for c in range(32):
        xd = to_dev(allx[16 * c:16 * c + 16], device)
        y = bits_of(twq.fused_linear_x(xd, w))
        assert np.array_equal(y, _two_call(twq, xd, w)), "chunk %d" % c
    _status_clean(twq)


def test_fused_x_zero_input_and_empty_batch(twq, device):
    import torch
    b, m, n, r = 4, 512, 128, 16
    _, R, L1, L2 = _operands(b, m, n, r, seed=24)
    w = _pack(twq, device, R, L1, L2)
    y = bits_of(twq.fused_linear_x(torch.zeros((b, m), dtype=torch.bfloat16, device=device), w))
    assert not (synth.bf16_to_f32(y) != 0).any()
    assert twq.fused_linear_x(torch.empty((0, m), dtype=torch.bfloat16, device=device), w).shape == (0, n)
    _status_clean(twq)


def test_fused_x_rejects_prefill_batches(twq, device):
    import torch
    b, m, n, r = 17, 512, 128, 16
    _, R, L1, L2 = _operands(b, m, n, r, seed=25)
    w = _pack(twq, device, R, L1, L2)
    with pytest.raises(twq.TwqError) as e:
        twq.fused_linear_x(torch.zeros((b, m), dtype=torch.bfloat16, device=device), w)
    assert e.value.status == 2


@pytest.mark.parametrize("b", [1, 4, 16])
def test_fused_x_decode_workload(twq, device, b):
    wl = synth.WORKLOADS["decode"]
    x = synth.make_x(wl, b=b)
    R, L1, L2 = synth.make_weights(wl)
    w = _pack(twq, device, R, L1, L2)
    xd = to_dev(x, device)
    y = bits_of(twq.fused_linear_x(xd, w))
    assert np.array_equal(y, _two_call(twq, xd, w))
    assert_y_close(y, oracle.layer(x, R, L1, L2, mode=oracle.FUSED)["y"], "decode b=%d" % b)
    _status_clean(twq)


@pytest.mark.parametrize("b,m,n,r", [(16, 4096, 512, 128), (3, 1024, 384, 48), (1, 2048, 256, 0)])
def test_host_step_matches_device_call(twq, device, b, m, n, r):
    """twq_fused_linear_x_host: host X in, host Y out, on two streams with their own
    buffers; Y bitwise equal to twq_fused_linear_x on the device copy of X."""
    import torch
    x, R, L1, L2 = _operands(b, m, n, r, seed=31)
    w = _pack(twq, device, R, L1, L2)
    ref = bits_of(twq.fused_linear_x(to_dev(x, device), w))
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    streams = [torch.cuda.Stream(device), torch.cuda.Stream(device)]
    bufs = [(torch.empty((b, m), dtype=torch.bfloat16, device=device),
             torch.empty((b, n), dtype=torch.bfloat16, device=device),
             torch.empty((b, n), dtype=torch.bfloat16).pin_memory()) for _ in streams]
    for i in range(6):
        xd, yd, yh = bufs[i % 2]
        yh.fill_(0)
        twq.fused_linear_x_host(xh, w, xd, yd, yh, stream=streams[i % 2])
    torch.cuda.synchronize()
    for _, _, yh in bufs:
        assert np.array_equal(yh.view(torch.int16).numpy().view(np.uint16), ref)
    _status_clean(twq)


def test_prepared_decode_step(twq, device):
    """twq.DecodeStep: the prepared form of the host call gives the same Y."""
    import torch
    b, m, n, r = 8, 2048, 384, 64
    x, R, L1, L2 = _operands(b, m, n, r, seed=33)
    w = _pack(twq, device, R, L1, L2)
    ref = bits_of(twq.fused_linear_x(to_dev(x, device), w))
    step = twq.DecodeStep(torch.empty((b, m), dtype=torch.bfloat16, device=device),
                          torch.empty((b, n), dtype=torch.bfloat16, device=device),
                          torch.zeros((b, n), dtype=torch.bfloat16).pin_memory())
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = step(xh, w)
    torch.cuda.synchronize()
    assert np.array_equal(yh.view(torch.int16).numpy().view(np.uint16), ref)
    with pytest.raises(ValueError):
        step(xh[: b - 1].contiguous(), w)
    _status_clean(twq)
