"""GPU parity of the W4A8 path (TwinQuant §5.1: 4-bit weights, 8-bit activations;
Eq. (1) with q_max = 127 for the activations) against the CPU oracle.

Codes and scales of twq_quantize_act_a8 must be bit-exact. Y of twq_fused_linear_a8
must meet the tolerance in helpers.py against the oracle, and twq_fused_linear_x_a8
(quantizer inside the layer kernel) must equal the two-call path bitwise."""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_y_close, bits_of, to_dev
from test_gpu_parity import ADVERSARIAL, _absmax_lanes, _bf16_exact, every_absmax

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def twq(device):
    from rank_residual_w4a4_b200 import _build, twq as binding
    _build.build()
    binding.load()
    return binding


def _status_clean(twq):
    assert twq.device_status() == 0, "a kernel's bounded wait ran out"


def ties_a8():
    # absmax 127 in lane 0 of each group (s = 1), k + 0.5 for every k in [-127, 126]
    halves = np.arange(-127, 127, dtype=np.float32) + np.float32(0.5)
    g = np.concatenate([[127.0], halves[:127]]).astype(np.float32)
    g2 = np.concatenate([[-127.0], halves[127:]]).astype(np.float32)
    return np.tile(np.stack([g, g2]), (2, 3))


def tie_sweep_a8(rows, m):
    """Groups whose absmax a runs over the 128 BF16 mantissas of [1, 2), the rest over
    BF16 values of [a/256, a] of both signs: v / s meets every half-integer below 127."""
    groups = rows * m // 128
    out = np.empty((groups, 128), np.float32)
    mags_all = np.array([np.float32((1.0 + j / 128.0) * 2.0 ** e) for e in range(-8, 1)
                         for j in range(128)], np.float32)
    for gidx in range(groups):
        k, chunk = gidx % 128, gidx // 128
        a = np.float32(1.0 + k / 128.0)
        mags = mags_all[(mags_all <= a) & (mags_all >= a / 256)]
        cand = np.concatenate([mags, -mags])
        idx = (np.arange(127) + chunk * 127) % cand.size
        out[gidx, 0] = a if chunk % 2 == 0 else -a
        out[gidx, 1:] = cand[idx]
    return out.reshape(rows, m)


CASES = dict(ADVERSARIAL)
CASES.pop("tie_sweep")
CASES["ties_a8"] = ties_a8
CASES["tie_sweep_a8"] = lambda: tie_sweep_a8(72, 4096)
CASES["every_absmax"] = lambda: every_absmax(256, 16384)


def _check_codes(twq, device, x):
    xq8, sx = twq.quantize_act_a8(to_dev(x, device))
    rq, rs = oracle.quantize_rows(x, a8=True)
    assert np.array_equal(xq8.cpu().numpy(), rq)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("case", list(CASES) + ["absmax_lanes"])
def test_quantize_act_a8_adversarial(twq, device, case):
    f = _absmax_lanes() if case == "absmax_lanes" else CASES[case]()
    _check_codes(twq, device, _bf16_exact(f))


@pytest.mark.parametrize("name,b", [("tiny", 16), ("decode", 1), ("decode", 16), ("tiny", 129),
                                    ("gateup", 2048)])
def test_quantize_act_a8_bitexact(twq, device, name, b):
    _check_codes(twq, device, synth.make_x(synth.WORKLOADS[name], b=b))


SHAPES = [  # b, m, n, r: clusters of 4 and 8, ragged splits, r = 0, a CTA with no groups
    (16, 4096, 512, 128), (7, 4096, 256, 128), (16, 8192, 256, 128), (5, 1024, 384, 48),
    (16, 128, 128, 16), (2, 640, 128, 32), (16, 4096, 128, 0), (1, 2048, 256, 64),
]


def _operands(b, m, n, r, seed):
    w = synth.WORKLOADS["tiny"]
    x = synth.fill(b, m, w.x_dist[0], w.x_dist[1], w.x_dist[2], seed, synth.ID_X)
    R, L1, L2 = synth.make_weights(w, seed=seed, m=m, n=n, r=r)
    return x, R, (L1 if r else None), (L2 if r else None)


def _pack(twq, dev, R, L1, L2):
    r = 0 if L1 is None else L1.shape[1]
    return twq.pack_weights(to_dev(R, dev), to_dev(L1, dev) if r else None,
                            to_dev(L2, dev) if r else None)


@pytest.mark.parametrize("b,m,n,r", SHAPES)
def test_w4a8_layer_matches_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=41)
    w = _pack(twq, device, R, L1, L2)
    xd = to_dev(x, device)
    y2 = bits_of(twq.fused_linear_a8(*twq.quantize_act_a8(xd), w))
    ref = oracle.layer(x, R, L1, L2, mode=oracle.FUSED if r else oracle.W4A4_ONLY, a8=True)["y"]
    assert_y_close(y2, ref, "W4A8 %s" % ((b, m, n, r),))
    y1 = bits_of(twq.fused_linear_x(xd, w, a8=True))
    assert np.array_equal(y1, y2), "fused_x_a8 != quantize_a8 + fused_a8 %s" % ((b, m, n, r),)
    _status_clean(twq)


def test_w4a8_decode_workload(twq, device):
    wl = synth.WORKLOADS["decode"]
    x = synth.make_x(wl, b=16, seed=3)
    R, L1, L2 = synth.make_weights(wl, seed=3)
    w = _pack(twq, device, R, L1, L2)
    y = bits_of(twq.fused_linear_x(to_dev(x, device), w, a8=True))
    assert_y_close(y, oracle.layer(x, R, L1, L2, a8=True)["y"], "W4A8 decode16")
    # 8-bit activations are closer to the unquantized-activation product than 4-bit ones
    y4 = bits_of(twq.fused_linear_x(to_dev(x, device), w))
    xf = synth.bf16_to_f32(x).astype(np.float64)
    qr, sr = oracle.quantize_cols(R)
    ql1, sl1 = oracle.quantize_cols(L1)
    G = R.shape[0] // 128
    Wr = (qr.reshape(-1, G, 128) * sr.T[:, :, None]).reshape(qr.shape).T.astype(np.float64)
    Wl = (ql1.reshape(-1, G, 128) * sl1.T[:, :, None]).reshape(ql1.shape).T.astype(np.float64)
    exact = xf @ Wr + (xf @ Wl) @ synth.bf16_to_f32(L2).astype(np.float64)
    e8 = np.abs(synth.bf16_to_f32(y).astype(np.float64) - exact).mean()
    e4 = np.abs(synth.bf16_to_f32(y4).astype(np.float64) - exact).mean()
    assert e8 < e4 / 4
    _status_clean(twq)


PREFILL_SHAPES = [  # b > 16: the tensor-core GEMM kernel; ragged rows, two H chunks, r = 0,
    # and CTA pairs (128 < r <= 256, even column-tile count)
    (17, 384, 256, 64), (129, 512, 384, 128), (200, 256, 256, 144), (64, 640, 128, 0),
    (300, 256, 1024, 256), (257, 384, 768, 160), (33, 1024, 512, 32),
]


@pytest.mark.parametrize("b,m,n,r", PREFILL_SHAPES)
def test_w4a8_prefill_matches_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=43)
    w = _pack(twq, device, R, L1, L2)
    y = bits_of(twq.fused_linear_a8(*twq.quantize_act_a8(to_dev(x, device)), w))
    ref = oracle.layer(x, R, L1, L2, mode=oracle.FUSED if r else oracle.W4A4_ONLY, a8=True)["y"]
    assert_y_close(y, ref, "W4A8 prefill %s" % ((b, m, n, r),))
    _status_clean(twq)


@pytest.mark.parametrize("name", ["gateup", "down"])
def test_w4a8_prefill_workload_sampled_rows(twq, device, name):
    wl = synth.WORKLOADS[name]
    x = synth.make_x(wl, seed=5)
    R, L1, L2 = synth.make_weights(wl, seed=5)
    w = _pack(twq, device, R, L1, L2)
    y = bits_of(twq.fused_linear_a8(*twq.quantize_act_a8(to_dev(x, device)), w))
    rows = synth.sample_rows(wl.b, 12, seed=13)
    ref = oracle.layer(x, R, L1, L2, rows=rows, a8=True)["y"]
    assert_y_close(y[rows], ref, "W4A8 %s rows" % name)
    _status_clean(twq)
