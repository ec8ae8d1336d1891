"""GPU parity of the INT4 stage 2 (TwinQuant §4.3: H requantized on chip to 4 bits,
multiplied by the 4-bit V = L2) against oracle.layer_s2q.

The packed L2 codes and scales must be bit-exact. Y is compared with the usual tolerance
plus an allowance for the one place floating point decides an integer differently on the
two sides: H is accumulated in fp32 per group on the GPU and in fp64 by the oracle, so
bf16(H) may differ in its last bit, and a value next to a rounding tie of Eq. (1) then
gets the neighbouring code. Each such flip moves Y[i, j] by s_H[i, g] * s_V[g, j] * |q_V|
<= s_H[i, g] * max|V[g, j]|; two flips per row and group are allowed, and the relative
Frobenius error must still meet the bound."""
import numpy as np
import pytest

import oracle
import synth
from helpers import FROB_TOL, ELEM_TOL, bf16_ulp, bits_of, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def twq(device):
    from rank_residual_w4a4_b200 import _build, twq as binding
    _build.build()
    binding.load()
    return binding


def _status_clean(twq):
    assert twq.device_status() == 0, "a kernel's bounded wait ran out"


def _operands(b, m, n, r, seed, wl="tiny"):
    w = synth.WORKLOADS[wl]
    x = synth.fill(b, m, *w.x_dist, seed, synth.ID_X)
    R, L1, L2 = synth.make_weights(w, seed=seed, m=m, n=n, r=r)
    return x, R, L1, L2


def _run(twq, device, x, R, L1, L2):
    w = twq.pack_weights(to_dev(R, device), to_dev(L1, device), to_dev(L2, device))
    l2q, sl2q = twq.pack_l2_int4(to_dev(L2, device))
    xq, sx = twq.quantize_act(to_dev(x, device))
    return bits_of(twq.fused_linear_s2q(xq, sx, w, l2q, sl2q)), l2q, sl2q


def _assert_s2q_close(y_bits, ref, L2, what):
    yd = synth.bf16_to_f32(y_bits).astype(np.float64)
    yr = synth.bf16_to_f32(ref["y"]).astype(np.float64)
    assert np.isfinite(yd).all(), what
    rms = np.sqrt(np.mean(yr ** 2))
    frob = np.linalg.norm(yd - yr) / max(np.linalg.norm(yr), 1e-300)
    assert frob <= FROB_TOL, "relative Frobenius error %.3g %s" % (frob, what)
    r = L2.shape[0]
    v = np.abs(synth.bf16_to_f32(L2).astype(np.float64)).reshape(r // 128, 128, -1).max(axis=1)
    flip = 2.0 * ref["sh"].astype(np.float64) @ v          # rows x n
    excess = np.abs(yd - yr) - (ELEM_TOL * rms + bf16_ulp(yr) + flip)
    assert excess.max() <= 0.0, "per-element bound exceeded by %.3g %s" % (excess.max(), what)


@pytest.mark.parametrize("r,n", [(128, 256), (256, 384)])
def test_pack_l2_int4_bitexact(twq, device, r, n):
    _, _, _, L2 = _operands(1, 128, n, r, seed=21)
    l2q, sl2q = twq.pack_l2_int4(to_dev(L2, device))
    qv, sv = oracle.quantize_cols(L2)
    assert np.array_equal(l2q.cpu().numpy(), oracle.pack_nibbles(qv))
    assert np.array_equal(sl2q.cpu().numpy().view(np.uint32), sv.view(np.uint32))


SHAPES = [  # b, m, n, r: one and two groups of r, ragged rows, a single token, several tiles
    (5, 256, 128, 128), (16, 512, 384, 128), (129, 384, 256, 256), (300, 128, 512, 128),
    (64, 640, 128, 256), (1, 128, 128, 128), (200, 1024, 256, 256),
]


@pytest.mark.parametrize("b,m,n,r", SHAPES)
def test_s2q_matches_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=22)
    y, _, _ = _run(twq, device, x, R, L1, L2)
    ref = oracle.layer_s2q(x, R, L1, L2, want=("y", "sh"))
    _assert_s2q_close(y, ref, L2, str((b, m, n, r)))
    _status_clean(twq)


@pytest.mark.parametrize("name", ["gateup", "down"])
def test_s2q_workload_sampled_rows(twq, device, name):
    wl = synth.WORKLOADS[name]
    x = synth.make_x(wl, seed=6)
    R, L1, L2 = synth.make_weights(wl, seed=6)
    y, _, _ = _run(twq, device, x, R, L1, L2)
    rows = synth.sample_rows(wl.b, 10, seed=17)
    ref = oracle.layer_s2q(x, R, L1, L2, rows=rows, want=("y", "sh"))
    _assert_s2q_close(y[rows], ref, L2, name)
    _status_clean(twq)


def test_s2q_differs_from_bf16_stage2_by_the_requantization_only(twq, device):
    """With L2 on an exact 4-bit grid (Q(V) = V), the two stage-2 forms differ only by
    the requantization of H: bounded by 1/2 code step of H times sum |V|."""
    b, m, n, r = 8, 256, 128, 128
    x, R, L1, _ = _operands(b, m, n, r, seed=23)
    rng = np.random.default_rng(4)
    steps = rng.integers(-7, 8, size=(r, n)).astype(np.float32)
    steps[0, :] = 7.0
    l2f = steps * np.float32(0.125)
    L2 = (l2f.view(np.uint32) >> 16).astype(np.uint16)
    y, _, _ = _run(twq, device, x, R, L1, L2)
    w = twq.pack_weights(to_dev(R, device), to_dev(L1, device), to_dev(L2, device))
    yb = bits_of(twq.fused_linear(*twq.quantize_act(to_dev(x, device)), w))
    ref = oracle.layer_s2q(x, R, L1, L2, want=("sh",))
    d = np.abs(synth.bf16_to_f32(y).astype(np.float64) - synth.bf16_to_f32(yb).astype(np.float64))
    bound = (0.5 * ref["sh"][:, :1].astype(np.float64) * np.abs(l2f).sum(axis=0)[None, :]
             + 2 * bf16_ulp(synth.bf16_to_f32(yb)) + 1e-6)
    assert (d <= bound).all()
    _status_clean(twq)


DECODE_SHAPES = [  # b <= 16, r = 128: the split-K decode kernel. Clusters of 4 (two 16-wide
    # units of r per CTA) and of 8 (one unit, K padded to 32), uneven group splits
    (1, 4096, 512, 128), (7, 4096, 256, 128), (16, 8192, 256, 128), (16, 1024, 384, 128),
    (5, 640, 128, 128),
]


@pytest.mark.parametrize("b,m,n,r", DECODE_SHAPES)
def test_s2q_decode_matches_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=24)
    y, _, _ = _run(twq, device, x, R, L1, L2)
    ref = oracle.layer_s2q(x, R, L1, L2, want=("y", "sh"))
    _assert_s2q_close(y, ref, L2, "decode %s" % ((b, m, n, r),))
    _status_clean(twq)


def test_s2q_decode_workload(twq, device):
    wl = synth.WORKLOADS["decode"]
    x = synth.make_x(wl, b=16, seed=7)
    R, L1, L2 = synth.make_weights(wl, seed=7)
    y, _, _ = _run(twq, device, x, R, L1, L2)
    _assert_s2q_close(y, oracle.layer_s2q(x, R, L1, L2, want=("y", "sh")), L2, "decode16")
    _status_clean(twq)
