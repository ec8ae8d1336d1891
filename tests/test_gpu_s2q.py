"""GPU parity of the INT4 stage 2 (TwinQuant §4.3: H requantized on chip to 4 bits,
multiplied by the 4-bit V = L2) against oracle.layer_s2q.

The packed L2 codes and scales must be bit-exact. Y is compared with the usual tolerance
plus an allowance for the one place floating point decides an integer differently on the
two sides: H is accumulated in fp32 on the GPU and in fp64 by the oracle, so bf16(H) may
differ in its last bit where the exact H lies within the fp32 accumulation error of a
BF16 rounding boundary, and such an element may then get the neighbouring code of
Eq. (1). The allowance is computed element by element: only the H elements whose error
interval [H - e, H + e] straddles a BF16 rounding boundary (e bounds the fp32 error of
the GPU's sum of G scaled group products) may change their code by one, which moves
Y[i, j] by s_H[i, g] s_V[g, j] |q_V[j, k]|; if such an element can reach the group's
absmax, s_H itself may change and every code of that (row, group) may move by one. All
other elements get no allowance, and the relative Frobenius error must still meet the
bound."""
import numpy as np
import pytest

import oracle
import synth
from helpers import FROB_TOL, ELEM_TOL, bf16_ulp, bits_of, block_rows, to_dev

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


def _bf16_rne(f32):
    u = np.ascontiguousarray(f32, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _flip_allowance(x, L1, L2, rows=None):
    """Per element of Y (rows x n): the change that code flips of Q_H can cause, counting
    only the H elements whose bf16 rounding the fp32-vs-fp64 accumulation can decide."""
    xr = x if rows is None else x[rows]
    qx, sx = oracle.quantize_rows(xr)
    ql1, sl1 = oracle.quantize_cols(L1)
    b, m = qx.shape
    G, r = m // 128, ql1.shape[0]
    T = np.zeros((b, r))
    for g in range(G):
        k = slice(g * 128, (g + 1) * 128)
        ig = qx[:, k].astype(np.int64) @ ql1[:, k].astype(np.int64).T
        T += np.abs(sx[:, g:g + 1].astype(np.float64) * sl1[g][None, :].astype(np.float64) * ig)
    h = oracle.linear(qx, sx, None, None, ql1, sl1, L2, mode=oracle.LOWRANK_ONLY, want=("h64", "hb"))
    h64, hb = h["h64"], h["hb"]
    # fp32 error of the GPU's H: two roundings per group product, G accumulation steps,
    # up to G more for summing split-K partials (each bounded by T in magnitude), x 2
    eps = (2 * G + 4) * 2.0 ** -24 * T
    lo, hi = _bf16_rne((h64 - eps).astype(np.float32)), _bf16_rne((h64 + eps).astype(np.float32))
    flip = lo != hi
    hi_abs = np.maximum(np.abs(synth.bf16_to_f32(lo)), np.abs(synth.bf16_to_f32(hi)))
    qh, sh = oracle.quantize_rows(hb)
    qv, sv = oracle.quantize_cols(L2)  # qv: n x r codes, sv: r/128 x n
    allow = np.zeros((b, qv.shape[0]))
    for g2 in range(r // 128):
        k = slice(g2 * 128, (g2 + 1) * 128)
        amax = np.abs(synth.bf16_to_f32(hb[:, k])).max(axis=1)
        unstable = (flip[:, k] & (hi_abs[:, k] >= amax[:, None])).any(axis=1)
        wgt = flip[:, k].astype(np.float64)
        wgt[unstable] = 1.1  # s_H may change: every code of the group may move (and s_H by 2^-8)
        allow += (sh[:, g2:g2 + 1].astype(np.float64) * sv[g2][None, :].astype(np.float64)
                  * (wgt @ np.abs(qv[:, k]).astype(np.float64).T))
    return allow, int(flip.sum())


def _assert_s2q_close(y_bits, ref, x, L1, L2, what, rows=None):
    yd = synth.bf16_to_f32(y_bits).astype(np.float64)
    yr = synth.bf16_to_f32(ref["y"]).astype(np.float64)
    assert np.isfinite(yd).all(), what
    rms = np.sqrt(np.mean(yr ** 2))
    frob = np.linalg.norm(yd - yr) / max(np.linalg.norm(yr), 1e-300)
    assert frob <= FROB_TOL, "relative Frobenius error %.3g %s" % (frob, what)
    allow, _ = _flip_allowance(x, L1, L2, rows)
    excess = np.abs(yd - yr) - (ELEM_TOL * rms + bf16_ulp(yr) + allow)
    assert excess.max() <= 0.0, "per-element bound exceeded by %.3g %s" % (excess.max(), what)


def test_flip_allowance_is_tied_to_rounding_boundaries():
    """The allowance is not blanket: under 1% of the H elements lie close enough to a
    BF16 rounding boundary to flip, and the mean allowance is a small fraction of two code
    flips per row and group."""
    x, R, L1, L2 = _operands(64, 1024, 256, 256, seed=25)
    allow, flips = _flip_allowance(x, L1, L2)
    assert flips < 0.01 * 64 * 256
    # a blanket allowance of two code flips per row and group of r, for comparison
    ref = oracle.layer_s2q(x, R, L1, L2, want=("sh",))
    v = np.abs(synth.bf16_to_f32(L2).astype(np.float64)).reshape(2, 128, -1).max(axis=1)
    blanket = 2.0 * ref["sh"].astype(np.float64) @ v
    assert allow.mean() < 0.5 * blanket.mean()


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
    # the CTA-pair kernel (b > 16, m >= 256, n % 256 == 0): r = 128 with an odd number of K
    # groups, ragged rows over several row blocks and column tiles, r = 256 with G odd
    (40, 384, 512, 128), (513, 512, 768, 128), (300, 1152, 512, 256),
]


@pytest.mark.parametrize("b,m,n,r", SHAPES)
def test_s2q_matches_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=22)
    y, _, _ = _run(twq, device, x, R, L1, L2)
    ref = oracle.layer_s2q(x, R, L1, L2, want=("y", "sh"))
    _assert_s2q_close(y, ref, x, L1, L2, str((b, m, n, r)))
    _status_clean(twq)


@pytest.mark.parametrize("name", ["gateup", "down"])
def test_s2q_workload_sampled_rows(twq, device, name):
    wl = synth.WORKLOADS[name]
    x = synth.make_x(wl, seed=6)
    R, L1, L2 = synth.make_weights(wl, seed=6)
    y, _, _ = _run(twq, device, x, R, L1, L2)
    rows = block_rows(wl.b, per_block=1, seed=17)
    ref = oracle.layer_s2q(x, R, L1, L2, rows=rows, want=("y", "sh"))
    _assert_s2q_close(y[rows], ref, x, L1, L2, name, rows=rows)
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
    _assert_s2q_close(y, ref, x, L1, L2, "decode %s" % ((b, m, n, r),))
    _status_clean(twq)


def test_s2q_decode_workload(twq, device):
    wl = synth.WORKLOADS["decode"]
    x = synth.make_x(wl, b=16, seed=7)
    R, L1, L2 = synth.make_weights(wl, seed=7)
    y, _, _ = _run(twq, device, x, R, L1, L2)
    _assert_s2q_close(y, oracle.layer_s2q(x, R, L1, L2, want=("y", "sh")), x, L1, L2, "decode16")
    _status_clean(twq)
