"""Pins of the CPU oracle against what TwinQuant's equations and plain mathematics fix.

Nothing here compares the oracle with itself: each check is a hand-worked value
of Eq. (1), an exhaustive property of Eq. (1) over all BF16 magnitudes, an
invariant of the layer, a library routine (numpy / torch) on a step that
reduces to one, or brute force (dequantize first, then multiply in fp64).
"""
import os
import struct

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "eq1_groups.txt")


def _f32_bits(x):
    return struct.unpack("<I", struct.pack("<f", float(x)))[0]


def _bf16_bits_of(values):
    """Exact BF16 bit patterns of values that BF16 holds exactly (checked)."""
    f = np.asarray(values, dtype=np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(synth.bf16_to_f32(bits), f), "value not exact in BF16"
    return bits


def _golden_cases():
    cases = []
    with open(GOLDEN) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, vals, codes, scale = [p.strip() for p in line.split("|")]
            cases.append((name, [float(v) for v in vals.split()], [int(c) for c in codes.split()],
                          int(scale, 16)))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c[0])
def test_eq1_hand_worked(case):
    name, vals, codes, scale_bits = case
    group = np.zeros(128, np.float32)
    group[:len(vals)] = vals
    # through the float entry point
    q, s = oracle.quant_group_f32(group)
    assert _f32_bits(s) == scale_bits
    assert q[:len(codes)].tolist() == codes
    assert not q[len(codes):].any()
    # and through the BF16 activation path (row-major, one token)
    x = _bf16_bits_of(group)[None, :]
    qx, sx = oracle.quantize_rows(x)
    assert _f32_bits(sx[0, 0]) == scale_bits
    assert qx[0, :len(codes)].tolist() == codes
    # and through the weight path (a column)
    qw, sw = oracle.quantize_cols(x.T.copy())
    assert _f32_bits(sw[0, 0]) == scale_bits
    assert qw[0, :len(codes)].tolist() == codes


def test_qmax_is_seven():
    # Eq. (1): q_max = 2^(k-1) - 1 with k = 4
    assert oracle.qmax() == 7


def test_all_equal_group_maps_to_pm7():
    for v in (-3.25, 0.015625, 1e-20):
        g = np.full(128, v, np.float32)
        q, s = oracle.quant_group_f32(g)
        assert (q == (7 if v > 0 else -7)).all()


def test_clamp_matters_only_below_bf16_range():
    # a = 10 * 2^-149 (a float32 subnormal): s = fl(a/7) = 2^-149, a/s = 10 -> clamped to 7.
    a = np.float32(10 * 2.0 ** -149)
    g = np.zeros(128, np.float32)
    g[0] = a
    q, s = oracle.quant_group_f32(g)
    assert s == np.float32(2.0 ** -149)
    assert q[0] == 7


def test_exhaustive_bf16_absmax_maps_to_7():
    """For every positive finite BF16 a: s = fl(a/7) != 0 and a/s rounds to exactly 7,
    so the group's absmax always gets code +-7 (never clamped, never 6)."""
    bits = np.arange(1, 0x7F80, dtype=np.uint16)  # all positive finite BF16 values
    n = bits.size
    x = np.zeros((2 * n, 128), np.uint16)
    x[:n, 0] = bits
    x[n:, 5] = bits | 0x8000  # negative absmax at another lane
    q, s = oracle.quantize_rows(x)
    assert (s[:, 0] > 0).all()
    assert (q[:n, 0] == 7).all()
    assert (q[n:, 5] == -7).all()
    assert (q[:n, 1:] == 0).all() and (q[n:, :5] == 0).all()


def test_code_range_and_absmax_positions():
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_x(wl)
    q, s = oracle.quantize_rows(x)
    assert q.min() >= -7 and q.max() <= 7
    xf = synth.bf16_to_f32(x).reshape(x.shape[0], -1, 128)
    qg = q.reshape(x.shape[0], -1, 128)
    a = np.abs(xf).max(axis=2, keepdims=True)
    at_max = np.abs(xf) == a
    assert (np.abs(qg[at_max]) == 7).all()
    assert (np.sign(qg[at_max]) == np.sign(xf[at_max])).all()
    # the scale is the float32 quotient a / 7
    assert np.array_equal(s, (a[..., 0] / np.float32(7)).astype(np.float32))


def test_group_axis_weights():
    """Weights are grouped along m (the reduction axis), one scale per column and group."""
    m, cols = 384, 5
    k = np.arange(m)
    w = np.zeros((m, cols), np.float32)
    for j in range(cols):
        w[:, j] = ((k % 128) - 63) * 2.0 ** (j + k // 128)
    q, s = oracle.quantize_cols(_bf16_bits_of(w))
    for g in range(3):
        for j in range(cols):
            assert s[g, j] == np.float32(np.float32(64 * 2.0 ** (j + g)) / np.float32(7))
    assert q.shape == (cols, m)
    assert (q[:, 127] == 7).all() and (q[:, 0] == -7).all()


def test_sign_and_power_of_two_equivariance_of_codes():
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_x(wl)
    q, s = oracle.quantize_rows(x)
    qn, sn = oracle.quantize_rows(x ^ np.uint16(0x8000))
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    x4 = _bf16_bits_of(synth.bf16_to_f32(x) * np.float32(4.0))
    q4, s4 = oracle.quantize_rows(x4)
    assert np.array_equal(q4, q) and np.array_equal(s4, s * np.float32(4.0))


def test_nibble_packing():
    assert oracle.pack_nibbles(np.array([-7, 7, -1, 0], np.int8)).tolist() == [0x79, 0x0F]
    codes = np.array([(a, b) for a in range(-7, 8) for b in range(-7, 8)], np.int8).reshape(-1)
    assert np.array_equal(oracle.unpack_nibbles(oracle.pack_nibbles(codes)), codes)
    # explicit byte layout: low nibble = even index
    p = oracle.pack_nibbles(codes)
    lo = (p & 0xF).astype(np.int16)
    lo[lo >= 8] -= 16
    assert np.array_equal(lo, codes[0::2])


def test_bf16_rounding_against_torch():
    torch = pytest.importorskip("torch")
    vals = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 3.0e38, 1e-40, -0.0,
                     65504.0, 1.00390625, 2.0 ** -133], np.float32)
    rnd = np.random.default_rng(0).standard_normal(4096).astype(np.float32) * 1e3
    vals = np.concatenate([vals, rnd])
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want)


def _tiny_operands(b, m, n, r, seed):
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_x(wl, b=b, seed=seed) if m == wl.m else synth.fill(b, m, 0, 0.0, 1.0, seed, 0)
    R, L1, L2 = synth.make_weights(wl, seed=seed, m=m, n=n, r=r)
    qx, sx = oracle.quantize_rows(x)
    qr, sr = oracle.quantize_cols(R)
    if r:
        ql1, sl1 = oracle.quantize_cols(L1)
    else:
        ql1 = sl1 = L2 = None
    return qx, sx, qr, sr, ql1, sl1, L2


@pytest.mark.parametrize("b,m,n,r", [(1, 128, 8, 0), (3, 256, 17, 1), (4, 128, 64, 16),
                                     (2, 256, 33, 16), (4, 256, 64, 1)])
@pytest.mark.parametrize("mode", [oracle.FUSED, oracle.W4A4_ONLY, oracle.LOWRANK_ONLY])
def test_brute_force_dequantize_then_matmul(b, m, n, r, mode):
    """Eq. (2) per group equals dequantize-first (s*q, Eq. (1)) then an ungrouped fp64 matmul."""
    ops = _tiny_operands(b, m, n, r, seed=3)
    y = oracle.linear(*ops, mode=mode, want=("y64",))["y64"]
    ref = oracle.dequant_matmul(*ops, mode=mode)
    scale = max(np.abs(ref).max(), 1e-30)
    assert np.abs(y - ref).max() <= 1e-12 * scale


@pytest.mark.parametrize("b,m,n,r", [(3, 256, 17, 1), (4, 128, 64, 16), (2, 384, 40, 32)])
@pytest.mark.parametrize("mode", [oracle.FUSED, oracle.W4A4_ONLY, oracle.LOWRANK_ONLY])
def test_brute_force_in_numpy(b, m, n, r, mode):
    """Outside the oracle's C code: dequantize with numpy (s*q per group, Eq. (1)), one
    ungrouped fp64 matmul per GEMM, and bf16(float32(H)) for stage 2. The oracle's H bits
    may differ from numpy's only where the two fp64 sums straddle a float32 rounding
    boundary; Y is then compared on the oracle's own BF16 H."""
    qx, sx, qr, sr, ql1, sl1, L2 = _tiny_operands(b, m, n, r, seed=31)
    out = oracle.linear(qx, sx, qr, sr, ql1, sl1, L2, mode=mode, want=("y64", "hb"))
    xd = qx.astype(np.float64) * np.repeat(sx.astype(np.float64), 128, axis=1)    # b x m
    rd = np.repeat(sr.astype(np.float64), 128, axis=0) * qr.T.astype(np.float64)   # m x n
    l1d = np.repeat(sl1.astype(np.float64), 128, axis=0) * ql1.T.astype(np.float64)  # m x r
    h = xd @ l1d
    hb_np = synth.f32_to_bf16(h.astype(np.float32))
    mism = np.flatnonzero(out["hb"] != hb_np) if mode != oracle.W4A4_ONLY else np.array([])
    assert mism.size <= max(1, h.size // 500)
    hb = synth.bf16_to_f32(out["hb"]).astype(np.float64) if mode != oracle.W4A4_ONLY else 0.0
    yres = xd @ rd
    ylr = hb @ synth.bf16_to_f32(L2).astype(np.float64) if mode != oracle.W4A4_ONLY else 0.0
    ref = {oracle.FUSED: yres + ylr, oracle.W4A4_ONLY: yres, oracle.LOWRANK_ONLY: ylr}[mode]
    assert np.abs(out["y64"] - ref).max() <= 1e-12 * max(np.abs(ref).max(), 1e-30)


def test_stage2_is_a_plain_matmul_of_bf16_h():
    """Y_lr = bf16(H) @ L2: checked with numpy's matmul on the oracle's own H bits, and
    H itself against the fp64 dequantized product (a second, ungrouped route)."""
    b, m, n, r = 5, 256, 48, 16
    qx, sx, qr, sr, ql1, sl1, L2 = _tiny_operands(b, m, n, r, seed=5)
    out = oracle.linear(qx, sx, qr, sr, ql1, sl1, L2, mode=oracle.LOWRANK_ONLY,
                        want=("y64", "h64", "hb"))
    xd = sx.repeat(128, axis=1).astype(np.float64) * qx
    l1d = (sl1.repeat(128, axis=0).astype(np.float64) * ql1.T)  # m x r
    h = xd @ l1d
    assert np.abs(out["h64"] - h).max() <= 1e-12 * np.abs(h).max()
    hb = synth.bf16_to_f32(out["hb"]).astype(np.float64)
    ylr = hb @ synth.bf16_to_f32(L2).astype(np.float64)
    assert np.abs(out["y64"] - ylr).max() <= 1e-12 * np.abs(ylr).max()


def test_final_rounding_is_bf16_of_float_sum():
    ops = _tiny_operands(4, 256, 40, 16, seed=9)
    out = oracle.linear(*ops, want=("y", "y64"))
    f = out["y64"].astype(np.float32)
    assert np.array_equal(out["y"], synth.f32_to_bf16(f))


def test_identities_r0_and_R0():
    b, m, n, r = 4, 256, 32, 16
    qx, sx, qr, sr, ql1, sl1, L2 = _tiny_operands(b, m, n, r, seed=11)
    y_w4 = oracle.linear(qx, sx, qr, sr, None, None, None, mode=oracle.W4A4_ONLY)["y"]
    y_r0 = oracle.linear(qx, sx, qr, sr, None, None, None, mode=oracle.FUSED)["y"]
    assert np.array_equal(y_w4, y_r0)
    zq = np.zeros_like(qr)
    zs = np.zeros_like(sr)
    y_R0 = oracle.linear(qx, sx, zq, zs, ql1, sl1, L2, mode=oracle.FUSED)["y"]
    y_lr = oracle.linear(qx, sx, qr, sr, ql1, sl1, L2, mode=oracle.LOWRANK_ONLY)["y"]
    assert np.array_equal(y_R0, y_lr)


def test_sign_scaling_and_in_group_permutation_of_y():
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_x(wl, b=6)
    R, L1, L2 = synth.make_weights(wl, n=64)
    y = oracle.layer(x, R, L1, L2)["y"]
    # Y(-X) = -Y(X), bitwise
    yn = oracle.layer(x ^ np.uint16(0x8000), R, L1, L2)["y"]
    assert np.array_equal(yn, y ^ np.uint16(0x8000))
    # Y(2X) = 2Y(X), bitwise
    x2 = _bf16_bits_of(synth.bf16_to_f32(x) * np.float32(2))
    y2 = oracle.layer(x2, R, L1, L2)["y"]
    assert np.array_equal(synth.bf16_to_f32(y2), synth.bf16_to_f32(y) * np.float32(2))
    # permuting k inside each group (X columns with W rows) leaves Y unchanged
    perm = np.concatenate([g * 128 + np.random.default_rng(g).permutation(128)
                           for g in range(wl.m // 128)])
    yp = oracle.layer(x[:, perm], R[perm], L1[perm], L2)["y"]
    assert np.array_equal(yp, y)


def test_row_subset_matches_full():
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_x(wl)
    R, L1, L2 = synth.make_weights(wl)
    full = oracle.layer(x, R, L1, L2)["y"]
    rows = np.array([0, 3, 15])
    sub = oracle.layer(x, R, L1, L2, rows=rows)["y"]
    assert np.array_equal(sub, full[rows])


def test_pack_weights_layout():
    wl = synth.WORKLOADS["tiny"]
    R, L1, L2 = synth.make_weights(wl, n=256)
    pw = oracle.pack_weights(R, L1, L2)
    qr, sr = oracle.quantize_cols(R)
    ql1, sl1 = oracle.quantize_cols(L1)
    assert np.array_equal(oracle.unpack_nibbles(pw["rq"]), qr)
    assert np.array_equal(pw["sr"], sr)
    assert np.array_equal(oracle.unpack_nibbles(pw["l1q"]), ql1)
    assert np.array_equal(pw["sl1"], sl1)
    assert np.array_equal(pw["l2t"], L2.T)


def test_weight_overhead_closed_form():
    """Observation 2 (§3): FP16 low-rank parameters relative to the 4-bit residual of a
    4096 x 4096 projection are r(m+n)*16 / (m*n*4): 6.25% at r = 32 and 50% at r = 256."""
    m = n = 4096
    for r, want in ((32, 0.0625), (256, 0.5)):
        assert r * (m + n) * 16 / (m * n * 4) == want
