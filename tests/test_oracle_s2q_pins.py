"""Pins of the oracle's INT4 stage 2 (TwinQuant §4.3: H requantized to 4 bits on chip,
multiplied by the 4-bit V), in the readings the oracle states: Eq. (1) with q_max = 7
on bf16(H) per token in groups of 128 along r, and on L2 per output column in groups
of 128 along r.

Each check stands outside the oracle's grouped GEMM: numpy re-derives the codes from
correctly rounded float32 division, and an ungrouped fp64 matmul of the dequantized
operands gives Y."""
import numpy as np
import pytest

import oracle
import synth


def _operands(b, m, n, r, seed):
    wl = synth.WORKLOADS["tiny"]
    x = synth.fill(b, m, *wl.x_dist, seed, synth.ID_X)
    R, L1, L2 = synth.make_weights(wl, seed=seed, m=m, n=n, r=r)
    return x, R, L1, L2


def _eq1_numpy(v, axis_groups):
    """Eq. (1) with numpy float32: v (rows x k) in groups of 128 along k."""
    rows, k = v.shape
    g = v.reshape(rows, k // 128, 128)
    a = np.abs(g).max(axis=2)
    s = (a / np.float32(7)).astype(np.float32)
    with np.errstate(invalid="ignore", divide="ignore"):
        t = (g / s[..., None]).astype(np.float32)
    q = np.where(s[..., None] == 0, 0, np.clip(np.rint(t), -7, 7)).astype(np.int8)
    return q.reshape(rows, k), s


def _dequant(q, s):
    rows, k = q.shape
    return (q.reshape(rows, k // 128, 128).astype(np.float64) * s[..., None]).reshape(rows, k)


@pytest.mark.parametrize("b,m,n,r", [(3, 256, 128, 128), (4, 384, 256, 256), (1, 128, 128, 128)])
def test_codes_and_brute_force(b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=11)
    o = oracle.layer_s2q(x, R, L1, L2, want=("y", "y64", "hb", "qh", "sh"))
    # Q_H: Eq. (1) on bf16(H), re-derived with numpy
    hb = synth.bf16_to_f32(o["hb"])
    qh, sh = _eq1_numpy(hb, r)
    assert np.array_equal(o["qh"], qh) and np.array_equal(o["sh"], sh)
    # Q_V: Eq. (1) on L2 columns (groups along r), re-derived with numpy
    qv, sv = _eq1_numpy(synth.bf16_to_f32(L2).T.copy(), r)   # n x r codes, n x (r/128) scales
    # Y = Y_res + dequant(Q_H) @ dequant(Q_V)^T, one ungrouped fp64 matmul each
    qx, sx = oracle.quantize_rows(x)
    qr, sr = oracle.quantize_cols(R)
    yres = _dequant(qx, sx) @ _dequant(qr, sr.T.copy()).T
    ylr = _dequant(qh, sh) @ _dequant(qv, sv).T
    ref = yres + ylr
    assert np.abs(o["y64"] - ref).max() <= 1e-12 * np.abs(ref).max()
    # the output is the BF16 of the float32 of that sum
    f = ref.astype(np.float32).view(np.uint32).astype(np.uint64)
    ybits = ((f + 0x7FFF + ((f >> 16) & 1)) >> 16).astype(np.uint16)
    mism = np.flatnonzero(o["y"] != ybits)
    # only where fp64 rounding order could move the float32 (checked to be rare and 1 ulp)
    assert mism.size <= max(1, o["y"].size // 1000)


def test_exact_v_reduces_to_dequantized_h_times_l2():
    """With L2 on a 4-bit grid whose column groups reach +-7 steps, Q(V) is exact, so
    Y_lr = dequant(Q_H) @ L2."""
    b, m, n, r = 2, 256, 128, 128
    x, R, L1, _ = _operands(b, m, n, r, seed=12)
    rng = np.random.default_rng(3)
    steps = rng.integers(-7, 8, size=(r, n)).astype(np.float32)
    steps[0, :] = 7.0
    l2f = steps * np.float32(0.25)
    L2 = (l2f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(synth.bf16_to_f32(L2), l2f)
    o = oracle.layer_s2q(x, R, L1, L2, want=("y64", "qh", "sh"))
    qx, sx = oracle.quantize_rows(x)
    qr, sr = oracle.quantize_cols(R)
    yres = _dequant(qx, sx) @ _dequant(qr, sr.T.copy()).T
    ref = yres + _dequant(o["qh"], o["sh"]) @ l2f.astype(np.float64)
    assert np.abs(o["y64"] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_two_groups_of_r_have_their_own_scales():
    """r = 256: the two halves of each H row are quantized with separate scales. With
    the second half of L1 = 64 x the first (a power of two, so every rounding commutes
    with it), the second half of H is exactly 64 x the first: its scale is exactly 64 x
    larger and its codes are the same."""
    b, m, n, r = 2, 128, 128, 256
    x, R, L1, L2 = _operands(b, m, n, r, seed=13)
    l1 = synth.bf16_to_f32(L1).copy()
    l1[:, 128:] = l1[:, :128] * np.float32(64.0)
    L1 = (l1.view(np.uint32) >> 16).astype(np.uint16)
    o = oracle.layer_s2q(x, R, L1, L2, want=("sh", "qh"))
    assert np.array_equal(o["sh"][:, 1], o["sh"][:, 0] * np.float32(64.0))
    assert np.array_equal(o["qh"][:, 128:], o["qh"][:, :128])
    assert (np.abs(o["qh"][:, :128]).max(axis=1) == 7).all()


def test_needs_whole_groups_of_r():
    x, R, L1, L2 = _operands(1, 128, 128, 64, seed=14)
    with pytest.raises(ValueError):
        oracle.layer_s2q(x, R, L1, L2)
