"""Pins of the oracle's W4A8 activation quantizer (TwinQuant §5.1, the quantization
settings: W4A8 is 4-bit weights with 8-bit activations; Eq. (1) with k = 8 gives
q_max = 2^7 - 1 = 127) and of the W4A8 layer.

Each check stands outside the oracle: hand-worked values of Eq. (1), an
exhaustive property over all BF16 magnitudes, numpy's correctly rounded float32
division and round-half-even, and brute force (dequantize first, then an fp64
matmul).
"""
import numpy as np
import pytest

import oracle
import synth


def _bf16(values):
    f = np.asarray(values, dtype=np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(synth.bf16_to_f32(bits), f), "value not exact in BF16"
    return bits


def test_qmax_a8_is_127():
    assert oracle.qmax_a8() == 127


def test_hand_worked_groups():
    # absmax 127: s = 1 exactly and every integer code is its own value
    g = np.zeros(128, np.float32)
    g[:9] = [127, -127, 0, 1, -1, 64, -100, 3, 126]
    q, s = oracle.quant_group_f32(g, a8=True)
    assert s == 1.0
    assert q[:9].tolist() == [127, -127, 0, 1, -1, 64, -100, 3, 126]
    # absmax 254: s = 2; odd values sit on ties and round half to even
    g[:] = 0
    g[:7] = [254, 1, 3, 5, -5, 7, -253]
    q, s = oracle.quant_group_f32(g, a8=True)
    assert s == 2.0
    assert q[:7].tolist() == [127, 0, 2, 2, -2, 4, -126]
    # the same group through the BF16 activation path
    qx, sx = oracle.quantize_rows(_bf16(g)[None, :], a8=True)
    assert sx[0, 0] == 2.0 and qx[0, :7].tolist() == [127, 0, 2, 2, -2, 4, -126]


def test_exhaustive_bf16_absmax_maps_to_127():
    """For every positive finite BF16 a: s = fl(a/127) > 0 and a/s rounds to 127, so the
    group's absmax always gets code +-127 (never clamped, never 126)."""
    bits = np.arange(1, 0x7F80, dtype=np.uint16)
    n = bits.size
    x = np.zeros((2 * n, 128), np.uint16)
    x[:n, 0] = bits
    x[n:, 9] = bits | 0x8000
    q, s = oracle.quantize_rows(x, a8=True)
    assert (s[:, 0] > 0).all()
    assert (q[:n, 0] == 127).all()
    assert (q[n:, 9] == -127).all()
    assert (q[:n, 1:] == 0).all() and (q[n:, :9] == 0).all()


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_codes_match_numpy_float32_division(name):
    """Eq. (1) restated with numpy: s = float32(a) / float32(127) and q = rint(v / s),
    both correctly rounded float32 divisions, round half to even."""
    wl = synth.WORKLOADS[name]
    x = synth.make_x(wl, b=4)
    q, s = oracle.quantize_rows(x, a8=True)
    xf = synth.bf16_to_f32(x).reshape(x.shape[0], -1, 128)
    a = np.abs(xf).max(axis=2)
    s_np = (a / np.float32(127)).astype(np.float32)
    assert np.array_equal(s, s_np)
    with np.errstate(invalid="ignore", divide="ignore"):
        t = (xf / s_np[..., None]).astype(np.float32)
    q_np = np.where(s_np[..., None] == 0, 0, np.clip(np.rint(t), -127, 127)).astype(np.int8)
    assert np.array_equal(q.reshape(q_np.shape), q_np)


def test_error_bound_half_step():
    """Away from the clamp, |v - s q| <= s/2 (plus the float32 rounding of v/s)."""
    x = synth.make_x(synth.WORKLOADS["tiny"], b=8)
    q, s = oracle.quantize_rows(x, a8=True)
    xf = synth.bf16_to_f32(x).astype(np.float64).reshape(8, -1, 128)
    sq = s.astype(np.float64)[..., None] * q.reshape(8, -1, 128)
    err = np.abs(xf - sq)
    assert (err <= s.astype(np.float64)[..., None] * (0.5 + 2.0 ** -20)).all()
    # and the 8-bit codes are finer than the 4-bit ones on the same input
    q4, s4 = oracle.quantize_rows(x)
    e4 = np.abs(xf - s4.astype(np.float64)[..., None] * q4.reshape(8, -1, 128))
    assert err.mean() < e4.mean() / 8


@pytest.mark.parametrize("b,m,n,r", [(2, 128, 16, 0), (3, 256, 24, 8), (4, 384, 40, 16)])
@pytest.mark.parametrize("mode", [oracle.FUSED, oracle.W4A4_ONLY])
def test_w4a8_layer_brute_force(b, m, n, r, mode):
    """Eq. (2) per group with 8-bit activation codes equals dequantize-first then an
    ungrouped fp64 matmul."""
    rng = np.random.default_rng(7)
    x = _bf16(np.round(rng.standard_normal((b, m)) * 64) / 64)
    R = _bf16(np.round(rng.standard_normal((m, n)) * 32) / 256)
    qx, sx = oracle.quantize_rows(x, a8=True)
    assert np.abs(qx).max() == 127
    qr, sr = oracle.quantize_cols(R)
    if r:
        L1 = _bf16(np.round(rng.standard_normal((m, r)) * 32) / 256)
        L2 = _bf16(np.round(rng.standard_normal((r, n)) * 32) / 256)
        ql1, sl1 = oracle.quantize_cols(L1)
    else:
        ql1 = sl1 = L2 = None
    out = oracle.linear(qx, sx, qr, sr, ql1, sl1, L2, mode=mode, want=("y64", "hb"))
    ref = oracle.dequant_matmul(qx, sx, qr, sr, ql1, sl1, L2, mode=mode)
    assert np.abs(out["y64"] - ref).max() <= 1e-12 * max(np.abs(ref).max(), 1e-30)
    # and outside the oracle's C code: numpy dequantization, ungrouped fp64 matmuls, stage 2
    # on the oracle's BF16 H (whose fp64 -> float32 -> BF16 chain numpy re-derives)
    xd = qx.astype(np.float64) * np.repeat(sx.astype(np.float64), 128, axis=1)
    rd = np.repeat(sr.astype(np.float64), 128, axis=0) * qr.T.astype(np.float64)
    ref_np = xd @ rd
    if r and mode == oracle.FUSED:
        l1d = np.repeat(sl1.astype(np.float64), 128, axis=0) * ql1.T.astype(np.float64)
        h = xd @ l1d
        assert np.flatnonzero(out["hb"] != synth.f32_to_bf16(h.astype(np.float32))).size <= 1
        ref_np = ref_np + (synth.bf16_to_f32(out["hb"]).astype(np.float64)
                           @ synth.bf16_to_f32(L2).astype(np.float64))
    assert np.abs(out["y64"] - ref_np).max() <= 1e-12 * max(np.abs(ref_np).max(), 1e-30)
