"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Codes and scales must be bit-exact; Y must meet the tolerance in helpers.py.
Small shapes span several tiles and ragged tails; the five workloads run at
full size in the launch configuration the benchmark uses, compared on seeded
row samples where the oracle would be too slow for every row.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_y_close, bits_of, block_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def twq(device):
    from rank_residual_w4a4_b200 import _build, twq as binding
    _build.build()
    binding.load()
    return binding


def _status_clean(twq):
    assert twq.device_status() == 0, "a kernel's bounded wait ran out"


def _pack(twq, dev, R, L1, L2):
    r = 0 if L1 is None else L1.shape[1]
    return twq.pack_weights(to_dev(R, dev), to_dev(L1, dev) if r else None,
                            to_dev(L2, dev) if r else None)


def _operands(b, m, n, r, seed=0, wl="tiny"):
    w = synth.WORKLOADS[wl]
    if m == w.m:
        x = synth.make_x(w, b=b, seed=seed)
    else:
        x = synth.fill(b, m, w.x_dist[0], w.x_dist[1], w.x_dist[2], seed, synth.ID_X)
    R, L1, L2 = synth.make_weights(w, seed=seed, m=m, n=n, r=r)
    if r == 0:
        L1 = L2 = None
    return x, R, L1, L2


# ------------------------------------------------------------- quantize / pack

ADVERSARIAL = {
    # ties: absmax 7 in lane 0 of each group, x.5 values elsewhere
    "ties": lambda: np.tile(np.concatenate([[7.0], np.tile(np.arange(-7, 7) + 0.5, 10)[:127]])
                            .astype(np.float32), (3, 4)),
    "zero_groups": lambda: np.zeros((5, 512), np.float32),
    "all_equal": lambda: np.full((4, 256), -0.375, np.float32),
    "subnormal": lambda: np.tile((np.arange(128) + 1) * np.float32(2.0 ** -133), (2, 2)),
    # scales above 2^125 (reciprocal not normal) and just inside the normal range
    "huge": lambda: np.tile(np.linspace(-1.5, 1.5, 128, dtype=np.float32) * np.float32(2.0 ** 126), (2, 2)),
    "tiny_normal": lambda: np.tile(np.linspace(-1.0, 1.0, 128, dtype=np.float32) * np.float32(2.0 ** -120), (2, 2)),
    "tie_sweep": lambda: tie_sweep(72, 2048),
    "every_absmax": lambda: every_absmax(256, 16384),
}


def tie_sweep(rows, m):
    """Groups of 128 whose absmax a runs over all 128 BF16 mantissas of [1, 2) and
    whose other elements run over every BF16 value of [a/16, a] of both signs, so
    that v / s falls on or next to every half-integer the codes can round at."""
    groups = rows * m // 128
    out = np.empty((groups, 128), np.float32)
    for gidx in range(groups):
        k, chunk = gidx % 128, gidx // 128
        a = np.float32(1.0 + k / 128.0)
        mags = np.array([np.float32((1.0 + j / 128.0) * 2.0 ** e) for e in range(-4, 1)
                         for j in range(128)], np.float32)
        mags = mags[(mags <= a) & (mags >= a / 16)]
        cand = np.concatenate([mags, -mags])
        idx = (np.arange(127) + chunk * 127) % cand.size
        out[gidx, 0] = a if chunk % 2 == 0 else -a
        out[gidx, 1:] = cand[idx]
    return out.reshape(rows, m)


def every_absmax(rows, m, seed=9):
    """Groups whose absmax runs over every non-negative finite BF16 value (32,640 of
    them, zero included), at a lane that moves from group to group, with the other
    elements below it; the leftover groups are zero."""
    groups = rows * m // 128
    assert groups >= 0x7F80
    rng = np.random.default_rng(seed)
    a = np.zeros(groups, np.float32)
    a[:0x7F80] = (np.arange(0x7F80, dtype=np.uint32) << 16).view(np.float32)
    f = (a[:, None] * rng.uniform(-1, 1, (groups, 128))).astype(np.float32)
    pos = (np.arange(groups) * 37) % 128
    sign = np.where(np.arange(groups) % 2 == 0, 1.0, -1.0).astype(np.float32)
    f[np.arange(groups), pos] = sign * a
    return f.reshape(rows, m)


def _absmax_lanes():
    # +-absmax at every lane position (one row per position and sign)
    rows = []
    rng = np.random.default_rng(5)
    for pos in range(128):
        for sign in (1.0, -1.0):
            v = rng.uniform(-1, 1, 128).astype(np.float32)
            v[pos] = sign * 3.0
            rows.append(v)
    return np.stack(rows)


def _bf16_exact(f):
    f = np.asarray(f, np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("case", list(ADVERSARIAL) + ["absmax_lanes"])
def test_quantize_act_adversarial(twq, device, case):
    f = _absmax_lanes() if case == "absmax_lanes" else ADVERSARIAL[case]()
    x = _bf16_exact(f)
    xq, sx = twq.quantize_act(to_dev(x, device))
    rq, rs = oracle.quantize_act(x)
    assert np.array_equal(xq.cpu().numpy(), rq)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("name,b", [("tiny", 16), ("decode", 1), ("decode", 4), ("decode", 16),
                                    ("gateup", 2048), ("down", 4096), ("large", 8192),
                                    ("tiny", 3), ("tiny", 129)])
def test_quantize_act_bitexact(twq, device, name, b):
    wl = synth.WORKLOADS[name]
    x = synth.make_x(wl, b=b)
    xq, sx = twq.quantize_act(to_dev(x, device))
    rq, rs = oracle.quantize_act(x)
    assert np.array_equal(xq.cpu().numpy(), rq)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    _status_clean(twq)


def test_pack_weights_every_absmax(twq, device):
    # every BF16 absmax as a (group, column) scale of R: m = 2048, n = 2048
    R = _bf16_exact(every_absmax(2048, 2048).reshape(2048, 16, 128).transpose(1, 2, 0)
                    .reshape(2048, 2048).copy())
    w = _pack(twq, device, R, None, None)
    ref = oracle.pack_weights(R, None, None)
    assert np.array_equal(w.rq.cpu().numpy(), ref["rq"])
    assert np.array_equal(w.sr.cpu().numpy().view(np.uint32), ref["sr"].view(np.uint32))
    _status_clean(twq)


def test_pack_weights_tie_sweep(twq, device):
    # the same near-tie groups along the columns of R and L1 (offline packing path)
    R = _bf16_exact(tie_sweep(128, 2048).T.copy())       # m = 2048, n = 128
    L1 = _bf16_exact(tie_sweep(16, 2048).T.copy())       # m = 2048, r = 16
    L2 = _bf16_exact(np.ones((16, 128), np.float32))
    w = _pack(twq, device, R, L1, L2)
    ref = oracle.pack_weights(R, L1, L2)
    assert np.array_equal(w.rq.cpu().numpy(), ref["rq"])
    assert np.array_equal(w.sr.cpu().numpy().view(np.uint32), ref["sr"].view(np.uint32))
    assert np.array_equal(w.l1q.cpu().numpy(), ref["l1q"])
    assert np.array_equal(w.sl1.cpu().numpy().view(np.uint32), ref["sl1"].view(np.uint32))
    _status_clean(twq)


@pytest.mark.parametrize("name", ["tiny", "decode", "gateup", "down", "large"])
def test_pack_weights_bitexact(twq, device, name):
    wl = synth.WORKLOADS[name]
    R, L1, L2 = synth.make_weights(wl)
    w = _pack(twq, device, R, L1, L2)
    ref = oracle.pack_weights(R, L1, L2)
    assert np.array_equal(w.rq.cpu().numpy(), ref["rq"])
    assert np.array_equal(w.sr.cpu().numpy().view(np.uint32), ref["sr"].view(np.uint32))
    assert np.array_equal(w.l1q.cpu().numpy(), ref["l1q"])
    assert np.array_equal(w.sl1.cpu().numpy().view(np.uint32), ref["sl1"].view(np.uint32))
    assert np.array_equal(bits_of(w.l2t), ref["l2t"])
    _status_clean(twq)


# ------------------------------------------------------------------ the layer

SHAPES = [  # b, m, n, r: several tiles, ragged b, one/two H chunks, r not a multiple of 64
    (16, 512, 512, 32), (1, 128, 128, 16), (3, 256, 384, 48), (17, 384, 256, 64),
    (129, 512, 384, 128), (200, 256, 256, 144), (64, 640, 128, 256), (300, 128, 512, 16),
    # CTA pairs sharing H (even column-tile count, 128 < r <= 256, r % 32 == 0): halves of
    # r/2 = 112 and 80 that straddle 64-column chunks, three pair items per row block, r = 256
    (129, 256, 512, 224), (200, 256, 256, 192), (257, 384, 768, 160), (300, 256, 1024, 256),
]


def _oracle_y(x, R, L1, L2, mode, rows=None):
    return oracle.layer(x, R, L1, L2, mode=mode, rows=rows)["y"]


@pytest.mark.parametrize("b,m,n,r", SHAPES)
def test_fused_matches_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=1)
    w = _pack(twq, device, R, L1, L2)
    xq, sx = twq.quantize_act(to_dev(x, device))
    y = twq.fused_linear(xq, sx, w)
    assert_y_close(bits_of(y), _oracle_y(x, R, L1, L2, oracle.FUSED), "fused %s" % ((b, m, n, r),))
    _status_clean(twq)


@pytest.mark.parametrize("b,m,n,r", SHAPES[:5])
def test_variants_match_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=2)
    w = _pack(twq, device, R, L1, L2)
    xq, sx = twq.quantize_act(to_dev(x, device))
    y4 = twq.w4a4_only(xq, sx, w)
    assert_y_close(bits_of(y4), _oracle_y(x, R, L1, L2, oracle.W4A4_ONLY), "w4a4_only")
    ylr = twq.lowrank_only(xq, sx, w)
    assert_y_close(bits_of(ylr), _oracle_y(x, R, L1, L2, oracle.LOWRANK_ONLY), "lowrank_only")
    _status_clean(twq)


def _decode_path(b, m, r):
    """Shapes the library runs on the split-K decode kernel (b <= 16, r <= 128, m <= 8192)."""
    return 1 <= b <= 16 and r <= 128 and m // 128 <= 64


@pytest.mark.parametrize("b,m,n,r", SHAPES)
def test_unfused_vs_fused(twq, device, b, m, n, r):
    """Same kernel family: bitwise equal. Decode shapes (split-K kernel for the fused
    call): equal within the Y tolerance."""
    x, R, L1, L2 = _operands(b, m, n, r, seed=3)
    w = _pack(twq, device, R, L1, L2)
    xq, sx = twq.quantize_act(to_dev(x, device))
    yu, yf = bits_of(twq.unfused_linear(xq, sx, w)), bits_of(twq.fused_linear(xq, sx, w))
    if _decode_path(b, m, r):
        assert_y_close(yf, yu, "decode fused vs unfused")
    else:
        assert np.array_equal(yu, yf)
    _status_clean(twq)


DECODE_SHAPES = [  # b, m, n, r: cluster of 4 (m <= 4096) and of 8 (4096 < m <= 8192),
    # uneven group and r-unit splits, a CTA with no groups (m = 128), r below one unit per CTA
    (1, 4096, 512, 128), (7, 4096, 256, 128), (16, 8192, 256, 128), (16, 5120, 256, 64),
    (5, 1024, 384, 48), (16, 128, 128, 16), (2, 640, 128, 32), (16, 4096, 128, 0),
]


@pytest.mark.parametrize("b,m,n,r", DECODE_SHAPES)
def test_decode_kernel_matches_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=8)
    w = _pack(twq, device, R, L1, L2)
    xq, sx = twq.quantize_act(to_dev(x, device))
    assert_y_close(bits_of(twq.fused_linear(xq, sx, w)), _oracle_y(x, R, L1, L2, oracle.FUSED),
                   "decode fused %s" % ((b, m, n, r),))
    assert_y_close(bits_of(twq.w4a4_only(xq, sx, w)), _oracle_y(x, R, L1, L2, oracle.W4A4_ONLY),
                   "decode w4a4 %s" % ((b, m, n, r),))
    if r:
        assert_y_close(bits_of(twq.lowrank_only(xq, sx, w)),
                       _oracle_y(x, R, L1, L2, oracle.LOWRANK_ONLY), "decode lowrank %s" % ((b, m, n, r),))
    _status_clean(twq)


def test_decode_identities(twq, device):
    x, R, L1, L2 = _operands(8, 1024, 256, 64, seed=12)
    xq, sx = twq.quantize_act(to_dev(x, device))
    w0 = _pack(twq, device, R, None, None)
    assert np.array_equal(bits_of(twq.fused_linear(xq, sx, w0)), bits_of(twq.w4a4_only(xq, sx, w0)))
    wz = _pack(twq, device, np.zeros_like(R), L1, L2)
    w = _pack(twq, device, R, L1, L2)
    assert np.array_equal(bits_of(twq.fused_linear(xq, sx, wz)), bits_of(twq.lowrank_only(xq, sx, w)))
    yn = bits_of(twq.w4a4_only(*twq.quantize_act(to_dev(x ^ np.uint16(0x8000), device)), w0))
    assert np.array_equal(yn, bits_of(twq.w4a4_only(xq, sx, w0)) ^ np.uint16(0x8000))
    _status_clean(twq)


def test_r0_is_w4a4_and_R0_is_lowrank(twq, device):
    x, R, L1, L2 = _operands(40, 512, 256, 32, seed=4)
    xq, sx = twq.quantize_act(to_dev(x, device))
    w0 = _pack(twq, device, R, None, None)
    assert np.array_equal(bits_of(twq.fused_linear(xq, sx, w0)), bits_of(twq.w4a4_only(xq, sx, w0)))
    wz = _pack(twq, device, np.zeros_like(R), L1, L2)
    w = _pack(twq, device, R, L1, L2)
    assert np.array_equal(bits_of(twq.fused_linear(xq, sx, wz)), bits_of(twq.lowrank_only(xq, sx, w)))


def test_sign_and_scaling_equivariance(twq, device):
    x, R, L1, L2 = _operands(24, 512, 256, 0, seed=6)
    w = _pack(twq, device, R, None, None)
    y = bits_of(twq.w4a4_only(*twq.quantize_act(to_dev(x, device)), w))
    yn = bits_of(twq.w4a4_only(*twq.quantize_act(to_dev(x ^ np.uint16(0x8000), device)), w))
    assert np.array_equal(yn, y ^ np.uint16(0x8000))
    x2 = _bf16_exact(synth.bf16_to_f32(x) * np.float32(2))
    y2 = bits_of(twq.w4a4_only(*twq.quantize_act(to_dev(x2, device)), w))
    assert np.array_equal(synth.bf16_to_f32(y2), synth.bf16_to_f32(y) * np.float32(2))


def test_degenerate_inputs(twq, device):
    b, m, n, r = 33, 256, 128, 16
    _, R, L1, L2 = _operands(b, m, n, r, seed=7)
    w = _pack(twq, device, R, L1, L2)
    xz = np.zeros((b, m), np.uint16)
    y = bits_of(twq.fused_linear(*twq.quantize_act(to_dev(xz, device)), w))
    assert not (synth.bf16_to_f32(y) != 0).any()
    # b == 0 is a no-op that returns an empty result
    import torch
    xq0 = torch.empty((0, m // 2), dtype=torch.uint8, device=device)
    sx0 = torch.empty((0, m // 128), dtype=torch.float32, device=device)
    assert twq.fused_linear(xq0, sx0, w).shape == (0, n)
    _status_clean(twq)


# --------------------------------------------------- the five workloads, full size

def _full(twq, device, name, b, rows, byte_codes=False):
    wl = synth.WORKLOADS[name]
    x = synth.make_x(wl, b=b)
    R, L1, L2 = synth.make_weights(wl)
    w = _pack(twq, device, R, L1, L2)
    xd = to_dev(x, device)
    xq, sx = twq.quantize_act(xd)
    y = bits_of(twq.fused_linear(xq, sx, w))
    rows = np.arange(b) if rows is None else rows
    ref = _oracle_y(x, R, L1, L2, oracle.FUSED, rows=rows)
    assert_y_close(y[rows], ref, "%s b=%d" % (name, b))
    if byte_codes:
        # the benchmark's step: the same codes one per byte, the layer on them; the whole Y
        # is bitwise that of the packed path checked above
        xq8, sx8 = twq.quantize_act_i8(xd)
        assert np.array_equal(sx8.cpu().numpy().view(np.uint32), sx.cpu().numpy().view(np.uint32))
        assert np.array_equal(bits_of(twq.fused_linear_i8(xq8, sx8, w)), y)
    _status_clean(twq)
    return y, rows


@pytest.mark.parametrize("name,b", [("tiny", 16), ("decode", 1), ("decode", 4), ("decode", 16)])
def test_workload_all_rows(twq, device, name, b):
    _full(twq, device, name, b, None)


@pytest.mark.parametrize("name", ["gateup", "down", "large"])
def test_workload_rows_of_every_row_block(twq, device, name):
    """Full-size prefill workloads: two seeded rows of every 128-row block (every row
    block of the persistent schedule, so every CTA's work), all columns; and the byte-code
    path the benchmark times, bitwise against the whole packed-code Y."""
    wl = synth.WORKLOADS[name]
    _full(twq, device, name, wl.b, block_rows(wl.b, per_block=2, seed=11), byte_codes=True)
