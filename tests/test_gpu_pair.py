"""The prefill kernel on CTA pairs (tcgen05 cta_group::2, 256 x 256 tiles) against the
oracle, and its bounded waits.

Shapes that the pair kernel takes (b > 16, m >= 256, n % 256 == 0): ragged row blocks,
an odd number of K groups (the last two-group copy half out of range), ranks whose half
(r/2) is not a multiple of 32 or of 64, several items per pair (the row block changes
inside a pair's run, so H is recomputed and the H tile rewritten), and the layer modes.
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


def _operands(b, m, n, r, seed):
    wl = synth.WORKLOADS["tiny"]
    x = synth.fill(b, m, *wl.x_dist, seed, synth.ID_X)
    R, L1, L2 = synth.make_weights(wl, seed=seed, m=m, n=n, r=r)
    return x, R, L1, L2


def _pack(twq, device, R, L1, L2):
    r = 0 if L1 is None else L1.shape[1]
    return twq.pack_weights(to_dev(R, device), to_dev(L1, device) if r else None,
                            to_dev(L2, device) if r else None)


PAIR_SHAPES = [  # b, m, n, r
    (17, 256, 256, 16), (40, 384, 512, 32), (100, 640, 256, 48), (257, 512, 512, 96),
    (300, 1152, 768, 128), (129, 896, 256, 160), (513, 1024, 1024, 256), (64, 256, 256, 208),
    (2048, 512, 2560, 64),  # 80 items: more than one per pair, row block changes inside a run
]


@pytest.mark.parametrize("b,m,n,r", PAIR_SHAPES)
def test_pair_fused_matches_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=41)
    w = _pack(twq, device, R, L1, L2)
    xq, sx = twq.quantize_act(to_dev(x, device))
    y = bits_of(twq.fused_linear(xq, sx, w))
    rows = None if b <= 600 else block_rows(b, per_block=2, seed=3)
    ref = oracle.layer(x, R, L1, L2, mode=oracle.FUSED, rows=rows)["y"]
    assert_y_close(y if rows is None else y[rows], ref, "pair fused %s" % ((b, m, n, r),))
    assert twq.device_status() == 0


@pytest.mark.parametrize("b,m,n,r", PAIR_SHAPES[:6])
def test_pair_modes_match_oracle(twq, device, b, m, n, r):
    x, R, L1, L2 = _operands(b, m, n, r, seed=42)
    w = _pack(twq, device, R, L1, L2)
    xq, sx = twq.quantize_act(to_dev(x, device))
    y4 = bits_of(twq.w4a4_only(xq, sx, w))
    assert_y_close(y4, oracle.layer(x, R, L1, L2, mode=oracle.W4A4_ONLY)["y"], "pair w4a4")
    ylr = bits_of(twq.lowrank_only(xq, sx, w))
    assert_y_close(ylr, oracle.layer(x, R, L1, L2, mode=oracle.LOWRANK_ONLY)["y"], "pair lowrank")
    # identities: r = 0 is the W4A4 layer, R = 0 the low-rank one (bitwise)
    w0 = _pack(twq, device, R, None, None)
    assert np.array_equal(bits_of(twq.fused_linear(xq, sx, w0)), y4)
    wz = _pack(twq, device, np.zeros_like(R), L1, L2)
    assert np.array_equal(bits_of(twq.fused_linear(xq, sx, wz)), ylr)
    assert twq.device_status() == 0


@pytest.mark.parametrize("b,m,n,r", [(300, 1152, 768, 128), (513, 1024, 1024, 256)])
def test_pair_unfused_comparator_agrees(twq, device, b, m, n, r):
    """The unfused comparator (H and the fp32 components in HBM) against the pair kernel:
    the same arithmetic per element, so the same Y within the tolerance (bitwise unless
    the tensor cores sum a stage-2 K step in another order for the pair MMA shape)."""
    x, R, L1, L2 = _operands(b, m, n, r, seed=43)
    w = _pack(twq, device, R, L1, L2)
    xq, sx = twq.quantize_act(to_dev(x, device))
    yf, yu = bits_of(twq.fused_linear(xq, sx, w)), bits_of(twq.unfused_linear(xq, sx, w))
    assert_y_close(yf, yu, "fused vs unfused")
    assert twq.device_status() == 0


def test_pair_repeated_calls_are_deterministic(twq, device):
    x, R, L1, L2 = _operands(700, 768, 1536, 128, seed=44)
    w = _pack(twq, device, R, L1, L2)
    xq, sx = twq.quantize_act(to_dev(x, device))
    y0 = bits_of(twq.fused_linear(xq, sx, w))
    for _ in range(3):
        assert np.array_equal(bits_of(twq.fused_linear(xq, sx, w)), y0)
    assert twq.device_status() == 0


def test_bounded_wait_runs_out_and_the_context_stays_usable(twq, device):
    """The self-test withholds the kernel's X copies with a 100 us wait limit: the waits
    on X run out, the kernel records the site, lets its copies land, frees its tensor
    memory and returns; the status word reports it, and a normal call afterwards on the
    same stream is correct."""
    x, R, L1, L2 = _operands(300, 512, 512, 0, seed=45)
    w = _pack(twq, device, R, None, None)
    xq, sx = twq.quantize_act(to_dev(x, device))
    twq.selftest_wait_timeout(xq, sx, w, wait_limit_ns=100000)
    code = twq.device_status()
    assert 41 <= code <= 52, code
    assert twq.device_status() == 0  # read and cleared
    y = bits_of(twq.w4a4_only(xq, sx, w))
    assert_y_close(y, oracle.layer(x, R, None, None, mode=oracle.W4A4_ONLY)["y"], "after self-test")
    assert twq.device_status() == 0


@pytest.mark.parametrize("b,m,n,r", [(300, 1152, 768, 128), (513, 1024, 1024, 256), (40, 384, 512, 32),
                                     (2048, 512, 2560, 64), (100, 640, 256, 0)])
def test_byte_codes_give_the_packed_result_bitwise(twq, device, b, m, n, r):
    """quantize_act_i8 stores the codes of quantize_act one per byte (same scales), and
    the layer on them is bitwise the layer on the packed codes: the accumulator holds
    16 x (instead of 256 x) each exact group dot product, a power of two that every
    later product and the final scaling carry through unchanged."""
    x, R, L1, L2 = _operands(b, m, n, r, seed=46)
    w = _pack(twq, device, R, L1 if r else None, L2 if r else None)
    xd = to_dev(x, device)
    xq, sx = twq.quantize_act(xd)
    xq8, sx8 = twq.quantize_act_i8(xd)
    assert np.array_equal(sx8.cpu().numpy().view(np.uint32), sx.cpu().numpy().view(np.uint32))
    codes = xq8.cpu().numpy()
    assert codes.min() >= -7 and codes.max() <= 7
    assert np.array_equal(oracle.pack_nibbles(codes), xq.cpu().numpy())
    y8 = bits_of(twq.fused_linear_i8(xq8, sx8, w))
    assert np.array_equal(y8, bits_of(twq.fused_linear(xq, sx, w)))
    rows = None if b <= 600 else block_rows(b, per_block=1, seed=5)
    ref = oracle.layer(x, R, L1 if r else None, L2 if r else None, mode=oracle.FUSED, rows=rows)["y"]
    assert_y_close(y8 if rows is None else y8[rows], ref, "byte codes %s" % ((b, m, n, r),))
    assert twq.device_status() == 0


def test_byte_codes_w8_path_matches_oracle(twq, device):
    """W4A8 prefill (8-bit codes) on the pair kernel against the oracle's W4A8 layer."""
    b, m, n, r = 300, 1024, 768, 128
    x, R, L1, L2 = _operands(b, m, n, r, seed=47)
    w = _pack(twq, device, R, L1, L2)
    xq8, sx8 = twq.quantize_act_a8(to_dev(x, device))
    y = bits_of(twq.fused_linear_a8(xq8, sx8, w))
    ref = oracle.layer(x, R, L1, L2, mode=oracle.FUSED, a8=True)["y"]
    assert_y_close(y, ref, "pair W4A8")
    assert twq.device_status() == 0
