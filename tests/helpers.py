"""Shared helpers of the GPU tests: device transfer of BF16 bit arrays and the Y tolerance."""
import numpy as np

import synth

# Tolerance on Y (BF16 output) against the oracle's BF16-rounded Y:
#   relative Frobenius error <= 2e-3, and per element
#   |dY| <= 1e-2 * rms(Y_oracle) + 1 BF16 ulp of Y_oracle[i, j].
# The extra ulp admits a legitimate one-ulp flip of the final BF16 rounding,
# which alone exceeds 1e-2 * rms for |Y| > ~2.6 rms.
FROB_TOL = 2e-3
ELEM_TOL = 1e-2


def block_rows(b, per_block=2, seed=0, block=128):
    """Seeded rows of a b-row output, `per_block` from every `block`-row block (so every
    row block of the kernels' schedules is compared), plus the last row."""
    rng = np.random.default_rng(seed)
    rows = []
    for r0 in range(0, b, block):
        hi = min(b, r0 + block)
        rows.extend(rng.choice(np.arange(r0, hi), size=min(per_block, hi - r0), replace=False))
    rows.append(b - 1)
    return np.unique(np.array(rows, dtype=np.int64))


def to_dev(a, dev):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(a).to(dev)


def bits_of(t):
    """BF16 tensor -> numpy uint16 bit patterns."""
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_ulp(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def y_errors(y_dev_bits, y_ref_bits):
    yd = synth.bf16_to_f32(y_dev_bits).astype(np.float64)
    yr = synth.bf16_to_f32(y_ref_bits).astype(np.float64)
    rms = np.sqrt(np.mean(yr ** 2)) if yr.size else 0.0
    frob = np.linalg.norm(yd - yr) / max(np.linalg.norm(yr), 1e-300)
    excess = np.abs(yd - yr) - (ELEM_TOL * rms + bf16_ulp(yr))
    return frob, float(excess.max()) if excess.size else 0.0, rms


def assert_y_close(y_dev_bits, y_ref_bits, what=""):
    assert y_dev_bits.shape == y_ref_bits.shape, (y_dev_bits.shape, y_ref_bits.shape)
    yd = synth.bf16_to_f32(y_dev_bits)
    assert np.isfinite(yd).all(), "non-finite output %s" % what
    frob, excess, rms = y_errors(y_dev_bits, y_ref_bits)
    if rms == 0.0:
        assert not yd.any(), "expected all zeros %s" % what
        return
    assert frob <= FROB_TOL, "relative Frobenius error %.3g > %.1g %s" % (frob, FROB_TOL, what)
    assert excess <= 0.0, "per-element bound exceeded by %.3g (rms %.3g) %s" % (excess, rms, what)
