"""The seeded input generator: determinism, thread independence and distributions."""
import numpy as np

import synth


def test_splitmix64_reference_vector():
    # splitmix64 started from state 0: first output (the published reference stream).
    assert synth.mix64(0x9E3779B97F4A7C15) == 0xE220A8397B1DCDAF


def test_deterministic_and_seed_sensitive():
    a = synth.fill(7, 33, synth.NORMAL, 0.0, 1.0, 0, 1)
    b = synth.fill(7, 33, synth.NORMAL, 0.0, 1.0, 0, 1)
    c = synth.fill(7, 33, synth.NORMAL, 0.0, 1.0, 1, 1)
    d = synth.fill(7, 33, synth.NORMAL, 0.0, 1.0, 0, 2)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)


def test_element_values_depend_only_on_index():
    big = synth.fill(64, 100, synth.STUDENT_T, 3.0, 0.02, 0, 1)
    small = synth.fill(3, 100, synth.STUDENT_T, 3.0, 0.02, 0, 1)
    assert np.array_equal(big[:3], small)


def test_uniforms_in_open_interval():
    u = synth.element_uniforms(1000, 0, 0, 12345)
    assert (u > 0).all() and (u < 1).all()
    assert abs(u.mean() - 0.5) < 0.05


def test_bf16_rounding_of_draws():
    bits, vals = synth.fill(50, 50, synth.NORMAL, 0.0, 1.0, 0, 3, with_values=True)
    f32 = vals.astype(np.float32)
    assert np.array_equal(bits, synth.f32_to_bf16(f32))


def test_normal_moments():
    x = synth.bf16_to_f32(synth.fill(400, 500, synth.NORMAL, 0.0, 0.03, 0, 2)).astype(np.float64)
    assert abs(x.mean()) < 1e-3 * 3
    assert abs(x.std() - 0.03) < 0.03 * 0.01


def test_student_t_variance_and_tails():
    from scipy import stats
    # Student-t(nu=5): variance nu/(nu-2) = 5/3
    x = synth.bf16_to_f32(synth.fill(500, 800, synth.STUDENT_T, 5.0, 1.0, 0, 1)).astype(np.float64)
    assert abs(x.var() - 5.0 / 3.0) < 0.05
    # two-sided tail masses and the median of |t| against the exact t distribution
    for nu in (2.5, 3.0):
        t = synth.bf16_to_f32(synth.fill(500, 800, synth.STUDENT_T, nu, 1.0, 0, 1)).astype(np.float64)
        for c in (2.0, 5.0):
            want = 2 * stats.t.sf(c, nu)
            got = (np.abs(t) > c).mean()
            assert abs(got - want) < 4 * np.sqrt(want / t.size) + 1e-3 * want
        assert abs(np.median(np.abs(t)) - stats.t.ppf(0.75, nu)) < 0.01


def test_outlier_channel_counts_and_factor():
    for name, want in (("tiny", 10), ("decode", 41), ("gateup", 41), ("down", 72), ("large", 51)):
        wl = synth.WORKLOADS[name]
        ch = synth.outlier_channels(wl.m, wl.x_outlier[0], 0)
        assert ch.size == want and np.unique(ch).size == want
    wl = synth.WORKLOADS["tiny"]
    x = synth.bf16_to_f32(synth.make_x(wl, b=200)).astype(np.float64)
    ch = synth.outlier_channels(wl.m, wl.x_outlier[0], 0)
    rest = np.setdiff1d(np.arange(wl.m), ch)
    ratio = x[:, ch].std() / x[:, rest].std()
    assert 17 < ratio < 23


def test_permutation_is_a_permutation():
    p = synth.permutation(1000, 0, 4)
    assert np.array_equal(np.sort(p), np.arange(1000))
    assert not np.array_equal(p, np.arange(1000))


def test_sample_rows():
    rows = synth.sample_rows(4096, 64, 0)
    assert rows[0] == 0 and rows[-1] == 4095 and len(rows) == 64
    assert np.all(np.diff(rows) > 0)
