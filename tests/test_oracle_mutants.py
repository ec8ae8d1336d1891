"""The oracle's pins catch plausible mistakes in it.

Each case plants one mistake in a copy of the oracle's C source (a reciprocal
instead of Eq. (1)'s division, rounding half away from zero, a wrong q_max, a
dropped or sign-flipped stage 2, a scale taken from the wrong group, a
transposed operand, a weight group read across columns, ...). The copy is
compiled on the CPU into a build folder, loaded in place of the oracle, and a
battery of checks that stand outside the oracle's code runs against it:

* the hand-worked Eq. (1) cases of tests/golden/eq1_groups.txt;
* the nibble layout (element 2p in the low nibble of byte p);
* Eq. (1) re-derived with numpy (correctly rounded float32 division, round
  half to even) for activations (q_max = 7 and 127) and weights, groups of 128
  along the reduction dimension;
* the layer re-derived with numpy: dequantize first, one ungrouped fp64 matmul
  per GEMM, BF16 rounding of H (TwinQuant Eq. (2), (3) and §4.3).

The unmodified oracle passes the battery; every mutant fails at least one
check. Every planted change keeps all memory accesses in bounds.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "twq_oracle.cpp")
OUT = os.path.join(ROOT, "_build", "oracle_mutants")
GOLDEN = os.path.join(ROOT, "tests", "golden", "eq1_groups.txt")

MUTANTS = {
    "reciprocal_instead_of_division": (
        "float t = v[k * stride] / s;", "float t = v[k * stride] * (1.0f / s);"),
    "round_half_away_from_zero": ("std::nearbyint(t)", "std::round(t)"),
    "qmax_off_by_one": ("float s = a / static_cast<float>(qmax);",
                        "float s = a / static_cast<float>(qmax + 1);"),
    "absmax_without_abs": ("float m = std::fabs(v[k * stride]);", "float m = v[k * stride];"),
    "a8_qmax_126": ("constexpr int kQmaxA8 = (1 << (8 - 1)) - 1;",
                    "constexpr int kQmaxA8 = (1 << (8 - 1)) - 2;"),
    "nibbles_swapped": ("out[p] = static_cast<uint8_t>(lo | (hi << 4));",
                        "out[p] = static_cast<uint8_t>(hi | (lo << 4));"),
    "weight_groups_across_columns": ("w[(g * kGroup + k) * cols + j]",
                                     "w[j * m + g * kGroup + k]"),
    "weight_group_offset_dropped": (
        "dot += static_cast<int64_t>(xi[g * kGroup + k]) * wj[g * kGroup + k];",
        "dot += static_cast<int64_t>(xi[g * kGroup + k]) * wj[k];"),
    "x_scale_of_group_0": (
        "acc += static_cast<double>(sx[i * G + g]) * static_cast<double>(sr[g * n + j]) *",
        "acc += static_cast<double>(sx[i * G]) * static_cast<double>(sr[g * n + j]) *"),
    "l1_scales_transposed": ("static_cast<double>(sl1[g * r + c])",
                             "static_cast<double>(sl1[c * G + g])"),
    "h_not_rounded_to_bf16": ("hb[c] = static_cast<double>(bf16_to_f32(hbits));", "hb[c] = acc;"),
    "l2_transposed": ("ylr += hb[c] * static_cast<double>(bf16_to_f32(l2[c * n + j]));",
                      "ylr += hb[c] * static_cast<double>(bf16_to_f32(l2[j * r + c]));"),
    "stage2_dropped": ("double total = use_res ? yres[j] + ylr : ylr;",
                       "double total = use_res ? yres[j] : ylr;"),
    "stage2_sign": ("double total = use_res ? yres[j] + ylr : ylr;",
                    "double total = use_res ? yres[j] - ylr : ylr;"),
}


# ------------------------------------------------------------------ the battery

def _golden_cases():
    cases = []
    with open(GOLDEN) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                name, vals, codes, scale = [p.strip() for p in line.split("|")]
                cases.append(([float(v) for v in vals.split()], [int(c) for c in codes.split()],
                              int(scale, 16)))
    return cases


def _check_golden():
    for vals, codes, scale_bits in _golden_cases():
        group = np.zeros(128, np.float32)
        group[:len(vals)] = vals
        q, s = oracle.quant_group_f32(group)
        if int(np.float32(s).view(np.uint32)) != scale_bits or q[:len(codes)].tolist() != codes:
            return False
        x = (group.view(np.uint32) >> 16).astype(np.uint16)[None, :]
        qx, sx = oracle.quantize_rows(x)
        if qx[0, :len(codes)].tolist() != codes:
            return False
        qw, sw = oracle.quantize_cols(x.T.copy())
        if qw[0, :len(codes)].tolist() != codes:
            return False
    return True


def _check_nibbles():
    return oracle.pack_nibbles(np.array([-7, 7, -1, 0], np.int8)).tolist() == [0x79, 0x0F]


def _eq1_numpy(v, qmax):
    """Eq. (1) in groups of 128 along the last axis of v (float32, rows x k)."""
    rows, k = v.shape
    g = v.reshape(rows, k // 128, 128)
    s = (np.abs(g).max(axis=2) / np.float32(qmax)).astype(np.float32)
    with np.errstate(invalid="ignore", divide="ignore"):
        t = (g / s[..., None]).astype(np.float32)
    q = np.where(s[..., None] == 0, 0, np.clip(np.rint(t), -qmax, qmax))
    return q.reshape(rows, k).astype(np.int8), s


def _operands(seed=41, b=3, m=256, n=24, r=16):
    wl = synth.WORKLOADS["tiny"]
    x = synth.fill(b, m, *wl.x_dist, seed, synth.ID_X)
    R, L1, L2 = synth.make_weights(wl, seed=seed, m=m, n=n, r=r)
    return x, R, L1, L2


def _check_eq1_numpy():
    x, R, L1, _ = _operands()
    xf = synth.bf16_to_f32(x)
    for a8, qmax in ((False, 7), (True, 127)):
        q, s = oracle.quantize_rows(x, a8=a8)
        qn, sn = _eq1_numpy(xf, qmax)
        if not (np.array_equal(q, qn) and np.array_equal(s.view(np.uint32), sn.view(np.uint32))):
            return False
    for w in (R, L1):
        q, s = oracle.quantize_cols(w)                      # cols x m codes, (m/128) x cols
        qn, sn = _eq1_numpy(synth.bf16_to_f32(w).T.copy(), 7)
        if not (np.array_equal(q, qn) and np.array_equal(s.T.view(np.uint32), sn.view(np.uint32))):
            return False
    return True


def _check_layer_numpy():
    x, R, L1, L2 = _operands()
    qx, sx = oracle.quantize_rows(x)
    qr, sr = oracle.quantize_cols(R)
    ql1, sl1 = oracle.quantize_cols(L1)
    xd = qx.astype(np.float64) * np.repeat(sx.astype(np.float64), 128, axis=1)
    rd = np.repeat(sr.astype(np.float64), 128, axis=0) * qr.T.astype(np.float64)
    l1d = np.repeat(sl1.astype(np.float64), 128, axis=0) * ql1.T.astype(np.float64)
    fused = oracle.linear(qx, sx, qr, sr, ql1, sl1, L2, mode=oracle.FUSED, want=("y64", "hb"))
    # H: numpy's ungrouped fp64 sum and the oracle's grouped one may straddle a float32
    # rounding boundary in rare elements, so a few BF16 bits may differ
    hb_np = synth.f32_to_bf16((xd @ l1d).astype(np.float32))
    if np.count_nonzero(fused["hb"] != hb_np) > max(1, hb_np.size // 500):
        return False
    # Y on the oracle's BF16 H
    hb = synth.bf16_to_f32(fused["hb"]).astype(np.float64)
    yres = xd @ rd
    ylr = hb @ synth.bf16_to_f32(L2).astype(np.float64)
    for mode, ref in ((oracle.FUSED, yres + ylr), (oracle.W4A4_ONLY, yres),
                      (oracle.LOWRANK_ONLY, ylr)):
        y64 = (fused if mode == oracle.FUSED else
               oracle.linear(qx, sx, qr, sr, ql1, sl1, L2, mode=mode, want=("y64",)))["y64"]
        if np.abs(y64 - ref).max() > 1e-12 * np.abs(ref).max():
            return False
    return True


BATTERY = {"golden": _check_golden, "nibbles": _check_nibbles, "eq1_numpy": _check_eq1_numpy,
           "layer_numpy": _check_layer_numpy}


def _failures():
    return [name for name, check in BATTERY.items() if not check()]


# ------------------------------------------------------------------ the tests

def test_the_oracle_passes_the_battery():
    assert _failures() == []


def _mutant_lib(name):
    old, new = MUTANTS[name]
    with open(SRC) as fh:
        src = fh.read()
    assert src.count(old) == 1, "the planted line is no longer in the oracle: %r" % old
    os.makedirs(OUT, exist_ok=True)
    cpp = os.path.join(OUT, name + ".cpp")
    so = os.path.join(OUT, "lib" + name + "_%d.so" % os.getpid())
    with open(cpp, "w") as fh:
        fh.write(src.replace(old, new))
    subprocess.check_call(oracle.CXX + ["-o", so, cpp])
    lib = oracle._load(so)
    os.remove(so)  # the loaded mapping stays valid
    return lib


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_a_planted_mistake_fails_a_pin(name, monkeypatch):
    monkeypatch.setattr(oracle, "_lib", _mutant_lib(name))
    failed = _failures()
    assert failed, "mutant %s passed every check" % name


# ------------------------------------------- mistakes in the Python-side oracle
# The INT4 stage 2 (layer_s2q) and the transform fold (fold_transforms) are written
# in oracle/__init__.py. A mistake is planted in a copy of that module's source,
# which runs in place of the oracle under the pins of test_oracle_s2q_pins.py and
# test_fold_oracle.py (numpy re-derivations, closed forms and identities).

PY_MUTANTS = {
    "s2q_residual_dropped": ("    total = res + ylr\n", "    total = ylr\n"),
    "s2q_sign": ("    total = res + ylr\n", "    total = res - ylr\n"),
    "s2q_h_codes_8bit": ("qh, sh = quantize_rows(hb)", "qh, sh = quantize_rows(hb, a8=True)"),
    "s2q_v_scales_dropped": ("ylr = linear(qh, sh, qv, sv,", "ylr = linear(qh, sh, qv, np.ones_like(sv),"),
    "s2q_h_scales_dropped": ("ylr = linear(qh, sh, qv, sv,", "ylr = linear(qh, np.ones_like(sh), qv, sv,"),
    "fold_q_not_transposed": ("l1 = q.T @ (u @ g)", "l1 = q @ (u @ g)"),
    "fold_g_inverse_on_u": ("l1 = q.T @ (u @ g)", "l1 = q.T @ (u @ np.linalg.inv(g))"),
    "fold_g_not_inverted": ("l2 = np.linalg.inv(g) @ v", "l2 = g @ v"),
    "fold_r_not_transposed": ("rr = q.T @ r", "rr = q @ r"),
}


def _python_pins():
    import test_fold_oracle as fold
    import test_oracle_s2q_pins as s2q
    return [
        ("s2q codes and brute force r=128", s2q, lambda: s2q.test_codes_and_brute_force(3, 256, 128, 128)),
        ("s2q codes and brute force r=256", s2q, lambda: s2q.test_codes_and_brute_force(4, 384, 256, 256)),
        ("s2q exact V", s2q, s2q.test_exact_v_reduces_to_dequantized_h_times_l2),
        ("s2q two groups of r", s2q, s2q.test_two_groups_of_r_have_their_own_scales),
        ("fold identities", fold, fold.test_identity_transforms_leave_the_factors_unchanged),
        ("fold signed permutations", fold, fold.test_signed_permutations_are_exact),
        ("fold preserves the layer", fold, fold.test_fold_preserves_the_layer_output),
    ]


def _python_failures(module, monkeypatch):
    failed = []
    for name, test_module, run in _python_pins():
        monkeypatch.setattr(test_module, "oracle", module)
        try:
            run()
        except (AssertionError, ValueError):
            failed.append(name)
    return failed


def _mutant_module(name):
    import types
    old, new = PY_MUTANTS[name]
    path = oracle.__file__
    with open(path) as fh:
        src = fh.read()
    assert src.count(old) == 1, "the planted line is no longer in the oracle: %r" % old
    mod = types.ModuleType("oracle_mutant_" + name)
    mod.__file__ = path
    exec(compile(src.replace(old, new), path, "exec"), mod.__dict__)
    return mod


def test_the_python_oracle_passes_its_pins(monkeypatch):
    assert _python_failures(oracle, monkeypatch) == []


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_a_planted_python_mistake_fails_a_pin(name, monkeypatch):
    assert _python_failures(_mutant_module(name), monkeypatch), "mutant %s passed every pin" % name
