"""GPU parity of twq_fold_transforms (TwinQuant §4.1, Eq. (6): U' = Q^-1 U G,
V' = G^-1 V, R' = Q^-1 R) against the oracle's fp64 fold.

The device accumulates in fp32 and inverts G in fp64, so each BF16 output may
differ from the oracle's by one rounding flip: the bound is 1 BF16 ulp of the
oracle value plus 1e-6 of the output's largest magnitude. Exact cases
(identities, signed permutations with power-of-two scales) must match bitwise."""
import numpy as np
import pytest

import oracle
import synth
from helpers import bits_of, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def twq(device):
    from rank_residual_w4a4_b200 import _build, twq as binding
    _build.build()
    binding.load()
    return binding


def _bf16(f):
    return synth.f32_to_bf16(np.asarray(f, np.float32))


def _factors(m, n, r, seed):
    rng = np.random.default_rng(seed)
    return (_bf16(rng.standard_normal((m, r)) * 0.05), _bf16(rng.standard_normal((r, n)) * 0.05),
            _bf16(rng.standard_normal((m, n)) * 0.02))


def _transforms(m, r, seed):
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(rng.standard_normal((m, m)))
    G = np.eye(r) + 0.25 * rng.standard_normal((r, r)) / np.sqrt(r)
    return Q.astype(np.float32), G.astype(np.float32)


def _run(twq, device, Q, G, U, V, R):
    import torch
    outs = twq.fold_transforms(torch.from_numpy(Q).to(device), torch.from_numpy(G).to(device),
                               to_dev(U, device), to_dev(V, device), to_dev(R, device))
    return [bits_of(o) for o in outs]


def _assert_close(got, ref, what):
    g = synth.bf16_to_f32(got).astype(np.float64)
    e = synth.bf16_to_f32(ref).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(e), 2.0 ** -126))) - 7)
    bound = ulp + 1e-6 * np.abs(e).max()
    excess = np.abs(g - e) - bound
    assert excess.max() <= 0, "%s: worst excess %.3g" % (what, excess.max())


def test_identity_is_bitwise(twq, device):
    m, n, r = 192, 160, 32
    U, V, R = _factors(m, n, r, 1)
    got = _run(twq, device, np.eye(m, dtype=np.float32), np.eye(r, dtype=np.float32), U, V, R)
    assert all(np.array_equal(a, b) for a, b in zip(got, (U, V, R)))


def test_signed_permutations_are_bitwise(twq, device):
    m, n, r = 128, 96, 16
    U, V, R = _factors(m, n, r, 2)
    rng = np.random.default_rng(3)
    Q = np.zeros((m, m), np.float32)
    Q[np.arange(m), rng.permutation(m)] = rng.choice([-1.0, 1.0], m)
    G = np.zeros((r, r), np.float32)
    G[np.arange(r), rng.permutation(r)] = rng.choice([0.5, 2.0, -4.0], r)
    got = _run(twq, device, Q, G, U, V, R)
    ref = oracle.fold_transforms(Q, G, U, V, R)
    assert all(np.array_equal(a, b) for a, b in zip(got, ref))


@pytest.mark.parametrize("m,n,r", [(512, 384, 64), (200, 150, 37), (1024, 1024, 128), (64, 2048, 256)])
def test_fold_matches_oracle(twq, device, m, n, r):
    U, V, R = _factors(m, n, r, 4)
    Q, G = _transforms(m, r, 5)
    got = _run(twq, device, Q, G, U, V, R)
    ref = oracle.fold_transforms(Q, G, U, V, R)
    for name, a, b in zip(("L1'", "L2'", "R'"), got, ref):
        _assert_close(a, b, "%s %s" % (name, (m, n, r)))


def test_singular_g_is_reported(twq, device):
    m, n, r = 64, 64, 8
    U, V, R = _factors(m, n, r, 6)
    G = np.eye(r, dtype=np.float32)
    G[3] = 0.0  # a zero row: no pivot in column 3 after elimination
    with pytest.raises(twq.TwqError) as e:
        _run(twq, device, np.eye(m, dtype=np.float32), G, U, V, R)
    assert e.value.status == 1
