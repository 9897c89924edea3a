"""The package's calibration routine against the oracle's, and against the closed form of the
synthetic anisotropic workload (CPU)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import sas_oracle as O
from synth import make_problem
from token_level_sparse_head_b200.calibrate import MomentAccumulator, calibrate, scoring_basis


def test_basis_matches_the_oracle_on_random_moments():
    rng = np.random.default_rng(3)
    d, r, Hkv = 32, 8, 3
    Gq = np.stack([(lambda A: A @ A.T)(rng.standard_normal((d, d))) for _ in range(Hkv)])
    Gk = np.stack([(lambda A: A @ A.T)(rng.standard_normal((d, 2 * d))) for _ in range(Hkv)])
    M = scoring_basis(torch.from_numpy(Gq), torch.from_numpy(Gk), r).double().numpy()
    for h in range(Hkv):
        ref = O.calibration_basis(Gq[h], Gk[h], r)
        np.testing.assert_allclose(M[h], ref, atol=1e-6)
        np.testing.assert_allclose(M[h] @ M[h].T, np.eye(r), atol=1e-6)


def test_population_moments_of_the_anisotropic_workload_give_the_closed_form():
    # E[q-bar q-bar^T] ~ I and E[k k^T] = diag(s^2), s_j = 0.97^j: the first r standard vectors
    d, r, Hkv = 64, 16, 2
    s2 = torch.tensor([0.97 ** (2 * j) for j in range(d)], dtype=torch.float64)
    Gq = torch.eye(d, dtype=torch.float64).expand(Hkv, d, d) * 0.25
    Gk = torch.diag(s2).expand(Hkv, d, d) * 7.0
    M = scoring_basis(Gq, Gk, r).double().numpy()
    for h in range(Hkv):
        np.testing.assert_array_equal(M[h], np.eye(d)[:r])


def test_sampled_moments_capture_the_leading_channels():
    p = make_problem(B=2, Hq=8, Hkv=2, d=64, r=16, seqlens=[4096, 3000], k=[64, 64], aniso=True, basis="eye", seed=4)
    acc = MomentAccumulator(p.Hkv, p.d)
    g = torch.Generator().manual_seed(9)
    acc.add_queries(torch.randn(20000, p.Hq, p.d, generator=g, dtype=torch.float64))
    for b in range(p.B):
        acc.add_keys(p.K[b], int(p.seqlens[b]))
    assert acc.nq == 20000 and acc.nk == 4096 + 3000
    M = calibrate(acc, p.r).double().numpy()
    for h in range(p.Hkv):
        np.testing.assert_allclose(M[h] @ M[h].T, np.eye(p.r), atol=1e-6)
        captured = (M[h][:, : p.r // 2] ** 2).sum(axis=0)   # |M e_j|^2 for the leading channels
        assert np.all(captured > 0.9), captured
