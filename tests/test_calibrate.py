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


def _oracle_recall(M, qbars, K, k):
    """Mean over queries of |top-k of (M q-bar).(M k_i)  ∩  top-k of q-bar.k_i| / k (oracle's
    own projection, scores and ranking)."""
    kp = O.project_keys(K, M)
    rec = []
    for qb in qbars:
        exact = set(O.top_k_positions(O.decision_keys(K @ qb), k).tolist())
        u = O.selection_scores(O.project_query(M, qb), kp, 1.0)
        sel = set(O.top_k_positions(O.decision_keys(u), k).tolist())
        rec.append(len(exact & sel) / k)
    return float(np.mean(rec))


def test_joint_basis_keeps_the_ranking_a_key_only_basis_loses():
    # JSSA page, sections 问题形式化 / 迹归一化: the basis must preserve query-key interaction,
    # not key reconstruction.  Keys vary most in channels 0-3, where queries are almost zero;
    # queries vary most in channels 4-7.  The scores live in channels 4-7: the joint basis
    # (trace-normalised query + key moments) finds them, the key-only principal basis does not.
    rng = np.random.default_rng(11)
    d, r, G, N, T, k = 32, 4, 4, 4096, 4000, 128
    sk = np.ones(d); sk[:4] = 3.0
    sq = np.full(d, 0.3); sq[:4] = 0.1; sq[4:8] = 3.0
    K = rng.standard_normal((N, d)) * sk
    q = rng.standard_normal((T, 1, G, d)) * sq            # [T][Hkv=1][G][d]
    acc = MomentAccumulator(1, d)
    acc.add_queries(torch.from_numpy(q.reshape(T, G, d)))
    acc.add_keys(torch.from_numpy(K[None]))
    M_joint = calibrate(acc, r).double().numpy()[0]
    w, V = np.linalg.eigh(acc.Gk[0].numpy())
    M_key = V[:, np.argsort(w)[::-1][:r]].T               # principal key directions
    np.testing.assert_allclose((M_joint[:, 4:8] ** 2).sum(axis=1), 1.0, atol=0.05)  # spans channels 4-7
    qbars = [O.group_mean_query(rng.standard_normal((G, d)) * sq) for _ in range(20)]
    rec_joint = _oracle_recall(M_joint, qbars, K, k)
    rec_key = _oracle_recall(M_key, qbars, K, k)
    assert rec_joint > 0.5 and rec_joint > rec_key + 0.3, (rec_joint, rec_key)


def test_trace_normalisation_keeps_the_query_side():
    # JSSA page, section 迹归一化 (Table 9): the key second moment's trace can exceed the query
    # side's by orders of magnitude; summing the raw moments then returns a key-reconstruction
    # basis.  Same channels as above with the keys 10x larger: the normalised basis is unchanged
    # (scale-free), the raw sum picks the key channels and loses the ranking.
    rng = np.random.default_rng(12)
    d, r, G, N, T, k = 32, 4, 4, 4096, 4000, 128
    sk = np.ones(d) * 10.0; sk[:4] = 30.0
    sq = np.full(d, 0.3); sq[:4] = 0.1; sq[4:8] = 3.0
    K = rng.standard_normal((N, d)) * sk
    q = rng.standard_normal((T, G, d)) * sq
    acc = MomentAccumulator(1, d)
    acc.add_queries(torch.from_numpy(q))
    acc.add_keys(torch.from_numpy(K[None]))
    Gq, Gk = acc.Gq[0].numpy() / acc.nq, acc.Gk[0].numpy() / acc.nk
    assert np.trace(Gk) / np.trace(Gq) > 100
    M_norm = calibrate(acc, r).double().numpy()[0]
    w, V = np.linalg.eigh(Gq + Gk)
    M_raw = V[:, np.argsort(w)[::-1][:r]].T
    qbars = [O.group_mean_query(rng.standard_normal((G, d)) * sq) for _ in range(20)]
    rec_norm = _oracle_recall(M_norm, qbars, K, k)
    rec_raw = _oracle_recall(M_raw, qbars, K, k)
    assert rec_norm > 0.5 and rec_norm > rec_raw + 0.3, (rec_norm, rec_raw)
