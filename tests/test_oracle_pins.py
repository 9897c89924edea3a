"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test pins one oracle step to a closed form, a brute force on tiny inputs, an invariant,
or an independent library routine, chosen so that a plausible slip (a dropped term, a wrong
sign or index, a transposed operand, a wrong rounding mode) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import sas_oracle as O
from synth import make_config, make_problem
from tests.helpers import f64, problem_arrays

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------------------- bf16 rounding
def test_bf16_round_hand_values():
    # bf16 has 7 stored fraction bits: the spacing just above 1.0 is 2**-7.
    cases = [
        (1.0, 1.0),
        (1.0 + 2.0 ** -8, 1.0),                      # exact tie -> even (1.0000000)
        (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),      # exact tie -> even (1.0000010)
        (1.0 + 2.0 ** -8 + 2.0 ** -20, 1.0 + 2.0 ** -7),  # just above the tie -> up
        (2.2, 2.203125),                             # 1.0001100|11.. x2 -> 1.0001101 x2
        (-2.2, -2.203125),
        (0.4, 0.400390625),
        (3 * 2.0 ** -134, 2.0 ** -132),              # subnormal tie 1.5 q -> 2 q (even)
        (2.0 ** -134, 0.0),                          # half the smallest subnormal -> 0 (even)
        (255 * 2.0 ** 120, 255 * 2.0 ** 120),        # largest finite bf16
        (2.0 ** 128 * (1 - 2.0 ** -10), math.inf),   # rounds up past the largest -> inf
        (-0.0, -0.0),
        (0.0, 0.0),
    ]
    x = np.array([c[0] for c in cases])
    want = np.array([c[1] for c in cases])
    got = O.bf16_round(x)
    assert np.array_equal(got, want), list(zip(x, got, want))
    assert np.signbit(O.bf16_round(np.array([-0.0])))[0]


def test_bf16_round_matches_torch_on_fp32_inputs():
    # For values representable in fp32, bf16 rounding is torch's fp32 -> bf16 conversion.
    bits = RNG.integers(0, 2 ** 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    xf = bits.view(np.float32)
    xf = xf[np.isfinite(xf)]
    want = torch.from_numpy(xf.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(xf.astype(np.float64))
    assert np.array_equal(got, want)


# ----------------------------------------------------------------------------- O1 projection
def test_project_keys_hand_example():
    M = np.array([[0.5, 0.5, 0.5, 0.5], [0.5, -0.5, 0.5, -0.5]])  # orthonormal rows
    K = np.array([
        [1.0, 2.0, 3.0, 4.0],          # ->  5,    -1
        [1.5, 0.25, 3.0, -7.0],        # -> -1.125, 5.625
        [1.0, 1.0 / 128, 0.0, 0.0],    # ->  0.50390625 (exact), 0.49609375 (exact)
        [1.0, 1.0 / 256, 0.0, 0.0],    # ->  0.501953125 (tie -> 0.5), 0.498046875 (exact)
    ])
    got = O.project_keys(K, M)
    assert got[0].tolist() == [5.0, -1.0]
    assert got[1].tolist() == [-1.125, 5.625]
    assert got[2].tolist() == [0.50390625, 0.49609375]
    # 0.5*(1+1/256) = 2^-1 * 1.00000001b: a tie at 7 fraction bits -> even -> 0.5
    # 0.5*(1-1/256) = 2^-2 * 1.1111111b: representable, unchanged
    assert got[3].tolist() == [0.5, 0.498046875]


def test_project_keys_identity_rows_is_exact_copy():
    p = make_config("8b-32k", N=300, k=20, B=1)
    K = f64(p.K)
    M = f64(p.M)
    got = O.project_keys(K[0, 3], M[3])
    assert np.array_equal(got, K[0, 3][:, : p.r])


def test_qr_basis_orthonormal_and_norm_preserving():
    p = make_config("tiny")
    M = f64(p.M)[0]
    assert np.abs(M @ M.T - np.eye(p.r)).max() < 1e-6
    # A full orthonormal basis (r = d) preserves key norms up to bf16 rounding.
    pfull = make_problem(B=1, Hq=4, Hkv=1, d=64, r=64, seqlens=[256], k=8, basis="qr", seed=5)
    Mf = f64(pfull.M)[0]
    K = f64(pfull.K)[0, 0]
    kp = O.project_keys(K, Mf)
    rel = np.abs(np.linalg.norm(kp, axis=1) / np.linalg.norm(K, axis=1) - 1)
    assert rel.max() < 2 ** -8


# ----------------------------------------------------------------------------- O2/O3 scores
def test_group_mean_hand_and_special_cases():
    q = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0], [7.0, 8.0]])
    assert O.group_mean_query(q).tolist() == [4.0, 5.0]
    one = np.array([[0.25, -3.0, 7.5]])
    assert O.group_mean_query(one).tolist() == one[0].tolist()
    same = np.tile(np.array([[1.5, -2.0, 0.125]]), (8, 1))
    assert O.group_mean_query(same).tolist() == same[0].tolist()


def test_projected_score_equals_qbar_P_k():
    # s-hat = q-bar^T (M^T M) k, formed with the d x d projector, against the factored
    # (M q-bar) . (M k) the oracle evaluates.
    d, r, G = 64, 16, 4
    M = np.linalg.qr(RNG.standard_normal((d, d)))[0][:r]
    qh = RNG.standard_normal((G, d))
    K = RNG.standard_normal((50, d))
    P = M.T @ M
    qbar = qh.mean(axis=0)
    want = np.array([qbar @ P @ k for k in K])
    got = O.selection_scores(O.project_query(M, O.group_mean_query(qh)), K @ M.T, 1.0)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    # projection is idempotent: P P = P (orthonormal rows), error q-bar^T (I-P) k
    assert np.allclose(P @ P, P, atol=1e-12)
    full = np.array([qbar @ k for k in K])
    err = np.array([qbar @ (np.eye(d) - P) @ k for k in K])
    assert np.allclose(full - got, err, atol=1e-10)


def test_full_rank_basis_scores_equal_exact_scores():
    d, G = 32, 4
    M = np.linalg.qr(RNG.standard_normal((d, d)))[0]  # r = d, orthogonal
    qh = RNG.standard_normal((G, d))
    K = RNG.standard_normal((40, d))
    sigma = O.softmax_scale(d)
    got = O.selection_scores(O.project_query(M, O.group_mean_query(qh)), K @ M.T, sigma)
    want = sigma * (K @ qh.mean(axis=0))
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_gate_term_and_scale():
    assert O.softmax_scale(64) == 0.125
    assert O.softmax_scale(128) == 1 / math.sqrt(128)
    qhat = RNG.standard_normal(8)
    kp = RNG.standard_normal((30, 8))
    lg = -np.abs(RNG.standard_normal(30)) * 5
    u0 = O.selection_scores(qhat, kp, 0.3)
    u1 = O.selection_scores(qhat, kp, 0.3, lam=1.7, log_g_rows=lg)
    assert np.allclose(u1 - u0, 1.7 * lg, atol=1e-12)
    assert np.array_equal(O.selection_scores(qhat, kp, 0.3, lam=0.0, log_g_rows=lg), u0)


# ----------------------------------------------------------------------------- O4 top-k
def _topk_by_counting(keys, k):
    """Brute force: i is selected iff fewer than k positions beat it, where j beats i when
    key_j > key_i, or key_j == key_i and j < i."""
    n = len(keys)
    sel = []
    for i in range(n):
        beats = sum(1 for j in range(n) if keys[j] > keys[i] or (keys[j] == keys[i] and j < i))
        if beats < k:
            sel.append(i)
    return np.array(sel, dtype=np.int64)


@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (33, 5), (64, 64), (100, 1), (100, 99), (257, 40)])
def test_top_k_matches_counting_brute_force(n, k):
    for trial in range(5):
        # few distinct values force many exact ties
        keys = RNG.integers(-4, 5, size=n).astype(np.float32) if trial % 2 else \
            RNG.standard_normal(n).astype(np.float32)
        got = O.top_k_positions(keys, k)
        assert np.array_equal(got, _topk_by_counting(keys, k))
        assert np.all(np.diff(got) > 0)


def test_top_k_is_the_max_sum_subset_for_distinct_keys():
    for n, k in [(6, 2), (8, 3), (9, 4)]:
        keys = RNG.permutation(n).astype(np.float32) * 0.37 - 1.0
        best = max(itertools.combinations(range(n), k), key=lambda s: sum(keys[list(s)]))
        assert O.top_k_positions(keys, k).tolist() == sorted(best)


def test_top_k_special_cases():
    keys = RNG.standard_normal(50).astype(np.float32)
    assert O.top_k_positions(keys, 50).tolist() == list(range(50))
    assert O.top_k_positions(keys, 80).tolist() == list(range(50))
    assert O.top_k_positions(keys, 1).tolist() == [int(np.argmax(keys))]
    assert O.top_k_positions(keys, 0).tolist() == []
    assert O.top_k_positions(keys, -3).tolist() == []
    eq = np.full(20, 2.5, np.float32)
    assert O.top_k_positions(eq, 6).tolist() == [0, 1, 2, 3, 4, 5]
    # -inf scores lose to every finite one
    keys2 = np.array([-np.inf, 0.0, -np.inf, -1.0], np.float32)
    assert O.top_k_positions(keys2, 2).tolist() == [1, 3]


def test_decision_keys_are_fp32_roundings():
    u = np.array([1.0 + 2.0 ** -30, 1.0 + 2.0 ** -23, -3.3])
    k = O.decision_keys(u)
    assert k.dtype == np.float32
    assert k.tolist() == [1.0, float(np.float32(1.0 + 2.0 ** -23)), float(np.float32(-3.3))]


# ----------------------------------------------------------------------------- O5/O6 attention
def test_attention_matches_torch_sdpa():
    G, d, n = 4, 64, 37
    q = RNG.standard_normal((G, d))
    K = RNG.standard_normal((n, d))
    V = RNG.standard_normal((n, d))
    sigma = O.softmax_scale(d)
    got = O.sparse_attention(q, K, V, sigma)
    tq = torch.from_numpy(q)[None, :, None, :]           # [1, G, 1, d]
    tk = torch.from_numpy(K)[None, None].expand(1, G, n, d)
    tv = torch.from_numpy(V)[None, None].expand(1, G, n, d)
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=sigma)[0, :, 0].numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attention_naive_softmax_and_special_cases():
    G, d, n = 2, 16, 9
    q = RNG.standard_normal((G, d)) * 0.3
    K = RNG.standard_normal((n, d)) * 0.3
    V = RNG.standard_normal((n, d))
    sigma = 0.25
    # naive: no max subtraction (logits small)
    e = np.exp(sigma * q @ K.T)
    naive = (e / e.sum(axis=1, keepdims=True)) @ V
    assert np.allclose(O.sparse_attention(q, K, V, sigma), naive, atol=1e-13)
    # K = 0: uniform weights -> mean of V
    assert np.allclose(O.sparse_attention(q, np.zeros_like(K), V, sigma), np.tile(V.mean(0), (G, 1)))
    # one dominant logit -> that row of V
    K2 = K.copy()
    K2[4] = 200.0 * q[0] / np.linalg.norm(q[0])
    out = O.sparse_attention(q[:1], K2, V, 1.0)
    assert np.allclose(out[0], V[4], atol=1e-12)
    # gate: lambda * log g with log g ~ 0 at one position and very negative elsewhere
    lg = np.full(n, -80.0)
    lg[6] = 0.0
    out = O.sparse_attention(q, K, V, sigma, lam=1.0, log_g_sel=lg)
    assert np.allclose(out, np.tile(V[6], (G, 1)), atol=1e-12)
    # empty selection -> zeros
    assert np.array_equal(O.sparse_attention(q, K[:0], V[:0], sigma), np.zeros((G, d)))
    # permuting the query heads permutes the outputs
    perm = [1, 0]
    assert np.allclose(O.sparse_attention(q[perm], K, V, sigma), O.sparse_attention(q, K, V, sigma)[perm])
    # the order of the selected rows does not matter
    pr = RNG.permutation(n)
    assert np.allclose(O.sparse_attention(q, K[pr], V[pr], sigma), O.sparse_attention(q, K, V, sigma))


def test_full_budget_equals_dense():
    p = make_config("tiny", k=512)
    a = problem_arrays(p)
    kp = O.build_proj_cache(a["K"], a["M"], a["seqlens"])
    res = O.decode_step(a["q"], kp, a["K"], a["V"], a["M"], a["seqlens"], a["k"])
    dense = O.dense_step(a["q"], a["K"], a["V"], a["seqlens"], p.Hkv)
    idx, out, _, _ = res[(0, 0)]
    assert idx.tolist() == list(range(512))
    assert np.allclose(out, dense[(0, 0)], atol=1e-13)


def test_selection_independent_per_kv_head_and_shared_by_group():
    # Changing the queries of KV head 1 changes only head 1's set and outputs.
    p = make_problem(B=1, Hq=8, Hkv=2, d=64, r=16, seqlens=[300], k=30, seed=9)
    a = problem_arrays(p)
    kp = O.build_proj_cache(a["K"], a["M"], a["seqlens"])
    r1 = O.decode_step(a["q"], kp, a["K"], a["V"], a["M"], a["seqlens"], a["k"])
    q2 = a["q"].copy()
    q2[0, 4:8] = RNG.standard_normal((4, 64))
    r2 = O.decode_step(q2, kp, a["K"], a["V"], a["M"], a["seqlens"], a["k"])
    assert np.array_equal(r1[(0, 0)][0], r2[(0, 0)][0])
    assert np.array_equal(r1[(0, 0)][1], r2[(0, 0)][1])
    assert not np.array_equal(r1[(0, 1)][0], r2[(0, 1)][0])


def test_paged_layout_equals_contiguous_layout():
    # The same logical cache stored contiguously and in permuted 64-token pages.
    pp = make_problem(B=3, Hq=8, Hkv=2, d=64, r=16, seqlens=[130, 64, 257], k=[20, 64, 300],
                      k_max=300, paged=True, seed=3)
    a = problem_arrays(pp)
    cap = pp.cap
    Kc = np.zeros((3, 2, cap, 64))
    Vc = np.zeros((3, 2, cap, 64))
    for b in range(3):
        for h in range(2):
            n = int(a["seqlens"][b])
            Kc[b, h, :n] = O.logical_rows(a["K"], b, h, n, a["page_table"])
            Vc[b, h, :n] = O.logical_rows(a["V"], b, h, n, a["page_table"])
    kp_paged = O.build_proj_cache(a["K"], a["M"], a["seqlens"], a["page_table"])
    kp_cont = O.build_proj_cache(Kc, a["M"], a["seqlens"])
    rp = O.decode_step(a["q"], kp_paged, a["K"], a["V"], a["M"], a["seqlens"], a["k"], page_table=a["page_table"])
    rc = O.decode_step(a["q"], kp_cont, Kc, Vc, a["M"], a["seqlens"], a["k"])
    for key in rp:
        assert np.array_equal(rp[key][0], rc[key][0])
        assert np.array_equal(rp[key][1], rc[key][1])
    # k_b >= N_b selects every position
    assert rp[(1, 0)][0].tolist() == list(range(64))


# A hand-written page table over three physical 64-token pages of two KV heads.  Every
# physical slot (page, head, row) holds the number 1000*page + 100*head + row, so a value
# read back names the slot it came from.  Sequence 0 (100 tokens) lives in page 2 (tokens
# 0..63) and then page 0 (tokens 64..99); sequence 1 (10 tokens) in page 1.  The expected
# logical rows below are written out from that description, not computed by the oracle.
HAND_PAGE_TABLE = np.array([[2, 0], [1, -1]])
HAND_SEQLENS = [100, 10]


def _hand_paged_cache(width):
    cache = np.zeros((3, 2, 64, width))
    for page in range(3):
        for head in range(2):
            for row in range(64):
                cache[page, head, row, :] = 1000 * page + 100 * head + row
    # make the channels distinguishable too: channel c adds c / 8 (exact in float64)
    cache += np.arange(width)[None, None, None, :] / 8.0
    return cache


def test_paged_logical_rows_follow_a_hand_written_page_table():
    cache = _hand_paged_cache(4)
    for head in range(2):
        want0 = [2000 + 100 * head + t for t in range(64)] + [0 + 100 * head + (t - 64) for t in range(64, 100)]
        got0 = O.logical_rows(cache, 0, head, 100, HAND_PAGE_TABLE)
        assert got0.shape == (100, 4)
        assert got0[:, 0].tolist() == want0
        assert got0[:, 3].tolist() == [v + 3 / 8.0 for v in want0]
        want1 = [1000 + 100 * head + t for t in range(10)]
        assert O.logical_rows(cache, 1, head, 10, HAND_PAGE_TABLE)[:, 0].tolist() == want1
    # the contiguous layout indexes [b][h][t] directly
    cont = np.arange(2 * 2 * 5 * 1, dtype=np.float64).reshape(2, 2, 5, 1)
    assert O.logical_rows(cont, 1, 0, 3)[:, 0].tolist() == [10.0, 11.0, 12.0]


def test_paged_build_scatters_rows_to_their_physical_slots():
    # Key channels (page, head, row, 0.5) of every physical slot: small integers, exact in bf16.
    K = np.zeros((3, 2, 64, 4))
    for page in range(3):
        for head in range(2):
            for row in range(64):
                K[page, head, row] = [page, head, row, 0.5]
    # one basis per KV head picking key channels 2, 0, 1: Kproj of a slot = (row, page, head)
    M = np.stack([np.eye(4)[[2, 0, 1]]] * 2)
    kp = O.build_proj_cache(K, M, HAND_SEQLENS, HAND_PAGE_TABLE)
    assert kp.shape == (3, 2, 64, 3)
    for head in range(2):
        # sequence 0: page 2 rows 0..63 and page 0 rows 0..35 are written
        for row in range(64):
            assert kp[2, head, row].tolist() == [row, 2, head]
        for row in range(36):
            assert kp[0, head, row].tolist() == [row, 0, head]
        # sequence 1: page 1 rows 0..9
        for row in range(10):
            assert kp[1, head, row].tolist() == [row, 1, head]
        # slots no logical token maps to stay zero
        assert not kp[0, head, 36:].any()
        assert not kp[1, head, 10:].any()


# ----------------------------------------------------------------------------- calibration
def test_calibration_closed_form_for_anisotropic_keys():
    # q ~ N(0, I): E[q-bar q-bar^T] = I / G ; K = Z diag(s): E[k k^T] = diag(s^2).
    d, r, G = 128, 32, 4
    s = 0.97 ** np.arange(d)
    M = O.calibration_basis(np.eye(d) / G, np.diag(s * s), r)
    assert np.array_equal(M, np.eye(d)[:r])


def test_calibration_bound_and_optimality():
    d, r = 24, 6
    for _ in range(20):
        A = RNG.standard_normal((d, d))
        Bm = RNG.standard_normal((d, 3 * d)) * np.linspace(2, 0.1, d)[:, None]
        Gq = O.trace_normalise(A @ A.T)
        Gk = O.trace_normalise(Bm @ Bm.T)
        M = O.calibration_basis(Gq, Gk, r)
        assert np.abs(M @ M.T - np.eye(r)).max() < 1e-10
        P = M.T @ M
        lsel = O.selection_objective(P, Gq, Gk)
        lmarg = O.marginal_objective(P, Gq, Gk)
        assert 0 <= lsel <= 0.25 * lmarg ** 2 + 1e-12
        # the spectral basis minimises L_marg: no random rank-r projector does better
        for _ in range(10):
            Q = np.linalg.qr(RNG.standard_normal((d, r)))[0]
            assert lmarg <= O.marginal_objective(Q @ Q.T, Gq, Gk) + 1e-12


def test_selection_objective_closed_forms():
    # Diagonal second moments and a coordinate projector onto the set S: the error of the
    # projected score comes only from the channels outside S, L_sel = sum_{j not in S} a_j b_j,
    # and L_marg = sum_{j not in S} (a_j + b_j).
    a = np.array([3.0, 0.5, 2.0, 1.5, 0.25])
    b = np.array([1.0, 4.0, 0.5, 2.0, 8.0])
    S = [0, 2]
    P = np.diag([1.0 if j in S else 0.0 for j in range(5)])
    rest = [j for j in range(5) if j not in S]
    assert O.selection_objective(P, np.diag(a), np.diag(b)) == sum(a[j] * b[j] for j in rest)  # 0.5*4 + 1.5*2 + 0.25*8
    assert O.marginal_objective(P, np.diag(a), np.diag(b)) == sum(a[j] + b[j] for j in rest)
    # A rank-1 complement I - P = v v^T with non-diagonal moments: L_sel = (v^T Gq v)(v^T Gk v).
    # P projects on (1, 1)/sqrt 2, v = (1, -1)/sqrt 2; by hand v^T Gq v = (2 - 2 + 2)/2 = 1 and
    # v^T Gk v = (1 - 2 + 3)/2 = 1.
    Gq = np.array([[2.0, 1.0], [1.0, 2.0]])
    Gk = np.array([[1.0, 1.0], [1.0, 3.0]])
    P = np.full((2, 2), 0.5)
    assert abs(O.selection_objective(P, Gq, Gk) - 1.0) < 1e-15
    assert abs(O.marginal_objective(P, Gq, Gk) - 2.0) < 1e-15
    # and with P = e1 e1^T the complement is e2: L_sel = Gq[1,1] * Gk[1,1] = 6 (not 7, which a
    # product missing the second (I - P) factor gives)
    P = np.diag([1.0, 0.0])
    assert O.selection_objective(P, Gq, Gk) == 6.0


# ------------------------------------------------------------------ FP8 E4M3 (projected cache)
def test_e4m3_round_hand_values():
    cases = {
        0.0: 0.0, 1.0: 1.0, 1.0625: 1.0, 1.1875: 1.25,   # spacing 1/8 in [1, 2); ties to even
        17.0: 16.0, 19.0: 20.0, 18.0: 18.0,               # spacing 2 in [16, 32)
        448.0: 448.0, 500.0: 448.0, -1000.0: -448.0,      # saturation at the finite maximum
        2.0 ** -9: 2.0 ** -9, 2.0 ** -10: 0.0, 3 * 2.0 ** -10: 2.0 ** -8,  # subnormal spacing 2**-9
        0.001: 2.0 ** -9, -0.53125: -0.5,
    }
    for x, want in cases.items():
        assert O.e4m3_round(x) == want, (x, O.e4m3_round(x), want)


def test_e4m3_round_matches_torch_in_range():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 1e-1, 1.0, 30.0, 150.0)])
    x = np.clip(x, -448.0, 448.0).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e4m3_round(x.astype(np.float64)), want)


def test_project_keys_fp8_identity_rows_round_the_scaled_channels():
    rng = np.random.default_rng(6)
    K = O.bf16_round(rng.standard_normal((64, 32)))
    M = np.eye(32)[:8]
    for scale in (2.0 ** -6, 1.0, 4.0):
        codes = O.project_keys_fp8(K, M, scale)
        np.testing.assert_array_equal(codes, O.e4m3_round(K[:, :8] / scale))
        # the scored value is scale * code: within half an FP8 quantum of the true projection
        err = np.abs(scale * codes - K[:, :8])
        _, e = np.frexp(K[:, :8] / scale)
        half_q = 0.5 * scale * np.ldexp(1.0, np.maximum(e - 4, -9))
        assert np.all(err <= half_q + 1e-300)
