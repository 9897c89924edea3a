"""Host logic of the benchmark's selection-recall report (CPU, no kernels): the fraction of the
exact full-dimension top-k (JSSA page, appendix B.5 oracle top-k recall) that a selection keeps."""
from types import SimpleNamespace

import pytest
import torch

import bench


def _fake(idx, q, K, seqlens, ks, lam=0.0, log_g=None, page_table=None):
    p = SimpleNamespace(paged=page_table is not None, B=q.shape[0], Hq=q.shape[1], Hkv=K.shape[1], q=q, K=K,
                        lam=lam, log_g=log_g, page_table=page_table)
    return SimpleNamespace(p=p, sess=SimpleNamespace(idx=idx), seqlens_h=seqlens, ks_h=ks)


def _problem(seed=0, B=2, Hkv=2, G=2, N=64, d=8):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hkv * G, d, generator=g)
    K = torch.randn(B, Hkv, N, d, generator=g)
    return q, K


def _exact(q, K, b, h, G, n, k):
    qbar = q[b, h * G:(h + 1) * G].mean(0)
    return torch.argsort(K[b, h, :n] @ qbar, descending=True)[:k]


@pytest.mark.parametrize("frac", [1.0, 0.5, 0.0])
def test_recall_counts_the_kept_share_of_the_exact_top_k(frac):
    B, Hkv, G, N, k = 2, 2, 2, 64, 8
    q, K = _problem(B=B, Hkv=Hkv, G=G, N=N)
    seqlens = [N, 40]
    idx = torch.zeros(B, Hkv, k, dtype=torch.int32)
    keep = int(frac * k)
    for b in range(B):
        for h in range(Hkv):
            order = _exact(q, K, b, h, G, seqlens[b], seqlens[b])
            picked = torch.cat([order[:keep], order[k:k + (k - keep)]])   # keep of the top-k, rest outside
            idx[b, h] = picked[torch.randperm(k)].to(torch.int32)         # order inside the set is free
    r = bench.selection_recall(torch, _fake(idx, q, K, seqlens, [k, k]))
    assert r == pytest.approx(frac)


def test_recall_skips_sequences_whose_budget_covers_them():
    B, Hkv, G, N, k = 2, 1, 2, 32, 8
    q, K = _problem(B=B, Hkv=Hkv, G=G, N=N)
    idx = torch.zeros(B, Hkv, N, dtype=torch.int32)
    order = _exact(q, K, 0, 0, G, N, N)
    idx[0, 0, :k] = order[k:2 * k].to(torch.int32)                       # recall 0 on the first sequence
    idx[1, 0, :] = torch.arange(N, dtype=torch.int32)                    # k >= N_b: every row, skipped
    r = bench.selection_recall(torch, _fake(idx, q, K, [N, N], [k, N]))
    assert r == 0.0
    assert bench.selection_recall(torch, _fake(idx, q, K, [N, N], [N, N])) is None


def _paged(K, seed=1):
    """The same rows in 64-row pages [P][Hkv][64][d] under a random page permutation."""
    B, Hkv, N, d = K.shape
    per = N // 64
    perm = torch.randperm(B * per, generator=torch.Generator().manual_seed(seed))
    Kp = torch.empty(B * per, Hkv, 64, d)
    table = torch.empty(B, per, dtype=torch.int32)
    for b in range(B):
        for j in range(per):
            pg = int(perm[b * per + j])
            Kp[pg] = K[b, :, j * 64:(j + 1) * 64]
            table[b, j] = pg
    return Kp, table


def test_recall_reads_paged_rows_through_the_page_table():
    B, Hkv, G, N, k = 2, 2, 2, 256, 16
    q, K = _problem(B=B, Hkv=Hkv, G=G, N=N)
    seqlens = [N, 150]
    idx = torch.zeros(B, Hkv, k, dtype=torch.int32)
    for b in range(B):
        for h in range(Hkv):
            order = _exact(q, K, b, h, G, seqlens[b], seqlens[b])
            idx[b, h] = torch.cat([order[:k // 4], order[k:k + 3 * k // 4]]).to(torch.int32)
    Kp, table = _paged(K)
    contiguous = bench.selection_recall(torch, _fake(idx, q, K, seqlens, [k, k]))
    paged = bench.selection_recall(torch, _fake(idx, q, Kp, seqlens, [k, k], page_table=table))
    assert contiguous == pytest.approx(0.25) and paged == pytest.approx(0.25)


def test_gated_recall_ranks_the_full_dimension_key_with_the_gate():
    B, Hkv, G, N, k = 1, 1, 2, 64, 4
    q, K = _problem(B=B, Hkv=Hkv, G=G, N=N)
    log_g = torch.full((B, Hkv, N), -40.0)
    log_g[0, 0, 10:10 + k] = 0.0                      # the gate alone decides the top-k at lambda = 1
    idx = torch.arange(10, 10 + k, dtype=torch.int32).view(1, 1, k)
    wl = _fake(idx, q, K, [N], [k], lam=1.0, log_g=log_g)
    assert bench.selection_recall(torch, wl) == 1.0
    ungated = set(_exact(q, K, 0, 0, G, N, k).tolist())
    assert bench.selection_recall(torch, wl, gate=False) == pytest.approx(len(ungated & set(range(10, 14))) / k)
