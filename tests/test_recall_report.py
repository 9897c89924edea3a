"""Host logic of the benchmark's selection-recall report (CPU, no kernels): the fraction of the
exact full-dimension top-k (JSSA page, appendix B.5 oracle top-k recall) that a selection keeps."""
from types import SimpleNamespace

import pytest
import torch

import bench


def _fake(idx, q, K, seqlens, ks):
    p = SimpleNamespace(paged=False, B=q.shape[0], Hq=q.shape[1], Hkv=K.shape[1], q=q, K=K)
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
