"""Calibration of the scoring basis M (offline, before decoding; not on the decode step).

JSSA page, sections 乘积边缘分布 / 迹归一化 / 闭式谱解 / 校准：一次前向 + 一次特征分解: from the
activations of a dense prefill, take per KV head the second moments of the group-mean query
and of the keys, normalise each to unit trace so neither marginal dominates, sum them, and keep
the eigenvectors of the r largest eigenvalues as the rows of M (orthonormal, M M^T = I_r).
Each row's largest-magnitude component is made positive (the pages fix no sign; the projector
M^T M does not depend on it).

Plain torch on the host or the device, in fp64; this is a one-off per layer, so library
matrix products and the symmetric eigensolver are used as they are.
"""
from __future__ import annotations

from typing import Optional

import torch


class MomentAccumulator:
    """Running sums of q-bar q-bar^T and k k^T per KV head (fp64)."""

    def __init__(self, Hkv: int, d: int, device="cpu"):
        self.Gq = torch.zeros(Hkv, d, d, dtype=torch.float64, device=device)
        self.Gk = torch.zeros(Hkv, d, d, dtype=torch.float64, device=device)
        self.nq = 0
        self.nk = 0

    def add_queries(self, q: torch.Tensor):
        """q: [T][Hq][d] query vectors of T positions; heads h*G .. h*G+G-1 belong to KV head h."""
        T, Hq, d = q.shape
        Hkv = self.Gq.shape[0]
        qbar = q.to(self.Gq.device, torch.float64).view(T, Hkv, Hq // Hkv, d).mean(dim=2)  # [T][Hkv][d]
        self.Gq += torch.einsum("thi,thj->hij", qbar, qbar)
        self.nq += T

    def add_keys(self, K: torch.Tensor, n: Optional[int] = None):
        """K: [Hkv][N][d] cached keys of one sequence (rows n.. are ignored when n is given)."""
        Kd = K.to(self.Gk.device, torch.float64)
        if n is not None:
            Kd = Kd[:, :n]
        self.Gk += torch.einsum("hti,htj->hij", Kd, Kd)
        self.nk += Kd.shape[1]


def scoring_basis(Gq: torch.Tensor, Gk: torch.Tensor, r: int) -> torch.Tensor:
    """M [Hkv][r][d] fp32 from second moments Gq, Gk [Hkv][d][d] (any positive scale)."""
    Gq = Gq.to(torch.float64)
    Gk = Gk.to(torch.float64)
    trq = torch.diagonal(Gq, dim1=-2, dim2=-1).sum(-1)[:, None, None]
    trk = torch.diagonal(Gk, dim1=-2, dim2=-1).sum(-1)[:, None, None]
    A = Gq / trq + Gk / trk
    A = 0.5 * (A + A.transpose(-1, -2))
    w, U = torch.linalg.eigh(A)                      # ascending eigenvalues
    order = torch.argsort(-w, dim=-1, stable=True)[:, :r]
    rows = torch.gather(U, 2, order[:, None, :].expand(-1, U.shape[1], -1)).transpose(1, 2)  # [Hkv][r][d]
    piv = torch.gather(rows, 2, rows.abs().argmax(dim=2, keepdim=True))
    rows = torch.where(piv < 0, -rows, rows)
    return rows.to(torch.float32).contiguous()


def calibrate(acc: MomentAccumulator, r: int) -> torch.Tensor:
    """The scoring basis from accumulated moments."""
    return scoring_basis(acc.Gq, acc.Gk, r)
