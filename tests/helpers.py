"""Test helpers: tensor conversion and the comparison rules for selected sets and outputs."""
from __future__ import annotations

import numpy as np
import torch

# Output tolerance per (sequence, query head): max-abs and relative L2.
OUT_MAX_ABS = 2e-3
OUT_REL_L2 = 1e-2
# Selection band: positions whose key lies within this relative distance of the k-th key
# may differ between the two sides; exact ties go to the lower position on both.
TIE_REL = 1e-5


def f64(t):
    """Exact float64 copy of a bf16/fp32 tensor (or int64 copy of an integer tensor)."""
    if t is None:
        return None
    t = t.detach().cpu()
    if t.dtype in (torch.int32, torch.int64):
        return t.to(torch.int64).numpy()
    return t.to(torch.float64).numpy()


def problem_arrays(p):
    """The oracle's view of a synth.DecodeProblem (numpy, exact)."""
    return dict(
        q=f64(p.q), K=f64(p.K), V=f64(p.V), M=f64(p.M), seqlens=f64(p.seqlens), k=f64(p.k),
        page_table=None if p.page_table is None else f64(p.page_table),
        log_g=None if p.log_g is None else f64(p.log_g), lam=p.lam,
    )


def tie_band(keys_o, idx_o, u_scale):
    """Absolute band half-width around the oracle's k-th key."""
    if len(idx_o) == 0:
        return 0.0
    kth = float(np.min(np.asarray(keys_o, np.float64)[idx_o]))
    return TIE_REL * max(abs(kth), u_scale)


def check_selection(idx_gpu, idx_oracle, keys_oracle, u_scale, k_eff):
    """GPU set vs oracle set: equal size k_eff, ascending, distinct, in range; any difference
    only among positions whose oracle key lies inside the tie band of the k-th key.
    Returns the number of differing positions."""
    idx_gpu = np.asarray(idx_gpu, np.int64)
    idx_oracle = np.asarray(idx_oracle, np.int64)
    assert len(idx_gpu) == k_eff == len(idx_oracle), (len(idx_gpu), k_eff, len(idx_oracle))
    if k_eff == 0:
        return 0
    assert np.all(np.diff(idx_gpu) > 0), "GPU indices not strictly ascending"
    assert idx_gpu[0] >= 0 and idx_gpu[-1] < len(keys_oracle)
    sg, so = set(idx_gpu.tolist()), set(idx_oracle.tolist())
    diff = sg ^ so
    if diff:
        band = tie_band(keys_oracle, idx_oracle, u_scale)
        kth = float(np.min(np.asarray(keys_oracle, np.float64)[idx_oracle]))
        bad = [i for i in diff if abs(float(keys_oracle[i]) - kth) > band]
        assert not bad, f"selection differs outside the tie band: {bad[:8]} (kth={kth}, band={band})"
    return len(diff)


def check_output(o_gpu, o_ref, what=""):
    """Per (query head) row: max-abs <= 2e-3 and relative L2 <= 1e-2."""
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    mx = err.max(axis=-1)
    rel = np.linalg.norm(o_gpu - o_ref, axis=-1) / np.maximum(np.linalg.norm(o_ref, axis=-1), 1e-6)
    assert np.all(mx <= OUT_MAX_ABS), f"{what}: max-abs {mx.max():.3e} > {OUT_MAX_ABS}"
    assert np.all(rel <= OUT_REL_L2), f"{what}: rel-L2 {rel.max():.3e} > {OUT_REL_L2}"
    return float(mx.max()), float(rel.max())
