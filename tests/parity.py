"""GPU-vs-oracle parity runners (used by the GPU tests and by the smoke check).

The CUDA path is reached only through the C ABI (token_level_sparse_head_b200.lib); the
oracle runs on the CPU on exact copies of the same inputs.  Neither side feeds the other:
the projected cache both sides score is the oracle's own O1 output for small problems; at
full sizes each side builds its own and the test checks that they agree bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import sas_oracle as O
from tests.helpers import check_output, check_selection, f64, problem_arrays
from token_level_sparse_head_b200 import DecodeSession, lib, shape_of

SCORE_REL = 1e-5  # |u_gpu - u_oracle| <= SCORE_REL * (sigma |q-hat| |Kproj_i| + |lambda log g_i|)
BUILD_ULP_FRAC_MAX = 0.02  # share of projected elements allowed one spacing away from the exact rounding


def _unit_rows(M):
    """Every basis row is a unit coordinate vector (each projected channel copies a key channel)."""
    M = np.asarray(M)
    return bool(np.all((M == 0.0) | (M == 1.0)) and np.all(M.sum(axis=-1) == 1.0))


def bf16_ulp_diff(a, b):
    """Distance in bf16 ulps between two arrays of bf16 values (given as floats)."""
    def ordered(x):
        bits = (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.int64)
        return np.where(bits & 0x8000, 0x8000 - bits, bits + 0x8000)
    return np.abs(ordered(a) - ordered(b))


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (2**(e-8) for x = m 2**e, 0.5 <= m < 1)."""
    _, e = np.frexp(np.abs(np.asarray(x, np.float64)))
    return np.ldexp(1.0, np.maximum(e - 8, -133))


def check_build_rows(kp_g, kp_o, a, p):
    """GPU projected rows vs the oracle's correctly rounded ones.

    The kernel accumulates d products in fp32 (error at most d * 2**-24 * sum_c |M_jc K_c|)
    and rounds once (to bf16, or to E4M3 after the exact division by a power-of-two scale),
    the oracle rounds the exact sum: they may differ by that error plus one spacing."""
    mask = _rows_mask(p, a)
    Kabs = np.abs(a["K"])[mask]                         # [rows, d]
    heads = np.nonzero(mask)[1]                         # KV head of each row
    Mabs = np.abs(a["M"])[heads]                        # [rows, r, d]
    acc_bound = p.d * 2.0 ** -24 * np.einsum("nrd,nd->nr", Mabs, Kabs)
    g, o = kp_g[mask], kp_o[mask]
    sc = _scales(p)
    if sc is None:
        tol = bf16_ulp(np.maximum(np.abs(g), np.abs(o))) + 1.01 * acc_bound
    else:
        tol = e4m3_quantum(np.maximum(np.abs(g), np.abs(o))) + 1.01 * acc_bound / sc[heads][:, None]
    assert np.all(np.abs(g - o) <= tol), f"build: worst {np.max(np.abs(g - o) / tol):.3f} of bound"


def kproj_tensor(kp_np, device, fp8=False):
    """The oracle's projected cache as the library stores it: bf16 values or FP8 E4M3 codes
    (both representable exactly, so the conversion is exact)."""
    dt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(kp_np)).to(torch.float32).to(dt).to(device)


def e4m3_quantum(x):
    """Spacing of E4M3 values at |x| (2**(e-4) for x = m 2**e, 0.5 <= m < 1; 2**-9 below)."""
    _, e = np.frexp(np.abs(np.asarray(x, np.float64)))
    return np.ldexp(1.0, np.maximum(e - 4, -9))


def _scales(p):
    return None if getattr(p, "kproj_scale", None) is None else f64(p.kproj_scale)


def _rows_mask(p, a):
    """Boolean mask over the cache layout of the rows holding tokens < N_b."""
    if not p.paged:
        m = np.zeros((p.B, p.Hkv, p.n_cap), bool)
        for b in range(p.B):
            m[b, :, : int(a["seqlens"][b])] = True
        return m
    m = np.zeros((p.num_pages, p.Hkv, 64), bool)
    for b in range(p.B):
        n = int(a["seqlens"][b])
        t = np.arange(n)
        m[a["page_table"][b, t // 64], :, t % 64] = True
    return m


def u_scale(qhat, kp_rows, sigma, lam, lg_rows):
    s = sigma * np.linalg.norm(qhat) * (np.linalg.norm(kp_rows, axis=1).max() if len(kp_rows) else 0.0)
    if lam != 0.0 and lg_rows is not None and len(lg_rows):
        s += abs(lam) * np.abs(lg_rows).max()
    return s * 2.0 ** -10


def compare_head(p, a, b, h, kp_rows, idx_g, out_g, scores_g=None):
    """Compare one (b, h) of the GPU results with the oracle.  Returns #band differences."""
    n = int(a["seqlens"][b])
    G = p.Hq // p.Hkv
    d = p.d
    sigma = O.softmax_scale(d)
    kr = O.logical_rows(a["K"], b, h, n, a["page_table"])
    vr = O.logical_rows(a["V"], b, h, n, a["page_table"])
    lg = None if p.lam == 0.0 else a["log_g"][b, h, :n]
    qh = a["q"][b, h * G:(h + 1) * G]
    k_eff = max(0, min(int(a["k"][b]), n))
    idx_o, out_o, u_o, keys_o = O.decode_head(qh, a["M"][h], kp_rows, kr, vr, k_eff, p.lam, lg)
    qhat = O.project_query(a["M"][h], O.group_mean_query(qh))
    if scores_g is not None and n > 0:
        bound = sigma * np.linalg.norm(qhat) * np.linalg.norm(kp_rows, axis=1)
        if lg is not None:
            bound = bound + abs(p.lam) * np.abs(lg)
        err = np.abs(scores_g[:n] - u_o)
        assert np.all(err <= SCORE_REL * bound + 1e-30), f"scores (b={b},h={h}): worst {np.max(err / (bound + 1e-30)):.3e} rel"
    ig = np.asarray(idx_g)
    sel = ig[:k_eff]
    assert np.all(ig[k_eff:] == -1), f"padding (b={b},h={h})"
    nd = check_selection(sel, idx_o, keys_o, u_scale(qhat, kp_rows, sigma, p.lam, lg), k_eff)
    lg_sel = None if lg is None else lg[sel]
    ref = O.sparse_attention(qh, kr[sel], vr[sel], sigma, p.lam, lg_sel)
    check_output(out_g, ref, f"out (b={b},h={h})")
    if nd == 0:
        check_output(out_g, out_o, f"out vs oracle set (b={b},h={h})")
    return nd


def run_small(p_cpu, device="cuda", dense=True, check_build=True):
    """Full comparison on a problem small enough for the oracle to run entirely."""
    a = problem_arrays(p_cpu)
    sc = _scales(p_cpu)
    kp_o = O.build_proj_cache(a["K"], a["M"], a["seqlens"], a["page_table"], kproj_scale=sc)
    p = p_cpu.to(device)
    shape = shape_of(p)
    sess = DecodeSession(shape, p.k_max, device=device)
    kp_in = kproj_tensor(kp_o, device, fp8=sc is not None)
    stats = {}

    if check_build:
        kp_g = torch.zeros_like(kp_in)
        lib.sas_build_proj_cache(shape, p.K, p.M, kp_g, p.page_table, p.seqlens)
        check_build_rows(f64(kp_g), kp_o, a, p)
        ulp = bf16_ulp_diff(f64(kp_g)[_rows_mask(p, a)], kp_o[_rows_mask(p, a)])
        frac = float((ulp > 0).mean()) if ulp.size else 0.0
        stats["build_ulp_frac"] = frac
        # Elements where fp32 accumulation and the exact sum round to different neighbours: only
        # those whose exact value lies within the accumulation error of a rounding midpoint, a
        # small fraction; none at all when every basis row is a unit vector (an exact copy).
        assert frac <= BUILD_ULP_FRAC_MAX, f"build: {frac:.4f} of the elements one spacing off"
        if _unit_rows(a["M"]):
            assert frac == 0.0, "unit basis rows must copy channels exactly"

    scores = torch.full((p.B, p.Hkv, p.cap), float("nan"), dtype=torch.float32, device=device)
    idx_sel = torch.full((p.B, p.Hkv, p.k_max), -7, dtype=torch.int32, device=device)
    sess.select(p.q, p.M, kp_in, p.page_table, p.seqlens, p.k, p.lam, p.log_g, idx=idx_sel, scores=scores)
    # the two halves of the selection, called separately, give the same index lists
    idx_split = torch.full((p.B, p.Hkv, p.k_max), -7, dtype=torch.int32, device=device)
    lib.sas_score_scan(shape, p.q, p.M, kp_in, p.page_table, p.seqlens, p.k, p.k_max, p.lam, p.log_g, None,
                       sess.workspace, sess.ws_bytes)
    lib.sas_select_from_scores(shape, p.seqlens, p.k, p.k_max, idx_split, sess.workspace, sess.ws_bytes)
    out = torch.full((p.B, p.Hq, p.d), float("nan"), dtype=torch.float32, device=device)
    idx = torch.full((p.B, p.Hkv, p.k_max), -7, dtype=torch.int32, device=device)
    sess.decode(p.q, p.M, kp_in, p.K, p.V, p.page_table, p.seqlens, p.k, p.lam, p.log_g, out=out, idx=idx)
    torch.cuda.synchronize()
    st, code, where = sess.check()
    assert code == 0, f"device check error {code} at {where}"
    assert torch.equal(idx, idx_sel), "decode_step and select_topk index lists differ"
    assert torch.equal(idx, idx_split), "score_scan + select_from_scores differ from decode_step"
    sc_k = _scales(p_cpu)
    sc, ix, ot = f64(scores), f64(idx), f64(out)
    G = p.Hq // p.Hkv
    ndiff = 0
    for b in range(p.B):
        n = int(a["seqlens"][b])
        for h in range(p.Hkv):
            kp_rows = O.logical_rows(kp_o, b, h, n, a["page_table"])
            if sc_k is not None:
                kp_rows = sc_k[h] * kp_rows                 # the values the codes stand for
            ndiff += compare_head(p, a, b, h, kp_rows, ix[b, h], ot[b, h * G:(h + 1) * G], sc[b, h])
    stats["band_diffs"] = ndiff

    if dense:
        dout = torch.full((p.B, p.Hq, p.d), float("nan"), dtype=torch.float32, device=device)
        sess.dense(p.q, p.K, p.V, p.page_table, p.seqlens, out=dout)
        torch.cuda.synchronize()
        ref = O.dense_step(a["q"], a["K"], a["V"], a["seqlens"], p.Hkv, a["page_table"])
        do = f64(dout)
        for (b, h), o in ref.items():
            check_output(do[b, h * G:(h + 1) * G], o, f"dense (b={b},h={h})")
    return stats


def run_sampled(p, heads, device="cuda", dense_heads=None):
    """Full-size run: the GPU builds Kproj and runs the decode step (the launch configuration
    the benchmark times); the oracle recomputes the listed (b, h) heads from the inputs."""
    shape = shape_of(p)
    sess = DecodeSession(shape, p.k_max, device=device)
    sc = _scales(p)
    kdt = torch.bfloat16 if sc is None else torch.float8_e4m3fn
    if p.paged:
        kp = torch.zeros(p.num_pages, p.Hkv, 64, p.r, dtype=kdt, device=device)
    else:
        kp = torch.zeros(p.B, p.Hkv, p.n_cap, p.r, dtype=kdt, device=device)
    lib.sas_build_proj_cache(shape, p.K, p.M, kp, p.page_table, p.seqlens)
    out, idx = sess.decode(p.q, p.M, kp, p.K, p.V, p.page_table, p.seqlens, p.k, p.lam, p.log_g)
    torch.cuda.synchronize()
    st, code, where = sess.check()
    assert code == 0, f"device check error {code} at {where}"
    seqlens = f64(p.seqlens)
    ks = f64(p.k)
    pt = None if p.page_table is None else f64(p.page_table)
    G = p.Hq // p.Hkv
    ndiff = 0
    for b, h in heads:
        n = int(seqlens[b])
        a = _head_arrays(p, b, h, n, pt, seqlens, ks)
        kp_rows_g = _head_rows(kp, b, h, n, pt)
        acc_bound = p.d * 2.0 ** -24 * (np.abs(a["K"][0, 0, :n]) @ np.abs(a["M"][0]).T)
        if sc is None:
            kp_rows_o = O.project_keys(a["K"][0, 0, :n], a["M"][0])
            tol = bf16_ulp(np.maximum(np.abs(kp_rows_g), np.abs(kp_rows_o))) + 1.01 * acc_bound
        else:
            kp_rows_o = O.project_keys_fp8(a["K"][0, 0, :n], a["M"][0], sc[h])
            tol = e4m3_quantum(np.maximum(np.abs(kp_rows_g), np.abs(kp_rows_o))) + 1.01 * acc_bound / sc[h]
        assert np.all(np.abs(kp_rows_g - kp_rows_o) <= tol), "build rows outside the fp32 bound"
        if np.array_equal(f64(p.M[h]), np.eye(p.d)[: p.r]):
            assert np.array_equal(kp_rows_g, kp_rows_o), "identity basis must copy channels exactly"
        if sc is not None:
            kp_rows_o = sc[h] * kp_rows_o                   # the values the codes stand for
        ndiff += compare_head(_HeadView(p), a, 0, 0, kp_rows_o, f64(idx[b, h]), f64(out[b, h * G:(h + 1) * G]))
    if dense_heads:
        dout = sess.dense(p.q, p.K, p.V, p.page_table, p.seqlens, out=torch.empty_like(out))
        torch.cuda.synchronize()
        for b, h in dense_heads:
            n = int(seqlens[b])
            a = _head_arrays(p, b, h, n, pt, seqlens, ks)
            ref = O.dense_attention(a["q"][0], a["K"][0, 0, :n], a["V"][0, 0, :n], O.softmax_scale(p.d))
            check_output(f64(dout[b, h * G:(h + 1) * G]), ref, f"dense (b={b},h={h})")
    return {"band_diffs": ndiff}


class _HeadView:
    """A one-sequence, one-KV-head contiguous view of a problem (for compare_head)."""

    def __init__(self, p):
        self.B, self.Hkv, self.Hq, self.d, self.r, self.lam = 1, 1, p.Hq // p.Hkv, p.d, p.r, p.lam
        self.paged = False


def _head_rows(t, b, h, n, pt):
    if pt is None:
        return f64(t[b, h, :n])
    pages = torch.as_tensor(pt[b, np.arange(n) // 64], device=t.device)
    tt = torch.as_tensor(np.arange(n) % 64, device=t.device)
    return f64(t[pages, h, tt])


def _head_arrays(p, b, h, n, pt, seqlens, ks):
    """Exact host copies of one (b, h): q [1][G][d], K/V [1][1][n][d], M [1][r][d], log_g."""
    G = p.Hq // p.Hkv
    return dict(
        q=f64(p.q[b:b + 1, h * G:(h + 1) * G]),
        K=_head_rows(p.K, b, h, n, pt)[None, None],
        V=_head_rows(p.V, b, h, n, pt)[None, None],
        M=f64(p.M[h:h + 1]),
        seqlens=np.array([n]), k=np.array([int(ks[b])]), page_table=None,
        log_g=None if p.log_g is None else f64(p.log_g[b:b + 1, h:h + 1, :n]),
    )
