"""Plain CPU oracle for one decode step of top-k token-level sparse attention under GQA.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the tests, the smoke check and the
benchmark's CPU-baseline / reference leg may import or run this module.  The CUDA library
never calls it, and it shares no code, table or helper with the CUDA library.

Arithmetic is numpy float64 on values read exactly from the bf16 / fp32 inputs.  Each
function restates one step of the method, in the order and notation of the pages it cites:

  [JSSA]  "JSSA 完全拆解：联合 query-key 子空间打分与 gather-free 内核，训练无关的 token
          级稀疏解码" (pinghaoyang.com.cn explainer of JSSA, arXiv 2610.19026).
  [SAS]   "SAS：用门控稀疏注意力把"上下文排序"端到端对齐 LM 损失" (papers.ananclaw.com
          explainer of arXiv 2609.13141).
  [NSA-viz] "稀疏注意力：每个 query 只挑一部分历史去读" (learn-llm.fim.ai notebook).
  [Survey] "Sparse Attention · 稀疏注意力机制" (yayajjiang.github.io PaperTrace).

Readings where the pages are silent (each also listed in the design notes):
  * softmax scale sigma = 1/sqrt(d) on attention logits ([NSA-viz], selection-score
    paragraph); the same sigma multiplies the selection score so that lambda weighs the
    gate identically in selection and attention;
  * the gate lambda*log g enters both the selection key and the attention logits ([SAS] 2.1);
  * query head h belongs to KV head h // G (contiguous groups);
  * the selection decision is taken on the fp32 rounding of the fp64 score (the kernel's
    precision; the pages fix none); exact ties go to the lower position;
  * a selected set of size min(k_b, N_b); an empty set gives a zero output;
  * no sink and no forced recent window ([JSSA] 局限与需要留意的地方).

Parity pins: every function here is checked by the CPU tests against closed forms,
brute force, invariants or an independent library routine (see tests/test_oracle_pins.py).
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------------------
# bfloat16 rounding (the storage format of K, V, q and the projected cache)
# ----------------------------------------------------------------------------------------
_BF16_MAX_EXP = 128  # values at or above 2**128 after rounding overflow to infinity


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even (returned as float64).

    bfloat16 keeps 8 significant bits with the fp32 exponent range: a value with
    frexp exponent e (x = m * 2**e, 0.5 <= |m| < 1) has quantum 2**(e-8); below the normal
    range (e <= -125) the quantum stays 2**-133 (subnormals).
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    qe = np.maximum(e.astype(np.int64) - 8, -133)
    y = np.ldexp(np.rint(np.ldexp(x, -qe)), qe)  # scaling by powers of two is exact
    with np.errstate(invalid="ignore"):
        big = np.abs(y) >= np.ldexp(1.0, _BF16_MAX_EXP)
    y = np.where(big, np.copysign(np.inf, x), y)
    return y


# ----------------------------------------------------------------------------------------
# FP8 E4M3 rounding (the storage format of the FP8 projected cache)
# ----------------------------------------------------------------------------------------
E4M3_MAX = 448.0  # largest finite E4M3 value


def e4m3_round(x) -> np.ndarray:
    """Round float64 values to the nearest FP8 E4M3 value, ties to even, saturating at +-448.

    E4M3 keeps 4 significant bits with exponent bias 7: a value x = m * 2**e (0.5 <= |m| < 1)
    has quantum 2**(e-4); below the normal range the quantum stays 2**-9 (subnormals).  The
    format has no infinity; magnitudes past 448 saturate (the finite-saturating conversion).
    """
    x = np.asarray(x, np.float64)
    _, e = np.frexp(x)
    qe = np.maximum(e.astype(np.int64) - 4, -9)
    y = np.ldexp(np.rint(np.ldexp(x, -qe)), qe)  # scaling by powers of two is exact
    return np.clip(y, -E4M3_MAX, E4M3_MAX)


# ----------------------------------------------------------------------------------------
# Cache layout: logical rows of one (sequence, KV head)
# ----------------------------------------------------------------------------------------
def logical_rows(cache, b, h, n, page_table=None, page_size=64):
    """Rows 0..n-1 of sequence b, KV head h, as an [n, width] array.

    Contiguous cache: [B][Hkv][cap][width].  Paged cache: [pages][Hkv][page_size][width]
    with page_table[b][t // page_size] holding the physical page of logical token t.
    """
    if page_table is None:
        return cache[b, h, :n]
    t = np.arange(n)
    pages = np.asarray(page_table)[b, t // page_size]
    return cache[pages, h, t % page_size]


# ----------------------------------------------------------------------------------------
# O1  projected score cache  Kproj = K M^T, stored as bf16   ([JSSA] 投影打分缓存 / 3.4)
# ----------------------------------------------------------------------------------------
def project_keys(K_rows, M):
    """Kproj rows = bf16( K_rows @ M^T ): each key projected on the r basis rows of M.

    K_rows: [n, d] (bf16 values as float64); M: [r, d] with orthonormal rows.
    """
    return bf16_round(np.asarray(K_rows, np.float64) @ np.asarray(M, np.float64).T)


def project_keys_fp8(K_rows, M, scale):
    """FP8 projected rows: codes = e4m3( (K_rows @ M^T) / scale ); the value scored is
    scale * code.  ([JSSA] FP8 打分缓存的影响可以忽略: the projected cache is stored in FP8;
    the per-KV-head scale is this implementation's reading, the pages leave it open.)"""
    y = np.asarray(K_rows, np.float64) @ np.asarray(M, np.float64).T
    return e4m3_round(y / float(scale))


# ----------------------------------------------------------------------------------------
# O2  group-mean query and its projection   ([JSSA] 打分误差的定义: q-bar = (1/G) sum q_g)
# ----------------------------------------------------------------------------------------
def group_mean_query(q_heads):
    """q-bar = (1/G) * sum over the G query heads of one KV head.  q_heads: [G, d]."""
    q_heads = np.asarray(q_heads, np.float64)
    return q_heads.sum(axis=0) / q_heads.shape[0]


def project_query(M, qbar):
    """q-hat = M q-bar (the query side of s-hat = q-bar^T M^T M k)."""
    return np.asarray(M, np.float64) @ np.asarray(qbar, np.float64)


# ----------------------------------------------------------------------------------------
# O3  selection score on the projected cache, with the optional gate
#     ([JSSA] 打分误差的定义: s-hat = q-bar^T P k, P = M^T M;  [SAS] 2.1: + lambda log g_i)
# ----------------------------------------------------------------------------------------
def selection_scores(qhat, kproj_rows, sigma, lam=0.0, log_g_rows=None):
    """u_i = sigma * (q-hat . Kproj_i) + lambda * log g_i for every candidate i (all N_b)."""
    u = sigma * (np.asarray(kproj_rows, np.float64) @ np.asarray(qhat, np.float64))
    if lam != 0.0:
        u = u + lam * np.asarray(log_g_rows, np.float64)
    return u


def decision_keys(u):
    """The selection decision is taken on fp32 scores (the kernel's precision)."""
    return np.asarray(u, np.float64).astype(np.float32)


# ----------------------------------------------------------------------------------------
# O4  per-KV-head top-k   ([JSSA] JSSA 的整体结构 / Figure 1: top-k positions per KV head,
#     shared by the G query heads of that KV head)
# ----------------------------------------------------------------------------------------
def top_k_positions(keys, k):
    """Ascending positions of the k largest keys; on exact ties the lower position wins.

    Stable order of (-key, position), first min(k, n) entries, returned sorted ascending.
    """
    keys = np.asarray(keys)
    n = keys.shape[0]
    k = max(0, min(int(k), n))
    order = np.lexsort((np.arange(n), -keys.astype(np.float64)))
    return np.sort(order[:k]).astype(np.int64)


# ----------------------------------------------------------------------------------------
# O5 / O6  softmax attention on raw full-dimension K, V
#     ([JSSA] JSSA 的整体结构: final attention uses the raw full-dimension q, k, v;
#      [SAS] 2.1: logit_i = q . k_i + lambda log g_i, attn = softmax(logit))
# ----------------------------------------------------------------------------------------
def sparse_attention(q_heads, K_sel, V_sel, sigma, lam=0.0, log_g_sel=None):
    """out[g] = sum_i softmax_i(z_g)_i V_i with z_g,i = sigma q_g . K_i + lambda log g_i.

    q_heads: [G, d]; K_sel, V_sel: [k, d] rows of the selected positions (any order).
    Max-subtracted softmax in float64.  An empty selection returns zeros.
    """
    q_heads = np.asarray(q_heads, np.float64)
    K_sel = np.asarray(K_sel, np.float64)
    V_sel = np.asarray(V_sel, np.float64)
    G, d = q_heads.shape
    if K_sel.shape[0] == 0:
        return np.zeros((G, V_sel.shape[1] if V_sel.ndim == 2 else d))
    z = sigma * (q_heads @ K_sel.T)
    if lam != 0.0:
        z = z + lam * np.asarray(log_g_sel, np.float64)[None, :]
    w = np.exp(z - z.max(axis=1, keepdims=True))
    return (w @ V_sel) / w.sum(axis=1, keepdims=True)


def dense_attention(q_heads, K_rows, V_rows, sigma):
    """Full-KV decode attention over every cached row ([Survey] N(i) = all positions)."""
    return sparse_attention(q_heads, K_rows, V_rows, sigma)


# ----------------------------------------------------------------------------------------
# Whole decode step, one (sequence, KV head) at a time
# ----------------------------------------------------------------------------------------
def softmax_scale(d):
    """sigma = 1/sqrt(d)  ([NSA-viz], scores = softmax(q . k / sqrt(head_size)))."""
    return 1.0 / np.sqrt(float(d))


def decode_head(q_heads, M_h, kproj_rows, K_rows, V_rows, k, lam=0.0, log_g_rows=None):
    """One KV head of one sequence: O2 -> O3 -> O4 -> O5.

    Returns (idx ascending, out [G, d], u fp64 scores, decision keys).
    """
    d = np.asarray(q_heads).shape[1]
    sigma = softmax_scale(d)
    qbar = group_mean_query(q_heads)
    qhat = project_query(M_h, qbar)
    u = selection_scores(qhat, kproj_rows, sigma, lam, log_g_rows)
    keys = decision_keys(u)
    idx = top_k_positions(keys, k)
    lg_sel = None if lam == 0.0 else np.asarray(log_g_rows, np.float64)[idx]
    out = sparse_attention(q_heads, np.asarray(K_rows)[idx], np.asarray(V_rows)[idx], sigma, lam, lg_sel)
    return idx, out, u, keys


def decode_step(q, Kproj, K, V, M, seqlens, k, lam=0.0, log_g=None, page_table=None,
                page_size=64, heads=None, kproj_scale=None):
    """Decode step over all (or the listed) (sequence, KV head) pairs.

    Arrays are numpy (bf16 values as float64, fp32 as float64, ints as int64):
      q [B][Hq][d]; Kproj/K/V in the contiguous or paged layout (see logical_rows);
      M [Hkv][r][d]; seqlens, k [B]; log_g [B][Hkv][cap] when lam != 0.
    kproj_scale: [Hkv] for an FP8 cache (Kproj holds the codes; the scored rows are
      kproj_scale[h] * codes), None for a bf16 cache.
    heads: optional list of (b, h) pairs to evaluate (default all).
    Returns dict (b, h) -> (idx, out [G, d], u, keys).
    """
    B, Hq, d = q.shape
    Hkv = M.shape[0]
    G = Hq // Hkv
    res = {}
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in pairs:
        n = int(seqlens[b])
        kp = logical_rows(Kproj, b, h, n, page_table, page_size)
        if kproj_scale is not None:
            kp = float(kproj_scale[h]) * np.asarray(kp, np.float64)
        kr = logical_rows(K, b, h, n, page_table, page_size)
        vr = logical_rows(V, b, h, n, page_table, page_size)
        lg = None if lam == 0.0 else np.asarray(log_g)[b, h, :n]
        res[(b, h)] = decode_head(q[b, h * G:(h + 1) * G], M[h], kp, kr, vr, int(k[b]), lam, lg)
    return res


def dense_step(q, K, V, seqlens, Hkv, page_table=None, page_size=64, heads=None):
    """Dense full-KV decode over all (or the listed) (sequence, KV head) pairs -> dict of [G, d]."""
    B, Hq, d = q.shape
    G = Hq // Hkv
    sigma = softmax_scale(d)
    res = {}
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in pairs:
        n = int(seqlens[b])
        kr = logical_rows(K, b, h, n, page_table, page_size)
        vr = logical_rows(V, b, h, n, page_table, page_size)
        res[(b, h)] = dense_attention(q[b, h * G:(h + 1) * G], kr, vr, sigma)
    return res


def build_proj_cache(K, M, seqlens, page_table=None, page_size=64, heads=None, kproj_scale=None):
    """O1 over whole caches: returns a Kproj array in the layout of K (rows past N_b are 0);
    with kproj_scale ([Hkv]) the FP8 codes of project_keys_fp8 instead of bf16 values."""
    K = np.asarray(K)
    r = M.shape[1]
    out = np.zeros(K.shape[:-1] + (r,), np.float64)
    B = len(seqlens)
    Hkv = M.shape[0]
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in pairs:
        n = int(seqlens[b])
        kr = logical_rows(K, b, h, n, page_table, page_size)
        rows = project_keys(kr, M[h]) if kproj_scale is None else project_keys_fp8(kr, M[h], kproj_scale[h])
        if page_table is None:
            out[b, h, :n] = rows
        else:
            t = np.arange(n)
            out[np.asarray(page_table)[b, t // page_size], h, t % page_size] = rows
    return out


# ----------------------------------------------------------------------------------------
# Calibration of the scoring basis (offline, not on the decode step)
#     ([JSSA] 迹归一化, 精确目标与它的上界, 闭式谱解)
# ----------------------------------------------------------------------------------------
def trace_normalise(Gm):
    """G / tr(G): unit-trace second moment, so neither marginal dominates the sum."""
    Gm = np.asarray(Gm, np.float64)
    return Gm / np.trace(Gm)


def calibration_basis(G_qbar, G_k, r):
    """M* = top-r eigenvectors (as rows) of tr-normalised E[q-bar q-bar^T] + E[k k^T].

    Rows ordered by descending eigenvalue; each row's largest-magnitude component is made
    positive (the pages fix no sign; P = M^T M does not depend on it).
    """
    A = trace_normalise(G_qbar) + trace_normalise(G_k)
    A = 0.5 * (A + A.T)
    w, U = np.linalg.eigh(A)
    order = np.argsort(-w, kind="stable")[:r]
    rows = U[:, order].T.copy()
    for j in range(rows.shape[0]):
        i = int(np.argmax(np.abs(rows[j])))
        if rows[j, i] < 0:
            rows[j] = -rows[j]
    return rows


def selection_objective(P, Gq, Gk):
    """L_sel(P) = tr((I - P) Gq (I - P) Gk), the expected squared score error."""
    I = np.eye(P.shape[0])
    return float(np.trace((I - P) @ Gq @ (I - P) @ Gk))


def marginal_objective(P, Gq, Gk):
    """L_marg(P) = tr((I - P)(Gq + Gk)); the pages bound L_sel <= L_marg**2 / 4."""
    I = np.eye(P.shape[0])
    return float(np.trace((I - P) @ (Gq + Gk)))
