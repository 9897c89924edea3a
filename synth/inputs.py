"""Seeded synthetic inputs for one decode step of top-k sparse attention under GQA.

This module is shared by the CUDA path's tests and benchmark and by the oracle's tests.
It holds none of the method's arithmetic: it draws random numbers, shapes them into the
cache layouts, and writes the projection basis M that the workload prescribes.  Scoring,
selection and attention live elsewhere (the CUDA library and, separately, the oracle).

Workloads follow the shapes the JSSA explainer page ("JSSA 完全拆解：联合 query-key 子空间
打分与 gather-free 内核", pinghaoyang.com.cn) measures on: 8B-class GQA heads (32 query
heads, 8 KV heads, head dim 128), a rank-32 scoring basis (section 投影打分缓存与校准成本 /
缓存尺寸), and 32K-128K contexts (section 吞吐：从 32K 到 128K).  No dataset is involved:
q, K and V are Gaussian draws rounded to bfloat16, with the channel scaling below.

Every tensor gets its own torch generator, seeded from (seed, tensor name), so a tensor's
values do not depend on the order in which the others are drawn.  The same seed on a CPU
and on a CUDA device gives different values (different generator algorithms); tests that
compare the CUDA path with the oracle always hand both sides the same tensors.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field
from typing import Optional

import torch

PAGE_SIZE = 64

# Named workloads.  "k" is the per-sequence budget; for the paged workload it is N_b // 32.
CONFIGS = {
    "tiny": dict(B=1, Hq=4, Hkv=1, d=64, r=16, N=512, k=64, basis="qr", aniso=False),
    "8b-32k": dict(B=1, Hq=32, Hkv=8, d=128, r=32, N=32768, k=2048, basis="eye", aniso=True),
    "long-128k-b1": dict(B=1, Hq=32, Hkv=8, d=128, r=32, N=131072, k=4096, basis="eye", aniso=True),
    "long-128k-b16": dict(B=16, Hq=32, Hkv=8, d=128, r=32, N=131072, k=4096, basis="eye", aniso=True),
    # the same with the projected cache in FP8 E4M3 (per-KV-head power-of-two scale)
    "long-128k-b16-fp8": dict(B=16, Hq=32, Hkv=8, d=128, r=32, N=131072, k=4096, basis="eye", aniso=True,
                              kproj_fp8=True),
    "paged-b16": dict(B=16, Hq=32, Hkv=8, d=128, r=32, N=None, n_lo=8192, n_hi=131072,
                      k=None, k_div=32, basis="eye", aniso=True, paged=True),
    "gated-b4-k256": dict(B=4, Hq=32, Hkv=8, d=128, r=32, N=65536, k=256, lam=1.0, basis="eye", aniso=True),
    "gated-b4-k1024": dict(B=4, Hq=32, Hkv=8, d=128, r=32, N=65536, k=1024, lam=1.0, basis="eye", aniso=True),
    "gated-b4-k4096": dict(B=4, Hq=32, Hkv=8, d=128, r=32, N=65536, k=4096, lam=1.0, basis="eye", aniso=True),
    "gated-b4-k16384": dict(B=4, Hq=32, Hkv=8, d=128, r=32, N=65536, k=16384, lam=1.0, basis="eye", aniso=True),
}

# Channel scale of the anisotropic keys: K = Z * diag(s), s_j = 0.97**j.
ANISO_BASE = 0.97
# Selector scores behind the gate are N(0, 2) (variance 2).
GATE_SCORE_VAR = 2.0


def stream_seed(seed: int, name: str) -> int:
    """Seed of the generator stream for tensor `name` under run seed `seed`."""
    return (int(seed) * 0x9E3779B1 + zlib.crc32(name.encode())) & 0x7FFF_FFFF_FFFF_FFFF


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(seed, name))
    return g


@dataclass
class DecodeProblem:
    """All inputs of one decode step, in the library's layouts.

    Contiguous layout: K, V are [B][Hkv][n_cap][d] bf16.  Paged layout: K, V are
    [num_pages][Hkv][64][d] bf16 with page_table [B][max_pages] int32 (-1 = unused).
    M is [Hkv][r][d] fp32 with orthonormal rows.  log_g (when lam != 0) is
    [B][Hkv][cap] fp32 indexed by logical position, cap = n_cap or max_pages*64.
    """

    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    d: int
    r: int
    paged: bool
    n_cap: int
    max_pages: int
    num_pages: int
    k_max: int
    lam: float
    seqlens: torch.Tensor
    k: torch.Tensor
    q: torch.Tensor
    K: torch.Tensor
    V: torch.Tensor
    M: torch.Tensor
    page_table: Optional[torch.Tensor] = None
    log_g: Optional[torch.Tensor] = None
    kproj_scale: Optional[torch.Tensor] = None  # [Hkv] fp32 power of two (FP8 projected cache) or None
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def cap(self) -> int:
        return self.max_pages * PAGE_SIZE if self.paged else self.n_cap

    @property
    def page_size(self) -> int:
        return PAGE_SIZE if self.paged else 0

    def to(self, device) -> "DecodeProblem":
        out = DecodeProblem(**{f: getattr(self, f) for f in self.__dataclass_fields__})
        for f in ("seqlens", "k", "q", "K", "V", "M", "page_table", "log_g", "kproj_scale"):
            t = getattr(self, f)
            if t is not None:
                setattr(out, f, t.to(device))
        return out


def _qr_basis(d: int, r: int, Hkv: int, seed: int) -> torch.Tensor:
    """First r rows of the orthogonal factor of a seeded Gaussian d x d, one per KV head.

    The orthogonal factor is made unique by a positive diagonal of R.  Drawn and factored
    in fp64 on the CPU, stored as fp32.
    """
    g = _gen(seed, "M", "cpu")
    out = torch.empty(Hkv, r, d, dtype=torch.float64)
    for h in range(Hkv):
        A = torch.randn(d, d, generator=g, dtype=torch.float64)
        Q, R = torch.linalg.qr(A)
        Q = Q * torch.sign(torch.diagonal(R))[None, :]
        out[h] = Q[:r, :]
    return out.to(torch.float32)


def _eye_basis(d: int, r: int, Hkv: int) -> torch.Tensor:
    """First r rows of the identity, for every KV head.

    For the anisotropic workload this is the closed-form scoring basis: q ~ N(0, I) gives a
    group-mean second moment proportional to I, and K = Z diag(s) gives diag(s^2); after unit
    trace normalisation their sum is diagonal with strictly decreasing entries, so its top-r
    eigenvectors are the first r standard basis vectors.  (The oracle's calibration routine
    reproduces this from the moments; a CPU test checks it.)
    """
    M = torch.zeros(Hkv, r, d, dtype=torch.float32)
    for j in range(r):
        M[:, j, j] = 1.0
    return M


def _gauss_bf16(shape, seed, name, device, scale=None, chunk_rows=1 << 22):
    """N(0,1) draws (optionally times a per-channel scale) rounded to bf16, drawn in chunks.

    Chunking only bounds the fp32 staging memory; each chunk takes its own generator stream
    (name#i), so the result is reproducible for a given shape.
    """
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1, shape[-1])
    rows = flat.shape[0]
    for i, r0 in enumerate(range(0, rows, chunk_rows)):
        r1 = min(rows, r0 + chunk_rows)
        g = _gen(seed, f"{name}#{i}", device)
        z = torch.randn(r1 - r0, shape[-1], generator=g, device=device, dtype=torch.float32)
        if scale is not None:
            z.mul_(scale)
        flat[r0:r1].copy_(z)  # fp32 -> bf16, round to nearest even
    return out


def make_problem(
    *,
    B: int,
    Hq: int,
    Hkv: int,
    d: int,
    r: int,
    seqlens,
    k,
    k_max: Optional[int] = None,
    paged: bool = False,
    n_cap: Optional[int] = None,
    lam: float = 0.0,
    basis: str = "qr",
    aniso: bool = False,
    seed: int = 0,
    device="cpu",
    name: str = "custom",
    poison_tail: bool = False,
    extra_pages: int = 0,
    kproj_fp8: bool = False,
) -> DecodeProblem:
    """Build a decode problem.

    seqlens, k: per-sequence cached length N_b and budget k_b (ints or lists).
    paged: 64-token pages, page table = a seeded random permutation of all physical pages.
    poison_tail: fill cache rows at positions >= N_b (and unused gate entries) with huge
        values / NaN, so that any read past a sequence's end shows in the result.
    extra_pages: physical pages beyond those the sequences use (never referenced).
    kproj_fp8: the projected cache is stored as FP8 E4M3 codes with a per-KV-head scale:
        a power of two no smaller than max_i |K_i|_2 / 448 over the cached rows (with
        orthonormal basis rows every projected element is at most |K_i|_2, so the codes stay
        within the E4M3 range).
    """
    assert Hq % Hkv == 0
    seqlens = [int(x) for x in (seqlens if hasattr(seqlens, "__len__") else [seqlens] * B)]
    kk = [int(x) for x in (k if hasattr(k, "__len__") else [k] * B)]
    assert len(seqlens) == B and len(kk) == B
    if k_max is None:
        k_max = max(1, max(kk))
    scale = None
    if aniso:
        scale = torch.tensor([ANISO_BASE ** j for j in range(d)], dtype=torch.float32, device=device)

    q = _gauss_bf16((B, Hq, d), seed, "q", device)
    page_table = None
    if paged:
        pages_per = [(n + PAGE_SIZE - 1) // PAGE_SIZE for n in seqlens]
        max_pages = max(1, max(pages_per))
        num_pages = max(1, sum(pages_per) + extra_pages)
        g = _gen(seed, "page_perm", "cpu")
        perm = torch.randperm(num_pages, generator=g)
        pt = torch.full((B, max_pages), -1, dtype=torch.int32)
        off = 0
        for b in range(B):
            pt[b, : pages_per[b]] = perm[off: off + pages_per[b]].to(torch.int32)
            off += pages_per[b]
        page_table = pt.to(device)
        kv_shape = (num_pages, Hkv, PAGE_SIZE, d)
        n_cap_eff = 0
    else:
        max_pages = 0
        num_pages = 0
        # default capacity: the longest sequence, rounded up to a multiple of 4 rows
        n_cap_eff = int(n_cap) if n_cap is not None else (max(1, max(seqlens)) + 3) // 4 * 4
        assert n_cap_eff >= max(seqlens)
        kv_shape = (B, Hkv, n_cap_eff, d)
    K = _gauss_bf16(kv_shape, seed, "K", device, scale=scale)
    V = _gauss_bf16(kv_shape, seed, "V", device)

    if basis == "qr":
        M = _qr_basis(d, r, Hkv, seed).to(device)
    elif basis == "eye":
        M = _eye_basis(d, r, Hkv).to(device)
    else:
        raise ValueError(basis)

    cap = max_pages * PAGE_SIZE if paged else n_cap_eff
    log_g = None
    if lam != 0.0:
        # Gate input: log g = log-softmax over positions 0..N_b-1 of selector scores
        # ~ N(0, 2), per (sequence, KV head); computed in fp64, stored as fp32.
        g = _gen(seed, "gate", device)
        s = torch.randn(B, Hkv, cap, generator=g, device=device, dtype=torch.float64)
        s.mul_(math.sqrt(GATE_SCORE_VAR))
        lg = torch.full((B, Hkv, cap), float("nan") if poison_tail else -1.0e4,
                        dtype=torch.float64, device=device)
        for b in range(B):
            n = seqlens[b]
            if n > 0:
                lg[b, :, :n] = torch.log_softmax(s[b, :, :n], dim=-1)
        log_g = lg.to(torch.float32)

    if poison_tail:
        big = torch.tensor(3.0e4, dtype=torch.bfloat16)
        if paged:
            for b in range(B):
                n = seqlens[b]
                if n % PAGE_SIZE:
                    last = int(page_table[b, n // PAGE_SIZE])
                    K[last, :, n % PAGE_SIZE:, :] = big
                    V[last, :, n % PAGE_SIZE:, :] = big
        else:
            for b in range(B):
                K[b, :, seqlens[b]:, :] = big
                V[b, :, seqlens[b]:, :] = big

    kproj_scale = None
    if kproj_fp8:
        kproj_scale = torch.empty(Hkv, dtype=torch.float32)
        for h in range(Hkv):
            norm = 0.0
            for b in range(B):
                n = seqlens[b]
                if n == 0:
                    continue
                if paged:
                    t = torch.arange(n, device=device)
                    rows = K[page_table[b, t // PAGE_SIZE].long(), h, t % PAGE_SIZE]
                else:
                    rows = K[b, h, :n]
                norm = max(norm, float(rows.double().norm(dim=-1).max()))
            kproj_scale[h] = 2.0 ** math.ceil(math.log2(max(norm, 1e-30) / 448.0))
        kproj_scale = kproj_scale.to(device)

    return DecodeProblem(
        name=name, seed=seed, B=B, Hq=Hq, Hkv=Hkv, d=d, r=r, paged=paged,
        n_cap=n_cap_eff, max_pages=max_pages, num_pages=num_pages, k_max=int(k_max),
        lam=float(lam),
        seqlens=torch.tensor(seqlens, dtype=torch.int32, device=device),
        k=torch.tensor(kk, dtype=torch.int32, device=device),
        q=q, K=K, V=V, M=M, page_table=page_table, log_g=log_g, kproj_scale=kproj_scale,
    )


def make_config(name: str, seed: int = 0, device="cpu", **over) -> DecodeProblem:
    """Build one of the named workloads in CONFIGS (keyword overrides allowed)."""
    c = dict(CONFIGS[name])
    c.update(over)
    B = c["B"]
    if c.get("paged"):
        g = _gen(seed, "seqlens", "cpu")
        seqlens = torch.randint(c["n_lo"], c["n_hi"] + 1, (B,), generator=g).tolist()
        k = [n // c["k_div"] for n in seqlens]
        k_max = max(k)
    else:
        seqlens = [c["N"]] * B
        k = [c["k"]] * B
        k_max = c["k"]
    return make_problem(
        B=B, Hq=c["Hq"], Hkv=c["Hkv"], d=c["d"], r=c["r"], seqlens=seqlens, k=k, k_max=k_max,
        paged=bool(c.get("paged", False)), lam=float(c.get("lam", 0.0)), basis=c["basis"],
        aniso=bool(c["aniso"]), seed=seed, device=device, name=name,
        poison_tail=bool(c.get("poison_tail", False)), kproj_fp8=bool(c.get("kproj_fp8", False)),
    )
