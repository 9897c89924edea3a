"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Small problems span several tiles, pages, stages and cluster CTAs with ragged tails; the
full-size workloads run in the benchmark's launch configuration and are checked on sampled
(sequence, KV head) pairs.  Tolerances: index sets exact except within the tie band of the
k-th key; outputs max-abs 2e-3 and relative L2 1e-2 per query head (tests/helpers.py).
"""
import numpy as np
import pytest
import torch

from synth import make_config, make_problem
from tests.parity import run_sampled, run_small

pytestmark = pytest.mark.gpu


def test_tiny(cuda_lib):
    run_small(make_config("tiny"))


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("lam", [0.0, 1.0])
def test_ragged_batch(cuda_lib, paged, lam):
    # three sequences: several stages and pages with ragged tails, one with k >= N, one N = 1
    p = make_problem(B=3, Hq=8, Hkv=2, d=128, r=32, seqlens=[5000, 777, 1], k=[300, 900, 5], k_max=900,
                     paged=paged, n_cap=None if paged else 5004, lam=lam, basis="qr", aniso=True, seed=11,
                     poison_tail=True)
    run_small(p)


@pytest.mark.parametrize("d,r,Hq,Hkv", [(64, 16, 4, 1), (64, 64, 2, 2), (64, 32, 4, 2), (128, 64, 8, 1),
                                        (128, 16, 6, 3), (128, 32, 16, 2)])
def test_head_shapes(cuda_lib, d, r, Hq, Hkv):
    p = make_problem(B=2, Hq=Hq, Hkv=Hkv, d=d, r=r, seqlens=[3001, 640], k=[257, 64], k_max=257,
                     basis="qr", seed=d + r + Hq, poison_tail=True)
    run_small(p)


@pytest.mark.parametrize("d,r,Hq,Hkv", [(64, 16, 8, 2), (128, 32, 4, 2), (128, 32, 8, 2)])
def test_split_merge_many_splits(cuda_lib, d, r, Hq, Hkv):
    # one sequence and two KV heads, so the split merge takes four CTAs per head group (a quarter
    # of the channels each); k = 6000 gives 47 sparse splits (two load steps per merge warp) and
    # the dense decode of 20000 rows more still; head groups of 4 and of 2 query heads
    p = make_problem(B=1, Hq=Hq, Hkv=Hkv, d=d, r=r, seqlens=[20000], k=[6000], basis="qr", aniso=True,
                     seed=d + Hq, poison_tail=True)
    run_small(p, check_build=False)


def test_multi_cta_clusters(cuda_lib):
    # capacity 40000 with 2 heads -> clusters of 16 CTAs; with 32 heads -> clusters of 4
    p = make_problem(B=1, Hq=8, Hkv=2, d=128, r=32, seqlens=[40000], k=[2500], basis="eye", aniso=True, seed=3)
    run_small(p, dense=False, check_build=False)
    p = make_problem(B=4, Hq=32, Hkv=8, d=128, r=32, seqlens=[5000, 4999, 2048, 64], k=[400, 1, 2048, 63],
                     k_max=2048, n_cap=5000, basis="eye", aniso=True, seed=4)
    run_small(p, dense=True, check_build=False)


def test_paged_gated_multi_cta(cuda_lib):
    p = make_problem(B=2, Hq=8, Hkv=2, d=128, r=32, seqlens=[30001, 9000], k=[1000, 281], k_max=1000,
                     paged=True, lam=1.0, basis="eye", aniso=True, seed=5, extra_pages=7, poison_tail=True)
    run_small(p, dense=True, check_build=False)


def test_edge_cases(cuda_lib):
    # N_b = 0, k_b = 0, k_b < 0, k_b > N_b, k_b == N_b, N_b = 1
    p = make_problem(B=6, Hq=4, Hkv=2, d=64, r=16, seqlens=[0, 100, 100, 50, 64, 1], k=[5, 0, -3, 80, 64, 1],
                     k_max=80, n_cap=128, basis="qr", seed=6, poison_tail=True)
    run_small(p)


def test_exact_ties_take_lowest_positions(cuda_lib):
    # every projected key equal: all scores tie, so the first k positions are selected
    p = make_problem(B=1, Hq=4, Hkv=1, d=64, r=16, seqlens=[3000], k=[700], basis="eye", seed=7)
    p.K[0, 0, :, :16] = 0.5
    p.K[0, 0, 1500:, :16] = 0.25  # second half strictly lower
    run_small(p, dense=False)


@pytest.mark.parametrize("n,k", [(512, 63), (512, 64), (512, 65), (512, 511), (512, 512), (512, 513),
                                 (511, 64), (513, 64), (512, 1), (512, 0)])
def test_selection_size_around_the_tiny_budget(cuda_lib, n, k):
    # the budget either ranks (0 < k < n), takes every position (k >= n) or takes none (k <= 0);
    # the tiny workload's k = 64, n = 512 and its neighbours, one head split over a cluster
    p = make_problem(B=1, Hq=4, Hkv=1, d=64, r=16, seqlens=[n], k=[k], k_max=max(k, 1), basis="qr", seed=n + k,
                     poison_tail=True)
    run_small(p, dense=False)


@pytest.mark.parametrize("B,Hkv,N", [(1, 2, 20000), (40, 2, 10000)])
def test_candidate_overflow_takes_the_slow_path(cuda_lib, B, Hkv, N):
    # more than 4096 keys share the k-th key's first digit (half the positions tie), so the
    # candidate list cannot hold them: clusters of CTAs per head (B=1) and one CTA per head
    # (80 heads) both fall back to re-reading the keys
    p = make_problem(B=B, Hq=2 * Hkv, Hkv=Hkv, d=64, r=16, seqlens=[N] * B, k=[700] * B, basis="eye", seed=8)
    p.K[:, :, :N // 2, :16] = 0.5
    p.K[:, :, N // 2:, :16] = 0.25
    run_small(p, dense=False)


def test_device_checks_set_the_error_word(cuda_lib):
    from token_level_sparse_head_b200 import DecodeSession, lib, shape_of

    p = make_problem(B=2, Hq=4, Hkv=1, d=64, r=16, seqlens=[100, 50], k=[10, 10], n_cap=128, seed=8).to("cuda")
    s = shape_of(p)
    sess = DecodeSession(s, p.k_max)
    kp = torch.zeros(p.B, p.Hkv, p.n_cap, p.r, dtype=torch.bfloat16, device="cuda")
    lib.sas_build_proj_cache(s, p.K, p.M, kp, None, p.seqlens)
    bad = torch.tensor([100, 129], dtype=torch.int32, device="cuda")   # 129 > capacity
    sess.decode(p.q, p.M, kp, p.K, p.V, None, bad, p.k)
    torch.cuda.synchronize()
    st, code, where = sess.check()
    assert st == lib.SAS_ERR_DEVICE_CHECK and code == 1 and where == 1
    big_k = torch.tensor([10, 11], dtype=torch.int32, device="cuda")  # 11 > k_max = 10
    sess.decode(p.q, p.M, kp, p.K, p.V, None, p.seqlens, big_k)
    torch.cuda.synchronize()
    st, code, where = sess.check()
    assert code == 4 and where == 1
    assert sess.check()[1] == 0  # cleared
    # a page id outside the physical pages
    pp = make_problem(B=1, Hq=4, Hkv=1, d=64, r=16, seqlens=[130], k=[10], paged=True, seed=9).to("cuda")
    sp = shape_of(pp)
    sess2 = DecodeSession(sp, pp.k_max)
    kp2 = torch.zeros(pp.num_pages, 1, 64, 16, dtype=torch.bfloat16, device="cuda")
    lib.sas_build_proj_cache(sp, pp.K, pp.M, kp2, pp.page_table, pp.seqlens)
    pt = pp.page_table.clone()
    pt[0, 1] = pp.num_pages + 5
    sess2.decode(pp.q, pp.M, kp2, pp.K, pp.V, pt, pp.seqlens, pp.k)
    torch.cuda.synchronize()
    assert sess2.check()[1] == 2


def test_append_matches_build(cuda_lib):
    from token_level_sparse_head_b200 import lib, shape_of

    for paged in (False, True):
        p = make_problem(B=3, Hq=8, Hkv=2, d=128, r=32, seqlens=[70, 1, 200], k=[8, 1, 8], paged=paged,
                         basis="qr", seed=12).to("cuda")
        s = shape_of(p)
        shp = (p.num_pages, p.Hkv, 64, p.r) if paged else (p.B, p.Hkv, p.n_cap, p.r)
        kp_build = torch.zeros(shp, dtype=torch.bfloat16, device="cuda")
        lib.sas_build_proj_cache(s, p.K, p.M, kp_build, p.page_table, p.seqlens)
        kp_app = kp_build.clone()
        # overwrite the last row of every sequence through the append path
        knew = torch.empty(p.B, p.Hkv, p.d, dtype=torch.bfloat16, device="cuda")
        for b in range(p.B):
            n = int(p.seqlens[b])
            for h in range(p.Hkv):
                if paged:
                    pg = int(p.page_table[b, (n - 1) // 64])
                    knew[b, h] = p.K[pg, h, (n - 1) % 64]
                    kp_app[pg, h, (n - 1) % 64] = 0
                else:
                    knew[b, h] = p.K[b, h, n - 1]
                    kp_app[b, h, n - 1] = 0
        lib.sas_append_proj(s, knew, p.M, kp_app, p.page_table, p.seqlens)
        torch.cuda.synchronize()
        assert torch.equal(kp_app, kp_build)


# ------------------------------------------------------- many heads with ragged lengths
def _many_heads_problem(paged, lam, seed, fp8=False):
    # 128 KV heads with ragged lengths, an empty sequence, N = 1, k >= N and k = 0 among them
    rng = np.random.default_rng(seed)
    seqlens = [int(x) for x in rng.integers(3000, 6000, size=16)]
    ks = [int(x) for x in rng.integers(40, 200, size=16)]
    seqlens[3], seqlens[5], seqlens[7] = 1, 150, 0
    ks[5], ks[9], ks[11] = 200, 0, 1
    return make_problem(B=16, Hq=32, Hkv=8, d=128, r=32, seqlens=seqlens, k=ks, k_max=200, paged=paged,
                        n_cap=None if paged else 6000, lam=lam, basis="eye", aniso=True, seed=seed,
                        poison_tail=True, kproj_fp8=fp8)


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("lam", [0.0, 1.0])
def test_many_heads(cuda_lib, paged, lam):
    # 128 heads: one CTA of the selection per head, scan shares spanning head boundaries
    p = _many_heads_problem(paged, lam, seed=41)
    run_small(p, dense=False, check_build=False)


def test_many_heads_fp8(cuda_lib):
    p = _many_heads_problem(False, 1.0, seed=42, fp8=True)
    run_small(p, dense=False, check_build=False)


def test_ties_and_rising_scores(cuda_lib):
    # sequence 0: every key equal, so the ties are cut by position; sequence 1: scores rising with
    # position in bf16 steps (plateaus of ties), the order a recency-biased head would show
    N = 40000
    p = make_problem(B=2, Hq=2, Hkv=1, d=64, r=16, seqlens=[N, N], k=[64, 64], basis="eye", seed=43)
    p.K[0, 0, :, :16] = 0.5
    p.K[1, 0, :, :16] = 0.0
    p.K[1, 0, :, 0] = torch.linspace(0.0, 4.0, N).to(torch.bfloat16)
    p.q[1, :, 0] = 1.0
    run_small(p, dense=False, check_build=False)


# ------------------------------------------------------------------ FP8 E4M3 projected cache
@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("lam", [0.0, 1.0])
def test_fp8_ragged_batch(cuda_lib, paged, lam):
    p = make_problem(B=3, Hq=8, Hkv=2, d=128, r=32, seqlens=[5000, 777, 1], k=[300, 900, 5], k_max=900,
                     paged=paged, n_cap=None if paged else 5004, lam=lam, basis="qr", aniso=True, seed=21,
                     poison_tail=True, kproj_fp8=True)
    run_small(p)


@pytest.mark.parametrize("d,r,Hq,Hkv", [(64, 16, 4, 1), (128, 64, 8, 2)])
def test_fp8_head_shapes(cuda_lib, d, r, Hq, Hkv):
    p = make_problem(B=2, Hq=Hq, Hkv=Hkv, d=d, r=r, seqlens=[1500, 333], k=[100, 64], basis="qr", seed=22,
                     kproj_fp8=True)
    run_small(p)


def test_fp8_append_matches_build(cuda_lib):
    from token_level_sparse_head_b200 import lib, shape_of

    for paged in (False, True):
        p = make_problem(B=3, Hq=8, Hkv=2, d=128, r=32, seqlens=[70, 1, 200], k=[8, 1, 8], paged=paged,
                         basis="qr", seed=23, kproj_fp8=True).to("cuda")
        s = shape_of(p)
        shp = (p.num_pages, p.Hkv, 64, p.r) if paged else (p.B, p.Hkv, p.n_cap, p.r)
        kp_build = torch.zeros(shp, dtype=torch.uint8, device="cuda")
        lib.sas_build_proj_cache(s, p.K, p.M, kp_build, p.page_table, p.seqlens)
        kp_app = kp_build.clone()
        knew = torch.empty(p.B, p.Hkv, p.d, dtype=torch.bfloat16, device="cuda")
        for b in range(p.B):
            n = int(p.seqlens[b])
            for h in range(p.Hkv):
                if paged:
                    pg = int(p.page_table[b, (n - 1) // 64])
                    knew[b, h] = p.K[pg, h, (n - 1) % 64]
                    kp_app[pg, h, (n - 1) % 64] = 0
                else:
                    knew[b, h] = p.K[b, h, n - 1]
                    kp_app[b, h, n - 1] = 0
        lib.sas_append_proj(s, knew, p.M, kp_app, p.page_table, p.seqlens)
        torch.cuda.synchronize()
        assert torch.equal(kp_app, kp_build)
        assert int(kp_build.count_nonzero()) > 0


# ------------------------------------------------------------- gather-then-attend (the foil)
@pytest.mark.parametrize("paged", [False, True])
def test_gather_then_dense_matches_gather_free(cuda_lib, paged):
    """Gathering the selected rows and running the dense decode over them gives the outputs of
    the gather-free attention (and of the oracle on the same rows)."""
    from oracle import sas_oracle as O
    from tests.helpers import check_output, f64
    from token_level_sparse_head_b200 import DecodeSession, lib, shape_of

    p = make_problem(B=3, Hq=8, Hkv=2, d=128, r=32, seqlens=[5000, 777, 1], k=[300, 900, 5], k_max=900,
                     paged=paged, n_cap=None if paged else 5004, basis="qr", aniso=True, seed=31).to("cuda")
    shape = shape_of(p)
    kshp = (p.num_pages, p.Hkv, 64, p.r) if paged else (p.B, p.Hkv, p.n_cap, p.r)
    kp = torch.zeros(kshp, dtype=torch.bfloat16, device="cuda")
    lib.sas_build_proj_cache(shape, p.K, p.M, kp, p.page_table, p.seqlens)
    sess = DecodeSession(shape, p.k_max)
    out_free, idx = sess.decode(p.q, p.M, kp, p.K, p.V, p.page_table, p.seqlens, p.k)
    Kg = torch.zeros(p.B, p.Hkv, p.k_max, p.d, dtype=torch.bfloat16, device="cuda")
    Vg = torch.zeros_like(Kg)
    counts = torch.full((p.B,), -1, dtype=torch.int32, device="cuda")
    lib.sas_gather_selected(shape, p.K, p.V, p.page_table, p.seqlens, idx, p.k, p.k_max, Kg, Vg, counts)
    gshape = lib.Shape(p.B, p.Hq, p.Hkv, p.d, p.r, p.k_max)
    gsess = DecodeSession(gshape, p.k_max)
    out_g = gsess.dense(p.q, Kg, Vg, None, counts, out=torch.empty_like(out_free))
    torch.cuda.synchronize()
    assert counts.tolist() == [300, 777, 1]
    G = p.Hq // p.Hkv
    of, og, ix = f64(out_free), f64(out_g), f64(idx)
    sigma = O.softmax_scale(p.d)
    for b in range(p.B):
        c = int(counts[b])
        for h in range(p.Hkv):
            sel = ix[b, h, :c]
            kr, vr = f64(Kg[b, h, :c]), f64(Vg[b, h, :c])
            ref = O.sparse_attention(f64(p.q[b, h * G:(h + 1) * G]), kr, vr, sigma)
            check_output(og[b, h * G:(h + 1) * G], ref, f"gathered (b={b},h={h})")
            check_output(of[b, h * G:(h + 1) * G], ref, f"gather-free (b={b},h={h})")
            # the gathered rows are the cache rows at the selected positions
            n = int(p.seqlens[b])
            rows = O.logical_rows(f64(p.K), b, h, n, None if p.page_table is None else f64(p.page_table))
            assert np.array_equal(kr, rows[sel])


# ------------------------------------------------------------------------ full-size workloads
def _heads(B, Hkv):
    pairs = {(0, 0), (B - 1, Hkv - 1), (B // 2, Hkv // 2)}
    return sorted(pairs)


@pytest.mark.parametrize("name", ["8b-32k", "long-128k-b1", "long-128k-b16", "paged-b16",
                                  "gated-b4-k256", "gated-b4-k1024", "gated-b4-k4096", "gated-b4-k16384",
                                  "long-128k-b16-fp8"])
def test_full_size_sampled(cuda_lib, name):
    torch.cuda.empty_cache()
    p = make_config(name, device="cuda")
    heads = _heads(p.B, p.Hkv)
    dense = heads[:1] if name in ("long-128k-b16", "8b-32k", "paged-b16") else None
    st = run_sampled(p, heads, dense_heads=dense)
    del p
    torch.cuda.empty_cache()
    assert st["band_diffs"] >= 0
