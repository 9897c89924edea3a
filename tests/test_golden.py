"""Stored fixtures under tests/golden/.

* cache_size_rule.json: a figure the JSSA page prints (FP8 projected cache = 6.25% of the bf16
  K/V cache at r = 32), checked against the byte accounting behind the benchmark's roofline.
* tiny_decode_oracle.json: the oracle's decode step on the tiny workload, written by
  tests/golden/make_golden.py (oracle only).  The CPU test guards the oracle against unintended
  change; the GPU test compares the CUDA path with the stored values.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(HERE, name)) as fh:
        return json.load(fh)


def test_cache_size_rule_matches_the_byte_accounting():
    import bench

    g = _load("cache_size_rule.json")
    N = 4096
    by = bench.roofline_bytes(B=1, Hq=4, Hkv=1, d=g["d"], r=g["r"], seqlens=[N], ks=[N], lam=0.0)
    bf16_ratio = by["kproj"] / by["kv"]                   # 2-byte projected cache, as stored here
    assert bf16_ratio == pytest.approx(g["ratio_bf16"], abs=0)
    fp8_ratio = (by["kproj"] * g["kproj_bytes_per_element_fp8"] / 2) / by["kv"]
    assert fp8_ratio == pytest.approx(g["ratio_fp8"], abs=0)


def test_oracle_reproduces_the_stored_tiny_decode():
    import importlib.util

    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    assert mg.compute() == _load("tiny_decode_oracle.json")


@pytest.mark.gpu
def test_cuda_path_matches_the_stored_tiny_decode(cuda_lib):
    import torch

    from oracle import sas_oracle as O
    from synth import make_config
    from tests.helpers import check_output
    from tests.parity import kproj_tensor
    from token_level_sparse_head_b200 import DecodeSession, shape_of

    g = _load("tiny_decode_oracle.json")
    p = make_config(g["workload"], seed=g["seed"])
    f = lambda t: t.detach().to(torch.float64).numpy()
    kp = O.build_proj_cache(f(p.K), f(p.M), p.seqlens.tolist())
    pd = p.to("cuda")
    sess = DecodeSession(shape_of(pd), pd.k_max)
    out, idx = sess.decode(pd.q, pd.M, kproj_tensor(kp, "cuda"), pd.K, pd.V, pd.page_table, pd.seqlens, pd.k)
    torch.cuda.synchronize()
    G = p.Hq // p.Hkv
    out_h, idx_h = out.cpu().double().numpy(), idx.cpu().numpy()
    for hd in g["heads"]:
        b, h = hd["b"], hd["h"]
        k_eff = len(hd["idx"])
        assert idx_h[b, h, :k_eff].tolist() == hd["idx"]
        ref = np.array([[float.fromhex(x) for x in row] for row in hd["out"]])
        check_output(out_h[b, h * G:(h + 1) * G], ref, f"tiny golden (b={b}, h={h})")
