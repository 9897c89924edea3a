"""sas_decode_step_static_scratch: the decode step on the library's fixed scratch array.

The GPU test compares two calls in a row against sas_decode_step with a caller workspace on
the same inputs (same kernels, so index lists must agree exactly and outputs within the
output tolerance).  The size-limit test runs on the host only: the check happens before any
CUDA call.
"""
from __future__ import annotations

import pytest
import torch

from synth import make_problem
from tests.helpers import check_output, f64
from token_level_sparse_head_b200 import DecodeSession, lib, shape_of


def _problems():
    # 8B-shaped heads, one 32K sequence; and a ragged, paged, gated batch with multi-CTA heads
    yield make_problem(B=1, Hq=32, Hkv=8, d=128, r=32, seqlens=[32768], k=[2048], basis="eye", aniso=True,
                       seed=11, name="8b-32k-b1")
    yield make_problem(B=3, Hq=8, Hkv=2, d=128, r=32, seqlens=[40000, 777, 0], k=[1250, 777, 5], k_max=1300,
                       paged=True, lam=1.0, seed=12, name="paged-gated-ragged")


@pytest.mark.gpu
@pytest.mark.parametrize("case", [0, 1])
def test_static_scratch_matches_workspace_call(cuda_lib, case):
    p = list(_problems())[case].to("cuda")
    shape = shape_of(p)
    assert lib.sas_decode_workspace_bytes(shape, p.k_max) <= lib.STATIC_SCRATCH_BYTES
    if p.paged:
        kp = torch.zeros(p.num_pages, p.Hkv, 64, p.r, dtype=torch.bfloat16, device="cuda")
    else:
        kp = torch.zeros(p.B, p.Hkv, p.n_cap, p.r, dtype=torch.bfloat16, device="cuda")
    lib.sas_build_proj_cache(shape, p.K, p.M, kp, p.page_table, p.seqlens)

    sess = DecodeSession(shape, p.k_max, dense=False)
    out_ref = torch.full((p.B, p.Hq, p.d), float("nan"), dtype=torch.float32, device="cuda")
    idx_ref = torch.full((p.B, p.Hkv, p.k_max), -7, dtype=torch.int32, device="cuda")
    sess.decode(p.q, p.M, kp, p.K, p.V, p.page_table, p.seqlens, p.k, p.lam, p.log_g, out=out_ref, idx=idx_ref)

    results = []
    for _ in range(2):
        out = torch.full_like(out_ref, float("nan"))
        idx = torch.full_like(idx_ref, -7)
        lib.sas_decode_step_static_scratch(shape, p.q, p.M, kp, p.K, p.V, p.page_table, p.seqlens, p.k, p.k_max,
                                           p.lam, p.log_g, out, idx)
        results.append((out, idx))
    torch.cuda.synchronize()
    st, code, where = sess.check()
    assert code == 0, f"device check error {code} at {where}"

    o_ref, i_ref = f64(out_ref), f64(idx_ref)
    for n, (out, idx) in enumerate(results):
        assert torch.equal(idx, idx_ref), f"call {n}: index lists differ from sas_decode_step"
        o = f64(out)
        for b in range(p.B):
            check_output(o[b], o_ref[b], f"call {n}, sequence {b}")


def test_static_scratch_rejects_oversized_shape():
    """B=16 at 131072 tokens needs 79,823,104 bytes (76.1 MiB) of scratch: rejected on the host,
    nothing launched."""
    lib.load()
    shape = lib.Shape(16, 32, 8, 128, 32, 131072)
    need = lib.sas_decode_workspace_bytes(shape, 4096)
    assert need > lib.STATIC_SCRATCH_BYTES
    with pytest.raises(lib.SasError) as ei:
        lib.sas_decode_step_static_scratch(shape, None, None, None, None, None, None, None, None, 4096, 0.0,
                                           None, None, None, stream=0)
    assert ei.value.status == lib.SAS_ERR_UNSUPPORTED
    msg = str(ei.value)
    assert str(need) in msg and str(lib.STATIC_SCRATCH_BYTES) in msg, msg
