"""The C ABI library loads, exports every declared symbol, and validates on the host.

No call here reaches the GPU: workspace sizing is host-only, and every invalid call below is
rejected by host-side validation before any CUDA call.
"""
import os
import re

import pytest

from token_level_sparse_head_b200 import lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(sas_[a-z_]+)\s*\(", txt))
    return names


def test_library_loads_and_exports_every_declared_symbol():
    lib = L.load()
    declared = _declared_functions()
    assert "sas_decode_step" in declared and "sas_dense_decode" in declared
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(L.EXPORTED) == declared, set(L.EXPORTED) ^ declared
    hdr = open(os.path.join(ROOT, "include", "sas.h")).read()
    assert L.sas_abi_version() == int(re.search(r"#define SAS_ABI_VERSION (\d+)", hdr).group(1))


def test_workspace_sizes_are_pure_and_sane():
    s = L.Shape(16, 32, 8, 128, 32, n_cap=131072)
    a = L.sas_decode_workspace_bytes(s, 4096)
    assert a > 0 and a == L.sas_decode_workspace_bytes(s, 4096)
    assert L.sas_decode_workspace_bytes(s, 16384) >= a
    assert L.sas_dense_workspace_bytes(s) > 0
    paged = L.Shape(16, 32, 8, 128, 32, 0, 64, 2048, 17000)
    assert L.sas_decode_workspace_bytes(paged, 4096) > 0
    assert L.sas_decode_workspace_bytes(L.Shape(1, 4, 1, 96, 16, n_cap=512), 64) == 0  # d unsupported
    assert L.sas_decode_workspace_bytes(s, 0) == 0                                        # k_max < 1
    assert L.sas_decode_workspace_bytes(L.Shape(1, 6, 4, 64, 16, n_cap=512), 8) == 0      # Hq % Hkv
    assert L.sas_decode_workspace_bytes(L.Shape(1, 4, 1, 64, 16, n_cap=262148), 8) == 0   # capacity


def _expect(status, fn, *args, **kw):
    with pytest.raises(L.SasError) as e:
        fn(*args, **kw)
    assert e.value.status == status, str(e.value)


def test_host_validation_rejects_before_launch():
    s = L.Shape(1, 4, 1, 64, 16, n_cap=512)
    ws = L.sas_decode_workspace_bytes(s, 64)
    P = 1 << 20  # a 16-byte-aligned dummy address; never dereferenced (validation fails first)
    args = dict(q=P, M=P, Kproj=P, K=P, V=P, page_table=None, seqlens=P, k=P, k_max=64, lam=0.0,
                log_g=None, out=P, idx_out=P, workspace=P, ws_bytes=ws)

    def step(shape=s, **over):
        a = dict(args)
        a.update(over)
        L.sas_decode_step(shape, a["q"], a["M"], a["Kproj"], a["K"], a["V"], a["page_table"], a["seqlens"],
                          a["k"], a["k_max"], a["lam"], a["log_g"], a["out"], a["idx_out"], a["workspace"],
                          a["ws_bytes"], stream=0)

    _expect(L.SAS_ERR_UNSUPPORTED, step, L.Shape(1, 4, 1, 96, 16, n_cap=512))
    _expect(L.SAS_ERR_UNSUPPORTED, step, L.Shape(1, 4, 1, 64, 24, n_cap=512))
    _expect(L.SAS_ERR_INVALID_ARG, step, L.Shape(1, 6, 4, 64, 16, n_cap=512))
    _expect(L.SAS_ERR_INVALID_ARG, step, L.Shape(1, 4, 1, 64, 16, n_cap=510))    # n_cap % 4
    _expect(L.SAS_ERR_UNSUPPORTED, step, L.Shape(1, 4, 1, 64, 16, 0, 32, 8, 8))  # page size
    _expect(L.SAS_ERR_INVALID_ARG, step, L.Shape(1, 4, 1, 64, 16, 0, 64, 8, 8))  # paged, no table
    _expect(L.SAS_ERR_INVALID_ARG, step, k_max=0)
    _expect(L.SAS_ERR_INVALID_ARG, step, q=None)
    _expect(L.SAS_ERR_INVALID_ARG, step, K=P + 8)                                # misaligned
    _expect(L.SAS_ERR_INVALID_ARG, step, lam=1.0)                                # gate without log_g
    _expect(L.SAS_ERR_INVALID_ARG, step, ws_bytes=ws - 1)
    _expect(L.SAS_ERR_INVALID_ARG, L.sas_workspace_init, None, 1024, 0)
    with pytest.raises(L.SasError):
        L.sas_dense_decode(s, P, P, P, None, P, P, P, 16, stream=0)             # workspace too small
    with pytest.raises(L.SasError):
        L.sas_build_proj_cache(s, P, None, P, None, P, stream=0)
    with pytest.raises(L.SasError):
        L.sas_append_proj(s, P, P, P, None, None, stream=0)
