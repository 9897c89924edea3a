"""Thin Python binding of libsas (the C ABI in include/sas.h).

Argument marshalling only: every step of the decode path runs in the CUDA library.  Tensors
are passed by data pointer, the stream is the current torch CUDA stream.  The entry points
have the C names; they raise SasError on a non-OK status.  If libsas.so is missing or cannot
be loaded, every entry point raises (there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsas.so")

SAS_OK, SAS_ERR_INVALID_ARG, SAS_ERR_UNSUPPORTED, SAS_ERR_CUDA, SAS_ERR_DEVICE_CHECK = range(5)
PAGE_SIZE = 64

# Exported symbols and their C signatures (kept in step with include/sas.h).
_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t


class sas_shape(ctypes.Structure):
    _fields_ = [("B", _i32), ("Hq", _i32), ("Hkv", _i32), ("d", _i32), ("r", _i32),
                ("n_cap", _i32), ("page_size", _i32), ("max_pages", _i32), ("num_pages", _i32),
                ("kproj_dtype", _i32), ("kproj_scale", _vp)]


SAS_KPROJ_BF16, SAS_KPROJ_FP8_E4M3 = 0, 1


_SIGS = {
    "sas_abi_version": (ctypes.c_int, []),
    "sas_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sas_last_error_detail": (ctypes.c_char_p, []),
    "sas_decode_workspace_bytes": (_sz, [ctypes.POINTER(sas_shape), _i32]),
    "sas_dense_workspace_bytes": (_sz, [ctypes.POINTER(sas_shape)]),
    "sas_workspace_init": (ctypes.c_int, [_vp, _sz, _vp]),
    "sas_check_workspace": (ctypes.c_int, [_vp, _sz, _vp, ctypes.POINTER(ctypes.c_uint32),
                                           ctypes.POINTER(ctypes.c_uint32)]),
    "sas_build_proj_cache": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp]),
    "sas_append_proj": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp]),
    "sas_decode_step": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _vp, _i32, _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sas_select_topk": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                       _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sas_score_scan": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp, _i32, _f32,
                                      _vp, _vp, _vp, _sz, _vp]),
    "sas_select_from_scores": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _i32, _vp, _vp, _sz, _vp]),
    "sas_sparse_attention": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp,
                                            _vp, _i32, _f32, _vp, _vp, _vp, _sz, _vp]),
    "sas_dense_decode": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _sz, _vp]),
    "sas_decode_step_static_scratch": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp,
                                                      _vp, _vp, _i32, _f32, _vp, _vp, _vp, _vp]),
    "sas_gather_selected": (ctypes.c_int, [ctypes.POINTER(sas_shape), _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                                           _vp, _vp]),
}
STATIC_SCRATCH_BYTES = 16 << 20  # SAS_STATIC_SCRATCH_BYTES
EXPORTED = tuple(_SIGS)


class SasError(RuntimeError):
    def __init__(self, status: int, detail: str, call: str):
        super().__init__(f"{call}: status {status} ({_status_name(status)}): {detail}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsas.so (once) and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"libsas.so not built at {path}; run python -m token_level_sparse_head_b200.build")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _status_name(s: int) -> str:
    try:
        return load().sas_status_string(s).decode()
    except Exception:
        return str(s)


def _check(status: int, call: str):
    if status != SAS_OK:
        raise SasError(status, load().sas_last_error_detail().decode(), call)


def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch

    return torch.cuda.current_stream().cuda_stream


@dataclass
class Shape:
    B: int
    Hq: int
    Hkv: int
    d: int
    r: int
    n_cap: int = 0
    page_size: int = 0
    max_pages: int = 0
    num_pages: int = 0
    kproj_dtype: int = 0
    kproj_scale: Optional[object] = None  # device fp32 [Hkv] (tensor or pointer) for FP8

    def c(self) -> sas_shape:
        return sas_shape(self.B, self.Hq, self.Hkv, self.d, self.r, self.n_cap, self.page_size,
                         self.max_pages, self.num_pages, self.kproj_dtype, _p(self.kproj_scale))

    @property
    def cap(self) -> int:
        return self.max_pages * self.page_size if self.page_size else self.n_cap


def shape_of(problem) -> Shape:
    """Shape of a synth.DecodeProblem-like object (fields B, Hq, Hkv, d, r, paged, ...)."""
    scale = getattr(problem, "kproj_scale", None)
    dt = SAS_KPROJ_FP8_E4M3 if scale is not None else SAS_KPROJ_BF16
    if problem.paged:
        return Shape(problem.B, problem.Hq, problem.Hkv, problem.d, problem.r, 0, PAGE_SIZE,
                     problem.max_pages, problem.num_pages, dt, scale)
    return Shape(problem.B, problem.Hq, problem.Hkv, problem.d, problem.r, problem.n_cap, 0, 0, 0, dt, scale)


# ------------------------------------------------------------------------------ entry points
def sas_abi_version() -> int:
    return load().sas_abi_version()


def sas_decode_workspace_bytes(shape: Shape, k_max: int) -> int:
    return int(load().sas_decode_workspace_bytes(ctypes.byref(shape.c()), int(k_max)))


def sas_dense_workspace_bytes(shape: Shape) -> int:
    return int(load().sas_dense_workspace_bytes(ctypes.byref(shape.c())))


def sas_workspace_init(workspace, ws_bytes: int, stream=None):
    _check(load().sas_workspace_init(_p(workspace), int(ws_bytes), _stream(stream)), "sas_workspace_init")


def sas_check_workspace(workspace, ws_bytes: int, stream=None):
    """Returns (status, code, where); does not raise on SAS_ERR_DEVICE_CHECK."""
    code, where = ctypes.c_uint32(0), ctypes.c_uint32(0)
    s = load().sas_check_workspace(_p(workspace), int(ws_bytes), _stream(stream), ctypes.byref(code),
                                   ctypes.byref(where))
    if s not in (SAS_OK, SAS_ERR_DEVICE_CHECK):
        _check(s, "sas_check_workspace")
    return s, code.value, where.value


def sas_build_proj_cache(shape: Shape, K, M, Kproj, page_table, seqlens, stream=None):
    _check(load().sas_build_proj_cache(ctypes.byref(shape.c()), _p(K), _p(M), _p(Kproj), _p(page_table),
                                       _p(seqlens), _stream(stream)), "sas_build_proj_cache")


def sas_append_proj(shape: Shape, K_new, M, Kproj, page_table, seqlens, stream=None):
    _check(load().sas_append_proj(ctypes.byref(shape.c()), _p(K_new), _p(M), _p(Kproj), _p(page_table),
                                  _p(seqlens), _stream(stream)), "sas_append_proj")


def sas_decode_step(shape: Shape, q, M, Kproj, K, V, page_table, seqlens, k, k_max: int, lam: float,
                    log_g, out, idx_out, workspace, ws_bytes: int, stream=None):
    _check(load().sas_decode_step(ctypes.byref(shape.c()), _p(q), _p(M), _p(Kproj), _p(K), _p(V),
                                  _p(page_table), _p(seqlens), _p(k), int(k_max), float(lam), _p(log_g),
                                  _p(out), _p(idx_out), _p(workspace), int(ws_bytes), _stream(stream)),
           "sas_decode_step")


def sas_select_topk(shape: Shape, q, M, Kproj, page_table, seqlens, k, k_max: int, lam: float, log_g,
                    idx_out, scores_out, workspace, ws_bytes: int, stream=None):
    _check(load().sas_select_topk(ctypes.byref(shape.c()), _p(q), _p(M), _p(Kproj), _p(page_table),
                                  _p(seqlens), _p(k), int(k_max), float(lam), _p(log_g), _p(idx_out),
                                  _p(scores_out), _p(workspace), int(ws_bytes), _stream(stream)),
           "sas_select_topk")


def sas_score_scan(shape: Shape, q, M, Kproj, page_table, seqlens, k, k_max: int, lam: float, log_g,
                   scores_out, workspace, ws_bytes: int, stream=None):
    _check(load().sas_score_scan(ctypes.byref(shape.c()), _p(q), _p(M), _p(Kproj), _p(page_table), _p(seqlens),
                                 _p(k), int(k_max), float(lam), _p(log_g), _p(scores_out), _p(workspace),
                                 int(ws_bytes), _stream(stream)), "sas_score_scan")


def sas_select_from_scores(shape: Shape, seqlens, k, k_max: int, idx_out, workspace, ws_bytes: int,
                           stream=None):
    _check(load().sas_select_from_scores(ctypes.byref(shape.c()), _p(seqlens), _p(k), int(k_max), _p(idx_out),
                                         _p(workspace), int(ws_bytes), _stream(stream)), "sas_select_from_scores")


def sas_sparse_attention(shape: Shape, q, K, V, page_table, seqlens, idx, k, k_max: int, lam: float,
                         log_g, out, workspace, ws_bytes: int, stream=None):
    _check(load().sas_sparse_attention(ctypes.byref(shape.c()), _p(q), _p(K), _p(V), _p(page_table),
                                       _p(seqlens), _p(idx), _p(k), int(k_max), float(lam), _p(log_g),
                                       _p(out), _p(workspace), int(ws_bytes), _stream(stream)),
           "sas_sparse_attention")


def sas_dense_decode(shape: Shape, q, K, V, page_table, seqlens, out, workspace, ws_bytes: int,
                     stream=None):
    _check(load().sas_dense_decode(ctypes.byref(shape.c()), _p(q), _p(K), _p(V), _p(page_table),
                                   _p(seqlens), _p(out), _p(workspace), int(ws_bytes), _stream(stream)),
           "sas_dense_decode")


def sas_decode_step_static_scratch(shape: Shape, q, M, Kproj, K, V, page_table, seqlens, k, k_max: int,
                                   lam: float, log_g, out, idx_out, stream=None):
    """sas_decode_step on the library's fixed scratch array (no workspace argument)."""
    _check(load().sas_decode_step_static_scratch(ctypes.byref(shape.c()), _p(q), _p(M), _p(Kproj), _p(K), _p(V),
                                                 _p(page_table), _p(seqlens), _p(k), int(k_max), float(lam),
                                                 _p(log_g), _p(out), _p(idx_out), _stream(stream)),
           "sas_decode_step_static_scratch")


def sas_gather_selected(shape: Shape, K, V, page_table, seqlens, idx, k, k_max: int, Kg, Vg, counts, stream=None):
    """Copies the selected K/V rows into contiguous buffers (the gather-then-attend foil)."""
    _check(load().sas_gather_selected(ctypes.byref(shape.c()), _p(K), _p(V), _p(page_table), _p(seqlens), _p(idx),
                                      _p(k), int(k_max), _p(Kg), _p(Vg), _p(counts), _stream(stream)),
           "sas_gather_selected")
