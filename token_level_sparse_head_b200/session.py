"""DecodeSession: owns the workspace for one problem shape and forwards to the C ABI.

PyTorch provides the device memory (workspace, outputs) and the stream; the library does
all the work.
"""
from __future__ import annotations

import torch

from . import lib


class DecodeSession:
    """Workspace + output buffers for repeated decode steps of one shape and budget bound."""

    def __init__(self, shape: lib.Shape, k_max: int, device="cuda", dense: bool = True):
        self.shape = shape
        self.k_max = int(k_max)
        nbytes = lib.sas_decode_workspace_bytes(shape, self.k_max)
        if dense:
            nbytes = max(nbytes, lib.sas_dense_workspace_bytes(shape))
        if nbytes == 0:
            raise ValueError("invalid shape for libsas")
        self.ws_bytes = nbytes
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        lib.sas_workspace_init(self.workspace, nbytes)
        self.out = torch.empty(shape.B, shape.Hq, shape.d, dtype=torch.float32, device=device)
        self.idx = torch.empty(shape.B, shape.Hkv, self.k_max, dtype=torch.int32, device=device)

    def decode(self, q, M, Kproj, K, V, page_table, seqlens, k, lam=0.0, log_g=None, out=None, idx=None):
        out = self.out if out is None else out
        idx = self.idx if idx is None else idx
        lib.sas_decode_step(self.shape, q, M, Kproj, K, V, page_table, seqlens, k, self.k_max, lam, log_g,
                            out, idx, self.workspace, self.ws_bytes)
        return out, idx

    def dense(self, q, K, V, page_table, seqlens, out=None):
        out = self.out if out is None else out
        lib.sas_dense_decode(self.shape, q, K, V, page_table, seqlens, out, self.workspace, self.ws_bytes)
        return out

    def select(self, q, M, Kproj, page_table, seqlens, k, lam=0.0, log_g=None, idx=None, scores=None):
        idx = self.idx if idx is None else idx
        lib.sas_select_topk(self.shape, q, M, Kproj, page_table, seqlens, k, self.k_max, lam, log_g, idx,
                            scores, self.workspace, self.ws_bytes)
        return idx

    def attend(self, q, K, V, page_table, seqlens, idx, k, lam=0.0, log_g=None, out=None):
        out = self.out if out is None else out
        lib.sas_sparse_attention(self.shape, q, K, V, page_table, seqlens, idx, k, self.k_max, lam, log_g,
                                 out, self.workspace, self.ws_bytes)
        return out

    def check(self):
        """(status, code, where) of the device-side checks since the last check (synchronises)."""
        return lib.sas_check_workspace(self.workspace, self.ws_bytes)
