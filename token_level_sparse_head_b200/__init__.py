"""Top-k token-level sparse GQA decode (JSSA-style) on B200: CUDA library + thin binding."""
from . import lib  # noqa: F401
from .lib import (  # noqa: F401
    Shape,
    SasError,
    shape_of,
    sas_abi_version,
    sas_append_proj,
    sas_build_proj_cache,
    sas_check_workspace,
    sas_decode_step,
    sas_decode_workspace_bytes,
    sas_dense_decode,
    sas_dense_workspace_bytes,
    sas_decode_step_static_scratch,
    sas_gather_selected,
    sas_score_scan,
    sas_select_from_scores,
    sas_select_topk,
    sas_sparse_attention,
    sas_workspace_init,
)
from .session import DecodeSession  # noqa: F401
from .calibrate import MomentAccumulator, calibrate, scoring_basis  # noqa: F401
