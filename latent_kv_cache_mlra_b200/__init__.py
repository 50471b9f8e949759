"""B200 (sm_100a) MLRA single-token decode attention.

The work happens in libmlra.so (C ABI in include/mlra.h, CUDA kernels in csrc/); this package
is its Python binding: ``decode`` / ``Decoder`` (step 2), ``decode_multi`` (several query tokens
per sequence), ``absorb`` and ``rope_append`` (step 1), ``project`` (step 3); ``tp`` holds the
branch-parallel step.
"""
from .mlra import (Decoder, MlraError, absorb, decode, decode_multi, dims_for, make_dims, pack_wuk,
                   pack_wuv, plan_host, project, query_plan, read_status, resolve_rows,
                   rope_append, status_string, workspace_size, workspace_size_multi)

__all__ = ["Decoder", "MlraError", "decode", "decode_multi", "absorb", "pack_wuk", "project",
           "pack_wuv", "rope_append", "dims_for", "make_dims", "plan_host", "query_plan",
           "read_status", "resolve_rows", "status_string", "workspace_size", "workspace_size_multi"]
