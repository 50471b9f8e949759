"""B200 (sm_100a) MLRA single-token decode attention.

The work happens in libmlra.so (C ABI in include/mlra.h, CUDA kernels in csrc/); this package
is its Python binding.  See ``mlra.decode`` and ``mlra.Decoder``.
"""
from .mlra import (Decoder, MlraError, decode, dims_for, make_dims, plan_host, query_plan,
                   read_status, resolve_rows, status_string, workspace_size)

__all__ = ["Decoder", "MlraError", "decode", "dims_for", "make_dims", "plan_host", "query_plan", "read_status",
           "resolve_rows", "status_string", "workspace_size"]
