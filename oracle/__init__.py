"""CPU float64 oracle for MLRA decode attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product package.
"""
from .mlra_oracle import (absorb, append_token, branch_probabilities, decode, decode_heads,
                          decode_multi, project, resolve_rows, rope, to_f64)

__all__ = ["decode", "decode_heads", "decode_multi", "project", "absorb", "rope", "append_token", "resolve_rows",
           "branch_probabilities", "to_f64"]
