"""B200 (sm_100a) DeepSeek Sparse Attention hot path: lightning indexer ->
per-query causal top-k -> sparse MLA attention (MQA mode), as hand-written CUDA
kernels behind the C interface in include/dsa.h.

Submodules:
  api     -- Python entry points named after the C functions (marshalling only)
  inputs  -- seeded synthetic workloads (no method arithmetic)
  build   -- in-tree nvcc build of libdsa_b200.so for sm_100a
  _lib    -- ctypes declarations of the C interface
The CUDA library is loaded on first use of an api function; a missing library
raises (there is no fallback).
"""
from . import api, inputs  # noqa: F401

__all__ = ["api", "inputs"]
