"""MSA (MiniMax Sparse Attention) hot path on B200: a C-ABI CUDA library
(``lib/libmsa.so``, built from ``csrc/`` for sm_100a) and a thin Python
binding.

  capi      -- ctypes calls with the C entry points' names
  pipeline  -- the five calls of one forward pass on one stream
  workloads -- seeded synthetic inputs (shared with tests and the benchmark)
"""
from . import capi, pipeline, workloads  # noqa: F401

__all__ = ["capi", "pipeline", "workloads"]
