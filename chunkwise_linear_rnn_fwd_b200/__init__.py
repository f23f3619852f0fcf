"""Chunkwise Gated Linear Attention (forward + backward) for NVIDIA B200 (sm_100a).

The computation lives in the in-tree CUDA library ``libgla_b200.so`` (C ABI in
``include/gla.h``); this package is its thin Python binding.
"""
from .gla import (GLAError, alloc_workspace, build_info, gla_bwd, gla_fwd, load, poll_status, timing_collect,
                  timing_enable, workspace_size)

__all__ = ["GLAError", "alloc_workspace", "build_info", "gla_bwd", "gla_fwd", "load", "poll_status",
           "timing_collect", "timing_enable", "workspace_size"]
