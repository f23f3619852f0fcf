"""Chunkwise Gated Linear Attention (forward + backward) for NVIDIA B200 (sm_100a).

The computation lives in the in-tree CUDA library ``libgla_b200.so`` (C ABI in
``include/gla.h``); this package is its thin Python binding.
"""
from .gla import (FLAG_REUSE_PREP, FLAG_SAVE_STATES, GLAError, alloc_workspace, build_info, gla_bwd,
                  gla_decode_step, epilogue_workspace_size, gla_epilogue_bwd, gla_epilogue_fwd, gla_fwd, gla_fwd_noalloc, load, poll_status, selftest_timeout, timing_collect,
                  timing_enable, workspace_size)

__all__ = ["FLAG_REUSE_PREP", "FLAG_SAVE_STATES", "GLAError", "alloc_workspace", "build_info", "gla_bwd",
           "gla_decode_step", "epilogue_workspace_size", "gla_epilogue_bwd", "gla_epilogue_fwd", "gla_fwd", "gla_fwd_noalloc", "load", "poll_status", "selftest_timeout",
           "timing_collect", "timing_enable", "workspace_size"]
