"""Chunkwise Gated Linear Attention (forward + backward) for NVIDIA B200 (sm_100a).

The computation lives in the in-tree CUDA library ``libgla_b200.so`` (C ABI in
``include/gla.h``); this package is its thin Python binding.  ``seqpar`` splits one
sequence over the ranks of a torch.distributed group.
"""
from .gla import (FLAG_REUSE_PREP, FLAG_REUSE_SEGMENTS, FLAG_SAVE_STATES, GLAError, alloc_workspace, build_info,
                  epilogue_workspace_size, general_workspace_size, gla_bwd, gla_bwd_general, gla_bwd_state, gla_decode_step, gla_epilogue_bwd,
                  gla_epilogue_fwd, gla_fwd, gla_fwd_epilogue, gla_fwd_general, gla_fwd_noalloc, gla_fwd_state, gla_state_scan, load, poll_status, poll_status_noalloc,
                  selftest_timeout, timing_collect, timing_enable, workspace_size)

__all__ = ["FLAG_REUSE_PREP", "FLAG_REUSE_SEGMENTS", "FLAG_SAVE_STATES", "GLAError", "alloc_workspace", "build_info",
           "epilogue_workspace_size", "general_workspace_size", "gla_bwd", "gla_bwd_general", "gla_bwd_state", "gla_decode_step", "gla_epilogue_bwd",
           "gla_epilogue_fwd", "gla_fwd", "gla_fwd_epilogue", "gla_fwd_general", "gla_fwd_noalloc", "gla_fwd_state", "gla_state_scan", "load",
           "poll_status", "poll_status_noalloc", "selftest_timeout", "timing_collect", "timing_enable", "workspace_size"]
