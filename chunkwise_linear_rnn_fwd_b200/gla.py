"""Thin Python binding of the C ABI in include/gla.h (ctypes; argument marshalling only).

Every step of the computation runs in the CUDA library ``libgla_b200.so`` built
in-tree from ``csrc/``.  There is no fallback: if the library is missing or a
call fails, an exception is raised.  PyTorch is used only to own device memory
(inputs, outputs and the workspace) and to name the CUDA stream.
"""
from __future__ import annotations

import ctypes
import functools
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgla_b200.so")

GLA_OK = 0
STATUS = {
    0: "GLA_OK", -1: "GLA_ERR_INVALID_ARG", -2: "GLA_ERR_UNSUPPORTED_SHAPE", -3: "GLA_ERR_MISALIGNED",
    -4: "GLA_ERR_WORKSPACE_TOO_SMALL", -5: "GLA_ERR_CUDA", -6: "GLA_ERR_TIMEOUT", -7: "GLA_ERR_GATE_RANGE",
    -8: "GLA_ERR_NO_DEVICE",
}
DTYPE = {torch.bfloat16: 0, torch.float32: 1}
GATE = {"vector": 0, "scalar": 1, "none": 2}
VARIANT = {"auto": 0, "fused": 1, "materialized": 2}
NOALLOC_SCRATCH_BYTES = 64 << 20  # GLA_NOALLOC_SCRATCH_BYTES in include/gla.h

# Every exported symbol of include/gla.h.
EXPORTS = ["gla_workspace_size", "gla_check", "gla_fwd", "gla_bwd", "gla_poll_status", "gla_status_string",
           "gla_timing_enable", "gla_timing_collect", "gla_kernel_name", "gla_build_info", "gla_fwd_noalloc",
           "gla_decode_step", "gla_selftest_timeout", "gla_epilogue_workspace_size", "gla_epilogue_fwd",
           "gla_epilogue_bwd", "gla_fwd_state", "gla_bwd_state", "gla_state_scan", "gla_general_workspace_size",
           "gla_fwd_general", "gla_bwd_general", "gla_poll_status_noalloc", "gla_last_cuda_error",
           "gla_fwd_epilogue"]


class GLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        extra = ""
        if code == -5:  # GLA_ERR_CUDA: name the CUDA error behind it
            extra = f"; CUDA: {load().gla_last_cuda_error().decode()}"
        super().__init__(f"{where} failed: {STATUS.get(code, code)} ({status_string(code)}{extra})")


class gla_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("dk", ctypes.c_int),
                ("dv", ctypes.c_int), ("dtype", ctypes.c_int), ("gate", ctypes.c_int), ("subchunk", ctypes.c_int),
                ("variant", ctypes.c_int), ("segments", ctypes.c_int), ("flags", ctypes.c_int),
                ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgla_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run chunkwise_linear_rnn_fwd_b200/build.py)")
    lib = ctypes.CDLL(path)
    vp, i, dp = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(gla_desc)
    lib.gla_workspace_size.argtypes = [dp, i, i]
    lib.gla_workspace_size.restype = ctypes.c_size_t
    lib.gla_check.argtypes = [dp, i]
    lib.gla_check.restype = i
    lib.gla_fwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i, vp]
    lib.gla_fwd.restype = i
    lib.gla_fwd_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i, vp]
    lib.gla_fwd_noalloc.restype = i
    lib.gla_poll_status_noalloc.argtypes = [vp]
    lib.gla_poll_status_noalloc.restype = i
    lib.gla_decode_step.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp]
    lib.gla_decode_step.restype = i
    lib.gla_selftest_timeout.argtypes = [vp, ctypes.c_uint, vp]
    lib.gla_selftest_timeout.restype = i
    f = ctypes.c_float
    lib.gla_epilogue_workspace_size.argtypes = [dp]
    lib.gla_epilogue_workspace_size.restype = ctypes.c_size_t
    lib.gla_epilogue_fwd.argtypes = [dp, vp, vp, vp, vp, f, vp, vp]
    lib.gla_epilogue_fwd.restype = i
    lib.gla_fwd_epilogue.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, i, vp]
    lib.gla_fwd_epilogue.restype = i
    lib.gla_epilogue_bwd.argtypes = [dp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp, vp]
    lib.gla_epilogue_bwd.restype = i
    lib.gla_fwd_state.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i, vp]
    lib.gla_fwd_state.restype = i
    lib.gla_bwd_state.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i, vp]
    lib.gla_bwd_state.restype = i
    lib.gla_state_scan.argtypes = [dp, i, i, i, vp, vp, vp, vp, vp]
    lib.gla_state_scan.restype = i
    lib.gla_general_workspace_size.argtypes = [dp, i, i]
    lib.gla_general_workspace_size.restype = ctypes.c_size_t
    lib.gla_fwd_general.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp]
    lib.gla_fwd_general.restype = i
    lib.gla_bwd_general.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp]
    lib.gla_bwd_general.restype = i
    lib.gla_bwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp]
    lib.gla_bwd.restype = i
    lib.gla_poll_status.argtypes = [dp, vp]
    lib.gla_poll_status.restype = i
    lib.gla_status_string.argtypes = [i]
    lib.gla_status_string.restype = ctypes.c_char_p
    lib.gla_timing_enable.argtypes = [i]
    lib.gla_timing_enable.restype = i
    lib.gla_timing_collect.argtypes = [i, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float)]
    lib.gla_timing_collect.restype = i
    lib.gla_kernel_name.argtypes = [i]
    lib.gla_kernel_name.restype = ctypes.c_char_p
    lib.gla_build_info.argtypes = []
    lib.gla_build_info.restype = ctypes.c_char_p
    lib.gla_last_cuda_error.argtypes = []
    lib.gla_last_cuda_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().gla_status_string(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the GLA library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream))


def _on_stream(fn):
    """Run a binding with `stream` (keyword argument) as torch's current stream, so that
    the tensors the binding allocates (outputs the caller did not pass, a temporary
    workspace) belong to the stream the library launches on: the caching allocator
    then cannot hand a temporary workspace to other work while the kernels that use
    it are still queued on that stream."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        stream = kwargs.get("stream")
        if stream is None or stream == torch.cuda.current_stream(stream.device):
            return fn(*args, **kwargs)
        with torch.cuda.stream(stream):
            return fn(*args, **kwargs)
    return wrapper


def _gate_of(log_alpha, gate):
    if gate is not None:
        return gate
    if log_alpha is None:
        return "none"
    return "vector" if log_alpha.dim() == 4 else "scalar"


FLAG_REUSE_PREP = 1
FLAG_SAVE_STATES = 2
FLAG_REUSE_SEGMENTS = 4


def make_desc(B, H, T, dk, dv, dtype, gate, *, subchunk=16, variant="auto", segments=0, flags=0,
              workspace: Optional[torch.Tensor] = None) -> gla_desc:
    d = gla_desc()
    d.B, d.H, d.T, d.dk, d.dv = int(B), int(H), int(T), int(dk), int(dv)
    d.dtype = DTYPE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    d.gate = GATE[gate] if isinstance(gate, str) else int(gate)
    d.subchunk = int(subchunk)
    d.variant = VARIANT[variant] if isinstance(variant, str) else int(variant)
    d.segments = int(segments)
    d.flags = int(flags)
    if workspace is not None:
        d.workspace = workspace.data_ptr()
        d.workspace_bytes = workspace.numel() * workspace.element_size()
    return d


def workspace_size(B, H, T, dk, dv, dtype, gate, chunk=64, for_bwd=False, **kw) -> int:
    d = make_desc(B, H, T, dk, dv, dtype, gate, **kw)
    n = load().gla_workspace_size(ctypes.byref(d), int(chunk), int(bool(for_bwd)))
    if n == 0:
        raise GLAError(load().gla_check(ctypes.byref(d), int(chunk)), "gla_workspace_size")
    return int(n)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A caller-owned workspace (PyTorch memory, 256-byte aligned by the allocator)."""
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


@_on_stream
def gla_fwd(q, k, v, log_alpha=None, h0=None, *, chunk=64, gate=None, subchunk=16, variant="auto", segments=0,
            o=None, h_final=None, want_final=True, workspace=None, stream=None, save_states=False,
            reuse_prep=False, reuse_segments=False):
    """Forward.  Returns (o, h_final or None).  See include/gla.h.
    save_states=True: also store the bf16 chunk states in `workspace` (sized for
    the backward) for a following gla_bwd(..., saved_states=True)
    (GLA_FLAG_SAVE_STATES).  reuse_prep / reuse_segments: `workspace` holds the prep
    outputs / segment contributions of a gla_fwd_state call on the same inputs and
    flags (GLA_FLAG_REUSE_PREP, GLA_FLAG_REUSE_SEGMENTS)."""
    lib = load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_of(log_alpha, gate)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if h_final is None and want_final:
        h_final = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    flags = ((FLAG_SAVE_STATES if save_states else 0) | (FLAG_REUSE_PREP if reuse_prep else 0)
             | (FLAG_REUSE_SEGMENTS if reuse_segments else 0))
    if workspace is None:
        workspace = alloc_workspace(workspace_size(B, H, T, dk, dv, q.dtype, gate, chunk, save_states,
                                                   subchunk=subchunk, variant=variant, segments=segments,
                                                   flags=flags), q.device)
    d = make_desc(B, H, T, dk, dv, q.dtype, gate, subchunk=subchunk, variant=variant, segments=segments,
                  flags=flags, workspace=workspace)
    r = lib.gla_fwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(h0), _ptr(o), _ptr(h_final),
                    int(chunk), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_fwd")
    return o, h_final


def general_workspace_size(B, H, T, dk, dv, dtype, gate, chunk=64, for_bwd=False) -> int:
    d = make_desc(B, H, T, dk, dv, dtype, gate)
    n = load().gla_general_workspace_size(ctypes.byref(d), int(chunk), int(bool(for_bwd)))
    if n == 0:
        raise GLAError(load().gla_check(ctypes.byref(d), int(chunk)), "gla_general_workspace_size")
    return int(n)


@_on_stream
def gla_fwd_general(q, k, v, log_alpha, log_beta, h0=None, *, chunk=64, gate=None, o=None, h_final=None,
                    want_final=True, workspace=None, stream=None):
    """Forward with the general gate alpha_t^T beta_t (log_beta [B,H,T,d_v]).
    Returns (o, h_final or None).  See include/gla.h."""
    lib = load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_of(log_alpha, gate)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if h_final is None and want_final:
        h_final = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(general_workspace_size(B, H, T, dk, dv, q.dtype, gate, chunk, False), q.device)
    d = make_desc(B, H, T, dk, dv, q.dtype, gate, workspace=workspace)
    r = lib.gla_fwd_general(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(log_beta), _ptr(h0),
                            _ptr(o), _ptr(h_final), int(chunk), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_fwd_general")
    return o, h_final


@_on_stream
def gla_bwd_general(q, k, v, log_alpha, log_beta, do, h0=None, dh_final=None, *, chunk=64, gate=None,
                    want_dh0=True, workspace=None, stream=None):
    """Backward of gla_fwd_general: (dq, dk, dv, dlog_alpha or None, dlog_beta, dh0 or None)."""
    lib = load()
    B, H, T, dk_ = q.shape
    dv_ = v.shape[-1]
    gate = _gate_of(log_alpha, gate)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dla = None if gate == "none" else torch.empty_like(log_alpha)
    dlb = torch.empty_like(log_beta)
    dh0 = torch.empty(B, H, dk_, dv_, dtype=torch.float32, device=q.device) if want_dh0 else None
    if workspace is None:
        workspace = alloc_workspace(general_workspace_size(B, H, T, dk_, dv_, q.dtype, gate, chunk, True), q.device)
    d = make_desc(B, H, T, dk_, dv_, q.dtype, gate, workspace=workspace)
    r = lib.gla_bwd_general(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(log_beta), _ptr(h0),
                            _ptr(do), _ptr(dh_final), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dla), _ptr(dlb), _ptr(dh0),
                            int(chunk), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_bwd_general")
    return dq, dk, dv, dla, dlb, dh0


@_on_stream
def gla_fwd_state(q, k, v, log_alpha=None, h0=None, *, chunk=64, gate=None, subchunk=16, segments=0,
                  delta=None, gamma=None, workspace=None, stream=None, save_states=False, reuse_prep=False):
    """Summary of this piece of the sequence: (delta, gamma) = (the state after the
    piece from h0, the product of its gates per key channel).  See include/gla.h.
    save_states: use the workspace layout of gla_fwd(..., save_states=True), so that
    call can reuse the prep outputs and segment contributions left here."""
    lib = load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_of(log_alpha, gate)
    if delta is None:
        delta = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    if gamma is None:
        gamma = torch.empty(B, H, dk, dtype=torch.float32, device=q.device)
    flags = (FLAG_SAVE_STATES if save_states else 0) | (FLAG_REUSE_PREP if reuse_prep else 0)
    if workspace is None:
        workspace = alloc_workspace(workspace_size(B, H, T, dk, dv, q.dtype, gate, chunk, bool(flags),
                                                   subchunk=subchunk, segments=segments, flags=flags), q.device)
    d = make_desc(B, H, T, dk, dv, q.dtype, gate, subchunk=subchunk, segments=segments, flags=flags,
                  workspace=workspace)
    r = lib.gla_fwd_state(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(h0), _ptr(delta),
                          _ptr(gamma), int(chunk), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_fwd_state")
    return delta, gamma


@_on_stream
def gla_bwd_state(q, k, log_alpha, do, dh_final=None, *, chunk=64, gate=None, subchunk=16, segments=0,
                  ddelta=None, gamma=None, want_gamma=True, workspace=None, stream=None, reuse_prep=False):
    """Reverse summary of this piece: (ddelta, gamma or None) = (the state adjoint
    before the piece given dh_final after it, the gate product).  See include/gla.h."""
    lib = load()
    B, H, T, dk = q.shape
    dv = do.shape[-1]
    gate = _gate_of(log_alpha, gate)
    if ddelta is None:
        ddelta = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    if gamma is None and want_gamma:
        gamma = torch.empty(B, H, dk, dtype=torch.float32, device=q.device)
    flags = FLAG_REUSE_PREP if reuse_prep else 0
    if workspace is None:
        workspace = alloc_workspace(workspace_size(B, H, T, dk, dv, q.dtype, gate, chunk, True, subchunk=subchunk,
                                                   segments=segments), q.device)
    d = make_desc(B, H, T, dk, dv, q.dtype, gate, subchunk=subchunk, segments=segments, flags=flags,
                  workspace=workspace)
    r = lib.gla_bwd_state(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(log_alpha), _ptr(do), _ptr(dh_final), _ptr(ddelta),
                          _ptr(gamma), int(chunk), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_bwd_state")
    return ddelta, gamma


@_on_stream
def gla_state_scan(gammas, deltas, seg, *, reverse=False, init=None, out=None, stream=None):
    """Fold of gathered piece summaries: gammas [P,B,H,dk], deltas [P,B,H,dk,dv] fp32.
    reverse=False: the state entering piece `seg` (pieces 0 .. seg-1 over init);
    reverse=True: the adjoint leaving piece `seg` (pieces P-1 .. seg+1 over init)."""
    lib = load()
    P, B, H, dk, dv = deltas.shape
    if out is None:
        out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=deltas.device)
    d = make_desc(B, H, 1, dk, dv, torch.bfloat16, "vector")
    r = lib.gla_state_scan(ctypes.byref(d), int(P), int(seg), int(bool(reverse)), _ptr(gammas), _ptr(deltas),
                           _ptr(init), _ptr(out), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_state_scan")
    return out


@_on_stream
def gla_fwd_noalloc(q, k, v, log_alpha=None, h0=None, *, chunk=64, gate=None, subchunk=16, variant="auto",
                    segments=0, o=None, h_final=None, want_final=True, stream=None):
    """Forward without a workspace, for callers that cannot allocate device memory:
    the library uses a fixed scratch array of its own (GLA_NOALLOC_SCRATCH_BYTES,
    shared by all calls; calls must not overlap on the GPU).  Returns (o, h_final)."""
    lib = load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_of(log_alpha, gate)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if h_final is None and want_final:
        h_final = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    d = make_desc(B, H, T, dk, dv, q.dtype, gate, subchunk=subchunk, variant=variant, segments=segments)
    r = lib.gla_fwd_noalloc(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(h0), _ptr(o),
                            _ptr(h_final), int(chunk), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_fwd_noalloc")
    return o, h_final


def poll_status_noalloc(stream=None) -> int:
    """Synchronise and read/clear the status word of gla_fwd_noalloc's scratch on the
    current device (GLA_OK = 0, GLA_ERR_TIMEOUT = -6, GLA_ERR_GATE_RANGE = -7)."""
    return int(load().gla_poll_status_noalloc(_stream_handle(stream)))


@_on_stream
def gla_decode_step(q, k, v, log_alpha, state, *, gate=None, o=None, stream=None):
    """One recurrent decode step per (batch, head): state <- diag(alpha) state + k^T v
    (in place), o = q state.  q, k [B,H,d_k]; v [B,H,d_v]; log_alpha [B,H,d_k] or
    [B,H] or None; state [B,H,d_k,d_v] fp32.  Returns o [B,H,d_v].  See include/gla.h."""
    lib = load()
    B, H, dk = q.shape
    dv = v.shape[-1]
    if gate is None:
        gate = "none" if log_alpha is None else ("vector" if log_alpha.dim() == 3 else "scalar")
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    d = make_desc(B, H, 1, dk, dv, q.dtype, gate)
    r = lib.gla_decode_step(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(state), _ptr(o),
                            _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_decode_step")
    return o


def epilogue_workspace_size(B, H, T, dv, dtype) -> int:
    """Bytes of the layer epilogue's workspace (status word + dw/db partial sums)."""
    d = make_desc(B, H, T, 1, dv, dtype, "none")
    return int(load().gla_epilogue_workspace_size(ctypes.byref(d)))


@_on_stream
def gla_epilogue_fwd(o, r, w=None, b=None, *, eps=1e-5, y=None, workspace=None, stream=None):
    """y = LayerNorm(o; w, b, eps) * Swish(r) per (batch, head, token) over d_v.
    o, r [B,H,T,d_v]; w, b [d_v] fp32 or None.  See include/gla.h."""
    lib = load()
    B, H, T, dv = o.shape
    if y is None:
        y = torch.empty_like(o)
    if workspace is None:
        workspace = alloc_workspace(256, o.device)
    d = make_desc(B, H, T, 1, dv, o.dtype, "none", workspace=workspace)
    r_ = lib.gla_epilogue_fwd(ctypes.byref(d), _ptr(o), _ptr(r), _ptr(w), _ptr(b), float(eps), _ptr(y),
                              _stream_handle(stream))
    if r_ != GLA_OK:
        raise GLAError(r_, "gla_epilogue_fwd")
    return y


@_on_stream
def gla_fwd_epilogue(q, k, v, log_alpha, r, w=None, b=None, h0=None, *, eps=1e-5, chunk=64, gate=None, subchunk=16,
                     variant="auto", segments=0, o=None, y=None, h_final=None, want_final=True, workspace=None,
                     stream=None, save_states=False, reuse_prep=False):
    """Forward with the layer epilogue fused into its output store.  Returns
    (o, y, h_final or None): o and h_final as gla_fwd, y = LayerNorm(o; w, b, eps)
    * Swish(r).  r [B,H,T,d_v] like v; w, b [d_v] fp32 or None.  See include/gla.h."""
    lib = load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_of(log_alpha, gate)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if y is None:
        y = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if h_final is None and want_final:
        h_final = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    flags = (FLAG_SAVE_STATES if save_states else 0) | (FLAG_REUSE_PREP if reuse_prep else 0)
    if workspace is None:
        workspace = alloc_workspace(workspace_size(B, H, T, dk, dv, q.dtype, gate, chunk, save_states,
                                                   subchunk=subchunk, variant=variant, segments=segments,
                                                   flags=flags), q.device)
    d = make_desc(B, H, T, dk, dv, q.dtype, gate, subchunk=subchunk, variant=variant, segments=segments,
                  flags=flags, workspace=workspace)
    r_ = lib.gla_fwd_epilogue(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(h0), _ptr(r), _ptr(w),
                              _ptr(b), float(eps), _ptr(o), _ptr(y), _ptr(h_final), int(chunk), _stream_handle(stream))
    if r_ != GLA_OK:
        raise GLAError(r_, "gla_fwd_epilogue")
    return o, y, h_final


@_on_stream
def gla_epilogue_bwd(o, r, dy, w=None, b=None, *, eps=1e-5, want_dwb=True, workspace=None, stream=None):
    """Backward of gla_epilogue_fwd: (do, dr, dw or None, db or None)."""
    lib = load()
    B, H, T, dv = o.shape
    do_, dr = torch.empty_like(o), torch.empty_like(r)
    dw = db = None
    if want_dwb:
        dw = torch.empty(dv, dtype=torch.float32, device=o.device)
        db = torch.empty(dv, dtype=torch.float32, device=o.device)
    if workspace is None:
        workspace = alloc_workspace(epilogue_workspace_size(B, H, T, dv, o.dtype) if want_dwb else 256, o.device)
    d = make_desc(B, H, T, 1, dv, o.dtype, "none", workspace=workspace)
    r_ = lib.gla_epilogue_bwd(ctypes.byref(d), _ptr(o), _ptr(r), _ptr(w), _ptr(b), float(eps), _ptr(dy), _ptr(do_),
                              _ptr(dr), _ptr(dw), _ptr(db), _stream_handle(stream))
    if r_ != GLA_OK:
        raise GLAError(r_, "gla_epilogue_bwd")
    return do_, dr, dw, db


@_on_stream
def gla_bwd(q, k, v, log_alpha, do, h0=None, dh_final=None, *, chunk=64, gate=None, subchunk=16, dq=None, dk=None,
            dv=None, dlog_alpha=None, dh0=None, want_dh0=True, workspace=None, stream=None, reuse_prep=False,
            saved_states=False, reuse_segments=False, segments=0, variant="auto"):
    """Backward.  Returns (dq, dk, dv, dlog_alpha or None, dh0 or None).  See include/gla.h.
    reuse_prep=True: `workspace` holds the prep outputs of a gla_fwd call on the same
    inputs with this workspace (GLA_FLAG_REUSE_PREP).  saved_states=True: it also
    holds the chunk states of a gla_fwd(..., save_states=True) call with the same
    segments and variant (GLA_FLAG_SAVE_STATES).  reuse_segments=True: it holds the
    segment contributions of a gla_bwd_state call (GLA_FLAG_REUSE_SEGMENTS)."""
    lib = load()
    B, H, T, dk_ = q.shape
    dv_ = v.shape[-1]
    gate = _gate_of(log_alpha, gate)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if dlog_alpha is None and gate != "none":
        dlog_alpha = torch.empty_like(log_alpha)
    if dh0 is None and want_dh0:
        dh0 = torch.empty(B, H, dk_, dv_, dtype=torch.float32, device=q.device)
    flags = ((FLAG_REUSE_PREP if reuse_prep else 0) | (FLAG_SAVE_STATES if saved_states else 0)
             | (FLAG_REUSE_SEGMENTS if reuse_segments else 0))
    if workspace is None:
        workspace = alloc_workspace(workspace_size(B, H, T, dk_, dv_, q.dtype, gate, chunk, True, subchunk=subchunk,
                                                   segments=segments, variant=variant, flags=flags), q.device)
    d = make_desc(B, H, T, dk_, dv_, q.dtype, gate, subchunk=subchunk, variant=variant, segments=segments,
                  workspace=workspace, flags=flags)
    r = lib.gla_bwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(h0), _ptr(do), _ptr(dh_final),
                    _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlog_alpha), _ptr(dh0), int(chunk), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_bwd")
    return dq, dk, dv, dlog_alpha, dh0


def poll_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and read/clear the device status word of a workspace (GLA_OK = 0)."""
    d = gla_desc()
    d.workspace = workspace.data_ptr()
    d.workspace_bytes = workspace.numel()
    return int(load().gla_poll_status(ctypes.byref(d), _stream_handle(stream)))


def selftest_timeout(workspace: torch.Tensor, limit_us: int = 20000, stream=None) -> None:
    """Enqueue the bounded-wait self-test: a kernel whose wait on an mbarrier that
    nothing completes runs out after limit_us and sets the timeout bit of the status
    word at the start of `workspace` (read it with poll_status)."""
    r = load().gla_selftest_timeout(ctypes.c_void_p(workspace.data_ptr()), int(limit_us), _stream_handle(stream))
    if r != GLA_OK:
        raise GLAError(r, "gla_selftest_timeout")


def timing_enable(on: bool = True) -> None:
    load().gla_timing_enable(int(bool(on)))


def timing_collect(max_launches: int = 65536):
    """[(kernel_name, ms), ...] for the launches recorded since the last collect."""
    lib = load()
    ids = (ctypes.c_int * max_launches)()
    ms = (ctypes.c_float * max_launches)()
    n = lib.gla_timing_collect(max_launches, ids, ms)
    return [(lib.gla_kernel_name(ids[i]).decode(), float(ms[i])) for i in range(n)]


def build_info() -> str:
    return load().gla_build_info().decode()
