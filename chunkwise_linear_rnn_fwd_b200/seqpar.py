"""Sequence (context) parallelism: one sequence split into consecutive pieces, piece r
on rank r of a torch.distributed group.

"Gated Linear Attention Transformers with Hardware-Efficient Training", sections 3.3
and 4.2: the chunk-level recurrence S_n = diag(gamma_n) S_{n-1} + dS_n composes affine
maps, so each piece needs only the summaries of the pieces before it (forward) or
after it (backward).  One exchange per direction:

  forward   (delta_r, gamma_r) = gla_fwd_state(piece r; rank 0 starts from h0)
            all-gather of (gamma, delta)
            h_in_r = fold of pieces 0 .. r-1 (gla_state_scan); rank 0: h0
            o, h_out = gla_fwd(piece r from h_in_r)
  backward  (ddelta_r, gamma_r) = gla_bwd_state(piece r; the last rank from dh_final)
            all-gather of (gamma, ddelta)
            dh_out_r = fold of pieces P-1 .. r+1, reverse; last rank: dh_final
            gla_bwd(piece r from h_in_r with dh_final = dh_out_r)

gla_bwd's gate gradient includes the final-state term sum_v h_out dh_out, which is
the contribution of every later piece's tokens to the reverse cumulative sum of
dlog alpha, so the pieces' dlog alpha concatenate to the whole sequence's.

All compute runs in the CUDA library (`ops` defaults to LibraryOps); the collective is
torch.distributed's all-gather (NCCL on GPUs).  The summaries are small (d_k x d_v
fp32 per head), so there is nothing to overlap with.
"""
from __future__ import annotations

import contextlib
from typing import Optional

import torch
import torch.distributed as dist


class LibraryOps:
    """The compute steps bound to the CUDA library, for one piece.  One workspace,
    sized for the backward, serves the piece's four calls, so a training step runs
    prep once and each walk pre-pass once, as without sequence parallelism:
      fwd_state  prep, zero-state contributions of every segment, their fold
      fwd        reuses both (GLA_FLAG_REUSE_PREP | REUSE_SEGMENTS), saves the chunk states
      bwd_state  reuses the prep; reverse contributions of every segment, their fold
      bwd        reuses prep, saved states and reverse contributions
    A call reuses only what an earlier call on this object left for it (a forward
    without fwd_state, e.g. on one rank, computes everything)."""

    def __init__(self, chunk: int = 64, stream=None):
        self.chunk, self.stream = chunk, stream
        self.ws, self._key = None, None
        self._state = self._fwd = self._bstate = False

    def _workspace(self, q, dv, la):
        from . import gla as G
        gate = G._gate_of(la, None)
        key = (tuple(q.shape), int(dv), q.dtype, gate, q.device)
        if key != self._key:
            B, H, T, dk = q.shape
            n = G.workspace_size(B, H, T, dk, dv, q.dtype, gate, self.chunk, True, flags=G.FLAG_SAVE_STATES)
            # the old workspace may still be in use by kernels queued on self.stream:
            # allocate (and so later free) on that stream
            ctx = torch.cuda.stream(self.stream) if self.stream is not None else contextlib.nullcontext()
            with ctx:
                self.ws, self._key = G.alloc_workspace(n, q.device), key
            self._state = self._fwd = self._bstate = False
        return self.ws

    def fwd_state(self, q, k, v, la, h0):
        from . import gla as G
        ws = self._workspace(q, v.shape[-1], la)
        out = G.gla_fwd_state(q, k, v, la, h0, chunk=self.chunk, workspace=ws, save_states=True, stream=self.stream)
        self._state, self._fwd, self._bstate = True, False, False
        return out

    def fwd(self, q, k, v, la, h0):
        from . import gla as G
        ws = self._workspace(q, v.shape[-1], la)
        out = G.gla_fwd(q, k, v, la, h0, chunk=self.chunk, workspace=ws, save_states=True, reuse_prep=self._state,
                        reuse_segments=self._state, stream=self.stream)
        self._state, self._fwd, self._bstate = False, True, False
        return out

    def bwd_state(self, q, k, la, do, dhT):
        from . import gla as G
        ws = self._workspace(q, do.shape[-1], la)
        out = G.gla_bwd_state(q, k, la, do, dhT, chunk=self.chunk, workspace=ws, reuse_prep=self._fwd,
                              stream=self.stream)
        self._bstate = True
        return out

    def bwd(self, q, k, v, la, do, h0, dhT):
        from . import gla as G
        ws = self._workspace(q, v.shape[-1], la)
        out = G.gla_bwd(q, k, v, la, do, h0, dhT, chunk=self.chunk, workspace=ws, reuse_prep=self._fwd,
                        saved_states=self._fwd, reuse_segments=self._bstate, stream=self.stream)
        self._state = self._fwd = self._bstate = False
        return out

    def state_scan(self, gammas, deltas, seg, reverse):
        from . import gla as G
        return G.gla_state_scan(gammas, deltas, seg, reverse=reverse, stream=self.stream)


def _rank_world(group) -> tuple[int, int]:
    """(rank, world size) of `group`; without an initialised process group the
    sequence is one piece on this process (0, 1)."""
    if not (dist.is_available() and dist.is_initialized()):
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def gather_summaries(gamma: torch.Tensor, delta: torch.Tensor, group) -> tuple[torch.Tensor, torch.Tensor]:
    """One all-gather of the packed (gamma, delta) of every rank: [P, *gamma.shape],
    [P, *delta.shape], piece-major."""
    world = dist.get_world_size(group)
    packed = torch.cat([gamma.reshape(-1), delta.reshape(-1)]).contiguous()
    parts = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(parts, packed, group=group)
    allp = torch.stack(parts)
    ng = gamma.numel()
    return (allp[:, :ng].reshape(world, *gamma.shape).contiguous(),
            allp[:, ng:].reshape(world, *delta.shape).contiguous())


def sp_gla_fwd(q, k, v, log_alpha=None, h0: Optional[torch.Tensor] = None, *, group=None, ops=None,
               chunk: int = 64, stream=None):
    """Forward of this rank's piece.  q, k [B,H,T_r,d_k], v [B,H,T_r,d_v], log_alpha
    [B,H,T_r,d_k] / [B,H,T_r] / None; h0: the sequence's initial state (read on rank 0
    only; None = zero).  Returns (o, h_out, h_in): the piece's output, the state after
    it (the sequence's h_final on the last rank) and the state entering it (pass it
    to sp_gla_bwd).  ops: the compute steps (a LibraryOps, kept for the backward of
    the same piece so that it reuses this call's work)."""
    ops = ops or LibraryOps(chunk, stream)
    rank, world = _rank_world(group)
    if world == 1:
        o, h_out = ops.fwd(q, k, v, log_alpha, h0)
        return o, h_out, h0
    delta, gamma = ops.fwd_state(q, k, v, log_alpha, h0 if rank == 0 else None)
    gammas, deltas = gather_summaries(gamma, delta, group)
    h_in = h0 if rank == 0 else ops.state_scan(gammas, deltas, rank, False)
    o, h_out = ops.fwd(q, k, v, log_alpha, h_in)
    return o, h_out, h_in


def sp_gla_bwd(q, k, v, log_alpha, do, h_in: Optional[torch.Tensor], dh_final: Optional[torch.Tensor] = None, *,
               group=None, ops=None, chunk: int = 64, stream=None):
    """Backward of this rank's piece.  h_in from sp_gla_fwd; dh_final: the adjoint of
    the sequence's final state (read on the last rank only; None = zero).  Returns
    (dq, dk, dv, dlog_alpha, dh_in): the piece's gradients and the adjoint of the
    state entering it (the sequence's dh0 on rank 0)."""
    ops = ops or LibraryOps(chunk, stream)
    rank, world = _rank_world(group)
    if world == 1:
        return ops.bwd(q, k, v, log_alpha, do, h_in, dh_final)
    last = rank == world - 1
    ddelta, gamma = ops.bwd_state(q, k, log_alpha, do, dh_final if last else None)
    gammas, ddeltas = gather_summaries(gamma, ddelta, group)
    dh_out = dh_final if last else ops.state_scan(gammas, ddeltas, rank, True)
    return ops.bwd(q, k, v, log_alpha, do, h_in, dh_out)
