"""Sequence parallelism on the CPU: the exchange protocol of
chunkwise_linear_rnn_fwd_b200.seqpar driven by the float64 oracle.

The compute steps (piece summaries, forward, backward) are the oracle's and the fold
is written out here, so these tests check the protocol itself on gloo ranks:
- which rank starts from h0 and which from dh_final;
- the order of the gathered pieces and the direction of each fold;
- the gate gradient's dependence on later pieces.
The pieces' results, concatenated, must equal the oracle on the whole sequence.
The CUDA steps are checked against the oracle on the GPU (tests/test_gpu_seqpar.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from chunkwise_linear_rnn_fwd_b200.synth import make_inputs

B, H, K, V = 1, 2, 8, 6


def _gamma(la, gate, T):
    """prod_t alpha_t per key channel: the definition of a piece's gate product."""
    if gate == "none":
        return torch.ones(B, H, K, dtype=torch.float64)
    s = la.double().sum(dim=2)
    if gate == "scalar":
        s = s[..., None].expand(B, H, K)
    return torch.exp(s).contiguous()


def oracle_ops(gate):
    from types import SimpleNamespace

    from oracle import oracle

    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a))
    n = lambda x: None if x is None else x.double().numpy()

    def fwd_state(q, k, v, la, h0):
        _, hT = oracle.fwd(n(q), n(k), n(v), n(la), h0=n(h0), gate=gate)
        return t(hT), _gamma(la, gate, q.shape[2])

    def bwd_state(q, k, la, do, dhT):
        zeros_v = np.zeros(do.shape)
        *_, dh0 = oracle.bwd(n(q), n(k), zeros_v, n(la), n(do), None, n(dhT), gate=gate)
        return t(dh0), _gamma(la, gate, q.shape[2])

    def state_scan(gammas, deltas, seg, reverse):
        S = torch.zeros_like(deltas[0])
        order = range(len(deltas) - 1, seg, -1) if reverse else range(seg)
        for s in order:
            S = gammas[s][..., None] * S + deltas[s]
        return S

    def fwd(q, k, v, la, h0):
        o, hT = oracle.fwd(n(q), n(k), n(v), n(la), h0=n(h0), gate=gate)
        return t(o), t(hT)

    def bwd(q, k, v, la, do, h0, dhT):
        return tuple(t(x) for x in oracle.bwd(n(q), n(k), n(v), n(la), n(do), n(h0), n(dhT), gate=gate))

    return SimpleNamespace(fwd_state=fwd_state, bwd_state=bwd_state, state_scan=state_scan, fwd=fwd, bwd=bwd)


def _inputs(T, gate, seed):
    x = make_inputs(B, H, T, K, V, dtype=torch.float64, gate=gate, seed=seed, with_h0=True, with_dh_final=True)
    la = None if x.log_alpha is None else x.log_alpha.double()
    return x.q, x.k, x.v, la, x.do, x.h0.double(), x.dh_final.double()


def _piece(t, lo, hi):
    return None if t is None else t[:, :, lo:hi].contiguous()


def test_summary_fold_pin(oracle_mod):
    """Without any process group: the state after a split sequence is the fold of the
    pieces' summaries, and the adjoint before it is the reverse fold (the affine-map
    composition that sequence parallelism rests on), against the whole-sequence oracle."""
    ops = oracle_ops("vector")
    q, k, v, la, do, h0, dhT = _inputs(130, "vector", seed=3)
    cuts = [0, 40, 41, 130]
    parts = [(cuts[i], cuts[i + 1]) for i in range(3)]
    summ = [ops.fwd_state(*(_piece(a, lo, hi) for a in (q, k, v, la)), h0 if i == 0 else None)
            for i, (lo, hi) in enumerate(parts)]
    gammas = torch.stack([g for _, g in summ])
    deltas = torch.stack([d for d, _ in summ])
    _, hT = ops.fwd(q, k, v, la, h0)
    h_end = ops.state_scan(gammas, deltas, 2, False)  # entering the last piece
    last = ops.fwd(*(_piece(a, 41, 130) for a in (q, k, v, la)), h_end)[1]
    assert torch.allclose(last, hT, rtol=1e-12, atol=1e-12)
    full = gammas[2][..., None] * h_end + deltas[2]
    assert torch.allclose(full, hT, rtol=1e-12, atol=1e-12)
    rsumm = [ops.bwd_state(*(_piece(a, lo, hi) for a in (q, k, la, do)), dhT if i == 2 else None)
             for i, (lo, hi) in enumerate(parts)]
    dd = torch.stack([d for d, _ in rsumm])
    dh0 = ops.bwd(q, k, v, la, do, h0, dhT)[4]
    d_out0 = ops.state_scan(gammas, dd, 0, True)  # leaving piece 0
    assert torch.allclose(gammas[0][..., None] * d_out0 + dd[0], dh0, rtol=1e-12, atol=1e-12)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, T, cuts, gate, out):
    import torch.distributed as dist

    from chunkwise_linear_rnn_fwd_b200 import seqpar
    from oracle import oracle
    oracle.build()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ops = oracle_ops(gate)
        q, k, v, la, do, h0, dhT = _inputs(T, gate, seed=11)
        lo, hi = cuts[rank], cuts[rank + 1]
        pq, pk, pv, pla, pdo = (_piece(a, lo, hi) for a in (q, k, v, la, do))
        # h0 and dh_final are passed on every rank; only rank 0 / the last rank may read them
        o, h_out, h_in = seqpar.sp_gla_fwd(pq, pk, pv, pla, h0, ops=ops)
        dq, dk, dv, dla, dh_in = seqpar.sp_gla_bwd(pq, pk, pv, pla, pdo, h_in, dhT, ops=ops)
        out[rank] = {"o": o.numpy(), "h_out": h_out.numpy(), "dq": dq.numpy(), "dk": dk.numpy(),
                     "dv": dv.numpy(), "dla": None if dla is None else dla.numpy(), "dh_in": dh_in.numpy()}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cuts,gate", [(2, [0, 64, 150], "vector"), (3, [0, 50, 51, 150], "scalar"),
                                             (2, [0, 77, 150], "none"), (4, [0, 30, 31, 100, 150], "vector")])
def test_sequence_parallel_matches_whole_sequence(oracle_mod, world, cuts, gate):
    T = 150
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, T, cuts, gate, out), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v, la, do, h0, dhT = _inputs(T, gate, seed=11)
    ops = oracle_ops(gate)
    o, hT = ops.fwd(q, k, v, la, h0)
    dq, dk, dv, dla, dh0 = ops.bwd(q, k, v, la, do, h0, dhT)
    cat = lambda key: np.concatenate([out[r][key] for r in range(world)], axis=2)
    close = lambda a, b: np.testing.assert_allclose(a, b.numpy(), rtol=1e-10, atol=1e-10)
    close(cat("o"), o)
    close(cat("dq"), dq)
    close(cat("dk"), dk)
    close(cat("dv"), dv)
    if gate != "none":
        close(cat("dla"), dla)
    close(out[world - 1]["h_out"], hT)
    close(out[0]["dh_in"], dh0)


def test_library_ops_reuse_chain(monkeypatch):
    """seqpar.LibraryOps passes each call exactly the reuse flags that an earlier call
    on its workspace has earned: fwd_state -> fwd reuses prep and segments; bwd_state
    reuses prep only after fwd; bwd reuses prep and saved states only after fwd and
    segments only after bwd_state; a call on a new shape starts over.  The CUDA
    binding is replaced by a recorder (no GPU)."""
    from chunkwise_linear_rnn_fwd_b200 import gla as G
    from chunkwise_linear_rnn_fwd_b200 import seqpar
    calls = []
    monkeypatch.setattr(G, "workspace_size", lambda *a, **k: 256)
    monkeypatch.setattr(G, "alloc_workspace", lambda n, dev: torch.empty(n, dtype=torch.uint8))

    def rec(name):
        def f(*a, **kw):
            calls.append((name, {k: v for k, v in kw.items() if k in ("save_states", "reuse_prep", "reuse_segments",
                                                                          "saved_states")}))
            return (None, None) if name in ("fwd_state", "bwd_state", "fwd") else (None,) * 5
        return f

    for name in ("fwd_state", "bwd_state"):
        monkeypatch.setattr(G, "gla_" + name, rec(name))
    monkeypatch.setattr(G, "gla_fwd", rec("fwd"))
    monkeypatch.setattr(G, "gla_bwd", rec("bwd"))
    q = torch.zeros(1, 1, 8, 4)
    v = torch.zeros(1, 1, 8, 4)
    la = torch.zeros(1, 1, 8, 4)
    ops = seqpar.LibraryOps()
    ops.fwd_state(q, q, v, la, None)
    ops.fwd(q, q, v, la, None)
    ops.bwd_state(q, q, la, v, None)
    ops.bwd(q, q, v, la, v, None, None)
    ops.bwd(q, q, v, la, v, None, None)          # nothing left to reuse
    ops.fwd(q, q, v, la, None)                   # a forward without its summary
    q2 = torch.zeros(1, 1, 9, 4)
    ops.bwd_state(q2, q2, torch.zeros(1, 1, 9, 4), torch.zeros(1, 1, 9, 4), None)  # new shape: new workspace
    assert calls == [
        ("fwd_state", {"save_states": True}),
        ("fwd", {"save_states": True, "reuse_prep": True, "reuse_segments": True}),
        ("bwd_state", {"reuse_prep": True}),
        ("bwd", {"reuse_prep": True, "saved_states": True, "reuse_segments": True}),
        ("bwd", {"reuse_prep": False, "saved_states": False, "reuse_segments": False}),
        ("fwd", {"save_states": True, "reuse_prep": False, "reuse_segments": False}),
        ("bwd_state", {"reuse_prep": False}),
    ], calls
