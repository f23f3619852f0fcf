"""GPU parity of sequence parallelism (gla_fwd_state, gla_bwd_state, gla_state_scan
through the C ABI).

1. Each summary against what it summarises:
   - a piece's delta equals gla_fwd's h_final, and its ddelta equals gla_bwd's dh0;
   - gamma equals exp of the summed log-gates, in float64;
   - the scan equals a float64 fold of the same gathered summaries.
2. The whole protocol, emulated on one GPU: the pieces of one sequence run one after
   another (the all-gather is a stack), and the concatenated results are held
   against the float64 oracle on the whole sequence at the bf16 bar
   (max|x - r| / max(1, max|r|) <= 2e-2).  The pieces are independent launches; no
   kernel waits on another."""
import numpy as np
import pytest
import torch

from tests.parity import rel_err

pytestmark = pytest.mark.gpu


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


def _piece(t, lo, hi):
    return None if t is None else t[:, :, lo:hi].contiguous()


def _gamma64(la, gate, B, H, K):
    if gate == "none":
        return torch.ones(B, H, K, dtype=torch.float64)
    s = la.double().cpu().sum(dim=2)
    return torch.exp(s[..., None].expand(B, H, K) if gate == "scalar" else s)


@pytest.mark.parametrize("gate,segments", [("vector", 0), ("vector", 1), ("scalar", 0), ("none", 0)])
def test_summaries_match_what_they_summarise(gate, segments):
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    B, H, T, K, V = 1, 3, 700, 256, 512
    x = make_inputs(B, H, T, K, V, gate=gate, seed=5, with_h0=True, with_dh_final=True)
    dev = torch.device("cuda")
    q, k, v, la, do, h0, dhT = (None if t is None else t.to(dev)
                                for t in (x.q, x.k, x.v, x.log_alpha, x.do, x.h0, x.dh_final))
    delta, gamma = pkg.gla_fwd_state(q, k, v, la, h0, segments=segments)
    _, hT = pkg.gla_fwd(q, k, v, la, h0, segments=segments)
    ddelta, gamma2 = pkg.gla_bwd_state(q, k, la, do, dhT, segments=segments)
    dh0 = pkg.gla_bwd(q, k, v, la, do, h0, dhT, segments=segments)[4]
    torch.cuda.synchronize()
    errs = {"delta": rel_err(_np(delta), _np(hT)), "ddelta": rel_err(_np(ddelta), _np(dh0)),
            # gamma is a product of ~T gates (1e-15 here): element-wise relative error
            "gamma": float(np.max(np.abs(_np(gamma) / _np(_gamma64(x.log_alpha, gate, B, H, K)) - 1.0))),
            # the reverse pass multiplies the segments' gate products in the opposite order
            "gamma_bwd": float(np.max(np.abs(_np(gamma2) / _np(gamma) - 1.0)))}
    print("summaries", gate, segments, {n: f"{e:.1e}" for n, e in errs.items()})
    assert errs["delta"] <= 1e-5 and errs["ddelta"] <= 1e-5, errs
    assert errs["gamma"] <= 1e-4 and errs["gamma_bwd"] <= 1e-6, errs


@pytest.mark.parametrize("reverse", [False, True])
def test_state_scan_is_the_fold(reverse):
    import chunkwise_linear_rnn_fwd_b200 as pkg
    g = torch.Generator().manual_seed(2)
    P, B, H, K, V = 5, 2, 3, 128, 192
    gammas = torch.rand(P, B, H, K, generator=g, dtype=torch.float64)
    deltas = torch.randn(P, B, H, K, V, generator=g, dtype=torch.float64)
    init = torch.randn(B, H, K, V, generator=g, dtype=torch.float64)
    dev = torch.device("cuda")
    gd, dd, idv = (t.float().to(dev) for t in (gammas, deltas, init))
    for seg in range(P):
        for use_init in (False, True):
            out = pkg.gla_state_scan(gd, dd, seg, reverse=reverse, init=idv if use_init else None)
            S = init.clone() if use_init else torch.zeros(B, H, K, V, dtype=torch.float64)
            for s in (range(P - 1, seg, -1) if reverse else range(seg)):
                S = gammas[s][..., None] * S + deltas[s]
            assert rel_err(_np(out), _np(S)) <= 1e-6, (seg, use_init)


class _FreshOps:
    """Every call on a fresh workspace: nothing reused."""

    def __init__(self, pkg):
        self.p = pkg

    def fwd_state(self, *a):
        return self.p.gla_fwd_state(*a)

    def fwd(self, *a):
        return self.p.gla_fwd(*a)

    def bwd_state(self, *a):
        return self.p.gla_bwd_state(*a)

    def bwd(self, *a):
        return self.p.gla_bwd(*a)


@pytest.mark.parametrize("gate,cuts,reuse", [("vector", [0, 320, 576, 1000], False),
                                             ("vector", [0, 320, 576, 1000], True),
                                             ("vector", [0, 100, 1000], True), ("scalar", [0, 448, 1000], True),
                                             ("scalar", [0, 448, 1000], False), ("none", [0, 500, 1000], True)])
def test_emulated_sequence_parallel_against_oracle(gate, cuts, reuse):
    """reuse: each piece's four calls share one workspace (seqpar.LibraryOps: prep,
    segment contributions and chunk states are computed once and reused)."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200 import seqpar
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    from oracle import oracle
    B, H, T, K, V = 1, 2, 1000, 256, 512
    x = make_inputs(B, H, T, K, V, gate=gate, seed=9, with_h0=True, with_dh_final=True)
    dev = torch.device("cuda")
    q, k, v, la, do, h0, dhT = (None if t is None else t.to(dev)
                                for t in (x.q, x.k, x.v, x.log_alpha, x.do, x.h0, x.dh_final))
    P = len(cuts) - 1
    pieces = [(cuts[r], cuts[r + 1]) for r in range(P)]
    cut = lambda t, r: _piece(t, *pieces[r])
    ops = [seqpar.LibraryOps() if reuse else _FreshOps(pkg) for _ in range(P)]
    # forward: summaries, gather (stack), fold, rerun
    summ = [ops[r].fwd_state(cut(q, r), cut(k, r), cut(v, r), cut(la, r), h0 if r == 0 else None)
            for r in range(P)]
    gammas = torch.stack([g for _, g in summ])
    deltas = torch.stack([d for d, _ in summ])
    h_in = [h0] + [pkg.gla_state_scan(gammas, deltas, r) for r in range(1, P)]
    outs = [ops[r].fwd(cut(q, r), cut(k, r), cut(v, r), cut(la, r), h_in[r]) for r in range(P)]
    # backward: reverse summaries, gather, reverse fold, rerun
    rsumm = [ops[r].bwd_state(cut(q, r), cut(k, r), cut(la, r), cut(do, r), dhT if r == P - 1 else None)
             for r in range(P)]
    dds = torch.stack([d for d, _ in rsumm])
    dh_out = [pkg.gla_state_scan(gammas, dds, r, reverse=True) for r in range(P - 1)] + [dhT]
    grads = [ops[r].bwd(cut(q, r), cut(k, r), cut(v, r), cut(la, r), cut(do, r), h_in[r], dh_out[r])
             for r in range(P)]
    torch.cuda.synchronize()
    cat = lambda ts: np.concatenate([_np(t) for t in ts], axis=2)
    ro, rhT = oracle.fwd(*(_np(t) for t in (x.q, x.k, x.v, x.log_alpha)), h0=_np(x.h0), gate=gate)
    rdq, rdk, rdv, rdla, rdh0 = oracle.bwd(*(_np(t) for t in (x.q, x.k, x.v, x.log_alpha, x.do)), _np(x.h0),
                                           _np(x.dh_final), gate=gate)
    errs = {"o": rel_err(cat([o for o, _ in outs]), ro), "h_final": rel_err(_np(outs[-1][1]), rhT),
            "dq": rel_err(cat([g[0] for g in grads]), rdq), "dk": rel_err(cat([g[1] for g in grads]), rdk),
            "dv": rel_err(cat([g[2] for g in grads]), rdv), "dh0": rel_err(_np(grads[0][4]), rdh0)}
    if gate != "none":
        errs["dlog_alpha"] = rel_err(cat([g[3] for g in grads]), rdla)
    print("sequence parallel (emulated)", gate, cuts, "reuse" if reuse else "fresh",
          {n: f"{e:.1e}" for n, e in errs.items()})
    assert all(e <= 2e-2 for e in errs.values()), errs
