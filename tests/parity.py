"""Shared parity machinery: run the CUDA path through the C ABI and the float64
oracle on the same seeded inputs and compare them element by element.

Tolerance metric, per output tensor:  max_i |x_i - r_i| / max(1, max_i |r_i|)
(the largest element-wise deviation, normalised by the tensor's scale floored at
1), <= 5e-3 for fp32 inputs and <= 2e-2 for bf16 inputs.  The purely
element-wise variant max_i |x_i - r_i| / max(1, |r_i|) is also computed and
reported (it is what the fp32 path is held to as well)."""
from __future__ import annotations

import numpy as np
import torch

TOL = {torch.float32: 5e-3, torch.bfloat16: 2e-2}

# Every run_case result of this session, (case description, tensor-scale errors,
# element-wise errors); tests/conftest.py prints them in pytest's terminal summary
# so that a run's log keeps both metrics.
RECORDS: list = []


def rel_err(x, ref) -> float:
    """max|x - ref| / max(1, max|ref|)"""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if x.size == 0:
        return 0.0
    return float(np.max(np.abs(x - ref)) / max(1.0, float(np.max(np.abs(ref)))))


def elem_err(x, ref) -> float:
    """max_i |x_i - ref_i| / max(1, |ref_i|)"""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if x.size == 0:
        return 0.0
    return float(np.max(np.abs(x - ref) / np.maximum(1.0, np.abs(ref))))


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


def run_case(B, H, T, K, V, *, dtype=torch.bfloat16, gate="vector", chunk=64, seed=0, z_mean=0.0, with_h0=False,
             with_dh_final=False, bwd=True, variant="auto", segments=0, gate_scale=None, log_alpha_const=None,
             sample_b=None, device="cuda", reuse_prep=False, save_states=False):
    """Returns {name: max rel err}.  sample_b: list of batch indices the oracle
    checks (all when None); the GPU always runs the full batch.  reuse_prep /
    save_states: the backward reads the forward's prep outputs / chunk states
    from a workspace the two calls share."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    from oracle import oracle

    x = make_inputs(B, H, T, K, V, dtype=dtype, gate=gate, seed=seed, z_mean=z_mean, with_h0=with_h0,
                    with_dh_final=with_dh_final, gate_scale=gate_scale, log_alpha_const=log_alpha_const)
    dev = torch.device(device)
    g = {n: (None if getattr(x, n) is None else getattr(x, n).to(dev))
         for n in ("q", "k", "v", "log_alpha", "do", "h0", "dh_final")}
    ws = None
    shared = dict(variant=variant, segments=segments)
    if reuse_prep or save_states:
        flags = (pkg.FLAG_REUSE_PREP if reuse_prep else 0) | (pkg.FLAG_SAVE_STATES if save_states else 0)
        ws = pkg.alloc_workspace(max(pkg.workspace_size(B, H, T, K, V, dtype, gate, chunk, False, **shared),
                                     pkg.workspace_size(B, H, T, K, V, dtype, gate, chunk, True, flags=flags,
                                                        **shared)), dev)
    o, hT = pkg.gla_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["h0"], chunk=chunk, gate=gate, workspace=ws,
                        save_states=save_states, **shared)
    out = {"o": o, "h_final": hT}
    if bwd:
        dq, dk, dv, dla, dh0 = pkg.gla_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["do"], g["h0"], g["dh_final"],
                                           chunk=chunk, gate=gate, workspace=ws, reuse_prep=reuse_prep,
                                           saved_states=save_states, **shared)
        out.update(dq=dq, dk=dk, dv=dv, dlog_alpha=dla, dh0=dh0)
    torch.cuda.synchronize()
    out = {k: _np(v) for k, v in out.items()}
    sel = slice(None) if sample_b is None else list(sample_b)

    def cut(a):
        return None if a is None else _np(a)[sel]

    ro, rhT = oracle.fwd(cut(x.q), cut(x.k), cut(x.v), cut(x.log_alpha), h0=cut(x.h0), gate=gate)
    ref = {"o": ro, "h_final": rhT}
    if bwd:
        rdq, rdk, rdv, rdla, rdh0 = oracle.bwd(cut(x.q), cut(x.k), cut(x.v), cut(x.log_alpha), cut(x.do),
                                               h0=cut(x.h0), dh_final=cut(x.dh_final), gate=gate)
        ref.update(dq=rdq, dk=rdk, dv=rdv, dlog_alpha=rdla, dh0=rdh0)
    errs = {}
    elem = {}
    for k, r in ref.items():
        if r is None:
            continue
        a = out[k][sel]
        assert np.all(np.isfinite(a)), f"{k} has non-finite values"
        errs[k] = rel_err(a, r)
        elem[k] = elem_err(a, r)
    errs["_elementwise"] = elem
    RECORDS.append((f"B={B} H={H} T={T} dk={K} dv={V} {str(dtype).replace('torch.', '')} gate={gate} "
                    f"variant={variant} seed={seed}" + (" save_states" if save_states else ""),
                    {k: v for k, v in errs.items() if k != "_elementwise"}, dict(elem)))
    print("parity", {k: f"{v:.2e}" for k, v in errs.items() if k != "_elementwise"},
          "elementwise", {k: f"{v:.2e}" for k, v in elem.items()})
    return errs


def assert_parity(errs, dtype, elementwise=None):
    """Check the tensor-scale metric; elementwise=True also holds the per-element
    metric to the same tolerance (the fp32 path)."""
    tol = TOL[dtype]
    if elementwise is None:
        elementwise = dtype == torch.float32
    main = {k: v for k, v in errs.items() if k != "_elementwise"}
    bad = {k: v for k, v in main.items() if not v <= tol}
    if elementwise:
        bad.update({f"{k}(elementwise)": v for k, v in errs["_elementwise"].items() if not v <= tol})
    assert not bad, f"parity failed (tol {tol}): {bad}; all: {main}"
