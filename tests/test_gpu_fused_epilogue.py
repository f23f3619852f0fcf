"""GPU parity of the forward with the layer epilogue fused into its output store
(gla_fwd_epilogue through the C ABI) against the float64 oracle: the recurrence's
output o (oracle.fwd) and y = LayerNorm(o) * Swish(r) (oracle/epilogue.py applied
to the oracle's o).  Metric per tensor: max|x - r| / max(1, max|r|) <= 2e-2 for
bf16 (5e-3 for fp32, which runs the two-pass form).  On the bf16 tensor-core path
the output walk's clusters exchange row statistics through DSMEM; o itself must
be bit-identical to gla_fwd's on the same segmentation."""
import numpy as np
import pytest
import torch

from tests.parity import RECORDS, elem_err, rel_err

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 5e-3}


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


def _case(B, H, T, K, V, *, dtype=torch.bfloat16, gate="vector", seed=0, z_mean=0.0, with_h0=False, affine=True,
          segments=0, sample_b=None, save_states=False):
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    from oracle import epilogue, oracle

    x = make_inputs(B, H, T, K, V, dtype=dtype, gate=gate, seed=seed, z_mean=z_mean, with_h0=with_h0)
    g = torch.Generator().manual_seed(seed + 1000)
    r = torch.randn(B, H, T, V, generator=g, dtype=torch.float64).to(dtype)
    w = b = None
    if affine:
        w = (1 + 0.3 * torch.randn(V, generator=g, dtype=torch.float64)).to(torch.float32)
        b = (0.2 * torch.randn(V, generator=g, dtype=torch.float64)).to(torch.float32)
    dev = torch.device("cuda")
    cu = lambda t: None if t is None else t.to(dev)
    q, k, v, la, h0 = cu(x.q), cu(x.k), cu(x.v), cu(x.log_alpha), cu(x.h0)
    o, y, hT = pkg.gla_fwd_epilogue(q, k, v, la, cu(r), cu(w), cu(b), h0, segments=segments, save_states=save_states)
    o_plain, hT_plain = pkg.gla_fwd(q, k, v, la, h0, segments=segments)
    torch.cuda.synchronize()
    bs = list(range(B)) if sample_b is None else sample_b
    n = lambda t: None if t is None else _np(t)[bs]
    ro, rh = oracle.fwd(n(x.q), n(x.k), n(x.v), n(x.log_alpha), h0=n(x.h0), gate=gate)
    ry = epilogue.fwd(ro, n(r), _np(w), _np(b))
    got = {"o": _np(o)[bs], "y": _np(y)[bs], "h_final": _np(hT)[bs]}
    ref = {"o": ro, "y": ry, "h_final": rh}
    errs = {k2: rel_err(got[k2], ref[k2]) for k2 in got}
    RECORDS.append((f"fused epilogue B={B} H={H} T={T} K={K} V={V} {dtype} {gate}", errs,
                    {k2: elem_err(got[k2], ref[k2]) for k2 in got}))
    print("fused epilogue parity", (B, H, T, K, V, str(dtype), gate), {k2: f"{e:.2e}" for k2, e in errs.items()})
    return errs, (o, hT, o_plain, hT_plain, y)


@pytest.mark.parametrize("B,H,T,K,V,gate,segments,with_h0,affine", [
    (1, 2, 300, 256, 512, "vector", 0, False, True),    # clusters of 4, ragged last chunk
    (2, 2, 150, 128, 256, "scalar", 2, True, False),    # clusters of 2, two segments, h0
    (1, 3, 65, 128, 128, "none", 0, False, True),       # clusters of 1 (one tile per token)
    (1, 1, 1, 256, 384, "vector", 0, True, True),       # a single token, clusters of 3
    (2, 1, 1000, 256, 512, "vector", 5, False, True),   # five segments of four chunk tiles each
    (1, 3, 200, 128, 512, "vector", 0, True, True),     # d_k = 128 with clusters of 4
    (1, 2, 4096, 256, 512, "vector", 0, False, True),   # more segments than resident clusters: capped
])
def test_fused_epilogue_parity(B, H, T, K, V, gate, segments, with_h0, affine):
    errs, (o, hT, o_plain, hT_plain, _) = _case(B, H, T, K, V, gate=gate, seed=T + V, segments=segments,
                                                with_h0=with_h0, affine=affine)
    assert all(e <= TOL[torch.bfloat16] for e in errs.values()), errs
    if segments:
        # same segmentation, same kernels for o: the fused store changes nothing in o
        assert torch.equal(o, o_plain) and torch.equal(hT, hT_plain)


def test_fused_epilogue_config4_full_size():
    """The 1.3B-layer shape B=2 H=4 T=4096 d_k=256 d_v=512, z~N(-1,1), saving the
    chunk states for a backward; the oracle checks every head of batch entry 1."""
    errs, _ = _case(2, 4, 4096, 256, 512, z_mean=-1.0, seed=3, sample_b=[1], save_states=True)
    assert all(e <= TOL[torch.bfloat16] for e in errs.values()), errs


@pytest.mark.parametrize("dtype,V", [(torch.bfloat16, 192), (torch.float32, 128)])
def test_two_pass_shapes(dtype, V):
    """d_v not a multiple of 128 (bf16) and the fp32 path: gla_fwd then the epilogue
    pass, same results."""
    errs, _ = _case(1, 2, 130, 128 if dtype == torch.bfloat16 else 64, V, dtype=dtype, seed=V)
    assert all(e <= TOL[dtype] for e in errs.values()), errs


def test_fused_matches_two_pass_on_gpu():
    """y from the fused store against gla_epilogue_fwd over gla_fwd's bf16 o: they
    differ only by the statistics being taken before o's rounding to bf16."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    B, H, T, K, V = 2, 4, 777, 256, 512
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate="vector", seed=21)
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(5)
    r = torch.randn(B, H, T, V, generator=g).to(torch.bfloat16).to(dev)
    w = (1 + 0.3 * torch.randn(V, generator=g)).to(dev)
    b = (0.2 * torch.randn(V, generator=g)).to(dev)
    q, k, v, la = (t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha))
    o, y, _ = pkg.gla_fwd_epilogue(q, k, v, la, r, w, b)
    y2 = pkg.gla_epilogue_fwd(o, r, w, b)
    torch.cuda.synchronize()
    d = (y.float() - y2.float()).abs().max().item() / max(1.0, y2.float().abs().max().item())
    assert d <= 2e-2, d
    assert torch.isfinite(y.float()).all()


def test_fused_epilogue_reports_gate_range():
    """A gate beyond the range the tensor-core path takes (log alpha = -10 per token)
    is reported through the status word of the fused call, as for gla_fwd."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    B, H, T, K, V = 1, 2, 128, 128, 256
    dev = torch.device("cuda")
    q = torch.randn(B, H, T, K, device=dev).to(torch.bfloat16)
    k = torch.randn(B, H, T, K, device=dev).to(torch.bfloat16)
    v = torch.randn(B, H, T, V, device=dev).to(torch.bfloat16)
    r = torch.randn(B, H, T, V, device=dev).to(torch.bfloat16)
    la = torch.full((B, H, T, K), -10.0, device=dev)
    ws = pkg.alloc_workspace(pkg.workspace_size(B, H, T, K, V, torch.bfloat16, "vector", 64, False), dev)
    pkg.gla_fwd_epilogue(q, k, v, la, r, workspace=ws)
    assert pkg.poll_status(ws) == -7  # GLA_ERR_GATE_RANGE


def test_fused_epilogue_forward_feeds_the_backward():
    """A training step through the fused forward: gla_fwd_epilogue saving the chunk
    states, then gla_bwd reading them and the forward's prep outputs from the same
    workspace.  The gradients match the oracle's back-propagation of the plain
    recurrence (the epilogue's own backward is the separate pass, tested elsewhere)."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    from oracle import oracle
    B, H, T, K, V = 1, 4, 1100, 256, 512
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate="vector", seed=17, z_mean=-1.0)
    dev = torch.device("cuda")
    q, k, v, la, do = (t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.do))
    r = torch.randn(B, H, T, V, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).to(dev)
    flags = pkg.FLAG_SAVE_STATES | pkg.FLAG_REUSE_PREP
    ws = pkg.alloc_workspace(pkg.workspace_size(B, H, T, K, V, torch.bfloat16, "vector", 64, True, flags=flags), dev)
    o, y, _ = pkg.gla_fwd_epilogue(q, k, v, la, r, workspace=ws, save_states=True)
    dq, dk, dv, dla, _ = pkg.gla_bwd(q, k, v, la, do, None, None, workspace=ws, reuse_prep=True, saved_states=True,
                                     want_dh0=False)
    torch.cuda.synchronize()
    assert pkg.poll_status(ws) == 0
    n = lambda t: t.double().numpy()
    ro, _ = oracle.fwd(n(x.q), n(x.k), n(x.v), n(x.log_alpha), gate="vector")
    rdq, rdk, rdv, rdla, _ = oracle.bwd(n(x.q), n(x.k), n(x.v), n(x.log_alpha), n(x.do), None, None, gate="vector")
    errs = {"o": rel_err(_np(o), ro), "dq": rel_err(_np(dq), rdq), "dk": rel_err(_np(dk), rdk),
            "dv": rel_err(_np(dv), rdv), "dlog_alpha": rel_err(_np(dla), rdla)}
    print("fused forward -> backward", {k2: f"{e:.2e}" for k2, e in errs.items()})
    assert all(e <= TOL[torch.bfloat16] for e in errs.values()), errs
