"""GPU parity of the general gate G_t = alpha_t^T beta_t (gla_fwd_general /
gla_bwd_general through the C ABI) against the float64 oracle, every output tensor
element by element: max|x - r| / max(1, max|r|) <= 2e-2 (bf16 tensors) or 5e-3
(fp32 tensors; dlog_alpha, dlog_beta, h_final, dh0 are fp32 in either case and are
held to the bar of the input dtype, like the alpha-only path)."""
import numpy as np
import pytest
import torch

from tests.parity import rel_err

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 5e-3}


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


@pytest.mark.parametrize("B,H,T,K,V,dtype,gate", [
    (1, 2, 200, 64, 64, torch.float32, "vector"),
    (2, 2, 333, 128, 96, torch.bfloat16, "vector"),
    (1, 3, 130, 32, 48, torch.float32, "scalar"),
    (1, 2, 100, 64, 32, torch.bfloat16, "none"),
    (1, 1, 1, 16, 8, torch.float32, "vector"),
])
def test_general_gate_parity(B, H, T, K, V, dtype, gate):
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    from oracle import oracle
    x = make_inputs(B, H, T, K, V, dtype=dtype, gate=gate, seed=T + K, with_h0=True, with_dh_final=True,
                    with_log_beta=True)
    dev = torch.device("cuda")
    q, k, v, la, lb, do, h0, dhT = (None if t is None else t.to(dev)
                                    for t in (x.q, x.k, x.v, x.log_alpha, x.log_beta, x.do, x.h0, x.dh_final))
    o, hT = pkg.gla_fwd_general(q, k, v, la, lb, h0)
    dq, dk, dv, dla, dlb, dh0 = pkg.gla_bwd_general(q, k, v, la, lb, do, h0, dhT)
    torch.cuda.synchronize()
    ins = [_np(t) for t in (x.q, x.k, x.v, x.log_alpha, x.log_beta)]
    ro, rhT = oracle.fwd_general(*ins, h0=_np(x.h0), gate=gate)
    rdq, rdk, rdv, rdla, rdlb, rdh0 = oracle.bwd_general(*ins, _np(x.do), _np(x.h0), _np(x.dh_final), gate=gate)
    errs = {"o": rel_err(_np(o), ro), "h_final": rel_err(_np(hT), rhT), "dq": rel_err(_np(dq), rdq),
            "dk": rel_err(_np(dk), rdk), "dv": rel_err(_np(dv), rdv), "dlog_beta": rel_err(_np(dlb), rdlb),
            "dh0": rel_err(_np(dh0), rdh0)}
    if gate != "none":
        errs["dlog_alpha"] = rel_err(_np(dla), rdla)
    print("general gate", dtype, gate, (B, H, T, K, V), {n: f"{e:.1e}" for n, e in errs.items()})
    assert all(e <= TOL[dtype] for e in errs.values()), errs


def test_unit_beta_matches_the_alpha_only_path():
    """log beta = 0: the general path equals gla_fwd / gla_bwd on the same fp32 inputs
    (both the CUDA-core path), and its dlog_beta is the oracle's."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    x = make_inputs(1, 2, 150, 64, 64, dtype=torch.float32, gate="vector", seed=3, with_h0=True, with_dh_final=True)
    dev = torch.device("cuda")
    q, k, v, la, do, h0, dhT = (t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.do, x.h0, x.dh_final))
    lb = torch.zeros(1, 2, 150, 64, device=dev)
    o1, h1 = pkg.gla_fwd(q, k, v, la, h0)
    o2, h2 = pkg.gla_fwd_general(q, k, v, la, lb, h0)
    g1 = pkg.gla_bwd(q, k, v, la, do, h0, dhT)
    g2 = pkg.gla_bwd_general(q, k, v, la, lb, do, h0, dhT)
    torch.cuda.synchronize()
    assert rel_err(_np(o1), _np(o2)) <= 1e-6 and rel_err(_np(h1), _np(h2)) <= 1e-6
    for a, b in zip(g1, (g2[0], g2[1], g2[2], g2[3], g2[5])):
        assert rel_err(_np(a), _np(b)) <= 1e-6
