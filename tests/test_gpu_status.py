"""The device status word: a gate beyond the bf16 rescaling range and a bounded
wait that runs out are reported by gla_poll_status, nothing faults, and the
context stays usable afterwards."""
import numpy as np
import pytest
import torch

from tests.parity import rel_err

pytestmark = pytest.mark.gpu

GLA_OK, GLA_ERR_TIMEOUT, GLA_ERR_GATE_RANGE = 0, -6, -7


def _small_forward_parity(pkg, ws=None):
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    from oracle import oracle
    x = make_inputs(1, 2, 150, 128, 128, dtype=torch.bfloat16, gate="vector", seed=21)
    dev = torch.device("cuda")
    o, hT = pkg.gla_fwd(x.q.to(dev), x.k.to(dev), x.v.to(dev), x.log_alpha.to(dev), None, chunk=64, workspace=ws)
    torch.cuda.synchronize()
    f = lambda a: a.double().cpu().numpy()
    ro, rhT = oracle.fwd(f(x.q), f(x.k), f(x.v), f(x.log_alpha))
    return max(rel_err(f(o.float()), ro), rel_err(f(hT), rhT))


def test_gate_beyond_range_is_reported():
    """log alpha = -10 per token: a 16-token sub-chunk decays by e^-160, below fp32, so
    the bf16 path's sub-chunk rescaling cannot represent it; the prep kernel flags it."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    B, H, T, K, V = 1, 2, 128, 128, 128
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate="vector", seed=20, log_alpha_const=-10.0)
    dev = torch.device("cuda")
    # sized for the larger of this call and the follow-up one (T = 150)
    ws = pkg.alloc_workspace(pkg.workspace_size(B, H, 150, K, V, torch.bfloat16, "vector", 64, False), dev)
    pkg.gla_fwd(x.q.to(dev), x.k.to(dev), x.v.to(dev), x.log_alpha.to(dev), None, chunk=64, workspace=ws)
    assert pkg.poll_status(ws) == GLA_ERR_GATE_RANGE
    assert pkg.poll_status(ws) == GLA_OK  # the poll cleared it
    # the same workspace serves a normal call, which reports OK and matches the oracle
    assert _small_forward_parity(pkg, ws) <= 2e-2
    assert pkg.poll_status(ws) == GLA_OK


def test_bounded_wait_runs_out_and_context_survives():
    """A wait on an mbarrier that nothing completes gives up after 20 ms and sets the
    timeout bit; the next calls on the same context run and are correct."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    dev = torch.device("cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    pkg.selftest_timeout(ws, limit_us=20000)
    assert pkg.poll_status(ws) == GLA_ERR_TIMEOUT
    assert pkg.poll_status(ws) == GLA_OK
    assert _small_forward_parity(pkg) <= 2e-2
    torch.cuda.synchronize()
