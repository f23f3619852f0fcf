"""GPU parity of the recurrent decode step (gla_decode_step, through the C ABI)
against the float64 oracle on the same seeded inputs: single steps for every gate
mode and element type, ragged and odd head sizes, and a chain of steps that must
reproduce the oracle's sequence forward.  Metric per output tensor:
max|x - r| / max(1, max|r|), <= 2e-2 for bf16 inputs and 5e-3 for fp32 inputs
(the carried state is fp32 either way and is held to 5e-3)."""
import numpy as np
import pytest
import torch

from tests.parity import rel_err

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32
TOL = {BF16: 2e-2, F32: 5e-3}


def _step_inputs(B, H, K, V, dtype, gate, seed):
    """One decode token per (batch, head) with the workload distributions (q, v ~ N(0,1),
    k ~ N(0,1)/sqrt(K), log alpha = logsigmoid(z)/16) and a state ~ N(0,1)/sqrt(K)."""
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    x = make_inputs(B, H, 1, K, V, dtype=dtype, gate=gate, seed=seed, with_h0=True)
    la = None if x.log_alpha is None else x.log_alpha[:, :, 0]
    return x.q[:, :, 0], x.k[:, :, 0], x.v[:, :, 0], la, x.h0


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


@pytest.mark.parametrize("dtype", [BF16, F32])
@pytest.mark.parametrize("gate", ["vector", "scalar", "none"])
@pytest.mark.parametrize("B,H,K,V", [(2, 3, 64, 48), (8, 4, 256, 512), (1, 2, 1, 100), (3, 1, 300, 4)])
def test_decode_step_parity(dtype, gate, B, H, K, V):
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from oracle import oracle
    q, k, v, la, S = _step_inputs(B, H, K, V, dtype, gate, seed=K + V)
    dev = torch.device("cuda")
    Sd = S.to(dev).contiguous()
    o = pkg.gla_decode_step(q.to(dev), k.to(dev), v.to(dev), None if la is None else la.to(dev), Sd, gate=gate)
    torch.cuda.synchronize()
    ro, rS = oracle.decode_step(_np(q), _np(k), _np(v), _np(la), _np(S), gate=gate)
    eo, eS = rel_err(_np(o), ro), rel_err(_np(Sd), rS)
    print("decode parity", dtype, gate, (B, H, K, V), f"o {eo:.2e} state {eS:.2e}")
    assert eo <= TOL[dtype] and eS <= 5e-3, (eo, eS)


@pytest.mark.parametrize("dtype", [BF16, F32])
def test_decode_chain_matches_sequence_forward(dtype):
    """T decode steps from h0 on the GPU (state carried in fp32 on the device) against
    the oracle's sequence forward over the same T tokens."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    from oracle import oracle
    B, H, T, K, V = 2, 2, 40, 128, 128
    x = make_inputs(B, H, T, K, V, dtype=dtype, gate="vector", seed=12, with_h0=True)
    dev = torch.device("cuda")
    S = x.h0.to(dev).contiguous()
    outs = []
    for t in range(T):
        outs.append(pkg.gla_decode_step(x.q[:, :, t].to(dev).contiguous(), x.k[:, :, t].to(dev).contiguous(),
                                        x.v[:, :, t].to(dev).contiguous(),
                                        x.log_alpha[:, :, t].to(dev).contiguous(), S))
    torch.cuda.synchronize()
    o = torch.stack(outs, dim=2)
    ro, rhT = oracle.fwd(_np(x.q), _np(x.k), _np(x.v), _np(x.log_alpha), h0=_np(x.h0))
    eo, eS = rel_err(_np(o), ro), rel_err(_np(S), rhT)
    print("decode chain", dtype, f"o {eo:.2e} state {eS:.2e}")
    assert eo <= TOL[dtype] and eS <= 5e-3, (eo, eS)


def test_decode_step_matches_forward_final_state():
    """A decode step continuing from gla_fwd's final state gives the same output as
    gla_fwd over the sequence extended by that token (the last row)."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    B, H, T, K, V = 2, 4, 257, 256, 512
    x = make_inputs(B, H, T + 1, K, V, dtype=BF16, gate="vector", seed=13)
    dev = torch.device("cuda")
    g = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "log_alpha")}
    o_full, _ = pkg.gla_fwd(g["q"], g["k"], g["v"], g["log_alpha"], None, chunk=64)
    _, hT = pkg.gla_fwd(*(g[n][:, :, :T].contiguous() for n in ("q", "k", "v", "log_alpha")), None, chunk=64)
    o_last = pkg.gla_decode_step(*(g[n][:, :, T].contiguous() for n in ("q", "k", "v", "log_alpha")), hT)
    torch.cuda.synchronize()
    e = rel_err(_np(o_last), _np(o_full[:, :, T]))
    print("decode after forward", f"{e:.2e}")
    assert e <= TOL[BF16], e
