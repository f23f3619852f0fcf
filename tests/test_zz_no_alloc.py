"""The workspace-free forward (gla_fwd_noalloc), for callers that cannot
allocate device memory: it runs the very kernels gla_fwd runs, on the same
inputs, so its outputs must be bit-identical to gla_fwd's with a caller-owned
workspace, call after call (its scratch array is shared and keeps the previous
call's contents); they must match the float64 oracle; errors found on the
device must reach the caller through gla_poll_status_noalloc; and problems
larger than its fixed scratch are refused before anything is enqueued.  This
file is collected last on purpose."""
import ctypes

import pytest
import torch

import chunkwise_linear_rnn_fwd_b200 as pkg
from chunkwise_linear_rnn_fwd_b200 import gla as G
from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu

GLA_OK, GLA_ERR_GATE_RANGE = 0, -7


def _on_gpu(x, dev):
    return [None if t is None else t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.h0)]


@pytest.mark.parametrize("dtype,K,V", [(torch.bfloat16, 128, 256), (torch.bfloat16, 256, 512), (torch.float32, 64, 64)])
def test_noalloc_matches_workspace_entry_point(dtype, K, V):
    dev = torch.device("cuda", 0)
    assert pkg.poll_status_noalloc() == GLA_OK
    # two calls in a row with different inputs and lengths: the second must not
    # see anything the first left in the shared scratch
    for seed, T in ((21, 333), (22, 200)):
        x = make_inputs(2, 2, T, K, V, dtype=dtype, gate="vector", seed=seed, with_h0=True)
        q, k, v, la, h0 = _on_gpu(x, dev)
        o_ref, h_ref = pkg.gla_fwd(q, k, v, la, h0, chunk=64)
        o_na, h_na = G.gla_fwd_noalloc(q, k, v, la, h0, chunk=64)
        torch.cuda.synchronize()
        assert torch.equal(o_na, o_ref)
        assert torch.equal(h_na, h_ref)
        assert pkg.poll_status_noalloc() == GLA_OK


def test_noalloc_matches_oracle():
    from oracle import oracle
    dev = torch.device("cuda", 0)
    x = make_inputs(1, 2, 257, 128, 128, dtype=torch.bfloat16, gate="vector", seed=23, with_h0=True)
    q, k, v, la, h0 = _on_gpu(x, dev)
    o, hT = G.gla_fwd_noalloc(q, k, v, la, h0, chunk=64)
    torch.cuda.synchronize()
    f = lambda a: a.double().cpu().numpy()
    ro, rhT = oracle.fwd(f(x.q), f(x.k), f(x.v), f(x.log_alpha), h0=f(x.h0))
    assert rel_err(f(o.float()), ro) <= TOL[torch.bfloat16]
    assert rel_err(f(hT), rhT) <= TOL[torch.bfloat16]
    assert pkg.poll_status_noalloc() == GLA_OK


def test_noalloc_reports_gate_range():
    """log alpha = -10 per token is beyond the bf16 path's sub-chunk rescaling (a
    16-token decay of e^-160); the no-allocation forward records it in its scratch's
    status word, and gla_poll_status_noalloc returns it (then the word is clear)."""
    dev = torch.device("cuda", 0)
    x = make_inputs(1, 2, 128, 128, 128, dtype=torch.bfloat16, gate="vector", seed=24, log_alpha_const=-10.0)
    q, k, v, la, h0 = _on_gpu(x, dev)
    G.gla_fwd_noalloc(q, k, v, la, None, chunk=64)
    assert pkg.poll_status_noalloc() == GLA_ERR_GATE_RANGE
    assert pkg.poll_status_noalloc() == GLA_OK
    # the next call on the same scratch is clean
    y = make_inputs(1, 2, 128, 128, 128, dtype=torch.bfloat16, gate="vector", seed=25)
    q, k, v, la, _ = _on_gpu(y, dev)
    o_na, _ = G.gla_fwd_noalloc(q, k, v, la, None, chunk=64)
    o_ref, _ = pkg.gla_fwd(q, k, v, la, None, chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(o_na, o_ref)
    assert pkg.poll_status_noalloc() == GLA_OK


def test_noalloc_rejects_oversize_problem():
    lib = pkg.load()
    d = G.make_desc(64, 16, 65536, 256, 512, torch.bfloat16, "vector")
    need = lib.gla_workspace_size(ctypes.byref(d), 64, 0)
    assert need > G.NOALLOC_SCRATCH_BYTES
    a = ctypes.c_void_p(4096)
    assert lib.gla_fwd_noalloc(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -4
