"""The workspace-free forward (gla_fwd_noalloc), for callers that cannot
allocate device memory: it must give the same result as gla_fwd with a
caller-owned workspace, call after call (its scratch array is shared and keeps
the previous call's contents), and must refuse problems larger than its fixed
scratch before enqueuing anything.  This file is collected last on purpose."""
import ctypes

import pytest
import torch

import chunkwise_linear_rnn_fwd_b200 as pkg
from chunkwise_linear_rnn_fwd_b200 import gla as G
from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu


def _on_gpu(x, dev):
    return [None if t is None else t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.h0)]


@pytest.mark.parametrize("dtype,K,V", [(torch.bfloat16, 128, 256), (torch.bfloat16, 256, 512), (torch.float32, 64, 64)])
def test_noalloc_matches_workspace_entry_point(dtype, K, V):
    dev = torch.device("cuda", 0)
    # two calls in a row with different inputs and lengths: the second must not
    # see anything the first left in the shared scratch
    for seed, T in ((21, 333), (22, 200)):
        x = make_inputs(2, 2, T, K, V, dtype=dtype, gate="vector", seed=seed, with_h0=True)
        q, k, v, la, h0 = _on_gpu(x, dev)
        o_ref, h_ref = pkg.gla_fwd(q, k, v, la, h0, chunk=64)
        o_na, h_na = G.gla_fwd_noalloc(q, k, v, la, h0, chunk=64)
        torch.cuda.synchronize()
        tol = TOL[dtype]
        assert rel_err(o_na.double().cpu(), o_ref.double().cpu()) <= tol
        assert rel_err(h_na.double().cpu(), h_ref.double().cpu()) <= tol


def test_noalloc_rejects_oversize_problem():
    lib = pkg.load()
    d = G.make_desc(64, 16, 65536, 256, 512, torch.bfloat16, "vector")
    need = lib.gla_workspace_size(ctypes.byref(d), 64, 0)
    assert need > G.NOALLOC_SCRATCH_BYTES
    a = ctypes.c_void_p(4096)
    assert lib.gla_fwd_noalloc(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -4
