"""GPU parity of the layer epilogue (gla_epilogue_fwd / gla_epilogue_bwd through
the C ABI) against the float64 oracle: y = LayerNorm(o) * Swish(r) and its
gradients do, dr, dw, db.  Metric per output tensor: max|x - r| / max(1, max|r|),
<= 2e-2 for bf16 and 5e-3 for fp32 tensors."""
import numpy as np
import pytest
import torch

from tests.parity import rel_err

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 5e-3}


def _inputs(B, H, T, V, dtype, seed, affine):
    g = torch.Generator().manual_seed(seed)
    o = (torch.randn(B, H, T, V, generator=g, dtype=torch.float64) * 2 + 0.5).to(dtype)
    r = torch.randn(B, H, T, V, generator=g, dtype=torch.float64).to(dtype)
    dy = torch.randn(B, H, T, V, generator=g, dtype=torch.float64).to(dtype)
    w = b = None
    if affine:
        w = (1 + 0.3 * torch.randn(V, generator=g, dtype=torch.float64)).to(torch.float32)
        b = (0.2 * torch.randn(V, generator=g, dtype=torch.float64)).to(torch.float32)
    return o, r, dy, w, b


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,H,T,V,affine", [(2, 4, 333, 512, True), (1, 3, 65, 256, False), (2, 2, 17, 8, True),
                                            (1, 2, 100, 1024, True), (1, 1, 1, 776, True)])
def test_epilogue_parity(dtype, B, H, T, V, affine):
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from oracle import epilogue
    o, r, dy, w, b = _inputs(B, H, T, V, dtype, seed=V + T, affine=affine)
    dev = torch.device("cuda")
    dv_ = lambda t: None if t is None else t.to(dev)
    y = pkg.gla_epilogue_fwd(dv_(o), dv_(r), dv_(w), dv_(b))
    do_, dr, dw, db = pkg.gla_epilogue_bwd(dv_(o), dv_(r), dv_(dy), dv_(w), dv_(b))
    torch.cuda.synchronize()
    ry = epilogue.fwd(_np(o), _np(r), _np(w), _np(b))
    rdo, rdr, rdw, rdb = epilogue.bwd(_np(o), _np(r), _np(dy), _np(w), _np(b))
    errs = {"y": rel_err(_np(y), ry), "do": rel_err(_np(do_), rdo), "dr": rel_err(_np(dr), rdr),
            # dw, db are fp32 sums over B*H*T rows: held to the fp32 bar relative to their scale
            "dw": rel_err(_np(dw), rdw), "db": rel_err(_np(db), rdb)}
    print("epilogue parity", dtype, (B, H, T, V, affine), {k: f"{v:.2e}" for k, v in errs.items()})
    tol = TOL[dtype]
    assert all(errs[k] <= tol for k in ("y", "do", "dr")), errs
    assert errs["dw"] <= 5e-3 and errs["db"] <= 5e-3, errs


def test_epilogue_backward_is_deterministic_and_optional():
    """dw, db are summed in a fixed order (two calls agree bit for bit); without them
    the call needs no workspace and gives the same do, dr."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    o, r, dy, w, b = _inputs(2, 4, 513, 512, torch.bfloat16, seed=41, affine=True)
    dev = torch.device("cuda")
    o, r, dy, w, b = (t.to(dev) for t in (o, r, dy, w, b))
    a = pkg.gla_epilogue_bwd(o, r, dy, w, b)
    c = pkg.gla_epilogue_bwd(o, r, dy, w, b)
    n = pkg.gla_epilogue_bwd(o, r, dy, w, b, want_dwb=False)
    torch.cuda.synchronize()
    assert torch.equal(a[2], c[2]) and torch.equal(a[3], c[3])
    assert n[2] is None and n[3] is None
    assert torch.equal(a[0], n[0]) and torch.equal(a[1], n[1])


@pytest.mark.parametrize("B,H,T,V,dtype", [(2, 4, 4096, 512, torch.bfloat16), (1, 4, 1000, 1024, torch.float32)])
def test_epilogue_full_size_and_status(B, H, T, V, dtype):
    """Every row at the layer's full output shape (bf16: 32768 rows, about 14 per warp,
    so each warp's ring of staged rows wraps several times; fp32 at d_v = 1024: two
    stages per warp), then a clean device status word."""
    import chunkwise_linear_rnn_fwd_b200 as pkg
    from oracle import epilogue
    o, r, dy, w, b = _inputs(B, H, T, V, dtype, seed=7, affine=True)
    dev = torch.device("cuda")
    ws = pkg.alloc_workspace(pkg.epilogue_workspace_size(B, H, T, V, dtype), dev)
    od, rd, dyd, wd, bd = (t.to(dev) for t in (o, r, dy, w, b))
    y = pkg.gla_epilogue_fwd(od, rd, wd, bd, workspace=ws)
    assert pkg.poll_status(ws) == 0
    do_, dr, dw, db = pkg.gla_epilogue_bwd(od, rd, dyd, wd, bd, workspace=ws)
    assert pkg.poll_status(ws) == 0
    ry = epilogue.fwd(_np(o), _np(r), _np(w), _np(b))
    rdo, rdr, rdw, rdb = epilogue.bwd(_np(o), _np(r), _np(dy), _np(w), _np(b))
    errs = {"y": rel_err(_np(y), ry), "do": rel_err(_np(do_), rdo), "dr": rel_err(_np(dr), rdr),
            "dw": rel_err(_np(dw), rdw), "db": rel_err(_np(db), rdb)}
    print("epilogue full size", dtype, (B, H, T, V), {k: f"{v:.2e}" for k, v in errs.items()})
    assert all(errs[k] <= TOL[dtype] for k in ("y", "do", "dr")), errs
    assert errs["dw"] <= 5e-3 and errs["db"] <= 5e-3, errs
