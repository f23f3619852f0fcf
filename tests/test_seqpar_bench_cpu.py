"""bench.py's sequence-parallel mode on the CPU: the piece bounds, the per-rank step
and the gather of the pieces, run on gloo ranks with the float64 oracle as the
compute steps (the same stand-in as tests/test_seqpar_cpu.py).  The gathered
pieces must equal the oracle on the whole sequence, and every rank must hold the
same gathered tensors."""
import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tests.test_seqpar_cpu import _free_port, _inputs, oracle_ops


def test_seqpar_bounds():
    import bench
    for T, world, C in [(4096, 8, 64), (4096, 3, 64), (150, 4, 16), (150, 10, 16), (64, 1, 64), (1, 1, 64)]:
        cuts = bench.seqpar_bounds(T, world, C)
        assert len(cuts) == world + 1 and cuts[0] == 0 and cuts[-1] == T
        lens = [cuts[r + 1] - cuts[r] for r in range(world)]
        assert all(n > 0 for n in lens)
        assert all(c % C == 0 for c in cuts[:-1])      # every piece starts on a chunk boundary
        n_chunks = [-(-n // C) for n in lens]
        assert max(n_chunks) - min(n_chunks) <= 1      # as equal as whole chunks allow
    assert bench.seqpar_bounds(4096, 8, 64) == [512 * r for r in range(9)]
    with pytest.raises(ValueError):
        bench.seqpar_bounds(100, 3, 64)                 # two chunks for three pieces


def test_tensor_rel_err():
    import bench
    b = torch.tensor([[1.0, -4.0], [2.0, 0.5]])
    assert bench.tensor_rel_err(b, b) == 0.0
    a = b.clone()
    a[1, 1] += 0.2
    assert bench.tensor_rel_err(a, b) == pytest.approx(0.2 / 4.0)
    assert bench.tensor_rel_err(torch.zeros(0), torch.zeros(0)) == 0.0


def _worker(rank, world, port, T, gate, out):
    import os

    import torch.distributed as dist

    import bench
    from oracle import oracle
    oracle.build()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ops = oracle_ops(gate)
        q, k, v, la, do, h0, dhT = _inputs(T, gate, seed=5)
        cuts = bench.seqpar_bounds(T, world, 16)
        lo, hi = cuts[rank], cuts[rank + 1]
        piece = [None if t is None else t[:, :, lo:hi].contiguous() for t in (q, k, v, la, do)]
        o, dq, dk, dv, dla, h_out, dh_in = bench.seqpar_step(ops, piece, h0, dhT)
        g = {name: None if t is None else bench.gather_pieces(t, cuts).numpy()
             for name, t in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv), ("dla", dla))}
        out[rank] = {**g, "h_out": h_out.numpy(), "dh_in": dh_in.numpy(), "cuts": cuts}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,gate", [(2, 150, "vector"), (3, 150, "scalar"), (4, 150, "vector")])
def test_bench_seqpar_step_matches_whole_sequence(oracle_mod, world, T, gate):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, T, gate, out), nprocs=world, join=True, start_method="spawn")
    q, k, v, la, do, h0, dhT = _inputs(T, gate, seed=5)
    ops = oracle_ops(gate)
    o, hT = ops.fwd(q, k, v, la, h0)
    dq, dk, dv, dla, dh0 = ops.bwd(q, k, v, la, do, h0, dhT)
    want = {"o": o, "dq": dq, "dk": dk, "dv": dv, "dla": dla}
    for r in range(world):
        for name, ref in want.items():
            np.testing.assert_allclose(out[r][name], ref.numpy(), rtol=1e-10, atol=1e-10, err_msg=f"{name} rank {r}")
    np.testing.assert_allclose(out[world - 1]["h_out"], hT.numpy(), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(out[0]["dh_in"], dh0.numpy(), rtol=1e-10, atol=1e-10)
    assert out[0]["cuts"][-1] == T and len(out[0]["cuts"]) == world + 1


def test_bench_seqpar_step_without_process_group(oracle_mod):
    """One process and no process group: the sequence is one piece and the step is
    the plain forward and backward."""
    import bench
    q, k, v, la, do, h0, dhT = _inputs(100, "vector", seed=2)
    ops = oracle_ops("vector")
    o, dq, dk, dv, dla, h_out, dh_in = bench.seqpar_step(ops, (q, k, v, la, do), h0, dhT)
    ro, rh = ops.fwd(q, k, v, la, h0)
    rdq, rdk, rdv, rdla, rdh0 = ops.bwd(q, k, v, la, do, h0, dhT)
    for a, b in ((o, ro), (h_out, rh), (dq, rdq), (dk, rdk), (dv, rdv), (dla, rdla), (dh_in, rdh0)):
        np.testing.assert_allclose(a.numpy(), b.numpy(), rtol=0, atol=0)
    cuts = bench.seqpar_bounds(100, 1, 16)
    assert bench.gather_pieces(o, cuts) is o
