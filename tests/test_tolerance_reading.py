"""Evidence for the tolerance reading of the bf16 parity bar (CPU only).

The bar is "max|delta| / max(1, |ref|) <= 2e-2 for bf16 inputs with fp32
accumulation".  Its numerator max|delta| is one number per tensor, so the tests
read the denominator as the tensor's scale: max_i |x_i - r_i| / max(1, max_i |r_i|).
The other reading, max_i (|x_i - r_i| / max(1, |r_i|)), divides each element's
deviation by that element's own size.

This file shows, without a GPU, that the element-wise reading is out of reach of
any implementation whose tensor-core operands are bf16, however exact its
accumulation: `simulate` evaluates the chunkwise algorithm (chunk 64, 16-token
sub-chunks with a reference point per sub-chunk pair, the diagonal sub-chunk
blocks in full precision, the closed-form gate gradient) in float64, rounding to
bf16 exactly the operands a tensor-core kernel must hand to its bf16 MMAs (the
gate-rescaled q and k, the chunk states and their adjoints, the intra-chunk
score matrices and their gradients) and nothing else.  With rounding switched
off it reproduces the float64 oracle to 1e-9, so the errors it shows with
rounding on come from the bf16 operands alone.

On one head of the 1.3B-layer workload (T = 4096, d_k = 256, d_v = 512, gates
z ~ N(-1, 1)) the tensor-scale errors sit near 3e-3, an order of magnitude under
the bar, while the element-wise error of dk exceeds it many times over (dk
reaches hundreds in size, so an entry near zero carries the absolute rounding
noise of terms that large).  The numbers are printed (pytest -s shows them).
"""
import numpy as np
import pytest
import torch

from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
from tests.parity import elem_err, rel_err

C, SUB = 64, 16


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def simulate(q, k, v, la, do, rnd=True):
    """Chunkwise forward + backward of one head in float64; `rnd` rounds the
    bf16 MMA operands.  q, k [T,K], v, do [T,V], la [T,K] (log alpha <= 0).
    Returns o, h_final, dq, dk, dv, dlog_alpha, dh0 (h0 = 0, dh_final = 0) and,
    for comparison, dlog_alpha from one reverse sum over the whole sequence."""
    bf = _bf16 if rnd else (lambda a: a)
    T, K = q.shape
    V = v.shape[1]
    N = -(-T // C)
    Tp = N * C
    pad = lambda a: np.concatenate([a, np.zeros((Tp - T, a.shape[1]))]) if Tp > T else a
    q, k, v, la, do = pad(q), pad(k), pad(v), pad(la), pad(do)
    causal = np.tril(np.ones((C, C)))

    per = []  # per chunk: (sl, b, qg, kg, gam, P)
    for n in range(N):
        sl = slice(n * C, (n + 1) * C)
        b = np.cumsum(la[sl], axis=0)                     # chunk-local cumulative log-gate
        bl = b[-1]
        qg, kg = bf(q[sl] * np.exp(b)), bf(k[sl] * np.exp(bl - b))
        P = np.zeros((C, C))
        for j in range(C // SUB):
            rows = slice(SUB * j, SUB * (j + 1))
            z = b[SUB * j - 1] if j > 0 else np.zeros(K)
            if j > 0:                                      # earlier key sub-chunks: reference z_j
                keys = slice(0, SUB * j)
                P[rows, keys] = bf(q[sl][rows] * np.exp(b[rows] - z)) @ bf(k[sl][keys] * np.exp(z - b[keys])).T
            qd, kd, bd = q[sl][rows], k[sl][rows], b[rows]  # diagonal block, full precision
            P[rows, rows] = np.einsum("tc,sc,tsc->ts", qd, kd, np.exp(bd[:, None, :] - bd[None, :, :])) * np.tril(
                np.ones((SUB, SUB)))
        per.append((sl, b, qg, kg, np.exp(bl), bf(P)))

    # forward: states carried in full precision, their bf16 copy feeds the output MMA
    S = np.zeros((K, V))
    o = np.zeros((Tp, V))
    hb = []
    for sl, b, qg, kg, gam, P in per:
        Sb = bf(S)
        hb.append(Sb)
        o[sl] = qg @ Sb + P @ v[sl]
        S = gam[:, None] * S + kg.T @ v[sl]
    h_final = S

    # backward: adjoints carried in reverse, their bf16 copy feeds dv and dk
    dS = np.zeros((K, V))
    dv = np.zeros((Tp, V))
    dhb = [None] * N
    for n in range(N - 1, -1, -1):
        sl, b, qg, kg, gam, P = per[n]
        dSb = bf(dS)
        dhb[n] = dSb
        dv[sl] = kg @ dSb + P.T @ do[sl]
        dS = gam[:, None] * dS + qg.T @ do[sl]
    dh0 = dS

    dq = np.zeros((Tp, K))
    dk = np.zeros((Tp, K))
    Gb = np.zeros((N, K))
    for n, (sl, b, qg, kg, gam, P) in enumerate(per):
        bl = b[-1]
        dP = (do[sl] @ v[sl].T) * causal
        dqi = np.zeros((C, K))
        dki = np.zeros((C, K))
        dPb = bf(dP)
        for j in range(C // SUB):
            rows = slice(SUB * j, SUB * (j + 1))
            z = b[SUB * j - 1] if j > 0 else np.zeros(K)
            if j > 0:  # dq from earlier key sub-chunks, reference z_j
                keys = slice(0, SUB * j)
                dqi[rows] += np.exp(b[rows] - z) * (dPb[rows, keys] @ bf(k[sl][keys] * np.exp(z - b[keys])))
            if j < C // SUB - 1:  # dk from later query sub-chunks, reference at the end of key sub-chunk j
                zk = b[SUB * (j + 1) - 1]
                qs = slice(SUB * (j + 1), C)
                dki[rows] += np.exp(zk - b[rows]) * (dPb[qs, rows].T @ bf(q[sl][qs] * np.exp(b[qs] - zk)))
            bd, dPd = b[rows], dP[rows, rows]
            E = np.exp(bd[:, None, :] - bd[None, :, :]) * np.tril(np.ones((SUB, SUB)))[:, :, None]
            dqi[rows] += np.einsum("ts,sc,tsc->tc", dPd, k[sl][rows], E)
            dki[rows] += np.einsum("ts,tc,tsc->sc", dPd, q[sl][rows], E)
        dkh = v[sl] @ dhb[n].T
        dq[sl] = np.exp(b) * (do[sl] @ hb[n].T) + dqi
        dk[sl] = np.exp(bl - b) * dkh + dki
        # the part of the suffix sum that lies beyond chunk n: sum_v S_n dS_n, with
        # S_n = gam h_n + kg^T V formed from the same operands as dq and dk
        Gb[n] = gam * np.sum(hb[n] * dhb[n], axis=1) + np.sum(k[sl] * np.exp(bl - b) * dkh, axis=0)
    dlb = q * dq - k * dk                                  # closed form (fp32 dq, dk, unrounded)
    dla = np.zeros((Tp, K))
    for n in range(N):                                     # suffix sums inside each chunk, plus G_n
        sl = slice(n * C, (n + 1) * C)
        dla[sl] = np.cumsum(dlb[sl][::-1], axis=0)[::-1] + Gb[n]
    dla_global = np.cumsum(dlb[::-1], axis=0)[::-1]        # one reverse sum over the whole sequence
    return o[:T], h_final, bf(dq[:T]), bf(dk[:T]), bf(dv[:T]), dla[:T], dh0, dla_global[:T]


@pytest.fixture(scope="module")
def head():
    from oracle import oracle
    oracle.build()
    x = make_inputs(1, 1, 4096, 256, 512, dtype=torch.bfloat16, gate="vector", seed=0, z_mean=-1.0)
    f = lambda a: a.double().numpy()
    q, k, v, la, do = f(x.q), f(x.k), f(x.v), f(x.log_alpha), f(x.do)
    ro, rhT = oracle.fwd(q, k, v, la)
    rdq, rdk, rdv, rdla, rdh0 = oracle.bwd(q, k, v, la, do)
    ref = dict(o=ro[0, 0], h_final=rhT[0, 0], dq=rdq[0, 0], dk=rdk[0, 0], dv=rdv[0, 0], dlog_alpha=rdla[0, 0],
               dh0=rdh0[0, 0])
    return (q[0, 0], k[0, 0], v[0, 0], la[0, 0], do[0, 0]), ref


NAMES = ("o", "h_final", "dq", "dk", "dv", "dlog_alpha", "dh0")


def test_simulation_without_rounding_is_the_oracle(head):
    inp, ref = head
    res = simulate(*inp, rnd=False)
    out = dict(zip(NAMES, res))
    for n in NAMES:
        assert rel_err(out[n], ref[n]) <= 1e-9, n
    assert rel_err(res[-1], ref["dlog_alpha"]) <= 1e-9


def test_bf16_operands_meet_tensor_scale_bar_not_elementwise(head):
    inp, ref = head
    res = simulate(*inp, rnd=True)
    out = dict(zip(NAMES, res))
    ts = {n: rel_err(out[n], ref[n]) for n in NAMES}
    el = {n: elem_err(out[n], ref[n]) for n in NAMES}
    glob = rel_err(res[-1], ref["dlog_alpha"])
    print("\nsimulated bf16-operand chunkwise path, one head of B=2 H=4 T=4096 d_k=256 d_v=512, z~N(-1,1):")
    for n in NAMES:
        print(f"  {n:11s} tensor-scale {ts[n]:.2e}   element-wise {el[n]:.2e}")
    print(f"  dlog_alpha as one reverse sum over the whole sequence: tensor-scale {glob:.2e}")
    assert max(ts.values()) <= 1e-2          # well inside the 2e-2 bar under the tensor-scale reading
    assert el["dk"] > 2e-2                    # the element-wise reading fails with exact accumulation
    assert max(el.values()) > 5 * max(ts.values())
    # the per-chunk boundary term keeps the gate gradient's error at the level of the
    # other outputs; a single reverse sum over 4096 tokens accumulates the dq, dk errors
    assert glob > 2 * ts["dlog_alpha"]
