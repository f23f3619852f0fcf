"""Pins of the float64 oracle against things other than itself.

Each check compares the oracle (literal token recurrence + BPTT, "Gated Linear
Attention Transformers with Hardware-Efficient Training", section 4.1) with a
different formulation the paper fixes, a closed form, an invariant, or finite
differences.  All run on the CPU in seconds.
"""
import json
import os

import numpy as np
import pytest

from oracle import forms

RNG = np.random.default_rng(1234)


def rand_head(T, K, V, gate_scale=1.0, rng=RNG):
    q = rng.standard_normal((T, K))
    k = rng.standard_normal((T, K)) / np.sqrt(K)
    v = rng.standard_normal((T, V))
    z = rng.standard_normal((T, K))
    la = gate_scale * np.log(1.0 / (1.0 + np.exp(-z))) / 16.0
    return q, k, v, la


def one(oracle, q, k, v, la, h0=None, gate="vector"):
    """Run the oracle on a single head given 2-D arrays."""
    def e(x):
        return None if x is None else x[None, None]
    o, hT = oracle.fwd(e(q), e(k), e(v), e(la), h0=e(h0), gate=gate)
    return o[0, 0], hT[0, 0]


# ---------------------------------------------------------------- forward pins

@pytest.mark.parametrize("T,K,V", [(1, 1, 1), (5, 3, 2), (8, 4, 4)])
def test_brute_force_tiny(oracle_mod, T, K, V):
    q, k, v, la = rand_head(T, K, V)
    h0 = RNG.standard_normal((K, V))
    for h in (None, h0):
        o, _ = one(oracle_mod, q, k, v, la, h)
        ref = forms.brute_force(q, k, v, la, h)
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_parallel_form(oracle_mod):
    """C = L: masked parallel form ((Q.B)(K/B)^T . M) V (section 4.1)."""
    q, k, v, la = rand_head(48, 8, 6)
    h0 = RNG.standard_normal((8, 6))
    o, _ = one(oracle_mod, q, k, v, la, h0)
    np.testing.assert_allclose(o, forms.parallel_form(q, k, v, la, h0), rtol=1e-11, atol=1e-11)
    o2, S2 = forms.chunkwise_two_level(q, k, v, la, C=48, c=16, h0=h0)
    np.testing.assert_allclose(o, o2, rtol=1e-11, atol=1e-11)


def test_chunk_size_one_is_recurrence(oracle_mod):
    """C = 1 chunkwise recovers the recurrent form (section 2.2)."""
    q, k, v, la = rand_head(37, 5, 7)
    o, hT = one(oracle_mod, q, k, v, la)
    o2, S2 = forms.chunkwise_two_level(q, k, v, la, C=1, c=1)
    np.testing.assert_allclose(o, o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(hT, S2, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T,C,c", [(64, 16, 4), (100, 32, 8), (130, 64, 16), (256, 64, 16), (77, 8, 8)])
def test_chunkwise_any_tiling(oracle_mod, T, C, c):
    """Any chunk / sub-chunk size (incl. a ragged tail) gives the recurrence."""
    q, k, v, la = rand_head(T, 12, 10, gate_scale=4.0)
    h0 = RNG.standard_normal((12, 10))
    o, hT = one(oracle_mod, q, k, v, la, h0)
    o2, S2 = forms.chunkwise_two_level(q, k, v, la, C=C, c=c, h0=h0)
    np.testing.assert_allclose(o, o2, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(hT, S2, rtol=1e-10, atol=1e-10)


def test_strong_gates_long_sequence(oracle_mod):
    """Decay products underflow in the naive parallel form; the oracle and the
    log-space chunkwise form stay finite and agree."""
    q, k, v, la = rand_head(300, 6, 5)
    la = np.full_like(la, -5.0)
    o, hT = one(oracle_mod, q, k, v, la)
    assert np.all(np.isfinite(o))
    o2, S2 = forms.chunkwise_two_level(q, k, v, la, C=64, c=16)
    np.testing.assert_allclose(o, o2, rtol=1e-10, atol=1e-10)


def test_ungated_is_linear_attention(oracle_mod):
    """alpha == 1 reduces to (Q K^T . M) V (section 2.1), in both the 'none'
    mode and a vector gate of exact zeros."""
    q, k, v, _ = rand_head(40, 6, 9)
    ref = forms.linear_attention(q, k, v)
    o, _ = one(oracle_mod, q, k, v, None, gate="none")
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-11)
    o, _ = one(oracle_mod, q, k, v, np.zeros_like(q))
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-11)


def test_constant_scalar_gate_is_retnet(oracle_mod):
    """A data-independent scalar decay gamma gives (Q K^T . D) V with
    D[t,n] = gamma^(t-n)."""
    q, k, v, _ = rand_head(50, 6, 4)
    gamma = 0.93
    la = np.full((50,), np.log(gamma))
    o, _ = one(oracle_mod, q, k, v, la, gate="scalar")
    np.testing.assert_allclose(o, forms.retnet_form(q, k, v, gamma), rtol=1e-11, atol=1e-11)


def test_scalar_mode_equals_broadcast_vector(oracle_mod):
    q, k, v, _ = rand_head(33, 5, 3)
    las = RNG.standard_normal(33) * 0.1 - 0.05
    o1, h1 = one(oracle_mod, q, k, v, las, gate="scalar")
    o2, h2 = one(oracle_mod, q, k, v, np.repeat(las[:, None], 5, axis=1))
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h1, h2, rtol=1e-13, atol=1e-13)


def test_segment_concatenation(oracle_mod):
    """h0 carries 'the previous segment's state' (section 2.2): running
    [0,T1) then [T1,T) from its final state equals one run."""
    q, k, v, la = rand_head(90, 7, 5)
    o, hT = one(oracle_mod, q, k, v, la)
    oa, ha = one(oracle_mod, q[:41], k[:41], v[:41], la[:41])
    ob, hb = one(oracle_mod, q[41:], k[41:], v[41:], la[41:], h0=ha)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hb, hT, rtol=1e-12, atol=1e-12)


def test_linearity_in_v_and_h0(oracle_mod):
    q, k, v, la = rand_head(30, 4, 6)
    v2 = RNG.standard_normal(v.shape)
    h0 = RNG.standard_normal((4, 6))
    h1 = RNG.standard_normal((4, 6))
    a, b = 0.7, -1.3
    o_ab, _ = one(oracle_mod, q, k, a * v + b * v2, la, a * h0 + b * h1)
    o_a, _ = one(oracle_mod, q, k, v, la, h0)
    o_b, _ = one(oracle_mod, q, k, v2, la, h1)
    np.testing.assert_allclose(o_ab, a * o_a + b * o_b, rtol=1e-12, atol=1e-12)


def test_golden_hand_computed(oracle_mod):
    """Values worked out by hand from the recurrence (tests/golden/*.json)."""
    gdir = os.path.join(os.path.dirname(__file__), "golden")
    files = sorted(f for f in os.listdir(gdir) if f.startswith("hand_") and f.endswith(".json"))
    assert files
    for f in files:
        case = json.load(open(os.path.join(gdir, f)))
        q = np.array(case["q"], float)
        k = np.array(case["k"], float)
        v = np.array(case["v"], float)
        la = np.log(np.array(case["alpha"], float))
        h0 = None if case.get("h0") is None else np.array(case["h0"], float)
        o, hT = one(oracle_mod, q, k, v, la, h0)
        np.testing.assert_allclose(o, np.array(case["o"], float), rtol=0, atol=1e-12)
        np.testing.assert_allclose(hT, np.array(case["h_final"], float), rtol=0, atol=1e-12)


def test_decode_steps_reproduce_golden(oracle_mod):
    """The decode step applied token by token reproduces the hand-computed outputs and
    final state of tests/golden/*.json (the state carried between calls)."""
    gdir = os.path.join(os.path.dirname(__file__), "golden")
    files = sorted(f for f in os.listdir(gdir) if f.startswith("hand_") and f.endswith(".json"))
    assert files
    for f in files:
        case = json.load(open(os.path.join(gdir, f)))
        q = np.array(case["q"], float)
        k = np.array(case["k"], float)
        v = np.array(case["v"], float)
        la = np.log(np.array(case["alpha"], float))
        K, V = q.shape[1], v.shape[1]
        S = np.zeros((1, 1, K, V)) if case.get("h0") is None else np.array(case["h0"], float)[None, None]
        for t in range(q.shape[0]):
            o, S = oracle_mod.decode_step(q[None, None, t], k[None, None, t], v[None, None, t],
                                          la[None, None, t], S)
            np.testing.assert_allclose(o[0, 0], np.array(case["o"], float)[t], rtol=0, atol=1e-12)
        np.testing.assert_allclose(S[0, 0], np.array(case["h_final"], float), rtol=0, atol=1e-12)


@pytest.mark.parametrize("gate", ["vector", "scalar", "none"])
def test_decode_steps_match_sequence_forward(oracle_mod, gate):
    """T decode steps from h0 equal one forward pass over the T tokens from h0, and the
    step leaves its input state untouched."""
    rng = np.random.default_rng(11)
    B, H, T, K, V = 2, 3, 5, 4, 3
    q, k, v = rng.normal(size=(B, H, T, K)), rng.normal(size=(B, H, T, K)), rng.normal(size=(B, H, T, V))
    la = None
    if gate == "vector":
        la = -rng.uniform(0.01, 2.0, size=(B, H, T, K))
    elif gate == "scalar":
        la = -rng.uniform(0.01, 2.0, size=(B, H, T))
    h0 = rng.normal(size=(B, H, K, V))
    o_ref, hT_ref = oracle_mod.fwd(q, k, v, la, h0=h0, gate=gate)
    S = h0.copy()
    for t in range(T):
        S_in, S_copy = S, S.copy()
        o, S = oracle_mod.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], None if la is None else la[:, :, t], S_in,
                                      gate=gate)
        np.testing.assert_array_equal(S_in, S_copy)
        np.testing.assert_allclose(o, o_ref[:, :, t], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S, hT_ref, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------- layer epilogue pins

def test_epilogue_normalisation_and_gate_closed_forms():
    """With w = 1, b = 0 each row of LN(o) has mean 0 and variance var/(var+eps);
    the Swish gate at r = 0 is 0 and for large r tends to r; w and b act affinely."""
    from oracle import epilogue
    rng = np.random.default_rng(31)
    o = rng.normal(size=(2, 3, 5, 16)) * 3 + 1
    ones = np.ones_like(o)
    n = epilogue.fwd(o, 50.0 * ones) / 50.0      # sigmoid(50) = 1 - 2e-22
    np.testing.assert_allclose(n.mean(axis=-1), 0.0, atol=1e-12)
    var = o.var(axis=-1)
    np.testing.assert_allclose(n.var(axis=-1), var / (var + 1e-5), rtol=1e-12)
    assert np.all(epilogue.fwd(o, 0.0 * ones) == 0.0)
    w, b = rng.normal(size=16), rng.normal(size=16)
    np.testing.assert_allclose(epilogue.fwd(o, 50.0 * ones, w, b) / 50.0, n * w + b, rtol=1e-12, atol=1e-12)
    # Swish against its definition evaluated with Python's math module
    import math
    r = np.array([-4.0, -0.5, 0.0, 0.3, 2.0])
    ref = [x / (1.0 + math.exp(-x)) for x in r]
    np.testing.assert_allclose(epilogue.fwd(np.array([[1.0, -1.0]]).repeat(5, 0), r[:, None].repeat(2, 1))[:, 0],
                               np.array(ref) * (1.0 / math.sqrt(1.0 + 1e-5)), rtol=1e-14)


def test_epilogue_gradients_finite_differences():
    """Every gradient of the epilogue against central differences of the forward."""
    from oracle import epilogue
    rng = np.random.default_rng(32)
    o, r, dy = rng.normal(size=(2, 3, 8)), rng.normal(size=(2, 3, 8)), rng.normal(size=(2, 3, 8))
    w, b = rng.normal(size=8), rng.normal(size=8)
    do, dr, dw, db = epilogue.bwd(o, r, dy, w, b)
    L = lambda o_, r_, w_, b_: float(np.sum(epilogue.fwd(o_, r_, w_, b_) * dy))
    h = 1e-6
    for name, x, g in (("o", o, do), ("r", r, dr), ("w", w, dw), ("b", b, db)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"o": o, "r": r, "w": w, "b": b}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (L(args_p["o"], args_p["r"], args_p["w"], args_p["b"])
                        - L(args_m["o"], args_m["r"], args_m["w"], args_m["b"])) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


# --------------------------------------------------------------- backward pins

def loss_of(oracle, q, k, v, la, h0, do, dhT, gate):
    o, hT = oracle.fwd(q, k, v, la, h0=h0, gate=gate)
    return float(np.sum(o * do) + np.sum(hT * dhT))


@pytest.mark.parametrize("gate", ["vector", "scalar", "none"])
def test_finite_differences(oracle_mod, gate):
    """Central differences (step 1e-6, float64) of L = <o,do> + <h_T,dh_T>
    against the BPTT gradients for every input."""
    rng = np.random.default_rng(7)
    B, H, T, K, V = 1, 2, 11, 3, 4
    q = rng.standard_normal((B, H, T, K))
    k = rng.standard_normal((B, H, T, K)) / np.sqrt(K)
    v = rng.standard_normal((B, H, T, V))
    if gate == "vector":
        la = -np.abs(rng.standard_normal((B, H, T, K))) * 0.3
    elif gate == "scalar":
        la = -np.abs(rng.standard_normal((B, H, T))) * 0.3
    else:
        la = None
    h0 = rng.standard_normal((B, H, K, V))
    do = rng.standard_normal((B, H, T, V))
    dhT = rng.standard_normal((B, H, K, V))
    dq, dk, dv, dla, dh0 = oracle_mod.bwd(q, k, v, la, do, h0=h0, dh_final=dhT, gate=gate)
    eps = 1e-6
    named = {"q": (q, dq), "k": (k, dk), "v": (v, dv), "h0": (h0, dh0)}
    if la is not None:
        named["la"] = (la, dla)
    for name, (x, g) in named.items():
        flat = x.reshape(-1)
        gflat = g.reshape(-1)
        idx = rng.choice(flat.size, size=min(flat.size, 25), replace=False)
        for i in idx:
            old = flat[i]
            flat[i] = old + eps
            lp = loss_of(oracle_mod, q, k, v, la, h0, do, dhT, gate)
            flat[i] = old - eps
            lm = loss_of(oracle_mod, q, k, v, la, h0, do, dhT, gate)
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - gflat[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, gflat[i])


@pytest.mark.parametrize("with_final", [False, True])
def test_closed_form_gate_gradient(oracle_mod, with_final):
    """The paper's closed form (section 4.3 / Appendix B): dlog b_t =
    q_t.dq_t - k_t.dk_t and dlog alpha_t = sum_{i>=t} dlog b_i, with the extra
    final-state term sum_j h_T[c,j] dh_T[c,j] when dh_T != 0 (derived from the
    same recurrence), equals back-propagation through the token loop."""
    rng = np.random.default_rng(11)
    B, H, T, K, V = 2, 1, 70, 5, 6
    q = rng.standard_normal((B, H, T, K))
    k = rng.standard_normal((B, H, T, K)) / np.sqrt(K)
    v = rng.standard_normal((B, H, T, V))
    la = np.log(1 / (1 + np.exp(-rng.standard_normal((B, H, T, K))))) / 16
    h0 = rng.standard_normal((B, H, K, V))
    do = rng.standard_normal((B, H, T, V))
    dhT = rng.standard_normal((B, H, K, V)) if with_final else None
    dq, dk, dv, dla, dh0 = oracle_mod.bwd(q, k, v, la, do, h0=h0, dh_final=dhT)
    dlogb = q * dq - k * dk
    if with_final:
        _, hT = oracle_mod.fwd(q, k, v, la, h0=h0)
        dlogb[:, :, -1, :] += np.sum(hT * dhT, axis=-1)
    closed = np.flip(np.cumsum(np.flip(dlogb, axis=2), axis=2), axis=2)
    np.testing.assert_allclose(dla, closed, rtol=1e-10, atol=1e-10)


def test_scalar_gate_gradient_sums_channels(oracle_mod):
    rng = np.random.default_rng(3)
    B, H, T, K, V = 1, 1, 20, 4, 3
    q = rng.standard_normal((B, H, T, K))
    k = rng.standard_normal((B, H, T, K))
    v = rng.standard_normal((B, H, T, V))
    las = -np.abs(rng.standard_normal((B, H, T))) * 0.2
    do = rng.standard_normal((B, H, T, V))
    _, _, _, dla_s, _ = oracle_mod.bwd(q, k, v, las, do, gate="scalar")
    _, _, _, dla_v, _ = oracle_mod.bwd(q, k, v, np.repeat(las[..., None], K, -1), do, gate="vector")
    np.testing.assert_allclose(dla_s, dla_v.sum(-1), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------ planted mistakes (CPU)

def _pins_pass(orc):
    """A compact run of the pins above against an oracle-like object."""
    try:
        test_brute_force_tiny(orc, 8, 4, 4)
        test_chunkwise_any_tiling(orc, 100, 32, 8)
        for gate in ("vector", "scalar"):
            test_finite_differences(orc, gate)
        test_closed_form_gate_gradient(orc, True)
    except AssertionError:
        return False
    return True


def test_pins_pass_on_oracle(oracle_mod):
    assert _pins_pass(oracle_mod)


@pytest.mark.parametrize("mutant", [1, 2, 3, 4])
def test_pins_catch_planted_mistakes(mutant):
    from oracle.oracle import Mutant
    assert not _pins_pass(Mutant(mutant))


# ------------------------------------------------------ general gate (appendix C)
# S_t = diag(alpha_t) S_{t-1} diag(beta_t) + k_t^T v_t, o_t = q_t S_t.

def _general_case(rng, T, K, V, with_state=True):
    q = rng.standard_normal((1, 1, T, K))
    k = rng.standard_normal((1, 1, T, K)) / np.sqrt(K)
    v = rng.standard_normal((1, 1, T, V))
    la = np.log(rng.uniform(0.6, 1.0, (1, 1, T, K)))
    lb = np.log(rng.uniform(0.6, 1.0, (1, 1, T, V)))
    h0 = rng.standard_normal((1, 1, K, V)) if with_state else None
    return q, k, v, la, lb, h0


def test_general_gate_with_unit_beta_is_the_alpha_only_oracle(oracle_mod):
    """log beta = 0 reduces the general recurrence to the paper's per-key gate."""
    rng = np.random.default_rng(21)
    q, k, v, la, lb, h0 = _general_case(rng, 37, 5, 4)
    do, dhT = rng.standard_normal((1, 1, 37, 4)), rng.standard_normal((1, 1, 5, 4))
    zero = np.zeros_like(lb)
    o1, h1 = oracle_mod.fwd(q, k, v, la, h0)
    o2, h2 = oracle_mod.fwd_general(q, k, v, la, zero, h0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(h1, h2)
    g1 = oracle_mod.bwd(q, k, v, la, do, h0, dhT)
    g2 = oracle_mod.bwd_general(q, k, v, la, zero, do, h0, dhT)
    for a, b in zip(g1, (g2[0], g2[1], g2[2], g2[3], g2[5])):
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)


def test_general_gate_parallel_form(oracle_mod):
    """The recurrence against the quadratic (parallel) form written with global
    cumulative log-gates Ag (per key channel) and Eg (per value channel):
    o_t[j] = sum_c q_t[c] e^{Ag_t[c]} h0[c,j] e^{Eg_t[j]}
           + sum_{s<=t} sum_c q_t[c] k_s[c] e^{Ag_t[c]-Ag_s[c]} v_s[j] e^{Eg_t[j]-Eg_s[j]}."""
    rng = np.random.default_rng(22)
    T, K, V = 20, 5, 4
    q, k, v, la, lb, h0 = _general_case(rng, T, K, V)
    o, hT = oracle_mod.fwd_general(q, k, v, la, lb, h0)
    Q, Kk, Vv, H0 = q[0, 0], k[0, 0], v[0, 0], h0[0, 0]
    Ag, Eg = np.cumsum(la[0, 0], axis=0), np.cumsum(lb[0, 0], axis=0)
    ref = np.zeros((T, V))
    for t in range(T):
        ref[t] = (Q[t] * np.exp(Ag[t])) @ H0 * np.exp(Eg[t])
        for s in range(t + 1):
            ref[t] += (Q[t] * Kk[s] * np.exp(Ag[t] - Ag[s])).sum() * Vv[s] * np.exp(Eg[t] - Eg[s])
    refT = np.exp(Ag[-1])[:, None] * H0 * np.exp(Eg[-1])[None, :]
    for s in range(T):
        refT += np.outer(Kk[s] * np.exp(Ag[-1] - Ag[s]), Vv[s] * np.exp(Eg[-1] - Eg[s]))
    np.testing.assert_allclose(o[0, 0], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hT[0, 0], refT, rtol=1e-12, atol=1e-12)


def test_general_gate_transpose_symmetry(oracle_mod):
    """S^T obeys the same recurrence with (k, alpha) and (v, beta) exchanged, so the
    final state of the exchanged problem is the transpose (a swapped alpha / beta
    in the state update fails this)."""
    rng = np.random.default_rng(23)
    T, K, V = 15, 4, 3
    q, k, v, la, lb, h0 = _general_case(rng, T, K, V)
    _, hT = oracle_mod.fwd_general(q, k, v, la, lb, h0)
    qv = rng.standard_normal((1, 1, T, V))
    _, hTt = oracle_mod.fwd_general(qv, v, k, lb, la, np.swapaxes(h0, 2, 3))
    np.testing.assert_allclose(hTt, np.swapaxes(hT, 2, 3), rtol=1e-12, atol=1e-12)


def test_general_gate_finite_differences(oracle_mod):
    """Every gradient of L = sum(o W) + sum(h_final U), log beta and h0 included,
    against central differences."""
    rng = np.random.default_rng(24)
    T, K, V = 6, 3, 2
    q, k, v, la, lb, h0 = _general_case(rng, T, K, V)
    W, U = rng.standard_normal((1, 1, T, V)), rng.standard_normal((1, 1, K, V))

    def loss(q, k, v, la, lb, h0):
        o, hT = oracle_mod.fwd_general(q, k, v, la, lb, h0)
        return float((o * W).sum() + (hT * U).sum())

    dq, dk, dv, dla, dlb, dh0 = oracle_mod.bwd_general(q, k, v, la, lb, W, h0, U)
    args = [q, k, v, la, lb, h0]
    for i, g in enumerate((dq, dk, dv, dla, dlb, dh0)):
        fd = np.zeros_like(args[i])
        for idx in np.ndindex(args[i].shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[i][idx] += 1e-6
            minus[i][idx] -= 1e-6
            fd[idx] = (loss(*plus) - loss(*minus)) / 2e-6
        np.testing.assert_allclose(g, fd, rtol=1e-6, atol=1e-8)


def test_general_gate_closed_form_gate_gradients(oracle_mod):
    """The closed forms the CUDA path uses, against back-propagation:
    dlog alpha_t[c] = sum_{i>=t} (q_i dq_i - k_i dk_i)[c] + sum_j hT[c,j] dhT[c,j]
    dlog beta_t[j]  = sum_{i>=t} (o_i do_i - v_i dv_i)[j] + sum_c hT[c,j] dhT[c,j]
    (log alpha_t enters through q_t e^{Ag_t} and k_t e^{-Ag_t}, log beta_t through
    o_t = e^{Eg_t} (...) and v_t e^{-Eg_t}; the h_final terms are the suffix beyond T)."""
    rng = np.random.default_rng(25)
    T, K, V = 50, 4, 5
    q, k, v, la, lb, h0 = _general_case(rng, T, K, V)
    do, dhT = rng.standard_normal((1, 1, T, V)), rng.standard_normal((1, 1, K, V))
    o, hT = oracle_mod.fwd_general(q, k, v, la, lb, h0)
    dq, dk, dv, dla, dlb, _ = oracle_mod.bwd_general(q, k, v, la, lb, do, h0, dhT)
    rev = lambda x: np.flip(np.cumsum(np.flip(x, axis=2), axis=2), axis=2)
    cla = rev(q * dq - k * dk) + (hT * dhT).sum(axis=3)[:, :, None, :]
    clb = rev(o * do - v * dv) + (hT * dhT).sum(axis=2)[:, :, None, :]
    np.testing.assert_allclose(dla, cla, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(dlb, clb, rtol=1e-10, atol=1e-10)


def _general_pins_pass(orc):
    """The general-gate pins above against an oracle-like object."""
    try:
        test_general_gate_parallel_form(orc)
        test_general_gate_transpose_symmetry(orc)
        test_general_gate_finite_differences(orc)
        test_general_gate_closed_form_gate_gradients(orc)
    except AssertionError:
        return False
    return True


def test_general_pins_pass_on_oracle(oracle_mod):
    assert _general_pins_pass(oracle_mod)


@pytest.mark.parametrize("mutant", [5, 6, 7])
def test_general_pins_catch_planted_mistakes(mutant):
    """Each planted general-gate mistake (beta after the outer product; dlog beta
    without alpha; the adjoint propagated without beta) fails a pin."""
    from oracle.oracle import Mutant
    assert not _general_pins_pass(Mutant(mutant))
