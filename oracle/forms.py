"""Independent float64 restatements of GLA used to pin the recurrent oracle.

TEST INFRASTRUCTURE ONLY (never imported by the product path).

Each function is a different formulation of the same map, written out from
"Gated Linear Attention Transformers with Hardware-Efficient Training"
(arXiv:2312.06635), single head, numpy float64, no blocking beyond what the
formulation itself states.  Shapes (one head): q,k [T,K]; v [T,V];
la [T,K] log-gates (vector mode; scalar / none modes are expanded by the
caller); h0 [K,V] or None.
"""
from __future__ import annotations

import numpy as np


def brute_force(q, k, v, la, h0=None):
    """Unrolled recurrence (section 4.1, "parallel form" before b_t is
    introduced): o_t = sum_{i<=t} (q_t (.) prod_{j=i+1..t} alpha_j) k_i^T v_i
    + (q_t (.) prod_{j=1..t} alpha_j) h0, with the decay products formed by
    explicit multiplication of the gates (no logs, no cumulative sums).
    Tiny inputs only (O(T^2 K V))."""
    T, K = q.shape
    V = v.shape[1]
    alpha = np.exp(la)
    o = np.zeros((T, V))
    for t in range(T):
        for i in range(t + 1):
            decay = np.ones(K)
            for j in range(i + 1, t + 1):
                decay = decay * alpha[j]
            w = float(np.sum(q[t] * decay * k[i]))
            o[t] += w * v[i]
        if h0 is not None:
            decay = np.ones(K)
            for j in range(0, t + 1):
                decay = decay * alpha[j]
            o[t] += (q[t] * decay) @ h0
    return o


def parallel_form(q, k, v, la, h0=None):
    """Masked parallel form O = ((Q (.) B)(K / B)^T (.) M) V with
    b_t = prod_{j<=t} alpha_j (section 4.1; Appendix C.1 with beta = 1),
    plus the h0 term (Q (.) B) h0.  Only valid while b_t does not underflow,
    i.e. for short sequences -- the paper's own reason for the log-space and
    chunkwise forms."""
    T = q.shape[0]
    Bm = np.exp(np.cumsum(la, axis=0))
    M = np.tril(np.ones((T, T)))
    A = ((q * Bm) @ (k / Bm).T) * M
    o = A @ v
    if h0 is not None:
        o = o + (q * Bm) @ h0
    return o


def linear_attention(q, k, v):
    """Ungated causal linear attention O = (Q K^T (.) M) V (section 2.1)."""
    T = q.shape[0]
    return ((q @ k.T) * np.tril(np.ones((T, T)))) @ v


def retnet_form(q, k, v, gamma):
    """Data-independent scalar decay: O = (Q K^T (.) D) V with
    D[t,n] = gamma^(t-n) for n <= t, else 0 (the RetNet special case the paper
    names in section 4 and Appendix C.2)."""
    T = q.shape[0]
    t = np.arange(T)
    diff = t[:, None] - t[None, :]
    D = np.where(diff >= 0, float(gamma) ** np.maximum(diff, 0), 0.0)
    return ((q @ k.T) * D) @ v


def chunkwise_two_level(q, k, v, la, C, c, h0=None):
    """Chunkwise form with secondary (sub-chunk) tiling, as described in
    section 4.2 / Figure 3 and the two-level chunked forward of Appendix B,
    written here as plain numpy (the chunk-local cumulative log-gate restarts at
    every chunk and is indexed per token), plus an initial state h0 and the
    final state.

    For chunk n with chunk-local inclusive cumulative log-gate G (rows = tokens):
      inter-chunk : O_n  = (Q_n (.) e^G) S
      state       : S    = diag(e^{G_last}) S + (K_n (.) e^{G_last - G})^T V_n
      intra-chunk : the C x C causal score matrix is assembled from c x c tiles;
        a tile on the diagonal is formed entry by entry in log space,
            A[m,n] = sum_d q_m[d] k_n[d] e^{G_m[d] - G_n[d]},   n <= m,
        a tile strictly below it (query tile a, key tile b < a) is one product
        of rescaled blocks with the reference point zeta = G at the first row
        of query tile a,
            A[a,b] = (Q_a (.) e^{G_a - zeta}) (K_b (.) e^{zeta - G_b})^T,
        and O_n += A V_n.
    T need not be a multiple of C: the tail is zero padded (q = k = v = 0 and
    la = 0 beyond T), which leaves S unchanged.
    Returns (o [T,V], S_final [K,V])."""
    T, K = q.shape
    V = v.shape[1]
    assert C % c == 0
    n_chunks = -(-T // C)
    total = n_chunks * C
    Q = np.zeros((total, K)); Q[:T] = q
    Kk = np.zeros((total, K)); Kk[:T] = k
    Vv = np.zeros((total, V)); Vv[:T] = v
    L = np.zeros((total, K)); L[:T] = la
    state = np.zeros((K, V)) if h0 is None else np.array(h0, dtype=np.float64)
    out = np.zeros((total, V))
    tiles = C // c
    for n in range(n_chunks):
        rows = np.arange(n * C, (n + 1) * C)
        Qn, Kn, Vn = Q[rows], Kk[rows], Vv[rows]
        G = np.cumsum(L[rows], axis=0)
        g_last = G[-1]
        out_n = (Qn * np.exp(G)) @ state
        state = np.exp(g_last)[:, None] * state + (Kn * np.exp(g_last - G)).T @ Vn
        A = np.zeros((C, C))
        for a in range(tiles):
            qa = slice(a * c, (a + 1) * c)
            # diagonal tile, pairwise in log space: expo[m, n, d] = G_m[d] - G_n[d]
            expo = G[qa][:, None, :] - G[qa][None, :, :]
            tile = np.einsum("md,nd,mnd->mn", Qn[qa], Kn[qa], np.exp(np.minimum(expo, 0.0)))
            A[qa, qa] = np.tril(tile)
            zeta = G[a * c]
            q_res = Qn[qa] * np.exp(G[qa] - zeta)
            for b in range(a):
                kb = slice(b * c, (b + 1) * c)
                A[qa, kb] = q_res @ (Kn[kb] * np.exp(zeta - G[kb])).T
        out[rows] = out_n + A @ Vn
    return out[:T], state
