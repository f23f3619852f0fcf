/*
 * gla_oracle.c -- float64 CPU oracle for chunkwise Gated Linear Attention (GLA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may link, load or call this file.  Only the tests, the
 * smoke check and the CPU-baseline leg of the benchmark use it.
 *
 * What it computes (Yang, Wang, Shen, Panda, Kim, "Gated Linear Attention
 * Transformers with Hardware-Efficient Training", arXiv:2312.06635, section 4.1
 * "recurrent form"): for every (batch, head) independently,
 *
 *     S_t = (alpha_t^T 1) (.) S_{t-1} + k_t^T v_t ,      o_t = q_t S_t ,
 *
 * with S_t a d_k x d_v matrix, alpha_t in (0,1)^{d_k} a per-key-channel gate
 * (row t of S is scaled by alpha_t[c]), S_0 = h0 (zero if absent), and the
 * output at step t reading the state *after* step t's update (the current token
 * attends to itself).  The gate is passed as its logarithm la_t = log alpha_t.
 * Gate modes: VECTOR (la [T,d_k]), SCALAR (la [T], shared by all key channels,
 * the Mamba-2 style gamma_t 1^T 1 of the same section) and NONE (alpha == 1,
 * plain linear attention of section 2.1).
 *
 * The backward is plain back-propagation through this token loop (it does NOT
 * use the paper's closed-form gate gradient, so that the closed form can be
 * checked against it).  S_{t-1} is never reconstructed by dividing by alpha
 * (unstable); instead the forward states are checkpointed every CKPT steps and
 * each segment is recomputed forward before it is walked backward.
 *
 * General gate (appendix C of the paper, G_t = alpha_t^T beta_t): the
 * gla_oracle_*_general entry points also take lb_t = log beta_t [T, d_v], a gate
 * on the value side, so that column j of S is scaled by beta_t[j] as well:
 *
 *     S_t = diag(alpha_t) S_{t-1} diag(beta_t) + k_t^T v_t ,   o_t = q_t S_t .
 *
 * lb == NULL is beta == 1 and runs exactly the alpha-only arithmetic.
 *
 * Layout: contiguous row-major [B,H,T,D] for q,k,v,o,do,dq,dk,dv, la/dla
 * ([B,H,T,d_k] vector, [B,H,T] scalar) and lb/dlb [B,H,T,d_v]; states [B,H,d_k,d_v].
 * All arithmetic is float64.  (b,h) pairs run in parallel with OpenMP.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define GLA_ORACLE_GATE_VECTOR 0
#define GLA_ORACLE_GATE_SCALAR 1
#define GLA_ORACLE_GATE_NONE 2

#define CKPT 64

/* Planted-mistake builds for the pin tests only (default 0 = the oracle):
 *  1: output read before the state update (o_t = q_t S_{t-1})
 *  2: gate applied after the outer product (S_t = diag(alpha)(S_{t-1} + k^T v))
 *  3: gate gradient taken with S_t in place of S_{t-1}
 *  4: dk taken before the output term q_t^T do_t is added to dS
 *  5: (general gate) beta applied after the outer product
 *     (S_t = diag(alpha) S_{t-1} diag(beta) + k^T v diag(beta))
 *  6: (general gate) dlog beta accumulated without the alpha factor
 *  7: (general gate) the adjoint propagated without beta (dS <- diag(alpha) dS) */
#ifndef GLA_ORACLE_MUTANT
#define GLA_ORACLE_MUTANT 0
#endif

/* log-gate of token t, key channel c */
static inline double gate_log(const double *la, int mode, long t, int K, int c) {
  if (mode == GLA_ORACLE_GATE_VECTOR) return la[t * K + c];
  if (mode == GLA_ORACLE_GATE_SCALAR) return la[t];
  return 0.0;
}

/* One recurrence step S <- diag(alpha_t) S diag(beta_t) + k_t^T v_t (section 4.1;
 * appendix C for beta).  lbt = log beta_t [V] or NULL (beta == 1). */
static void step_state(double *S, const double *lbt, const double *kt, const double *vt,
                       const double *la, int mode, long t, int K, int V) {
  if (lbt) {
    for (int c = 0; c < K; ++c) {
      const double a = exp(gate_log(la, mode, t, K, c));
      double *row = S + (long)c * V;
#if GLA_ORACLE_MUTANT == 5
      for (int j = 0; j < V; ++j) row[j] = (a * row[j] + kt[c] * vt[j]) * exp(lbt[j]);
#else
      for (int j = 0; j < V; ++j) row[j] = a * row[j] * exp(lbt[j]) + kt[c] * vt[j];
#endif
    }
    return;
  }
  for (int c = 0; c < K; ++c) {
    const double a = exp(gate_log(la, mode, t, K, c));
    double *row = S + (long)c * V;
    const double kc = kt[c];
#if GLA_ORACLE_MUTANT == 2
    for (int j = 0; j < V; ++j) row[j] = a * (row[j] + kc * vt[j]);
#else
    for (int j = 0; j < V; ++j) row[j] = a * row[j] + kc * vt[j];
#endif
  }
}

/* o_t = q_t S_t */
static void read_out(const double *S, const double *qt, double *ot, int K, int V) {
  for (int j = 0; j < V; ++j) ot[j] = 0.0;
  for (int c = 0; c < K; ++c) {
    const double qc = qt[c];
    const double *row = S + (long)c * V;
    for (int j = 0; j < V; ++j) ot[j] += qc * row[j];
  }
}

static long la_head_stride(int mode, long T, int K) {
  if (mode == GLA_ORACLE_GATE_VECTOR) return T * K;
  if (mode == GLA_ORACLE_GATE_SCALAR) return T;
  return 0;
}

/*
 * Forward.  h0 may be NULL (zero state); hT may be NULL (not written); lb may be
 * NULL (beta == 1).
 */
void gla_oracle_fwd_general(int B, int H, long T, int K, int V, int mode,
                            const double *q, const double *k, const double *v, const double *la,
                            const double *lb, const double *h0, double *o, double *hT) {
  const long BH = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bh = 0; bh < BH; ++bh) {
    double *S = (double *)malloc(sizeof(double) * K * V);
    if (h0) memcpy(S, h0 + bh * K * V, sizeof(double) * K * V);
    else memset(S, 0, sizeof(double) * K * V);
    const double *qh = q + bh * T * K, *kh = k + bh * T * K, *vh = v + bh * T * V;
    const double *lah = la ? la + bh * la_head_stride(mode, T, K) : NULL;
    const double *lbh = lb ? lb + bh * T * V : NULL;
    double *oh = o + bh * T * V;
    for (long t = 0; t < T; ++t) {
      const double *lbt = lbh ? lbh + t * V : NULL;
#if GLA_ORACLE_MUTANT == 1
      read_out(S, qh + t * K, oh + t * V, K, V);
      step_state(S, lbt, kh + t * K, vh + t * V, lah, mode, t, K, V);
#else
      step_state(S, lbt, kh + t * K, vh + t * V, lah, mode, t, K, V);
      read_out(S, qh + t * K, oh + t * V, K, V);
#endif
    }
    if (hT) memcpy(hT + bh * K * V, S, sizeof(double) * K * V);
    free(S);
  }
}

void gla_oracle_fwd(int B, int H, long T, int K, int V, int mode,
                    const double *q, const double *k, const double *v, const double *la,
                    const double *h0, double *o, double *hT) {
  gla_oracle_fwd_general(B, H, T, K, V, mode, q, k, v, la, NULL, h0, o, hT);
}

/*
 * Backward by back-propagation through the token loop.
 *   dS <- dh_final (zero if NULL)
 *   for t = T..1:
 *     dS += q_t^T do_t                         (o_t = q_t S_t)
 *     dq_t[c]  = sum_j S_t[c,j] do_t[j]
 *     dk_t[c]  = sum_j dS[c,j] v_t[j]           (S_t = ... + k_t^T v_t)
 *     dv_t[j]  = sum_c k_t[c] dS[c,j]
 *     dla_t[c] = alpha_t[c] sum_j S_{t-1}[c,j] beta_t[j] dS[c,j]
 *     dlb_t[j] = beta_t[j] sum_c alpha_t[c] S_{t-1}[c,j] dS[c,j]
 *     dS      <- diag(alpha_t) dS diag(beta_t)
 *   dh0 = dS
 * Scalar mode returns dla_t = sum_c dla_t[c]; NONE mode writes no dla.
 * dh_final, dla, dh0 may be NULL; lb == NULL is beta == 1 (dlb then unused).
 */
void gla_oracle_bwd_general(int B, int H, long T, int K, int V, int mode,
                            const double *q, const double *k, const double *v, const double *la,
                            const double *lb, const double *h0, const double *dout, const double *dhT,
                            double *dq, double *dk, double *dv, double *dla, double *dlb, double *dh0) {
  const long BH = (long)B * H;
  const long nck = (T + CKPT - 1) / CKPT;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bh = 0; bh < BH; ++bh) {
    const long KV = (long)K * V;
    const double *qh = q + bh * T * K, *kh = k + bh * T * K, *vh = v + bh * T * V;
    const double *lah = la ? la + bh * la_head_stride(mode, T, K) : NULL;
    const double *lbh = lb ? lb + bh * T * V : NULL;
    double *dlbh = (lb && dlb) ? dlb + bh * T * V : NULL;
    const double *doh = dout + bh * T * V;
    double *dqh = dq + bh * T * K, *dkh = dk + bh * T * K, *dvh = dv + bh * T * V;
    double *dlah = (dla && mode != GLA_ORACLE_GATE_NONE) ? dla + bh * la_head_stride(mode, T, K) : NULL;

    /* checkpoints: ck[i] = state before token i*CKPT (S_{i*CKPT} in 1-based terms) */
    double *ck = (double *)malloc(sizeof(double) * KV * (nck + 1));
    double *S = (double *)malloc(sizeof(double) * KV);
    if (h0) memcpy(S, h0 + bh * KV, sizeof(double) * KV);
    else memset(S, 0, sizeof(double) * KV);
    for (long t = 0; t < T; ++t) {
      if (t % CKPT == 0) memcpy(ck + (t / CKPT) * KV, S, sizeof(double) * KV);
      step_state(S, lbh ? lbh + t * V : NULL, kh + t * K, vh + t * V, lah, mode, t, K, V);
    }

    /* seg holds S after each token of the current segment: seg[i] = state after token t0+i */
    double *seg = (double *)malloc(sizeof(double) * KV * CKPT);
    double *dS = (double *)malloc(sizeof(double) * KV);
    if (dhT) memcpy(dS, dhT + bh * KV, sizeof(double) * KV);
    else memset(dS, 0, sizeof(double) * KV);
    double *dla_vec = (double *)malloc(sizeof(double) * K);

    for (long ci = nck - 1; ci >= 0; --ci) {
      const long t0 = ci * CKPT;
      const long t1 = (t0 + CKPT < T) ? t0 + CKPT : T;
      /* recompute the segment forward from its checkpoint */
      memcpy(S, ck + ci * KV, sizeof(double) * KV);
      for (long t = t0; t < t1; ++t) {
        step_state(S, lbh ? lbh + t * V : NULL, kh + t * K, vh + t * V, lah, mode, t, K, V);
        memcpy(seg + (t - t0) * KV, S, sizeof(double) * KV);
      }
      for (long t = t1 - 1; t >= t0; --t) {
        const double *St = seg + (t - t0) * KV;                              /* S_t     */
        const double *Sp = (t > t0) ? seg + (t - t0 - 1) * KV : ck + ci * KV; /* S_{t-1} */
        const double *qt = qh + t * K, *kt = kh + t * K, *vt = vh + t * V, *dot = doh + t * V;
#if GLA_ORACLE_MUTANT == 4
        for (int c = 0; c < K; ++c) {
          double acck = 0.0;
          for (int j = 0; j < V; ++j) acck += dS[(long)c * V + j] * vt[j];
          dla_vec[c] = acck;
        }
#endif
        /* o_t = q_t S_t */
        for (int c = 0; c < K; ++c) {
          double *drow = dS + (long)c * V;
          const double *srow = St + (long)c * V;
          double acc = 0.0;
          for (int j = 0; j < V; ++j) {
            drow[j] += qt[c] * dot[j];
            acc += srow[j] * dot[j];
          }
          dqh[t * K + c] = acc;
        }
        /* S_t = diag(alpha_t) S_{t-1} diag(beta_t) + k_t^T v_t */
        const double *lbt = lbh ? lbh + t * V : NULL;
        for (int j = 0; j < V; ++j) dvh[t * V + j] = 0.0;
        if (dlbh)
          for (int j = 0; j < V; ++j) dlbh[t * V + j] = 0.0;
        for (int c = 0; c < K; ++c) {
          const double *drow = dS + (long)c * V;
          const double *prow = Sp + (long)c * V;
          const double a = exp(gate_log(lah, mode, t, K, c));
          double acck = 0.0, accg = 0.0;
          for (int j = 0; j < V; ++j) {
            acck += drow[j] * vt[j];
            dvh[t * V + j] += kt[c] * drow[j];
            const double bj = lbt ? exp(lbt[j]) : 1.0;
            accg += prow[j] * bj * drow[j];
#if GLA_ORACLE_MUTANT == 6
            if (dlbh) dlbh[t * V + j] += prow[j] * bj * drow[j];
#else
            if (dlbh) dlbh[t * V + j] += a * prow[j] * bj * drow[j];
#endif
          }
#if GLA_ORACLE_MUTANT == 4
          dkh[t * K + c] = dla_vec[c];
#else
          dkh[t * K + c] = acck;
#endif
#if GLA_ORACLE_MUTANT == 3
          accg = 0.0;
          for (int j = 0; j < V; ++j) accg += St[(long)c * V + j] * drow[j];
#endif
          dla_vec[c] = a * accg;
        }
        if (dlah) {
          if (mode == GLA_ORACLE_GATE_VECTOR) {
            for (int c = 0; c < K; ++c) dlah[t * K + c] = dla_vec[c];
          } else {
            double s = 0.0;
            for (int c = 0; c < K; ++c) s += dla_vec[c];
            dlah[t] = s;
          }
        }
        for (int c = 0; c < K; ++c) {
          const double a = exp(gate_log(lah, mode, t, K, c));
          double *drow = dS + (long)c * V;
#if GLA_ORACLE_MUTANT == 7
          if (0)
#else
          if (lbt)
#endif
            for (int j = 0; j < V; ++j) drow[j] *= a * exp(lbt[j]);
          else
            for (int j = 0; j < V; ++j) drow[j] *= a;
        }
      }
    }
    if (dh0) memcpy(dh0 + bh * KV, dS, sizeof(double) * KV);
    free(ck);
    free(S);
    free(seg);
    free(dS);
    free(dla_vec);
  }
}

void gla_oracle_bwd(int B, int H, long T, int K, int V, int mode,
                    const double *q, const double *k, const double *v, const double *la,
                    const double *h0, const double *dout, const double *dhT,
                    double *dq, double *dk, double *dv, double *dla, double *dh0) {
  gla_oracle_bwd_general(B, H, T, K, V, mode, q, k, v, la, NULL, h0, dout, dhT, dq, dk, dv, dla, NULL, dh0);
}

/* Threads OpenMP will use for the (b,h) loop. */
int gla_oracle_max_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
