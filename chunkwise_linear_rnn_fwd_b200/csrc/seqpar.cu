// seqpar.cu -- the two small kernels of sequence (context) parallelism.
//
// "Gated Linear Attention Transformers with Hardware-Efficient Training",
// section 3.3 / 4.2: the chunk-level recurrence S_n = diag(gamma_n) S_{n-1} + dS_n
// is a composition of affine maps, so a sequence split into consecutive pieces
// (one per GPU) needs, per piece, only its summary: the gate product
// gamma = prod_t alpha_t (per key channel) and the state it produces from zero.
// The state entering piece r is the fold of the summaries of pieces 0 .. r-1 over
// the initial state; in the backward, the state adjoint leaving piece r is the
// fold of the reverse summaries of pieces r+1 .. P-1.
//
//   k_fold_segments  a piece's summary from the walk's segment contributions: the
//                    zero-state pre-pass runs every segment of the piece in parallel
//                    (contributions delta_p [BH][P][K/4][V][4], gate products gseg_p);
//                    out = fold over p of S <- diag(gseg_p) S + delta_p
//   k_segment_starts the start state of every segment of a walk from the same
//                    contributions: S = h0; S <- diag(gseg_p) S + delta_p, stored after
//                    each p as the start of the next segment ([BH][P][K/4][V][4])
//                    from h0 (dh_final in reverse), gamma = prod_p gseg_p
//   k_state_scan     out = fold over the selected pieces of S <- diag(gamma_s) S + D_s
//                    (elementwise per (bh, c, v), HBM-bound: one read of every D_s)
#include "tc_common.cuh"

namespace gla {
namespace {

// Segment contributions and start states are [BH][P][K/4][V] float4 groups (the
// four channels 4 c4 .. 4 c4 + 3 of value column v in one float4, as the walk
// stores them).  Thread (bh, c4, v), v fastest: those are read and written as
// 512 contiguous bytes per warp, the [K][V] states (h0, out) as 128 per channel.
__global__ void __launch_bounds__(256) k_fold_segments(long BH, int K, int V, int P, int reverse,
                                                       const float4 *__restrict__ gseg,
                                                       const float4 *__restrict__ delta,
                                                       const float *__restrict__ h0, float *__restrict__ out,
                                                       float4 *__restrict__ gamma) {
  const int K4 = K / 4;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;  // index in [BH][K/4][V]
  if (i >= BH * K4 * V) return;
  const int v = (int)(i % V);
  const int c4 = (int)((i / V) % K4);
  const long bh = i / ((long)V * K4);
  const long o = (bh * K + 4 * c4) * (long)V + v;  // element (4 c4, v) of [BH][K][V]
  float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
  if (h0) S = make_float4(__ldg(h0 + o), __ldg(h0 + o + V), __ldg(h0 + o + 2L * V), __ldg(h0 + o + 3L * V));
  float4 gp = make_float4(1.f, 1.f, 1.f, 1.f);
  for (int j0 = 0; j0 < P; j0 += 4) {  // the loads of four segments in flight together
    float4 g[4], d[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u, p = reverse ? P - 1 - j : j;
      g[u] = j < P ? __ldg(gseg + (bh * P + p) * K4 + c4) : make_float4(1.f, 1.f, 1.f, 1.f);
      d[u] = j < P ? __ldg(delta + ((bh * P + p) * K4 + c4) * V + v) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      S.x = g[u].x * S.x + d[u].x;
      S.y = g[u].y * S.y + d[u].y;
      S.z = g[u].z * S.z + d[u].z;
      S.w = g[u].w * S.w + d[u].w;
      gp.x *= g[u].x;
      gp.y *= g[u].y;
      gp.z *= g[u].z;
      gp.w *= g[u].w;
    }
  }
  out[o] = S.x;
  out[o + V] = S.y;
  out[o + 2L * V] = S.z;
  out[o + 3L * V] = S.w;
  if (gamma && v == 0) gamma[bh * K4 + c4] = gp;
}

// Start states of the segments of one walk: thread (bh, c4, v) folds the
// contributions in walk order (forward: 0 .. P-2; reverse: P-1 .. 1) from h0
// ([BH][K][V] or zero) and stores the state after each as the next segment's
// start (the segment that begins from h0 is not written).
__global__ void __launch_bounds__(256) k_segment_starts(long BH, int K, int V, int P, int reverse,
                                                        const float4 *__restrict__ gseg,
                                                        const float4 *__restrict__ delta,
                                                        const float *__restrict__ h0, float4 *__restrict__ starts) {
  // launched with programmatic stream serialization: wait for the walk that wrote
  // the contributions, let the next walk's CTAs be scheduled early
  dev::pdl_launch_dependents();
  dev::pdl_wait();
  const int K4 = K / 4;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;  // index in [BH][K/4][V]
  if (i >= BH * K4 * V) return;
  const int v = (int)(i % V);
  const int c4 = (int)((i / V) % K4);
  const long bh = i / ((long)V * K4);
  float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
  if (h0) {
    const long o = (bh * K + 4 * c4) * (long)V + v;
    S = make_float4(__ldg(h0 + o), __ldg(h0 + o + V), __ldg(h0 + o + 2L * V), __ldg(h0 + o + 3L * V));
  }
  for (int j0 = 0; j0 + 1 < P; j0 += 4) {  // the loads of four segments in flight together
    float4 g[4], d[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u, p = reverse ? P - 1 - j : j;
      if (j + 1 < P) {
        g[u] = __ldg(gseg + (bh * P + p) * K4 + c4);
        d[u] = __ldg(delta + ((bh * P + p) * K4 + c4) * V + v);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u, p = reverse ? P - 1 - j : j;  // segment folded in
      if (j + 1 < P) {
        S.x = g[u].x * S.x + d[u].x;
        S.y = g[u].y * S.y + d[u].y;
        S.z = g[u].z * S.z + d[u].z;
        S.w = g[u].w * S.w + d[u].w;
        starts[((bh * P + (reverse ? p - 1 : p + 1)) * K4 + c4) * V + v] = S;  // the segment it starts
      }
    }
  }
}
// Pieces s in [s_lo, s_hi), ascending (forward) or descending (reverse).
__global__ void __launch_bounds__(256) k_state_scan(long BH, int K, int V, int s_lo, int s_hi, int reverse,
                                                    const float *__restrict__ gammas,
                                                    const float4 *__restrict__ deltas,
                                                    const float4 *__restrict__ init, float4 *__restrict__ out) {
  const long n4 = BH * K * (V / 4);
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;  // float4 index in [BH][K][V/4]
  if (i >= n4) return;
  const long row = i / (V / 4);  // bh * K + c
  float4 S = init ? __ldg(init + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  const int cnt = s_hi - s_lo;
  for (int j0 = 0; j0 < cnt; j0 += 4) {  // the loads of four pieces in flight together
    float g[4];
    float4 d[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u, s = reverse ? s_hi - 1 - j : s_lo + j;
      g[u] = j < cnt ? __ldg(gammas + (long)s * BH * K + row) : 1.f;
      d[u] = j < cnt ? __ldg(deltas + (long)s * n4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      S.x = g[u] * S.x + d[u].x;
      S.y = g[u] * S.y + d[u].y;
      S.z = g[u] * S.z + d[u].z;
      S.w = g[u] * S.w + d[u].w;
    }
  }
  out[i] = S;
}

}  // namespace

int fold_segments(long BH, int K, int V, int P, int reverse, const float *gseg, const float *delta, const float *h0,
                  float *out, float *gamma, cudaStream_t st) {
  const long n = BH * (K / 4) * V;
  GLA_LAUNCH(K_FOLD_SEGMENTS, st,
             (k_fold_segments<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
                 BH, K, V, P, reverse, (const float4 *)gseg, (const float4 *)delta, h0, out, (float4 *)gamma)));
  return GLA_OK;
}

int segment_starts(long BH, int K, int V, int P, int reverse, const float *gseg, const float *delta, const float *h0,
                   float *starts, cudaStream_t st) {
  const long n = BH * (K / 4) * V;
  GLA_LAUNCH(K_SEG_STARTS, st,
             if (launch_pdl(k_segment_starts, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, BH, K, V, P,
                            reverse, (const float4 *)gseg, (const float4 *)delta, h0, (float4 *)starts) != cudaSuccess)
                 return GLA_ERR_CUDA);
  return GLA_OK;
}

int state_scan(long BH, int K, int V, int nseg, int seg, int reverse, const float *gammas, const float *deltas,
               const float *init, float *out, cudaStream_t st) {
  const int s_lo = reverse ? seg + 1 : 0;
  const int s_hi = reverse ? nseg : seg;
  const long n4 = BH * K * (V / 4);
  GLA_LAUNCH(K_STATE_SCAN, st,
             (k_state_scan<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(
                 BH, K, V, s_lo, s_hi, reverse, gammas, (const float4 *)deltas, (const float4 *)init,
                 (float4 *)out)));
  return GLA_OK;
}

}  // namespace gla
