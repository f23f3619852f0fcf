// f32_path.cu -- fp32 CUDA-core implementation of chunkwise GLA (forward + backward).
//
// This is the library's path for fp32 inputs.  It follows the chunkwise form of
// "Gated Linear Attention Transformers with Hardware-Efficient Training",
// section 4.2, with every chunk-level state materialised (section 3.3,
// Figure 1b-c) and the intra-chunk scores formed pair by pair in log space
// (exp(B_t - B_s) with B the chunk-local cumulative log-gate, s <= t), so it is
// stable for any gate strength.  All arithmetic is fp32 on CUDA cores.
//
// Kernels (grid-parallel over heads and chunks except the two state scans,
// which are parallel over heads and state elements and sequential over chunks):
//   prep     B[t,c]   chunk-local inclusive cumsum of log_alpha
//   states   H[n]     state before chunk n (H[N] = final state): each chunk's
//                     contribution as a tiled fp32 GEMM over its tokens, then a scan
//   scores   P[n]     C x C causal intra-chunk scores (pairs staged in shared memory)
//   out      o        (q (.) e^B) H[n] + P V
//   dstates  dH[n]    adjoint of the state after chunk n (GEMMs, then a reverse scan)
//   dscores  dP[n]    dO V^T (causal part)
//   dqk      dq, dk, dlog_alpha (inter terms as tiled GEMMs over d_v; closed form,
//            section 4.3, with the chunk
//            boundary term sum_v S_n[c,v] dS_n[c,v])
//   dv       dv
//
// General gate (appendix C, G_t = alpha_t^T beta_t): with log beta [B,H,T,V] the
// state is also scaled per value channel, S_t = diag(alpha_t) S_{t-1} diag(beta_t)
// + k_t^T v_t.  Every kernel then takes E[t,v], the chunk-local cumulative log beta
// (null: beta == 1, the arithmetic above unchanged), and the factors
// exp(E_t[v] - E_s[v]) join the pairs (s, t) exactly as exp(B_t[c] - B_s[c]) do on
// the key side.  The gate gradient of beta has the same closed form as alpha's on
// the other index: dlog beta_t[v] = sum_{i>=t} (o_i[v] do_i[v] - v_i[v] dv_i[v])
// with the chunk boundary term sum_c S_n[c,v] dS_n[c,v] (kernel k_dlb; o is
// recomputed in fp32 for it).
#include <cuda_bf16.h>

#include "internal.h"

namespace gla {
namespace {

template <typename T>
__device__ __forceinline__ float ld(const T *p);
template <>
__device__ __forceinline__ float ld<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

template <typename T>
__device__ __forceinline__ void st(T *p, float x);
template <>
__device__ __forceinline__ void st<float>(float *p, float x) { *p = x; }
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

struct Dims {
  int T, K, V, C, N, gate;
  long Tp;
};

constexpr int kQkTile = 64, kQkRed = 32;  // output tile and staged reduction tile of the fp32 GEMMs

// ---------------------------------------------------------------- forward

// Bc[bh, t, c] = sum_{j in chunk(t), j <= t} log_alpha[bh, j, c]; rows t >= T add 0.
__global__ void k_prep(const float *__restrict__ la, Dims d, float *__restrict__ Bc) {
  const int c = threadIdx.x;
  if (c >= d.K) return;
  const long bh = blockIdx.y;
  const int n = blockIdx.x;
  float acc = 0.f;
  for (int j = 0; j < d.C; ++j) {
    const long t = (long)n * d.C + j;
    float g = 0.f;
    if (t < d.T) {
      if (d.gate == GLA_GATE_VECTOR) g = la[(bh * d.T + t) * d.K + c];
      else if (d.gate == GLA_GATE_SCALAR) g = la[bh * d.T + t];
    }
    acc += g;
    Bc[(bh * d.Tp + t) * d.K + c] = acc;
  }
}

// E[bh, t, v] = chunk-local inclusive cumsum of log_beta (rows t >= T add 0).
__global__ void k_prep_beta(const float *__restrict__ lb, Dims d, float *__restrict__ Ec) {
  const long bh = blockIdx.y;
  const int n = blockIdx.x;
  for (int v = threadIdx.x; v < d.V; v += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < d.C; ++j) {
      const long t = (long)n * d.C + j;
      if (t < d.T) acc += lb[(bh * d.T + t) * d.V + v];
      Ec[(bh * d.Tp + t) * d.V + v] = acc;
    }
  }
}

// H[bh, n] = state before chunk n; H[bh, N] = final state: the chunk contributions
// by k_chunk_kv<MODE 0>, composed by k_states_scan.

// Chunk contributions over the chunk's tokens, a tiled fp32 GEMM per (chunk, head):
//   MODE 0 (states):  D_n[c, v] = sum_t k_t[c] e^{B_last[c] - B_t[c]} v_t[v] e^{E_last[v] - E_t[v]},
//                     written to Hs slot n + 1 (k_states_scan composes it)
//   MODE 1 (adjoints): D_n[c, v] = sum_t q_t[c] e^{B_t[c]} do_t[v] e^{E_t[v]},
//                     written to dHs slot n (k_dstates_scan composes it)
// CTA = 64 key x 64 value channels; token tiles of 32 staged in shared memory with
// coalesced loads, each exp factor applied once per staged element; 256 threads,
// 4 x 4 outputs each.  grid: x = chunk, y = channel tile, z = head.
template <typename T, int MODE>
__global__ void __launch_bounds__(256) k_chunk_kv(const T *__restrict__ a, const T *__restrict__ b,
                                                  const float *__restrict__ Bc, const float *__restrict__ Ec, Dims d,
                                                  float *__restrict__ out) {
  __shared__ float Xs[kQkRed][kQkTile + 1];  // [t][c]
  __shared__ float Ys[kQkRed][kQkTile + 1];  // [t][v]
  const int n = blockIdx.x;
  const int ctiles = (d.K + kQkTile - 1) / kQkTile;
  const int c0 = (blockIdx.y % ctiles) * kQkTile, v0 = (blockIdx.y / ctiles) * kQkTile;
  const long bh = blockIdx.z;
  const long KV = (long)d.K * d.V;
  const long last = bh * d.Tp + (long)n * d.C + d.C - 1;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int j0 = 0; j0 < d.C; j0 += kQkRed) {
    for (int idx = threadIdx.x; idx < kQkRed * kQkTile; idx += 256) {
      const int j = idx / kQkTile, r = idx % kQkTile;
      const long t = (long)n * d.C + j0 + j;
      const bool ok = j0 + j < d.C && t < d.T;
      float x = 0.f, y = 0.f;
      if (ok && c0 + r < d.K) {
        const float Bt = Bc[(bh * d.Tp + t) * d.K + c0 + r];
        x = ld(a + (bh * d.T + t) * d.K + c0 + r) * __expf(MODE == 0 ? Bc[last * d.K + c0 + r] - Bt : Bt);
      }
      if (ok && v0 + r < d.V) {
        y = ld(b + (bh * d.T + t) * d.V + v0 + r);
        if (Ec) {
          const float Et = Ec[(bh * d.Tp + t) * d.V + v0 + r];
          y *= __expf(MODE == 0 ? Ec[last * d.V + v0 + r] - Et : Et);
        }
      }
      Xs[j][r] = x;
      Ys[j][r] = y;
    }
    __syncthreads();
#pragma unroll 8
    for (int j = 0; j < kQkRed; ++j) {
      float xa[4], ya[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) xa[u] = Xs[j][4 * ty + u], ya[u] = Ys[j][4 * tx + u];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] += xa[u] * ya[w];
    }
    __syncthreads();
  }
  float *D = out + (MODE == 0 ? bh * (d.N + 1) + n + 1 : bh * d.N + n) * KV;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = c0 + 4 * ty + u;
    if (c >= d.K) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int vv = v0 + 4 * tx + w;
      if (vv < d.V) D[(long)c * d.V + vv] = acc[u][w];
    }
  }
}

// Forward scan over chunks, in place: Hs[0] = h0; Hs[n+1] = e^{B_last+E_last} Hs[n] + D_n.
__global__ void k_states_scan(const float *__restrict__ Bc, const float *__restrict__ Ec,
                              const float *__restrict__ h0, Dims d, float *__restrict__ Hs,
                              float *__restrict__ hT) {
  const long KV = (long)d.K * d.V;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;  // c * V + v
  const long bh = blockIdx.y;
  if (i >= KV) return;
  const int c = (int)(i / d.V), vi = (int)(i % d.V);
  float *H = Hs + bh * (d.N + 1) * KV + i;
  float S = h0 ? h0[bh * KV + i] : 0.f;
  H[0] = S;
  for (int n = 0; n < d.N; ++n) {
    const long last = bh * d.Tp + (long)n * d.C + d.C - 1;
    const float g = Bc[last * d.K + c] + (Ec ? Ec[last * d.V + vi] : 0.f);
    S = __expf(g) * S + H[(long)(n + 1) * KV];
    H[(long)(n + 1) * KV] = S;
  }
  if (hT) hT[bh * KV + i] = S;
}

// Reverse scan, in place: dHs[n] holds D_n on entry; dHs[N-1] = dh_final,
// dHs[n-1] = e^{B_last,n + E_last,n} dHs[n] + D_n, dh0 = e^{...0} dHs[0] + D_0.
__global__ void k_dstates_scan(const float *__restrict__ Bc, const float *__restrict__ Ec,
                               const float *__restrict__ dhT, Dims d, float *__restrict__ dHs,
                               float *__restrict__ dh0) {
  const long KV = (long)d.K * d.V;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long bh = blockIdx.y;
  if (i >= KV) return;
  const int c = (int)(i / d.V), vi = (int)(i % d.V);
  float *dH = dHs + bh * d.N * KV + i;
  float dS = dhT ? dhT[bh * KV + i] : 0.f;
  for (int n = d.N - 1; n >= 0; --n) {
    const float Dn = dH[(long)n * KV];
    dH[(long)n * KV] = dS;
    const long last = bh * d.Tp + (long)n * d.C + d.C - 1;
    const float g = Bc[last * d.K + c] + (Ec ? Ec[last * d.V + vi] : 0.f);
    dS = __expf(g) * dS + Dn;
  }
  if (dh0) dh0[bh * KV + i] = dS;
}

// Causal pair sums of one chunk, staged in shared memory:
//   MODE 0 (scores):  P[t, s]  = sum_c q_t[c] k_s[c] e^{B_t[c] - B_s[c]}      (c < d_k)
//   MODE 1 (dscores): dP[t, s] = sum_v do_t[v] v_s[v] (e^{E_t[v] - E_s[v]})   (v < d_v)
// for s <= t (0 elsewhere), every pair in log space as before.  CTA = a 64 x 64 tile
// of the chunk's (t, s) pairs; slices of 32 channels of both operands and of the
// cumulative gates staged with coalesced loads; 256 threads, 4 x 4 pairs each; tiles
// and micro-tiles wholly above the diagonal skip the arithmetic.
template <typename T, int MODE>
__global__ void __launch_bounds__(256) k_pairs(const T *__restrict__ a, const T *__restrict__ b,
                                               const float *__restrict__ G, Dims d, float *__restrict__ out) {
  __shared__ float As[kQkRed][kQkTile + 1], Bs[kQkRed][kQkTile + 1];  // [channel][row]
  __shared__ float Ga[kQkRed][kQkTile + 1], Gb[kQkRed][kQkTile + 1];
  const int W = MODE == 0 ? d.K : d.V;
  const int tiles = (d.C + kQkTile - 1) / kQkTile;
  const int n = blockIdx.x / (tiles * tiles);
  const int t0 = ((blockIdx.x / tiles) % tiles) * kQkTile, s0 = (blockIdx.x % tiles) * kQkTile;
  const long bh = blockIdx.y;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float *Pc = out + (bh * d.N + n) * (long)d.C * d.C;
  float acc[4][4] = {};
  const bool tile_live = s0 <= t0 + kQkTile - 1;
  const bool live = tile_live && s0 + 4 * tx <= t0 + 4 * ty + 3;
  if (tile_live) {
    for (int c0 = 0; c0 < W; c0 += kQkRed) {
      for (int idx = threadIdx.x; idx < kQkTile * kQkRed; idx += 256) {
        const int r = idx / kQkRed, c = idx % kQkRed;
        const long t = (long)n * d.C + t0 + r, s = (long)n * d.C + s0 + r;
        const bool okc = c0 + c < W;
        const bool okt = okc && t0 + r < d.C && t < d.T, oks = okc && s0 + r < d.C && s < d.T;
        As[c][r] = okt ? ld(a + (bh * d.T + t) * W + c0 + c) : 0.f;
        Bs[c][r] = oks ? ld(b + (bh * d.T + s) * W + c0 + c) : 0.f;
        if (G) {
          Ga[c][r] = okt ? G[(bh * d.Tp + t) * W + c0 + c] : 0.f;
          Gb[c][r] = oks ? G[(bh * d.Tp + s) * W + c0 + c] : 0.f;
        }
      }
      __syncthreads();
      if (live) {
#pragma unroll 4
        for (int c = 0; c < kQkRed; ++c) {
          float xa[4], xb[4], ga[4], gb[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            xa[u] = As[c][4 * ty + u];
            xb[u] = Bs[c][4 * tx + u];
            ga[u] = G ? Ga[c][4 * ty + u] : 0.f;
            gb[u] = G ? Gb[c][4 * tx + u] : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[u][w] += G ? xa[u] * xb[w] * __expf(ga[u] - gb[w]) : xa[u] * xb[w];
        }
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int ti = t0 + 4 * ty + u;
    if (ti >= d.C) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int si = s0 + 4 * tx + w;
      if (si < d.C) Pc[(long)ti * d.C + si] = (si <= ti && (long)n * d.C + ti < d.T) ? acc[u][w] : 0.f;
    }
  }
}

// o[t, v] = e^{E_t[v]} sum_c q_t[c] e^{B_t[c]} H[n][c, v]
//         + sum_{s<=t} P[t, s] v_s[v] e^{E_t[v] - E_s[v]}          (E null: no E factors)
// CTA = 64 tokens x 64 value channels of one chunk; the first term a staged GEMM over
// d_k, the second over the chunk's tokens with P, v and E staged; the causal mask is
// applied before the exponential (for s > t, E_t - E_s > 0 could overflow).  256
// threads, 4 x 4 outputs each.  grid: x = chunk x token tile x value tile, y = head.
template <typename T, typename TO>
__global__ void __launch_bounds__(256) k_out(const T *__restrict__ q, const T *__restrict__ v,
                                             const float *__restrict__ Bc, const float *__restrict__ Ec,
                                             const float *__restrict__ Hs, const float *__restrict__ P, Dims d,
                                             TO *__restrict__ o) {
  __shared__ float Xs[kQkRed][kQkTile + 1], Ys[kQkRed][kQkTile + 1], Zs[kQkRed][kQkTile + 1];
  const int ttiles = (d.C + kQkTile - 1) / kQkTile, vtiles = (d.V + kQkTile - 1) / kQkTile;
  const int n = blockIdx.x / (ttiles * vtiles);
  const int t0 = ((blockIdx.x / vtiles) % ttiles) * kQkTile, v0 = (blockIdx.x % vtiles) * kQkTile;
  const long bh = blockIdx.y;
  const long KV = (long)d.K * d.V;
  const float *H = Hs + (bh * (d.N + 1) + n) * KV;
  const float *Pc = P + (bh * d.N + n) * (long)d.C * d.C;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  // inter: staged q e^{B} [c][t] and H [c][v]
  for (int c0 = 0; c0 < d.K; c0 += kQkRed) {
    for (int idx = threadIdx.x; idx < kQkTile * kQkRed; idx += 256) {
      const int r = idx / kQkRed, c = idx % kQkRed;
      const long t = (long)n * d.C + t0 + r;
      const bool okc = c0 + c < d.K;
      Xs[c][r] = (okc && t0 + r < d.C && t < d.T)
                     ? ld(q + (bh * d.T + t) * d.K + c0 + c) * __expf(Bc[(bh * d.Tp + t) * d.K + c0 + c])
                     : 0.f;
      const int cc = idx / kQkTile, vv = idx % kQkTile;  // H slice, coalesced along v
      Ys[cc][vv] = (c0 + cc < d.K && v0 + vv < d.V) ? H[(long)(c0 + cc) * d.V + v0 + vv] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kQkRed; ++c) {
      float xa[4], ya[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) xa[u] = Xs[c][4 * ty + u], ya[u] = Ys[c][4 * tx + u];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] += xa[u] * ya[w];
    }
    __syncthreads();
  }
  float Et[4][4] = {};
  if (Ec) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long t = (long)n * d.C + t0 + 4 * ty + u;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int vv = v0 + 4 * tx + w;
        Et[u][w] = (t0 + 4 * ty + u < d.C && t < d.T && vv < d.V) ? Ec[(bh * d.Tp + t) * d.V + vv] : 0.f;
        acc[u][w] *= __expf(Et[u][w]);
      }
    }
  }
  // intra: staged P [s][t], v [s][v] and E [s][v] over the chunk's tokens s
  const int s_end = min(d.C, t0 + kQkTile);
  for (int s0 = 0; s0 < s_end; s0 += kQkRed) {
    for (int idx = threadIdx.x; idx < kQkTile * kQkRed; idx += 256) {
      const int r = idx % kQkTile, j = idx / kQkTile;  // P slice: row t = t0 + r, column s0 + j
      const int sj = s0 + j;
      const long sg = (long)n * d.C + sj;
      Xs[j][r] = (sj < d.C && t0 + r < d.C) ? Pc[(long)(t0 + r) * d.C + sj] : 0.f;
      const bool oks = sj < d.C && sg < d.T && v0 + r < d.V;
      Ys[j][r] = oks ? ld(v + (bh * d.T + sg) * d.V + v0 + r) : 0.f;
      // an absent token's factor e^{E_t - E_s} must be 0, not 0 * overflow
      if (Ec) Zs[j][r] = oks ? Ec[(bh * d.Tp + sg) * d.V + v0 + r] : INFINITY;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < kQkRed; ++j) {
      const int sj = s0 + j;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (sj > t0 + 4 * ty + u) continue;  // causal: s <= t
        const float pv = Xs[j][4 * ty + u];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float x = pv * Ys[j][4 * tx + w];
          acc[u][w] += Ec ? x * __expf(Et[u][w] - Zs[j][4 * tx + w]) : x;
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int ti = t0 + 4 * ty + u;
    const long t = (long)n * d.C + ti;
    if (ti >= d.C || t >= d.T) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int vv = v0 + 4 * tx + w;
      if (vv < d.V) st(o + (bh * d.T + t) * d.V + vv, acc[u][w]);
    }
  }
}

// ---------------------------------------------------------------- backward

// dH[bh, n] = adjoint of the state after chunk n (through chunks > n and dh_final):
// the chunk contributions by k_chunk_kv<MODE 1>, composed by k_dstates_scan.

// Inter-chunk terms of dq and dk, contractions over the d_v channels per chunk n:
//   A1[t, c] = sum_v do_t[v] e^{E_t[v]} H[n][c, v]
//   A2[t, c] = sum_v v_t[v] e^{E_last[v] - E_t[v]} dH[n][c, v]
// (E null: no factors).  A tiled fp32 GEMM: CTA = 64 tokens x 64 channels of one
// chunk, head and term; operand tiles of 32 value channels staged in shared memory
// with coalesced loads (each exp factor applied once per staged element); 256
// threads, 4 x 4 outputs each.
template <typename T>
__global__ void __launch_bounds__(256) k_inter_qk(const T *__restrict__ dout, const T *__restrict__ v,
                                                  const float *__restrict__ Ec, const float *__restrict__ Hs,
                                                  const float *__restrict__ dHs, Dims d, float *__restrict__ A1,
                                                  float *__restrict__ A2) {
  __shared__ float Xs[kQkRed][kQkTile + 1];  // [j][t]
  __shared__ float Ys[kQkRed][kQkTile + 1];  // [j][c]
  const int tpc = (d.C + kQkTile - 1) / kQkTile;  // token tiles per chunk
  // grid: x = chunk x token tile, y = channel tile x term, z = head
  const int n = blockIdx.x / tpc, t0 = (blockIdx.x % tpc) * kQkTile;
  const long bh = blockIdx.z;
  const int which = blockIdx.y & 1;  // 0: A1 (do, H), 1: A2 (v, dH)
  const int c0 = (blockIdx.y >> 1) * kQkTile;
  const long KV = (long)d.K * d.V;
  const T *X = which ? v : dout;
  const float *M = which ? dHs + (bh * d.N + n) * KV : Hs + (bh * (d.N + 1) + n) * KV;
  const float *El = Ec ? Ec + (bh * d.Tp + (long)n * d.C + d.C - 1) * d.V : nullptr;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int j0 = 0; j0 < d.V; j0 += kQkRed) {
    for (int idx = threadIdx.x; idx < kQkTile * kQkRed; idx += 256) {
      const int r = idx / kQkRed, j = idx % kQkRed;
      const int ti = t0 + r;
      const long t = (long)n * d.C + ti;
      float x = 0.f;
      if (ti < d.C && t < d.T && j0 + j < d.V) {
        x = ld(X + (bh * d.T + t) * d.V + j0 + j);
        if (Ec) {
          const float Et = Ec[(bh * d.Tp + t) * d.V + j0 + j];
          x *= __expf(which ? El[j0 + j] - Et : Et);
        }
      }
      Xs[j][r] = x;
      Ys[j][r] = (c0 + r < d.K && j0 + j < d.V) ? M[(long)(c0 + r) * d.V + j0 + j] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int j = 0; j < kQkRed; ++j) {
      float xa[4], ya[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) xa[u] = Xs[j][4 * ty + u], ya[u] = Ys[j][4 * tx + u];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] += xa[u] * ya[w];
    }
    __syncthreads();
  }
  float *A = which ? A2 : A1;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int ti = t0 + 4 * ty + u;
    if (ti >= d.C) continue;
    const long t = (long)n * d.C + ti;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int c = c0 + 4 * tx + w;
      if (c < d.K) A[(bh * d.Tp + t) * d.K + c] = acc[u][w];
    }
  }
}

// One block per (chunk, head), one thread per key channel c:
//   dq_t = e^{B_t} (do_t H[n]^T) + sum_{s<=t} dP[t,s] k_s e^{B_t - B_s}
//   dk_t = e^{B_last - B_t} (v_t dH[n]^T) + sum_{s>=t} dP[s,t] q_s e^{B_s - B_t}
// with the two contractions over d_v (A1, A2) from k_inter_qk
//   dlog b_t = q_t dq_t - k_t dk_t   (closed form, section 4.3)
//   dlog alpha_t = sum_{i >= t in chunk} dlog b_i + G_n,  G_n[c] = sum_v S_n[c,v] dS_n[c,v]
// (S_n = H[n+1] the state after chunk n, dS_n = dH[n] its adjoint), which is the
// suffix of dlog b beyond the chunk, so no cross-chunk scan is needed.
template <typename T>
__global__ void k_dqk(const T *__restrict__ q, const T *__restrict__ k,
                      const float *__restrict__ Bc, const float *__restrict__ Hs, const float *__restrict__ dHs,
                      const float *__restrict__ dP, const float *__restrict__ A1, const float *__restrict__ A2, Dims d,
                      T *__restrict__ dq, T *__restrict__ dk, float *__restrict__ dgv) {
  __shared__ float Gs[256];  // d_k <= 256
  const int c = threadIdx.x;
  const long bh = blockIdx.y;
  const int n = blockIdx.x;
  const long KV = (long)d.K * d.V;
  // G[c] = sum_v S_n[c, v] dS_n[c, v]: each warp reduces whole rows, lanes along v
  // (coalesced), every thread of the block taking part
  {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const float *Hn = Hs + (bh * (d.N + 1) + n + 1) * KV;
    const float *dH = dHs + (bh * d.N + n) * KV;
    for (int r = warp; r < d.K; r += nw) {
      float acc = 0.f;
      for (int j = lane; j < d.V; j += 32) acc += Hn[(long)r * d.V + j] * dH[(long)r * d.V + j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) Gs[r] = acc;
    }
  }
  __syncthreads();
  if (c >= d.K) return;
  const float *dPc = dP + (bh * d.N + n) * (long)d.C * d.C;
  const float blast = Bc[(bh * d.Tp + (long)n * d.C + d.C - 1) * d.K + c];
  const float G = Gs[c];
  // pass 1: dlog b per token into dgv, dq and dk stored
  for (int ti = 0; ti < d.C; ++ti) {
    const long t = (long)n * d.C + ti;
    if (t >= d.T) break;
    const float Bt = Bc[(bh * d.Tp + t) * d.K + c];
    const float a1 = A1[(bh * d.Tp + t) * d.K + c], a2 = A2[(bh * d.Tp + t) * d.K + c];
    float dqv = __expf(Bt) * a1;
    float dkv = __expf(blast - Bt) * a2;
    for (int si = 0; si <= ti; ++si) {
      const long s = (long)n * d.C + si;
      dqv += dPc[ti * d.C + si] * ld(k + (bh * d.T + s) * d.K + c) * __expf(Bt - Bc[(bh * d.Tp + s) * d.K + c]);
    }
    for (int si = ti; si < d.C; ++si) {
      const long s = (long)n * d.C + si;
      if (s >= d.T) break;
      dkv += dPc[si * d.C + ti] * ld(q + (bh * d.T + s) * d.K + c) * __expf(Bc[(bh * d.Tp + s) * d.K + c] - Bt);
    }
    st(dq + (bh * d.T + t) * d.K + c, dqv);
    st(dk + (bh * d.T + t) * d.K + c, dkv);
    dgv[(bh * d.Tp + t) * d.K + c] = ld(q + (bh * d.T + t) * d.K + c) * dqv - ld(k + (bh * d.T + t) * d.K + c) * dkv;
  }
  // pass 2: reverse cumulative sum within the chunk plus the boundary term
  float run = G;
  for (int ti = d.C - 1; ti >= 0; --ti) {
    const long t = (long)n * d.C + ti;
    if (t >= d.T) continue;
    run += dgv[(bh * d.Tp + t) * d.K + c];
    dgv[(bh * d.Tp + t) * d.K + c] = run;
  }
}

// dv_t = e^{E_last - E_t} (k_t (.) e^{B_last - B_t}) dH[n] + sum_{s>=t} P[s,t] do_s e^{E_s - E_t}
// (E null: no E factors), tiled like k_out: the first term a staged GEMM over d_k, the
// second over the chunk's tokens s >= t (mask before the exponential).  dvf, if not
// null, receives dv in fp32 for the beta gradient.
template <typename T>
__global__ void __launch_bounds__(256) k_dv(const T *__restrict__ k, const T *__restrict__ dout,
                                            const float *__restrict__ Bc, const float *__restrict__ Ec,
                                            const float *__restrict__ dHs, const float *__restrict__ P, Dims d,
                                            T *__restrict__ dv, float *__restrict__ dvf) {
  __shared__ float Xs[kQkRed][kQkTile + 1], Ys[kQkRed][kQkTile + 1], Zs[kQkRed][kQkTile + 1];
  const int ttiles = (d.C + kQkTile - 1) / kQkTile, vtiles = (d.V + kQkTile - 1) / kQkTile;
  const int n = blockIdx.x / (ttiles * vtiles);
  const int t0 = ((blockIdx.x / vtiles) % ttiles) * kQkTile, v0 = (blockIdx.x % vtiles) * kQkTile;
  const long bh = blockIdx.y;
  const long KV = (long)d.K * d.V;
  const float *dH = dHs + (bh * d.N + n) * KV;
  const float *Pc = P + (bh * d.N + n) * (long)d.C * d.C;
  const long last = bh * d.Tp + (long)n * d.C + d.C - 1;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int c0 = 0; c0 < d.K; c0 += kQkRed) {
    for (int idx = threadIdx.x; idx < kQkTile * kQkRed; idx += 256) {
      const int r = idx / kQkRed, c = idx % kQkRed;
      const long t = (long)n * d.C + t0 + r;
      Xs[c][r] = (c0 + c < d.K && t0 + r < d.C && t < d.T)
                     ? ld(k + (bh * d.T + t) * d.K + c0 + c) *
                           __expf(Bc[last * d.K + c0 + c] - Bc[(bh * d.Tp + t) * d.K + c0 + c])
                     : 0.f;
      const int cc = idx / kQkTile, vv = idx % kQkTile;
      Ys[cc][vv] = (c0 + cc < d.K && v0 + vv < d.V) ? dH[(long)(c0 + cc) * d.V + v0 + vv] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kQkRed; ++c) {
      float xa[4], ya[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) xa[u] = Xs[c][4 * ty + u], ya[u] = Ys[c][4 * tx + u];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] += xa[u] * ya[w];
    }
    __syncthreads();
  }
  float Et[4][4] = {};
  if (Ec) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long t = (long)n * d.C + t0 + 4 * ty + u;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int vv = v0 + 4 * tx + w;
        const bool ok = t0 + 4 * ty + u < d.C && t < d.T && vv < d.V;
        Et[u][w] = ok ? Ec[(bh * d.Tp + t) * d.V + vv] : 0.f;
        acc[u][w] *= ok ? __expf(Ec[last * d.V + vv] - Et[u][w]) : 0.f;
      }
    }
  }
  for (int s0 = t0; s0 < d.C; s0 += kQkRed) {
    for (int idx = threadIdx.x; idx < kQkTile * kQkRed; idx += 256) {
      const int r = idx % kQkTile, j = idx / kQkTile;  // P slice: row s0 + j, column t0 + r
      const int sj = s0 + j;
      const long sg = (long)n * d.C + sj;
      Xs[j][r] = (sj < d.C && t0 + r < d.C) ? Pc[(long)sj * d.C + t0 + r] : 0.f;
      const bool oks = sj < d.C && sg < d.T && v0 + r < d.V;
      Ys[j][r] = oks ? ld(dout + (bh * d.T + sg) * d.V + v0 + r) : 0.f;
      // an absent token's factor e^{E_s - E_t} must be 0, not 0 * overflow
      if (Ec) Zs[j][r] = oks ? Ec[(bh * d.Tp + sg) * d.V + v0 + r] : -INFINITY;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < kQkRed; ++j) {
      const int sj = s0 + j;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (sj < t0 + 4 * ty + u) continue;  // s >= t
        const float pv = Xs[j][4 * ty + u];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float x = pv * Ys[j][4 * tx + w];
          acc[u][w] += Ec ? x * __expf(Zs[j][4 * tx + w] - Et[u][w]) : x;
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int ti = t0 + 4 * ty + u;
    const long t = (long)n * d.C + ti;
    if (ti >= d.C || t >= d.T) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int vv = v0 + 4 * tx + w;
      if (vv >= d.V) continue;
      st(dv + (bh * d.T + t) * d.V + vv, acc[u][w]);
      if (dvf) dvf[(bh * d.T + t) * d.V + vv] = acc[u][w];
    }
  }
}

// dlog beta[bh, t, v] = sum_{i >= t in chunk} (o_i[v] do_i[v] - v_i[v] dv_i[v])
//                      + sum_c S_n[c, v] dS_n[c, v]
// (o and dv in fp32; S_n = H[n+1] the state after chunk n, dS_n = dH[n] its
// adjoint: the suffix beyond the chunk, so no cross-chunk scan).  Thread = (v, chunk).
template <typename T>
__global__ void k_dlb(const T *__restrict__ v, const T *__restrict__ dout, const float *__restrict__ of,
                      const float *__restrict__ dvf, const float *__restrict__ Hs, const float *__restrict__ dHs,
                      Dims d, float *__restrict__ dlb) {
  const int vi = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = blockIdx.y;
  const long bh = blockIdx.z;
  if (vi >= d.V) return;
  const long KV = (long)d.K * d.V;
  const float *Hn = Hs + (bh * (d.N + 1) + n + 1) * KV + vi;
  const float *dH = dHs + (bh * d.N + n) * KV + vi;
  float run = 0.f;
  for (int c = 0; c < d.K; ++c) run += Hn[(long)c * d.V] * dH[(long)c * d.V];
  for (int ti = d.C - 1; ti >= 0; --ti) {
    const long t = (long)n * d.C + ti;
    if (t >= d.T) continue;
    const long i = (bh * d.T + t) * d.V + vi;
    run += of[i] * ld(dout + i) - ld(v + i) * dvf[i];
    dlb[i] = run;
  }
}

// Copy (vector gate) or channel-sum (scalar gate) the per-channel gate gradient.
__global__ void k_dg_out(const float *__restrict__ dgv, Dims d, float *__restrict__ dla) {
  const long bh = blockIdx.y;
  const long t = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= d.T) return;
  if (d.gate == GLA_GATE_VECTOR) {
    for (int c = 0; c < d.K; ++c) dla[(bh * d.T + t) * d.K + c] = dgv[(bh * d.Tp + t) * d.K + c];
  } else {
    float s = 0.f;
    for (int c = 0; c < d.K; ++c) s += dgv[(bh * d.Tp + t) * d.K + c];
    dla[bh * d.T + t] = s;
  }
}

Dims dims_of(const Problem &p) { return Dims{p.T, p.K, p.V, p.C, p.N, p.gate, p.Tp}; }

struct F32Ws {
  float *Bc, *Hs, *P, *dHs, *dP, *dgv, *A1, *A2;
  float *Ec, *of, *dvf;  // general gate only
  size_t bytes;
};

F32Ws carve(const Problem &p, void *ws, bool bwd, bool general) {
  Carve cv(ws);
  F32Ws w{};
  w.Bc = cv.take<float>((size_t)p.BH * p.Tp * p.K);
  w.Hs = cv.take<float>((size_t)p.BH * (p.N + 1) * p.K * p.V);
  w.P = cv.take<float>((size_t)p.BH * p.N * p.C * p.C);
  if (bwd) {
    w.dHs = cv.take<float>((size_t)p.BH * p.N * p.K * p.V);
    w.dP = cv.take<float>((size_t)p.BH * p.N * p.C * p.C);
    w.dgv = cv.take<float>((size_t)p.BH * p.Tp * p.K);
    w.A1 = cv.take<float>((size_t)p.BH * p.Tp * p.K);
    w.A2 = cv.take<float>((size_t)p.BH * p.Tp * p.K);
  }
  if (general) {
    w.Ec = cv.take<float>((size_t)p.BH * p.Tp * p.V);
    if (bwd) {
      w.of = cv.take<float>((size_t)p.BH * p.T * p.V);
      w.dvf = cv.take<float>((size_t)p.BH * p.T * p.V);
    }
  }
  w.bytes = cv.bytes();
  return w;
}

// Grid of k_out / k_dv: x = chunk x 64-token tile x 64-channel value tile, y = head.
dim3 tv_grid(const Problem &p) {
  const int ttiles = (p.C + kQkTile - 1) / kQkTile, vtiles = (p.V + kQkTile - 1) / kQkTile;
  return dim3((unsigned)(p.N * ttiles * vtiles), (unsigned)p.BH);
}

// Grid of k_pairs: x = chunk x 64 x 64 pair tile, y = head.
dim3 pair_grid(const Problem &p) {
  const int tiles = (p.C + kQkTile - 1) / kQkTile;
  return dim3((unsigned)(p.N * tiles * tiles), (unsigned)p.BH);
}

// States (Hs, and h_final if hT) and state adjoints (dHs, dh0): per-chunk GEMMs, then scans.
template <typename T>
int launch_states(const Problem &p, const Dims &d, const T *k, const T *v, const F32Ws &w, const float *h0,
                  float *hT, cudaStream_t st) {
  const dim3 grid(p.N, ((p.K + kQkTile - 1) / kQkTile) * ((p.V + kQkTile - 1) / kQkTile), p.BH);
  GLA_LAUNCH(K_F32_STATES, st, (k_chunk_kv<T, 0><<<grid, 256, 0, st>>>(k, v, w.Bc, w.Ec, d, w.Hs)));
  const long KV = (long)p.K * p.V;
  GLA_LAUNCH(K_F32_STATES, st,
             (k_states_scan<<<dim3((unsigned)((KV + 255) / 256), p.BH), 256, 0, st>>>(w.Bc, w.Ec, h0, d, w.Hs, hT)));
  return GLA_OK;
}

template <typename T>
int launch_dstates(const Problem &p, const Dims &d, const T *q, const T *dout, const F32Ws &w, const float *dhT,
                   float *dh0, cudaStream_t st) {
  const dim3 grid(p.N, ((p.K + kQkTile - 1) / kQkTile) * ((p.V + kQkTile - 1) / kQkTile), p.BH);
  GLA_LAUNCH(K_F32_DSTATES, st, (k_chunk_kv<T, 1><<<grid, 256, 0, st>>>(q, dout, w.Bc, w.Ec, d, w.dHs)));
  const long KV = (long)p.K * p.V;
  GLA_LAUNCH(K_F32_DSTATES, st,
             (k_dstates_scan<<<dim3((unsigned)((KV + 255) / 256), p.BH), 256, 0, st>>>(w.Bc, w.Ec, dhT, d, w.dHs,
                                                                                       dh0)));
  return GLA_OK;
}

template <typename T>
int fwd_impl(const Problem &p, const T *q, const T *k, const T *v, const float *la, const float *lb, const float *h0,
             T *o, float *hT, void *ws, cudaStream_t st) {
  const Dims d = dims_of(p);
  F32Ws w = carve(p, ws, false, lb != nullptr);
  const int kth = (p.K + 31) / 32 * 32;
  GLA_LAUNCH(K_F32_PREP, st, (k_prep<<<dim3(p.N, p.BH), kth, 0, st>>>(la, d, w.Bc)));
  if (lb) GLA_LAUNCH(K_F32_PREP, st, (k_prep_beta<<<dim3(p.N, p.BH), 256, 0, st>>>(lb, d, w.Ec)));
  if (const int r = launch_states<T>(p, d, k, v, w, h0, hT, st)) return r;
  GLA_LAUNCH(K_F32_SCORES, st, (k_pairs<T, 0><<<pair_grid(p), 256, 0, st>>>(q, k, w.Bc, d, w.P)));
  GLA_LAUNCH(K_F32_OUT, st,
             (k_out<T, T><<<tv_grid(p), 256, 0, st>>>(q, v, w.Bc, w.Ec, w.Hs, w.P, d, o)));
  return GLA_OK;
}

template <typename T>
int bwd_impl(const Problem &p, const T *q, const T *k, const T *v, const float *la, const float *lb, const float *h0,
             const T *dout, const float *dhT, T *dq, T *dk, T *dv, float *dla, float *dlb, float *dh0, void *ws,
             cudaStream_t st) {
  const Dims d = dims_of(p);
  F32Ws w = carve(p, ws, true, lb != nullptr);
  const int kth = (p.K + 31) / 32 * 32;
  GLA_LAUNCH(K_F32_PREP, st, (k_prep<<<dim3(p.N, p.BH), kth, 0, st>>>(la, d, w.Bc)));
  if (lb) GLA_LAUNCH(K_F32_PREP, st, (k_prep_beta<<<dim3(p.N, p.BH), 256, 0, st>>>(lb, d, w.Ec)));
  if (const int r = launch_states<T>(p, d, k, v, w, h0, nullptr, st)) return r;
  GLA_LAUNCH(K_F32_SCORES, st, (k_pairs<T, 0><<<pair_grid(p), 256, 0, st>>>(q, k, w.Bc, d, w.P)));
  if (const int r = launch_dstates<T>(p, d, q, dout, w, dhT, dh0, st)) return r;
  GLA_LAUNCH(K_F32_DSCORES, st, (k_pairs<T, 1><<<pair_grid(p), 256, 0, st>>>(dout, v, w.Ec, d, w.dP)));
  GLA_LAUNCH(K_F32_DQK, st,
             (k_inter_qk<T><<<dim3(p.N * ((p.C + kQkTile - 1) / kQkTile), 2 * ((p.K + kQkTile - 1) / kQkTile), p.BH), 256,
                              0, st>>>(dout, v, w.Ec, w.Hs, w.dHs, d, w.A1, w.A2)));
  GLA_LAUNCH(K_F32_DQK, st,
             (k_dqk<T><<<dim3(p.N, p.BH), kth, 0, st>>>(q, k, w.Bc, w.Hs, w.dHs, w.dP, w.A1, w.A2, d, dq, dk,
                                                         w.dgv)));
  GLA_LAUNCH(K_F32_DV, st,
             (k_dv<T><<<tv_grid(p), 256, 0, st>>>(k, dout, w.Bc, w.Ec, w.dHs, w.P, d, dv, w.dvf)));
  if (p.gate != GLA_GATE_NONE)
    GLA_LAUNCH(K_F32_DG_SCALAR, st, (k_dg_out<<<dim3((p.T + 127) / 128, p.BH), 128, 0, st>>>(w.dgv, d, dla)));
  if (lb) {
    // o in fp32 for the beta gradient, then the closed form
    GLA_LAUNCH(K_F32_OUT, st,
               (k_out<T, float><<<tv_grid(p), 256, 0, st>>>(q, v, w.Bc, w.Ec, w.Hs, w.P, d, w.of)));
    GLA_LAUNCH(K_F32_DLB, st,
               (k_dlb<T><<<dim3((p.V + 63) / 64, p.N, p.BH), 64, 0, st>>>(v, dout, w.of, w.dvf, w.Hs, w.dHs, d, dlb)));
  }
  return GLA_OK;
}

}  // namespace

size_t f32_workspace(const Problem &p, bool bwd) { return carve(p, nullptr, bwd, false).bytes; }
size_t f32_general_workspace(const Problem &p, bool bwd) { return carve(p, nullptr, bwd, true).bytes; }

int f32_fwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *lb,
            const float *h0, void *o, float *hT, void *ws, cudaStream_t st) {
  if (p.dtype == GLA_DTYPE_FP32)
    return fwd_impl<float>(p, (const float *)q, (const float *)k, (const float *)v, la, lb, h0, (float *)o, hT, ws,
                           st);
  using bf = __nv_bfloat16;
  return fwd_impl<bf>(p, (const bf *)q, (const bf *)k, (const bf *)v, la, lb, h0, (bf *)o, hT, ws, st);
}

int f32_bwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *lb,
            const float *h0, const void *dout, const float *dhT, void *dq, void *dk, void *dv, float *dla,
            float *dlb, float *dh0, void *ws, cudaStream_t st) {
  if (p.dtype == GLA_DTYPE_FP32)
    return bwd_impl<float>(p, (const float *)q, (const float *)k, (const float *)v, la, lb, h0, (const float *)dout,
                           dhT, (float *)dq, (float *)dk, (float *)dv, dla, dlb, dh0, ws, st);
  using bf = __nv_bfloat16;
  return bwd_impl<bf>(p, (const bf *)q, (const bf *)k, (const bf *)v, la, lb, h0, (const bf *)dout, dhT, (bf *)dq,
                      (bf *)dk, (bf *)dv, dla, dlb, dh0, ws, st);
}

}  // namespace gla
