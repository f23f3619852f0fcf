// epilogue.cu -- the GLA layer's output epilogue on CUDA cores.
//
// "Gated Linear Attention Transformers with Hardware-Efficient Training", the
// GLA layer: each head's output o_t is normalised by a LayerNorm over its d_v
// channels and multiplied by the Swish output gate r_t before the output
// projection:
//     y = (w (.) (o - mean) / sqrt(var + eps) + b) (.) r sigmoid(r)
// with one weight w and bias b of size d_v shared by every head.  The walk that
// produces o tiles d_v across CTAs, so the row statistics cannot be formed in its
// output store; the epilogue is its own pass, bound by HBM bandwidth (read o and
// r once, write y once; the backward reads o, r, dy and writes do, dr).
//
// One warp per row (batch, head, token): lane l holds the 8-element chunks
// l, l + 32, ... of the row (d_v <= 1024, a multiple of 8) in registers, so the
// mean and the variance are two passes over registers with warp shuffles.  The
// gradients of w and b are reduced deterministically: every CTA writes its
// partial sums to the caller's workspace and a second kernel adds them in order.
#include <cuda_bf16.h>

#include "internal.h"

namespace gla {
namespace {

constexpr int kEpiThreads = 256;        // 8 warps
constexpr int kEpiRowsPerWarp = 8;      // backward: rows per warp (per-CTA partials of dw, db)

__device__ __forceinline__ void ld8(const float *p, float *x) {
  const float4 a = __ldg(reinterpret_cast<const float4 *>(p)), b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void ld8(const __nv_bfloat16 *p, float *x) {
  const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void st8(float *p, const float *x) {
  reinterpret_cast<float4 *>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
  reinterpret_cast<float4 *>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void st8(__nv_bfloat16 *p, const float *x) {
  uint4 u;
  uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  *reinterpret_cast<uint4 *>(p) = u;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }

// Row statistics: mean and 1/sqrt(var + eps) of the row held in x (NCH chunks of 8
// per lane; chunk i of lane l is element 8 (l + 32 i) .. +8, valid if < V).
template <int NCH>
__device__ __forceinline__ void row_stats(const float (&x)[NCH][8], int lane, int V, float eps, float &mu,
                                          float &rstd) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NCH; ++i)
    if (8 * (lane + 32 * i) < V)
#pragma unroll
      for (int e = 0; e < 8; ++e) s += x[i][e];
  mu = warp_sum(s) / (float)V;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NCH; ++i)
    if (8 * (lane + 32 * i) < V)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = x[i][e] - mu;
        q += d * d;
      }
  rstd = rsqrtf(warp_sum(q) / (float)V + eps);
}

template <typename T, int NCH>
__global__ void __launch_bounds__(kEpiThreads)
    k_epi_fwd(long rows, int V, float eps, const T *__restrict__ o, const T *__restrict__ r,
              const float *__restrict__ w, const float *__restrict__ b, T *__restrict__ y) {
  const int lane = threadIdx.x & 31;
  const long row = (long)blockIdx.x * (kEpiThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  // o and r of the row are requested together, before the statistics need o
  float x[NCH][8], rr[NCH][8];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = 8 * (lane + 32 * i);
    if (c < V) {
      ld8(o + row * V + c, x[i]);
      ld8(r + row * V + c, rr[i]);
    }
  }
  float mu, rstd;
  row_stats<NCH>(x, lane, V, eps, mu, rstd);
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = 8 * (lane + 32 * i);
    if (c < V) {
      float ww[8], bb[8], out[8];
      if (w) ld8(w + c, ww);
      if (b) ld8(b + c, bb);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float n = (x[i][e] - mu) * rstd * (w ? ww[e] : 1.f) + (b ? bb[e] : 0.f);
        out[e] = n * (rr[i][e] * sigmoidf_(rr[i][e]));
      }
      st8(y + row * V + c, out);
    }
  }
}

// Backward; every warp takes kEpiRowsPerWarp consecutive rows and the CTA writes
// its partial sums of dw (= sum dn xhat) and db (= sum dn) to part[blockIdx.x][2][V].
template <typename T, int NCH>
__global__ void __launch_bounds__(kEpiThreads)
    k_epi_bwd(long rows, int V, float eps, const T *__restrict__ o, const T *__restrict__ r,
              const float *__restrict__ w, const float *__restrict__ b, const T *__restrict__ dy,
              T *__restrict__ dout, T *__restrict__ dr, float *__restrict__ part) {
  extern __shared__ float spart[];  // [8 warps][2][V]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float pw[NCH][8], pb[NCH][8];
#pragma unroll
  for (int i = 0; i < NCH; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) pw[i][e] = pb[i][e] = 0.f;
  const long row0 = ((long)blockIdx.x * (kEpiThreads / 32) + warp) * kEpiRowsPerWarp;
#pragma unroll 1
  for (int rr_ = 0; rr_ < kEpiRowsPerWarp; ++rr_) {
    const long row = row0 + rr_;
    if (row >= rows) break;
    float x[NCH][8];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = 8 * (lane + 32 * i);
      if (c < V) ld8(o + row * V + c, x[i]);
    }
    float mu, rstd;
    row_stats<NCH>(x, lane, V, eps, mu, rstd);
    // dxhat = dn w with dn = dy g; keep dxhat in x's registers after xhat is formed
    float dxh[NCH][8];
    float m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = 8 * (lane + 32 * i);
      if (c < V) {
        float rv[8], gy[8], ww[8], bb[8], drv[8];
        ld8(r + row * V + c, rv);
        ld8(dy + row * V + c, gy);
        if (w) ld8(w + c, ww);
        if (b) ld8(b + c, bb);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xh = (x[i][e] - mu) * rstd;
          const float we = w ? ww[e] : 1.f;
          const float n = xh * we + (b ? bb[e] : 0.f);
          const float sg = sigmoidf_(rv[e]);
          const float dn = gy[e] * (rv[e] * sg);
          drv[e] = gy[e] * n * (sg * (1.f + rv[e] * (1.f - sg)));
          pw[i][e] += dn * xh;
          pb[i][e] += dn;
          dxh[i][e] = dn * we;
          x[i][e] = xh;
          m1 += dxh[i][e];
          m2 += dxh[i][e] * xh;
        }
        st8(dr + row * V + c, drv);
      }
    }
    m1 = warp_sum(m1) / (float)V;
    m2 = warp_sum(m2) / (float)V;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = 8 * (lane + 32 * i);
      if (c < V) {
        float d[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) d[e] = rstd * (dxh[i][e] - m1 - x[i][e] * m2);
        st8(dout + row * V + c, d);
      }
    }
  }
  if (!part) return;
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = 8 * (lane + 32 * i);
    if (c < V)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        spart[(warp * 2) * V + c + e] = pw[i][e];
        spart[(warp * 2 + 1) * V + c + e] = pb[i][e];
      }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 2 * V; idx += kEpiThreads) {
    float s = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kEpiThreads / 32; ++w8) s += spart[w8 * 2 * V + idx];
    part[(long)blockIdx.x * 2 * V + idx] = s;
  }
}

// dw[c] = sum over CTAs of part[cta][0][c], db[c] likewise.  A CTA of 256 threads
// takes 32 consecutive entries of [dw | db]; warp w adds the partials w, w + 8, ...
// of its lane's entry and the 8 warp sums are added in warp order: a fixed order,
// so the result does not depend on scheduling.
__global__ void __launch_bounds__(256) k_epi_reduce(int nparts, int V, const float *__restrict__ part,
                                                    float *__restrict__ dw, float *__restrict__ db) {
  __shared__ float sred[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int idx = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (idx < 2 * V)
    for (int p = warp; p < nparts; p += 8) s += part[(long)p * 2 * V + idx];
  sred[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && idx < 2 * V) {
    float t = sred[0][lane];
#pragma unroll
    for (int w8 = 1; w8 < 8; ++w8) t += sred[w8][lane];
    if (idx < V) {
      if (dw) dw[idx] = t;
    } else if (db) {
      db[idx - V] = t;
    }
  }
}

template <int NCH>
int epi_fwd_n(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps, void *y,
              cudaStream_t st) {
  const long rows = (long)d->B * d->H * d->T;
  const unsigned grid = (unsigned)((rows + kEpiThreads / 32 - 1) / (kEpiThreads / 32));
  if (d->dtype == GLA_DTYPE_BF16)
    GLA_LAUNCH(K_EPI_FWD, st,
               (k_epi_fwd<__nv_bfloat16, NCH><<<grid, kEpiThreads, 0, st>>>(
                   rows, d->dv, eps, (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)r, w, b, (__nv_bfloat16 *)y)));
  else
    GLA_LAUNCH(K_EPI_FWD, st,
               (k_epi_fwd<float, NCH><<<grid, kEpiThreads, 0, st>>>(rows, d->dv, eps, (const float *)o,
                                                                    (const float *)r, w, b, (float *)y)));
  return GLA_OK;
}

template <int NCH>
int epi_bwd_n(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
              const void *dy, void *dout, void *dr, float *dw, float *db, cudaStream_t st) {
  const long rows = (long)d->B * d->H * d->T;
  const long per_cta = (long)(kEpiThreads / 32) * kEpiRowsPerWarp;
  const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
  float *part = (dw || db) ? (float *)d->workspace : nullptr;
  const size_t smem = (dw || db) ? (size_t)(kEpiThreads / 32) * 2 * d->dv * sizeof(float) : 0;
  if (smem > 48 * 1024) {  // the attribute belongs to the current device, so it is set on every such call
    const cudaError_t e = d->dtype == GLA_DTYPE_BF16
                              ? cudaFuncSetAttribute(k_epi_bwd<__nv_bfloat16, NCH>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                              : cudaFuncSetAttribute(k_epi_bwd<float, NCH>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return GLA_ERR_CUDA;
  }
  if (d->dtype == GLA_DTYPE_BF16)
    GLA_LAUNCH(K_EPI_BWD, st,
               (k_epi_bwd<__nv_bfloat16, NCH><<<grid, kEpiThreads, smem, st>>>(
                   rows, d->dv, eps, (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)r, w, b,
                   (const __nv_bfloat16 *)dy, (__nv_bfloat16 *)dout, (__nv_bfloat16 *)dr, part)));
  else
    GLA_LAUNCH(K_EPI_BWD, st,
               (k_epi_bwd<float, NCH><<<grid, kEpiThreads, smem, st>>>(rows, d->dv, eps, (const float *)o,
                                                                       (const float *)r, w, b, (const float *)dy,
                                                                       (float *)dout, (float *)dr, part)));
  if (part)
    GLA_LAUNCH(K_EPI_REDUCE, st,
               (k_epi_reduce<<<(2 * d->dv + 31) / 32, 256, 0, st>>>((int)grid, d->dv, part, dw, db)));
  return GLA_OK;
}

}  // namespace

size_t epilogue_workspace(const gla_desc *d) {
  const long rows = (long)d->B * d->H * d->T;
  const long per_cta = (long)(kEpiThreads / 32) * kEpiRowsPerWarp;
  return (size_t)((rows + per_cta - 1) / per_cta) * 2 * d->dv * sizeof(float);
}

int epilogue_fwd(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
                 void *y, cudaStream_t st) {
  const int nch = (d->dv + 255) / 256;
  if (nch == 1) return epi_fwd_n<1>(d, o, r, w, b, eps, y, st);
  if (nch == 2) return epi_fwd_n<2>(d, o, r, w, b, eps, y, st);
  if (nch == 3) return epi_fwd_n<3>(d, o, r, w, b, eps, y, st);
  return epi_fwd_n<4>(d, o, r, w, b, eps, y, st);
}

int epilogue_bwd(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
                 const void *dy, void *dout, void *dr, float *dw, float *db, cudaStream_t st) {
  const int nch = (d->dv + 255) / 256;
  if (nch == 1) return epi_bwd_n<1>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
  if (nch == 2) return epi_bwd_n<2>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
  if (nch == 3) return epi_bwd_n<3>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
  return epi_bwd_n<4>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
}

}  // namespace gla
