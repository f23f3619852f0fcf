// decode.cu -- the recurrent decode step: one token per (batch, head).
//
// "Gated Linear Attention Transformers with Hardware-Efficient Training",
// section 4.1 (the recurrent form, used for generation): with the carried fp32
// state S (d_k x d_v) of a head,
//     S <- diag(alpha) S + k^T v ,     o = q S   (o reads the updated state).
// Each step reads and rewrites the whole state, so the step is bound by HBM
// bandwidth on S (2 * d_k * d_v * 4 bytes per head); it runs on CUDA cores.
//
// CTA = (64-column tile of S, head), 256 threads: thread (row group g, column
// quad j) owns columns [4j, 4j + 4) of the tile and rows g, g + 16, g + 32, ...
// A warp therefore reads and writes two 256-byte row segments per instruction,
// and every thread keeps its rows' loads in flight together.  The reduction of
// o over the rows goes through shared memory.
#include <cuda_bf16.h>

#include "internal.h"

namespace gla {
namespace {

constexpr int kDecCols = 64;                   // columns of S per CTA
constexpr int kDecThreads = 256;
constexpr int kDecQuads = kDecCols / 4;        // 16 column quads
constexpr int kDecRG = kDecThreads / kDecQuads;  // 16 row groups

__device__ __forceinline__ float ld1(const float *p) { return __ldg(p); }
__device__ __forceinline__ float ld1(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

__device__ __forceinline__ float4 ld4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ void st4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void st4(__nv_bfloat16 *p, float4 v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t *>(&a);
  u.y = *reinterpret_cast<const uint32_t *>(&b);
  *reinterpret_cast<uint2 *>(p) = u;
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads)
    k_decode(int K, int V, int gate, const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
             const float *__restrict__ la, float *__restrict__ S, T *__restrict__ o) {
  extern __shared__ float sdec[];  // q, k, alpha of this head: 3 * K floats
  __shared__ float4 red[kDecRG][kDecQuads];
  float *sq = sdec, *sk = sdec + K, *sa = sdec + 2 * K;
  const long bh = blockIdx.y;
  const int tid = threadIdx.x, jq = tid % kDecQuads, rg = tid / kDecQuads;
  for (int r = tid; r < K; r += kDecThreads) {
    sq[r] = ld1(q + bh * K + r);
    sk[r] = ld1(k + bh * K + r);
    float a = 1.f;
    if (gate == GLA_GATE_VECTOR) a = expf(__ldg(la + bh * K + r));
    else if (gate == GLA_GATE_SCALAR) a = expf(__ldg(la + bh));
    sa[r] = a;
  }
  __syncthreads();
  const int col = blockIdx.x * kDecCols + 4 * jq;
  const bool on = col < V;  // V % 4 == 0
  const float4 vv = on ? ld4(v + bh * V + col) : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float *Sh = S + bh * (long)K * V + col;
  if (on) {
#pragma unroll 8
    for (int r = rg; r < K; r += kDecRG) {
      float4 *p = reinterpret_cast<float4 *>(Sh + (long)r * V);
      float4 s = *p;
      const float a = sa[r], kr = sk[r], qr = sq[r];
      s.x = fmaf(a, s.x, kr * vv.x);
      s.y = fmaf(a, s.y, kr * vv.y);
      s.z = fmaf(a, s.z, kr * vv.z);
      s.w = fmaf(a, s.w, kr * vv.w);
      *p = s;
      acc.x = fmaf(qr, s.x, acc.x);
      acc.y = fmaf(qr, s.y, acc.y);
      acc.z = fmaf(qr, s.z, acc.z);
      acc.w = fmaf(qr, s.w, acc.w);
    }
  }
  red[rg][jq] = acc;
  __syncthreads();
  if (tid < kDecQuads) {
    const int c = blockIdx.x * kDecCols + 4 * tid;
    if (c < V) {
      float4 sum = red[0][tid];
#pragma unroll
      for (int g = 1; g < kDecRG; ++g) {
        const float4 x = red[g][tid];
        sum.x += x.x;
        sum.y += x.y;
        sum.z += x.z;
        sum.w += x.w;
      }
      st4(o + bh * V + c, sum);
    }
  }
}

}  // namespace

int decode_step(const gla_desc *d, const void *q, const void *k, const void *v, const float *la, float *state,
                void *o, cudaStream_t st) {
  const long BH = (long)d->B * d->H;
  const dim3 grid((d->dv + kDecCols - 1) / kDecCols, (unsigned)BH);
  const size_t smem = 3 * (size_t)d->dk * sizeof(float);
  if (d->dtype == GLA_DTYPE_BF16) {
    GLA_LAUNCH(K_DECODE, st,
               (k_decode<__nv_bfloat16><<<grid, kDecThreads, smem, st>>>(
                   d->dk, d->dv, d->gate, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                   (const __nv_bfloat16 *)v, la, state, (__nv_bfloat16 *)o)));
  } else {
    GLA_LAUNCH(K_DECODE, st,
               (k_decode<float><<<grid, kDecThreads, smem, st>>>(d->dk, d->dv, d->gate, (const float *)q,
                                                                  (const float *)k, (const float *)v, la, state,
                                                                  (float *)o)));
  }
  return GLA_OK;
}

}  // namespace gla
