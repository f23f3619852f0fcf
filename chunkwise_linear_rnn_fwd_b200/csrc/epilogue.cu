// epilogue.cu -- the GLA layer's output epilogue on CUDA cores.
//
// "Gated Linear Attention Transformers with Hardware-Efficient Training", the
// GLA layer: each head's output o_t is normalised by a LayerNorm over its d_v
// channels and multiplied by the Swish output gate r_t before the output
// projection:
//     y = (w (.) (o - mean) / sqrt(var + eps) + b) (.) r sigmoid(r)
// with one weight w and bias b of size d_v shared by every head.  The walk that
// produces o tiles d_v across CTAs, so the row statistics cannot be formed in its
// output store alone; this file is the epilogue as its own pass, bound by HBM
// bandwidth (read o and r once, write y once; the backward reads o, r, dy and
// writes do, dr).  gla_fwd_epilogue fuses the forward into the output walk where
// the shape allows (its CTAs of one head form a cluster that exchanges the row
// statistics); this pass serves the backward and the other shapes.
//
// Persistent grid (SMs x resident CTAs); every warp owns the rows
// gw, gw + nw, gw + 2 nw, ... (gw its global warp index, nw the warp count) and a
// ring of S shared-memory stages.  Lane 0 fills a stage with one bulk copy
// (cp.async.bulk, the TMA engine) per input row and tensor, completing on the
// stage's mbarrier; the warp waits on it (bounded), works on the row and lane 0
// refills the stage with the row S steps ahead, so S - 1 rows per warp are in
// flight while one is computed.  No stage is shared between warps, so there are
// no block-wide barriers in the row loop.  Lane l holds the 8-element chunks
// l, l + 32, ... of a row (d_v <= 1024, a multiple of 8): the mean and the
// variance are two passes over registers with warp shuffles, the elementwise
// arithmetic runs on packed fp32 pairs (f32x2 add / mul / fma: one instruction per
// two values), and the outputs leave as coalesced 16-byte stores.  The gradients of w and b are reduced
// deterministically: every CTA writes its partial sums to the caller's workspace
// and a second kernel adds them in order.
#include <cuda_bf16.h>

#include "internal.h"
#include "tc_common.cuh"

namespace gla {
namespace {

constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kEpiMaxStages = 4;
constexpr int kEpiRingBudget = 24 * 1024;  // bytes of one warp's ring (stages x tensors x row)
constexpr long kEpiMaxGrid = 1024;         // bound on CTAs, hence on the partial sums of dw, db

struct EpiArgs {
  long rows;
  int V, S;
  float eps;
  const void *o, *r, *dy;
  const float *w, *b;
  void *out0, *out1;  // forward: y; backward: do, dr
  float *part;        // backward: per-CTA partial sums [grid][2][V], or null
  unsigned *status;
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// packed fp32 pairs and the one-instruction tanh (tc_common.cuh)
using dev::add2;
using dev::bf16pair;
using dev::f2;
using dev::fma2;
using dev::hsum;
using dev::mul2;
using dev::pk;
using dev::tanh_approx;
using dev::upk;

// 8 consecutive elements as 4 pairs: from shared memory (the staged row) ...
__device__ __forceinline__ void lds8p(const __nv_bfloat16 *p, f2 *x) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  x[0] = bf16pair(u.x);
  x[1] = bf16pair(u.y);
  x[2] = bf16pair(u.z);
  x[3] = bf16pair(u.w);
}
__device__ __forceinline__ void lds8p(const float *p, f2 *x) {
  const ulonglong2 a = reinterpret_cast<const ulonglong2 *>(p)[0], b = reinterpret_cast<const ulonglong2 *>(p)[1];
  x[0] = a.x;
  x[1] = a.y;
  x[2] = b.x;
  x[3] = b.y;
}
// ... from global memory (w, b) ...
__device__ __forceinline__ void ldg8p(const float *p, f2 *x) {
  const ulonglong2 a = __ldg(reinterpret_cast<const ulonglong2 *>(p)), b = __ldg(reinterpret_cast<const ulonglong2 *>(p) + 1);
  x[0] = a.x;
  x[1] = a.y;
  x[2] = b.x;
  x[3] = b.y;
}
// ... and back out (global or shared memory)
__device__ __forceinline__ void st8p(float *p, const f2 *x) {
  reinterpret_cast<ulonglong2 *>(p)[0] = make_ulonglong2(x[0], x[1]);
  reinterpret_cast<ulonglong2 *>(p)[1] = make_ulonglong2(x[2], x[3]);
}
__device__ __forceinline__ void st8p(__nv_bfloat16 *p, const f2 *x) {
  uint4 u;
  uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float lo, hi;
    upk(x[i], lo, hi);
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    w[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  *reinterpret_cast<uint4 *>(p) = u;
}

// Swish gate of a pair r: rs = r sigmoid(r) and sg = sigmoid(r).  bf16 rows:
// h = r/2, t = tanh(h), sigmoid = (1 + t)/2, r sigmoid(r) = h + h t; fp32 rows:
// the fast exponential and divide per element.
template <typename T>
__device__ __forceinline__ void gate2(f2 r, f2 &rs, f2 &sg) {
  float lo, hi;
  upk(r, lo, hi);
  sg = pk(__fdividef(1.f, 1.f + __expf(-lo)), __fdividef(1.f, 1.f + __expf(-hi)));
  rs = mul2(r, sg);
}
template <>
__device__ __forceinline__ void gate2<__nv_bfloat16>(f2 r, f2 &rs, f2 &sg) {
  const f2 half = pk(0.5f, 0.5f);
  const f2 h = mul2(r, half);
  float lo, hi;
  upk(h, lo, hi);
  const f2 t = pk(tanh_approx(lo), tanh_approx(hi));
  rs = fma2(h, t, h);
  sg = fma2(t, half, half);
}

// Row statistics over packed chunks: mean, then 1/sqrt(biased variance + eps).
template <int NCH>
__device__ __forceinline__ void row_stats2(const f2 (&x)[NCH][4], int lane, int V, float inv_v, float eps, float &mu,
                                           float &rstd) {
  f2 s = pk(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < NCH; ++i)
    if (8 * (lane + 32 * i) < V)
#pragma unroll
      for (int e = 0; e < 4; ++e) s = add2(s, x[i][e]);
  mu = warp_sum(hsum(s)) * inv_v;
  const f2 nmu = pk(-mu, -mu);
  f2 q = pk(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < NCH; ++i)
    if (8 * (lane + 32 * i) < V)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const f2 d = add2(x[i][e], nmu);
        q = fma2(d, d, q);
      }
  rstd = rsqrtf(warp_sum(hsum(q)) * inv_v + eps);
}

// Global -> shared bulk copy (no multicast) completing on an mbarrier.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dev::smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(dev::smem_u32(bar))
               : "memory");
}

// One warp's staged row stream: NT tensors, S stages of one row each.
template <typename T, int NT>
struct RowRing {
  uint8_t *ring;  // [S][NT][V] elements of T
  uint64_t *bar;  // [S]
  const T *src[NT];
  long gw, nw, mine;  // first row, row stride, rows of this warp
  int S;
  uint32_t rowb;

  __device__ uint8_t *stage(int s) const { return ring + (size_t)s * NT * rowb; }
  // lane 0 only: row j of this warp into stage s (= j mod S)
  __device__ void issue(long j, int s) const {
    const long row = gw + j * nw;
    uint8_t *st = stage(s);
    dev::mbar_arrive_expect_tx(&bar[s], NT * rowb);
#pragma unroll
    for (int t = 0; t < NT; ++t) bulk_g2s(st + t * rowb, src[t] + row * (rowb / sizeof(T)), rowb, &bar[s]);
  }
  // every lane: wait for stage s to complete phase ph; false (warp-uniform) once
  // the wait has run out
  __device__ bool wait(int s, uint32_t ph, unsigned *status) const {
    const bool ok = dev::mbar_wait(&bar[s], ph, status);
    return __all_sync(0xffffffffu, ok);
  }
  // lane 0, after the wait for row j (stage s, phase ph) ran out: let the copies
  // still in flight land
  __device__ void drain(long j, int s, uint32_t ph, unsigned *status) const {
    const long end = j + S < mine ? j + S : mine;
    for (long i = j; i < end; ++i) {
      dev::mbar_wait(&bar[s], ph, status);
      if (++s == S) s = 0, ph ^= 1u;
    }
  }
};

// Shared memory: the warps' rings [8][S][NT][V], then scratch_b bytes per warp,
// then the mbarriers [8][kEpiMaxStages].
template <typename T, int NT>
__device__ __forceinline__ RowRing<T, NT> make_ring(const EpiArgs &a, uint8_t *smem, const T *const (&src)[NT],
                                                    uint32_t scratch_b = 0) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  RowRing<T, NT> q;
  q.rowb = (uint32_t)(a.V * sizeof(T));
  q.S = a.S;
  q.ring = smem + (size_t)warp * a.S * NT * q.rowb;
  q.bar = reinterpret_cast<uint64_t *>(smem + (size_t)kEpiWarps * (a.S * NT * q.rowb + scratch_b)) +
          warp * kEpiMaxStages;
#pragma unroll
  for (int t = 0; t < NT; ++t) q.src[t] = src[t];
  q.nw = (long)gridDim.x * kEpiWarps;
  q.gw = (long)blockIdx.x * kEpiWarps + warp;
  q.mine = q.gw < a.rows ? (a.rows - 1 - q.gw) / q.nw + 1 : 0;
  if (lane == 0) {
    for (int s = 0; s < a.S; ++s) dev::mbar_init(&q.bar[s], 1);
    dev::fence_mbar_init();
  }
  __syncwarp();
  if (lane == 0)
    for (int j = 0; j < q.mine && j < a.S; ++j) q.issue(j, j);
  return q;
}

template <typename T, int NCH>
__global__ void __launch_bounds__(kEpiThreads) k_epi_fwd(EpiArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int V = a.V;
  const T *const src[2] = {(const T *)a.o, (const T *)a.r};
  const RowRing<T, 2> q = make_ring<T, 2>(a, smem, src);
  T *y = (T *)a.out0;
  f2 wv[NCH][4], bv[NCH][4];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = 8 * (lane + 32 * i);
#pragma unroll
    for (int e = 0; e < 4; ++e) wv[i][e] = pk(1.f, 1.f), bv[i][e] = pk(0.f, 0.f);
    if (c < V) {
      if (a.w) ldg8p(a.w + c, wv[i]);
      if (a.b) ldg8p(a.b + c, bv[i]);
    }
  }
  const float inv_v = 1.f / (float)V;
  int s = 0;
  uint32_t ph = 0;
  for (long j = 0; j < q.mine; ++j) {
    if (!q.wait(s, ph, a.status)) {
      if (lane == 0) q.drain(j, s, ph, a.status);
      return;
    }
    const long row = q.gw + j * q.nw;
    const T *so = reinterpret_cast<const T *>(q.stage(s)), *sr = so + V;
    f2 x[NCH][4];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = 8 * (lane + 32 * i);
      if (c < V) lds8p(so + c, x[i]);
    }
    float mu, rstd;
    row_stats2<NCH>(x, lane, V, inv_v, a.eps, mu, rstd);
    const f2 nmu = pk(-mu, -mu), rs2 = pk(rstd, rstd);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = 8 * (lane + 32 * i);
      if (c < V) {
        f2 rr[4], out[4];
        lds8p(sr + c, rr);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const f2 n = fma2(mul2(add2(x[i][e], nmu), rs2), wv[i][e], bv[i][e]);
          f2 rsw, sg;
          gate2<T>(rr[e], rsw, sg);
          out[e] = mul2(n, rsw);
        }
        st8p(y + row * V + c, out);
      }
    }
    __syncwarp();  // every lane has read the stage
    if (lane == 0 && j + q.S < q.mine) {
      dev::fence_proxy_async_smem();
      q.issue(j + q.S, s);
    }
    if (++s == q.S) s = 0, ph ^= 1u;
  }
}

// Backward.  With dn = dy r sigmoid(r) (the gradient at the LayerNorm output),
// x^ = (o - mean) rstd and g = dn w:  do = rstd (g - mean(g) - x^ mean(g x^)),
// dr = dy n sigmoid(r) (1 + r (1 - sigmoid(r))), dw += dn x^, db += dn.
template <typename T, int NCH>
__global__ void __launch_bounds__(kEpiThreads) k_epi_bwd(EpiArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int V = a.V;
  const T *const src[3] = {(const T *)a.o, (const T *)a.r, (const T *)a.dy};
  const RowRing<T, 3> q = make_ring<T, 3>(a, smem, src, 4u * V);
  // this warp's fp32 row of g = dn w, written in pass 1 and read in pass 2
  float *gs = reinterpret_cast<float *>(smem + (size_t)kEpiWarps * a.S * 3 * q.rowb) + (threadIdx.x >> 5) * V;
  T *dout = (T *)a.out0, *dr = (T *)a.out1;
  f2 pw[NCH][4], pb[NCH][4];
#pragma unroll
  for (int i = 0; i < NCH; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) pw[i][e] = pb[i][e] = pk(0.f, 0.f);
  const f2 one = pk(1.f, 1.f), zero = pk(0.f, 0.f);
  const float inv_v = 1.f / (float)V;
  int s = 0;
  uint32_t ph = 0;
  for (long j = 0; j < q.mine; ++j) {
    if (!q.wait(s, ph, a.status)) {
      if (lane == 0) q.drain(j, s, ph, a.status);
      break;
    }
    const long row = q.gw + j * q.nw;
    const T *so = reinterpret_cast<const T *>(q.stage(s)), *sr = so + V, *sd = so + 2 * V;
    f2 x[NCH][4];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = 8 * (lane + 32 * i);
      if (c < V) lds8p(so + c, x[i]);
    }
    float mu, rstd;
    row_stats2<NCH>(x, lane, V, inv_v, a.eps, mu, rstd);
    const f2 nmu = pk(-mu, -mu), rs2 = pk(rstd, rstd);
    // pass 1: dr, g (parked in gs), the dw / db partials and the row means of g
    // and g x^; x is replaced by x^
    f2 m1 = zero, m2 = zero;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = 8 * (lane + 32 * i);
      if (c < V) {
        f2 rv[4], gy[4], ww[4], bb[4], drv[4], gg[4];
        lds8p(sr + c, rv);
        lds8p(sd + c, gy);
#pragma unroll
        for (int e = 0; e < 4; ++e) ww[e] = one, bb[e] = zero;
        if (a.w) ldg8p(a.w + c, ww);
        if (a.b) ldg8p(a.b + c, bb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const f2 xh = mul2(add2(x[i][e], nmu), rs2);
          const f2 n = fma2(xh, ww[e], bb[e]);
          f2 rsw, sg;
          gate2<T>(rv[e], rsw, sg);
          const f2 dn = mul2(gy[e], rsw);
          // d(r sigmoid(r))/dr = sigmoid (1 + r (1 - sigmoid))
          const f2 dsw = mul2(sg, fma2(rv[e], add2(one, mul2(sg, pk(-1.f, -1.f))), one));
          drv[e] = mul2(mul2(gy[e], n), dsw);
          pw[i][e] = fma2(dn, xh, pw[i][e]);
          pb[i][e] = add2(pb[i][e], dn);
          gg[e] = mul2(dn, ww[e]);
          m1 = add2(m1, gg[e]);
          m2 = fma2(gg[e], xh, m2);
          x[i][e] = xh;
        }
        st8p(dr + row * V + c, drv);
        st8p(gs + c, gg);
      }
    }
    const float m1s = warp_sum(hsum(m1)) * inv_v, m2s = warp_sum(hsum(m2)) * inv_v;
    // pass 2: do = rstd g - rstd m1 - x^ (rstd m2), each lane reading back only its g
    const f2 c1 = pk(-rstd * m1s, -rstd * m1s), c2 = pk(-rstd * m2s, -rstd * m2s);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = 8 * (lane + 32 * i);
      if (c < V) {
        f2 gg[4], d[4];
        lds8p(gs + c, gg);
#pragma unroll
        for (int e = 0; e < 4; ++e) d[e] = fma2(x[i][e], c2, fma2(gg[e], rs2, c1));
        st8p(dout + row * V + c, d);
      }
    }
    __syncwarp();
    if (lane == 0 && j + q.S < q.mine) {
      dev::fence_proxy_async_smem();
      q.issue(j + q.S, s);
    }
    if (++s == q.S) s = 0, ph ^= 1u;
  }
  if (!a.part) return;
  // The CTA's partial sums: every warp parks its lanes' sums in its own ring (idle
  // now; a ring holds 3 S d_v >= 6 d_v elements of T, at least 2 d_v floats), then
  // the CTA adds the 8 warps in order.  A warp that gave up on a wait parks its
  // sums too; the status word already marks the call as failed.
  float *mine = reinterpret_cast<float *>(q.ring);
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = 8 * (lane + 32 * i);
    if (c < V) {
      st8p(mine + c, pw[i]);
      st8p(mine + V + c, pb[i]);
    }
  }
  __syncthreads();
  const size_t ring_floats = (size_t)a.S * 3 * q.rowb / sizeof(float);
  const float *all = reinterpret_cast<const float *>(smem);
  for (int idx = threadIdx.x; idx < 2 * V; idx += kEpiThreads) {
    float sum = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kEpiWarps; ++w8) sum += all[w8 * ring_floats + idx];
    a.part[(long)blockIdx.x * 2 * V + idx] = sum;
  }
}

// dw[c] = sum over CTAs of part[cta][0][c], db[c] likewise.  A CTA of 1024 threads
// owns 32 consecutive entries of the 2 d_v sums: warp w adds the partials
// w, w + 32, ... for its lane's entry, then warp 0 adds the 32 warp sums in order.
constexpr int kReduceWarps = 32;
__global__ void __launch_bounds__(32 * kReduceWarps) k_epi_reduce(int nparts, int V, const float *__restrict__ part,
                                                                  float *__restrict__ dw, float *__restrict__ db) {
  __shared__ float sred[kReduceWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int idx = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (idx < 2 * V)
#pragma unroll 4
    for (int p = warp; p < nparts; p += kReduceWarps) s += part[(long)p * 2 * V + idx];
  sred[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && idx < 2 * V) {
    float t = sred[0][lane];
#pragma unroll
    for (int w = 1; w < kReduceWarps; ++w) t += sred[w][lane];
    if (idx < V) {
      if (dw) dw[idx] = t;
    } else if (db) {
      db[idx - V] = t;
    }
  }
}

// Stages per warp, dynamic shared memory and the persistent grid of a launch.
struct EpiShape {
  int S;
  size_t smem;
  unsigned grid;
};

size_t stage_bytes(const gla_desc *d, int nt) { return (size_t)nt * d->dv * (d->dtype == GLA_DTYPE_BF16 ? 2 : 4); }

int stages_for(size_t per_stage) {
  const int S = (int)(kEpiRingBudget / per_stage);
  return S < 2 ? 2 : (S > kEpiMaxStages ? kEpiMaxStages : S);
}

template <typename Kern>
int epi_shape(Kern kernel, const gla_desc *d, int nt, size_t scratch_b, EpiShape *sh) {
  const long rows = (long)d->B * d->H * d->T;
  const size_t per_stage = stage_bytes(d, nt);
  sh->S = stages_for(per_stage);
  sh->smem = (size_t)kEpiWarps * (sh->S * per_stage + scratch_b) + (size_t)kEpiWarps * kEpiMaxStages * sizeof(uint64_t);
  // the attribute belongs to the current device, so it is set on every call that needs it
  if (sh->smem > 48 * 1024 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh->smem) != cudaSuccess)
    return GLA_ERR_CUDA;
  int dev = 0, nsm = 0, occ = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kEpiThreads, sh->smem) != cudaSuccess)
    return GLA_ERR_CUDA;
  if (occ < 1) return GLA_ERR_UNSUPPORTED_SHAPE;
  long g = (rows + kEpiWarps - 1) / kEpiWarps;
  if (g > (long)nsm * occ) g = (long)nsm * occ;
  if (g > kEpiMaxGrid) g = kEpiMaxGrid;
  sh->grid = (unsigned)g;
  return GLA_OK;
}

template <typename T, int NCH>
int epi_fwd_n(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps, void *y,
              cudaStream_t st) {
  EpiShape sh;
  if (const int e = epi_shape(k_epi_fwd<T, NCH>, d, 2, 0, &sh)) return e;
  const EpiArgs a{(long)d->B * d->H * d->T, d->dv, sh.S, eps, o, r, nullptr, w, b, y, nullptr, nullptr,
                  (unsigned *)d->workspace};
  GLA_LAUNCH(K_EPI_FWD, st, (k_epi_fwd<T, NCH><<<sh.grid, kEpiThreads, sh.smem, st>>>(a)));
  return GLA_OK;
}

template <typename T, int NCH>
int epi_bwd_n(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
              const void *dy, void *dout, void *dr, float *dw, float *db, cudaStream_t st) {
  EpiShape sh;
  if (const int e = epi_shape(k_epi_bwd<T, NCH>, d, 3, (size_t)4 * d->dv, &sh)) return e;
  float *part = (dw || db) ? (float *)((char *)d->workspace + kStatusBytes) : nullptr;
  const EpiArgs a{(long)d->B * d->H * d->T, d->dv, sh.S, eps, o, r, dy, w, b, dout, dr, part,
                  (unsigned *)d->workspace};
  GLA_LAUNCH(K_EPI_BWD, st, (k_epi_bwd<T, NCH><<<sh.grid, kEpiThreads, sh.smem, st>>>(a)));
  if (part)
    GLA_LAUNCH(K_EPI_REDUCE, st,
               (k_epi_reduce<<<(2 * d->dv + 31) / 32, 32 * kReduceWarps, 0, st>>>((int)sh.grid, d->dv, part, dw, db)));
  return GLA_OK;
}

template <int NCH>
int epi_fwd_t(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps, void *y,
              cudaStream_t st) {
  return d->dtype == GLA_DTYPE_BF16 ? epi_fwd_n<__nv_bfloat16, NCH>(d, o, r, w, b, eps, y, st)
                                    : epi_fwd_n<float, NCH>(d, o, r, w, b, eps, y, st);
}

template <int NCH>
int epi_bwd_t(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
              const void *dy, void *dout, void *dr, float *dw, float *db, cudaStream_t st) {
  return d->dtype == GLA_DTYPE_BF16 ? epi_bwd_n<__nv_bfloat16, NCH>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st)
                                    : epi_bwd_n<float, NCH>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
}

}  // namespace

size_t epilogue_workspace(const gla_desc *d) {
  const long rows = (long)d->B * d->H * d->T;
  long g = (rows + kEpiWarps - 1) / kEpiWarps;
  if (g > kEpiMaxGrid) g = kEpiMaxGrid;
  return kStatusBytes + (size_t)g * 2 * d->dv * sizeof(float);
}

int epilogue_fwd(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
                 void *y, cudaStream_t st, bool clear_status) {
  if (clear_status && cudaMemsetAsync(d->workspace, 0, kStatusBytes, st) != cudaSuccess) return GLA_ERR_CUDA;
  switch ((d->dv + 255) / 256) {
    case 1: return epi_fwd_t<1>(d, o, r, w, b, eps, y, st);
    case 2: return epi_fwd_t<2>(d, o, r, w, b, eps, y, st);
    case 3: return epi_fwd_t<3>(d, o, r, w, b, eps, y, st);
    default: return epi_fwd_t<4>(d, o, r, w, b, eps, y, st);
  }
}

int epilogue_bwd(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
                 const void *dy, void *dout, void *dr, float *dw, float *db, cudaStream_t st) {
  if (cudaMemsetAsync(d->workspace, 0, kStatusBytes, st) != cudaSuccess) return GLA_ERR_CUDA;
  switch ((d->dv + 255) / 256) {
    case 1: return epi_bwd_t<1>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
    case 2: return epi_bwd_t<2>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
    case 3: return epi_bwd_t<3>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
    default: return epi_bwd_t<4>(d, o, r, w, b, eps, dy, dout, dr, dw, db, st);
  }
}

}  // namespace gla
