// tc_bwd.cuh -- per-chunk backward kernel of the bf16 tensor-core path.
//
// One CTA per (chunk n, head, half of the key channels): 128 threads, one per key
// channel c of its half.  Inputs: the chunk state h_n (state before chunk n) and
// adjoint dh_n (gradient w.r.t. the state after chunk n), both bf16 in the walk's
// chunk-state layout (state_chunk_off): per 64-column d_v tile and channel half a
// contiguous 16 KB block of 8 x 8 core matrices [8 v-groups][16 c-groups][8 v][8 c],
// fetched with one bulk copy and read as the no-swizzle MN-major operand; gam from
// the prep kernel; q, k, V, dO and log_alpha.  (dv comes from the reverse walk, which holds dh_n on chip.)
// With B the chunk-local cumulative log-gate:
//   phase 1 (loop over d_v tiles of 64, accumulating in TMEM):
//     dqh^T = h_n dO^T          dkh^T = dh_n V^T         dP = dO V^T
//     R[c]  = sum_v h_n[c,v] dh_n[c,v]
//   phase 2 (intra-chunk, secondary chunking):
//     strictly-lower sub-chunk blocks on tcgen05 with reference points
//       dq_off[t] = u_t (.) sum_{s in earlier sub-chunks} dP[t,s] k_s e^{z_j(t) - B_s}
//       dk_off[s] = w_s (.) sum_{t in later sub-chunks}  dP[t,s] q_t e^{B_t - z_j(s)+1}
//     diagonal 16 x 16 blocks in fp32 on CUDA cores (one thread per key channel),
//       with the same fp32 pair factor q_t k_s e^{B_t - B_s} on the dq and the dk
//       side, so the pair terms cancel exactly in the closed-form gate gradient
//   epilogue per key channel:
//     dq = e^{B} (.) dqh + dq_intra ,  dk = e^{B_63 - B} (.) dkh + dk_intra
//     dlog b_t = q_t dq_t - k_t dk_t                       (section 4.3)
//     dlog alpha_t = sum_{i>=t in chunk} dlog b_i + G_n,
//     G_n = gam_n R + sum_t k_t (.) e^{B_63-B_t} dkh_t  ( = sum_v S_n dS_n, the
//           part of the suffix sum that lies beyond the chunk).
// A CTA needs 256 TMEM columns and ~100 KB of shared memory, so two share an SM
// and one's load phase overlaps the other's CUDA-core phase.  dP is formed by both
// halves of a chunk (it is tiny); with a scalar gate the two halves' channel sums
// of dlog alpha meet in one atomic add onto a zeroed output (exact: 0 + a + b).
#pragma once

#include "tc_kernels.cuh"

namespace gla {
namespace tc {

constexpr int kBwdKH = 128;  // key channels per backward CTA
#ifndef GLA_BWD_STAGGER_NS
#define GLA_BWD_STAGGER_NS 8000
#endif
constexpr unsigned kBwdStaggerNs = GLA_BWD_STAGGER_NS;

struct BwdArgs {
  int T, N, V, gate;
  long Tp;
  const bf16 *q, *k;
  const float *la;
  const float *gam;
  const bf16 *hb, *dhb;  // chunk states / adjoints, [BH][N][K/128][V/8][128][8]
  bf16 *dq, *dk;
  float *dla;
  unsigned *status;
  // CTAs with linear index in [stagger0, stagger1) start stagger_ns later, so
  // that half of the first wave is loading while the other half computes
  int stagger0, stagger1;
  unsigned stagger_ns;
};

struct BwdSmem {
  static constexpr int BVb = 64;
  static constexpr int kTileH = kBwdKH * BVb * 2;         // h or dh half-tile, [8][16][8 v][8 c] bf16
  static constexpr int kTileV = 64 * BVb * 2;             // V or dO tile, SW128
  static constexpr int kStage = 2 * kTileH + 2 * kTileV;  // h, dh, V, dO
  static constexpr int kPhase1End = 2 * kStage;
  // phase 2 (aliases the phase-1 stages)
  static constexpr int kRowsW = 96;
  static constexpr int kKh = 0;                               // key windows  [96][128]
  static constexpr int kQh = kKh + kRowsW * kBwdKH * 2;       // query windows [96][128]
  static constexpr int kdP = kQh + kRowsW * kBwdKH * 2;       // dP, strictly-lower blocks  [t][s]
  static constexpr int kdPT = kdP + 64 * 64 * 2;              // the same, transposed [s][t]
  static constexpr int kdPd = kdPT + 64 * 64 * 2;             // fp32 diagonal blocks [64][16]
  static constexpr int kQt = kdPd + 64 * 16 * 4;              // q tile [64][128] bf16 (TMA, after phase 1)
  static constexpr int kKt = kQt + 64 * kBwdKH * 2;           // k tile [64][128] bf16
  static constexpr int kPhase2End = kKt + 64 * kBwdKH * 2;
  // epilogue (aliases the windows and dP tiles, dead once the phase-2 MMAs are done):
  // dq, dk [2 column halves][64 t][64 c] bf16 and dlog alpha [2][64 t][64 c] fp32,
  // each column half one TMA store box
  static constexpr int kSDq = 0;
  static constexpr int kSDk = kSDq + 64 * kBwdKH * 2;
  static constexpr int kSDla = kSDk + 64 * kBwdKH * 2;
  static_assert(kSDla + 64 * kBwdKH * 4 <= kdPd, "epilogue staging stays clear of the diagonal blocks");
  static constexpr int kRed = (kPhase1End > kPhase2End ? kPhase1End : kPhase2End);  // scalar-gate sums [4][64]
  static constexpr int kRed2 = kRed + 4 * 64 * 4;            // sums of h (.) dh [128]
  static constexpr int kBar = kRed2 + kBwdKH * 4;
  static constexpr int kBytes = kBar + 128;
};

template <int K>
__global__ void __launch_bounds__(kBwdKH, 2)
    k_bwd_main(BwdArgs a, const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
               const __grid_constant__ CUtensorMap tmQin, const __grid_constant__ CUtensorMap tmKin,
               const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
               const __grid_constant__ CUtensorMap tmDLA) {
  using L = BwdSmem;
  constexpr int BVb = L::BVb;
  constexpr int kH = K / kBwdKH;  // CTAs per chunk
  constexpr int cDQ = 0, cDK = 64, cDP = 128;
  constexpr int cQI = cDP, cKI = 192;
  constexpr int kTmemCols = 256;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *full = (uint64_t *)(smem + L::kBar);  // [0],[1] stages
  uint64_t *mma_bar = full + 2;   // phase-1 MMAs, three issuing threads
  uint64_t *qk_bar = full + 3;
  uint64_t *mma2_bar = full + 4;  // phase-2 MMAs, two issuing threads
  uint32_t *tslot = (uint32_t *)(full + 5);
  float *red = (float *)(smem + L::kRed);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid (K/128, N, BH): the two channel halves of a chunk are neighbours in
  // launch order and share the chunk's V and dO tiles through L2
  const int half = blockIdx.x;
  const int n = blockIdx.y;
  const long bh = blockIdx.z;
  const int c0 = half * kBwdKH;
  const int nvt = a.V / BVb;
  const long hrow = bh * a.N + n;

  if (tid == 0) {
    dev::mbar_init(&full[0], 1);
    dev::mbar_init(&full[1], 1);
    dev::mbar_init(mma_bar, 3);
    dev::mbar_init(qk_bar, 1);
    dev::mbar_init(mma2_bar, 2);
    dev::fence_mbar_init();
    dev::prefetch_tmap(&tmV);
    dev::prefetch_tmap(&tmDO);
  }
  dev::pdl_launch_dependents();
  {
    const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    if (lin >= a.stagger0 && lin < a.stagger1) {  // bounded: stagger_ns < 1 ms
      const uint64_t t0 = dev::globaltimer();
      while (dev::globaltimer() - t0 < a.stagger_ns) __nanosleep(256);
    }
  }
  dev::pdl_wait();
  if (warp == 0) dev::tmem_alloc(tslot, kTmemCols);
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tslot;

  // this CTA's 16 KB block of h_n / dh_n for d_v tile i: ((hrow * V/64 + i) * K/128 + half) * 8192 elements
  const bf16 *h_src = a.hb + (hrow * (a.V / 64) * kH + half) * (long)(kBwdKH * BVb);
  const bf16 *dh_src = a.dhb + (hrow * (a.V / 64) * kH + half) * (long)(kBwdKH * BVb);
  const long tile_step = (long)K * BVb;  // elements from one d_v tile to the next
  auto stage = [&](int s) { return smem + s * L::kStage; };
  auto issue_tile = [&](int i) {
    const int s = i & 1;
    uint8_t *st = stage(s);
    const int v0 = i * BVb;
    dev::mbar_arrive_expect_tx(&full[s], (uint32_t)L::kStage);
    dev::bulk_load(st, h_src + i * tile_step, (uint32_t)L::kTileH, &full[s]);
    dev::bulk_load(st + L::kTileH, dh_src + i * tile_step, (uint32_t)L::kTileH, &full[s]);
    dev::tma_load_3d(st + 2 * L::kTileH, &tmV, v0, n * kC, (int)bh, &full[s]);
    dev::tma_load_3d(st + 2 * L::kTileH + L::kTileV, &tmDO, v0, n * kC, (int)bh, &full[s]);
  };
  if (tid == 0) {
    issue_tile(0);
    if (nvt > 1) issue_tile(1);
  }

  const int cl = tid;     // key channel within this CTA's half
  const int c = c0 + cl;  // key channel
  // partial sums of h (.) dh: thread -> channel group cg = 4 warp + lane / 8 (channels
  // 8 cg .. 8 cg + 7 of this half) and value columns v = 8 r + lane % 8 of every d_v
  // tile (core matrix (r, cg)); a warp reads 512 contiguous bytes (no bank conflict)
  const int cg = 4 * warp + (lane >> 3), vs = lane & 7;
  const uint32_t r_off = (uint32_t)(cg * 128 + vs * 16);
  float Racc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  bool ok = true;

  // per key channel: sub-chunk boundary values of the cumulative log-gate (their 64
  // gate loads are issued here, so that they complete while phase 1 streams); the 16
  // values inside sub-chunk j are rebuilt from log_alpha when needed
  float z[5], Gam[4], E[4], Gafter[4];
  const long qrow0 = bh * a.T + (long)n * kC;  // first token row of this chunk
  const uint32_t sQt = dev::smem_u32(smem + L::kQt), sKt = dev::smem_u32(smem + L::kKt);
  auto qk_at = [&](int t, float &qf, float &kf) {
    uint16_t qb, kb;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(qb) : "r"(sQt + dev::sw128_off(64, t, cl)));
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(kb) : "r"(sKt + dev::sw128_off(64, t, cl)));
    qf = __bfloat162float(*reinterpret_cast<const bf16 *>(&qb));
    kf = __bfloat162float(*reinterpret_cast<const bf16 *>(&kb));
  };
  // log_alpha of token t of this chunk (0 beyond T)
  auto gate_at = [&](int t) -> float {
    if ((long)n * kC + t >= a.T) return 0.f;
    if (a.gate == GLA_GATE_VECTOR) return __ldg(a.la + (qrow0 + t) * K + c);
    if (a.gate == GLA_GATE_SCALAR) return __ldg(a.la + qrow0 + t);
    return 0.f;
  };
  // g[e] = log_alpha of token 16 j + e; Bc[e] = z_j + g[0] + ... + g[e] (cumulative log-gate)
  auto load16 = [&](int j, float *g) {
#pragma unroll
    for (int e = 0; e < 16; ++e) g[e] = gate_at(16 * j + e);
  };
  auto cumsum16 = [&](const float *g, float zj, float *Bc) {
    float acc = zj;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      acc += g[e];
      Bc[e] = acc;
    }
  };
  const uint32_t lanebase = 32 * warp;
  // the 64 gate loads are issued now and first used after phase 1
  float gpre[kC];
#pragma unroll
  for (int t = 0; t < kC; ++t) gpre[t] = gate_at(t);
  // ============================ phase 1 ============================
  for (int i = 0; i < nvt; ++i) {
    const int s = i & 1;
    uint8_t *st = stage(s);
    if (ok) ok = dev::mbar_wait(&full[s], (i >> 1) & 1, a.status);
    // issue this tile's MMAs (lane 0 of warps 0, 1, 2: one accumulator each, since
    // a tcgen05.mma costs its issuing thread tens of cycles), then sum h (.) dh from
    // the same shared-memory tiles while they run
    if (lane == 0 && warp < 3 && ok) {
      const uint32_t sH = dev::smem_u32(st), sDH = sH + L::kTileH, sV = sDH + L::kTileH, sDO = sV + L::kTileV;
      constexpr uint32_t id_kk128 = dev::idesc_bf16(128, 64, true, false);  // A = h / dh MN-major
      constexpr uint32_t id_kk64 = dev::idesc_bf16(64, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < BVb / 16; ++kk) {
        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
        // h / dh as MN-major A without swizzle: 8 (v) x 16-byte (8 c) core matrices;
        // in this layout type the leading byte offset steps along K (8 value
        // columns: 2048 bytes) and the stride byte offset along M (8 channels: 128)
        if (warp == 0)
          dev::umma_bf16(tmem + cDQ, dev::sdesc_noswz(sH + (uint32_t)(kk * 4096), 2048u, 128u),
                         dev::desc_kmajor(sDO, 64, 0, kk * 16), id_kk128, acc);
        else if (warp == 1)
          dev::umma_bf16(tmem + cDK, dev::sdesc_noswz(sDH + (uint32_t)(kk * 4096), 2048u, 128u),
                         dev::desc_kmajor(sV, 64, 0, kk * 16), id_kk128, acc);
        else
          dev::umma_bf16(tmem + cDP, dev::desc_kmajor(sDO, 64, 0, kk * 16), dev::desc_kmajor(sV, 64, 0, kk * 16),
                         id_kk64, acc);
      }
      dev::umma_commit(mma_bar);
    }
    {
      const uint32_t sh = dev::smem_u32(st) + r_off, sdh = sh + L::kTileH;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        uint4 x, y;
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                     : "r"(sh + (uint32_t)(r * 2048)));
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(y.x), "=r"(y.y), "=r"(y.z), "=r"(y.w)
                     : "r"(sdh + (uint32_t)(r * 2048)));
        const __nv_bfloat162 *xh = reinterpret_cast<const __nv_bfloat162 *>(&x);
        const __nv_bfloat162 *yh = reinterpret_cast<const __nv_bfloat162 *>(&y);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 xf = __bfloat1622float2(xh[e]), yf = __bfloat1622float2(yh[e]);
          Racc[2 * e] += xf.x * yf.x;
          Racc[2 * e + 1] += xf.y * yf.y;
        }
      }
    }
    if (ok) ok = dev::mbar_wait(mma_bar, i & 1, a.status);
    dev::tc_fence_after();
    __syncthreads();  // every thread has finished reading stage s (R sums)
    if (tid == 0 && ok && i + 2 < nvt) issue_tile(i + 2);
  }

  // R[c] = sum_v h[c,v] dh[c,v]: the 8 lanes of a channel group add their partial
  // sums, then each channel's thread reads its total
  float *red2 = (float *)(smem + L::kRed2);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float x = Racc[e];
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    if (vs == 0) red2[8 * cg + e] = x;
  }
  __syncthreads();
  const float R = red2[cl];

  {
    float acc = 0.f;
    z[0] = 0.f;
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      acc += gpre[t];
      if ((t & 15) == 15) z[(t >> 4) + 1] = acc;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      Gam[j] = __expf(z[j + 1] - z[j]);
      E[j] = __expf(z[j]);
    }
    Gafter[3] = 1.f;
    Gafter[2] = Gam[3];
    Gafter[1] = Gam[3] * Gam[2];
    Gafter[0] = Gam[3] * Gam[2] * Gam[1];
  }

  // ============================ phase 2 ============================
  // q and k columns of this half into the space phase 1 no longer uses
  if (tid == 0) {
    dev::fence_proxy_async_smem();
    dev::mbar_arrive_expect_tx(qk_bar, (uint32_t)(2 * 64 * kBwdKH * 2));
#pragma unroll
    for (int cb = 0; cb < kBwdKH / 64; ++cb) {
      dev::tma_load_3d(smem + L::kQt + cb * 64 * 128, &tmQin, c0 + cb * 64, n * kC, (int)bh, qk_bar);
      dev::tma_load_3d(smem + L::kKt + cb * 64 * 128, &tmKin, c0 + cb * 64, n * kC, (int)bh, qk_bar);
    }
  }
  // dP (rows t, TMEM M = 64 layout) -> bf16 tiles of its strictly-lower sub-chunk
  // blocks, dP[t][s] and dP^T[s][t], and fp32 copies of the four diagonal blocks.
  const uint32_t sdP = dev::smem_u32(smem + L::kdP), sdPT = dev::smem_u32(smem + L::kdPT);
  float *dPd = (float *)(smem + L::kdPd);
  {
    const int t = 16 * warp + lane;
    float row[kC];
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) dev::tmem_ld16(dev::tmem_addr(tmem, 32 * warp, cDP + 16 * cb), row + 16 * cb);
    dev::tmem_wait_ld();
    if (lane < 16) {
      const int jt = warp;  // sub-chunk of t
#pragma unroll
      for (int s8 = 0; s8 < 8; ++s8) {
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = ((s8 * 8 + e) < 16 * jt && ok) ? row[s8 * 8 + e] : 0.f;
        dev::st_shared_v4(sdP + dev::sw128_chunk(64, t, s8), dev::pack_bf16(m8[0], m8[1]),
                          dev::pack_bf16(m8[2], m8[3]), dev::pack_bf16(m8[4], m8[5]), dev::pack_bf16(m8[6], m8[7]));
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const bf16 b = __float2bfloat16_rn(m8[e]);
          dev::st_shared_u16(sdPT + dev::sw128_off(64, s8 * 8 + e, t), *reinterpret_cast<const uint16_t *>(&b));
        }
      }
      float dg[16];
      dev::take16(row, jt, dg);  // the diagonal block's 16 entries of this row
#pragma unroll
      for (int e = 0; e < 16; ++e) dPd[t * 16 + e] = (16 * jt + e <= t && ok) ? dg[e] : 0.f;
    }
  }

  if (!dev::mbar_wait(qk_bar, 0, a.status)) ok = false;

  // window construction + boundary term G_n = gam_n R + sum_t k_t dk_inter_t
  float Gb = a.gam[(bh * a.N + n) * K + c] * R;
  {
    const uint32_t sKh = dev::smem_u32(smem + L::kKh), sQh = dev::smem_u32(smem + L::kQh);
    const int wK[4] = {0, 0, 16, 48};    // key window j >= 1: row wK[j] + s, s in [0, 16j)
    const int wQ[4] = {-16, 16, 32, 0};  // query window u <= 2: row wQ[u] + t, t in [16(u+1), 64)
    float gnext[16];
    load16(0, gnext);
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      float Bc[16], xk[16];
      const float zj = dev::sel4(j, z[0], z[1], z[2], z[3]);
      cumsum16(gnext, zj, Bc);
      if (j < 3) load16(j + 1, gnext);  // prefetch the next sub-chunk's gates
      dev::tmem_ld16(dev::tmem_addr(tmem, lanebase, cDK + 16 * j), xk);
      dev::tmem_wait_ld();
      const float zj1 = dev::sel4(j, z[1], z[2], z[3], z[4]);
      const float GAj = dev::sel4(j, Gafter[0], Gafter[1], Gafter[2], Gafter[3]);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int t = 16 * j + e;
        float qf, kf;
        qk_at(t, qf, kf);
        const float u = __expf(Bc[e] - zj);
        const float w = __expf(zj1 - Bc[e]);
        Gb += kf * w * GAj * xk[e];
        // key operand k_t e^{z_jq - B_t} for later query sub-chunks jq > j
        float f = kf * w;
#pragma unroll
        for (int jq = 1; jq < 4; ++jq) {
          if (jq > j) {
            const bf16 b = __float2bfloat16_rn(f);
            dev::st_shared_u16(sKh + dev::sw128_off(L::kRowsW, wK[jq] + t, cl),
                               *reinterpret_cast<const uint16_t *>(&b));
            f *= Gam[jq];
          }
        }
        // query operand q_t e^{B_t - z_{uu+1}} for earlier key sub-chunks uu < j
        float g2 = qf * u;
#pragma unroll
        for (int uu = 2; uu >= 0; --uu) {
          if (uu < j) {
            const bf16 b = __float2bfloat16_rn(g2);
            dev::st_shared_u16(sQh + dev::sw128_off(L::kRowsW, wQ[uu] + t, cl),
                               *reinterpret_cast<const uint16_t *>(&b));
            g2 *= Gam[uu];
          }
        }
      }
    }
  }
  dev::fence_proxy_async_smem();
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  if (lane == 0 && warp < 2 && ok) {  // dq blocks from warp 0, dk blocks from warp 1
    const uint32_t sKh = dev::smem_u32(smem + L::kKh), sQh = dev::smem_u32(smem + L::kQh);
    const int wK[4] = {0, 0, 16, 48};
    const int wQ[4] = {-16, 16, 32, 0};
    constexpr uint32_t id = dev::idesc_bf16(128, 16, true, false);
    if (warp == 0) {
#pragma unroll
      for (int j = 1; j < 4; ++j)
#pragma unroll
        for (int kk = 0; kk < j; ++kk)
          dev::umma_bf16(tmem + cQI + 16 * j, dev::desc_mnmajor(sKh, L::kRowsW, wK[j] + 16 * kk, 0),
                         dev::desc_kmajor(sdP, 64, 16 * j, 16 * kk), id, kk > 0 ? 1u : 0u);
    } else {
#pragma unroll
      for (int u = 0; u < 3; ++u)
#pragma unroll
        for (int kk = u + 1; kk < 4; ++kk)
          dev::umma_bf16(tmem + cKI + 16 * u, dev::desc_mnmajor(sQh, L::kRowsW, wQ[u] + 16 * kk, 0),
                         dev::desc_kmajor(sdPT, 64, 16 * u, 16 * kk), id, kk > u + 1 ? 1u : 0u);
    }
    dev::umma_commit(mma2_bar);
  }
  if (ok) ok = dev::mbar_wait(mma2_bar, 0, a.status);
  dev::tc_fence_after();

  // ============================ epilogue ============================
  // reverse over sub-chunks and tokens: dq, dk, dlog b and its suffix sum, staged in
  // shared memory for three TMA stores
  const uint32_t sDq = dev::smem_u32(smem + L::kSDq), sDk = dev::smem_u32(smem + L::kSDk),
                 sDla = dev::smem_u32(smem + L::kSDla);
  float run = Gb;
  float gnext[16];
  load16(3, gnext);
#pragma unroll 1
  for (int j = 3; j >= 0; --j) {
    float xq[16], xk[16], xqi[16], xki[16];
    dev::tmem_ld16(dev::tmem_addr(tmem, lanebase, cDQ + 16 * j), xq);
    dev::tmem_ld16(dev::tmem_addr(tmem, lanebase, cDK + 16 * j), xk);
    dev::tmem_ld16(dev::tmem_addr(tmem, lanebase, cQI + 16 * j), xqi);
    dev::tmem_ld16(dev::tmem_addr(tmem, lanebase, cKI + 16 * j), xki);
    dev::tmem_wait_ld();
    float Bc[16];
    const float zj = dev::sel4(j, z[0], z[1], z[2], z[3]);
    cumsum16(gnext, zj, Bc);
    if (j > 0) load16(j - 1, gnext);  // prefetch the previous sub-chunk's gates
    const float zj1 = dev::sel4(j, z[1], z[2], z[3], z[4]);
    const float Ej = dev::sel4(j, E[0], E[1], E[2], E[3]);
    const float invGj = 1.f / dev::sel4(j, Gam[0], Gam[1], Gam[2], Gam[3]);
    const float GAj = dev::sel4(j, Gafter[0], Gafter[1], Gafter[2], Gafter[3]);
    const float offq_on = (j > 0) ? 1.f : 0.f;  // no off-diagonal MMA wrote sub-chunk 0's dq columns
    const float offk_on = (j < 3) ? 1.f : 0.f;  // ... nor sub-chunk 3's dk columns
    // diagonal block of sub-chunk j in fp32:
    //   a_t = q_t e^{B_t - z_j},  b_s = k_s e^{z_j - B_s}
    //   dq_t += e^{B_t - z_j} sum_{s<=t} dP[t,s] b_s ,  dk_s += e^{z_j - B_s} sum_{t>=s} dP[t,s] a_t
    float uu[16], ww[16], qv[16], kv[16], av[16], bv[16], dqd[16], dkd[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      qk_at(16 * j + e, qv[e], kv[e]);
      uu[e] = __expf(Bc[e] - zj);
      ww[e] = __expf(zj1 - Bc[e]);
      av[e] = qv[e] * uu[e];
      bv[e] = kv[e] * ww[e] * invGj;
      dqd[e] = 0.f;
      dkd[e] = 0.f;
    }
    // dP rows hold zeros beyond the diagonal, so pairs (f, f+1) may run one past e
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float4 *rowp = reinterpret_cast<const float4 *>(dPd + (16 * j + e) * 16);
      float pr[16];
#pragma unroll
      for (int x4 = 0; x4 < 4; ++x4) {
        const float4 v4 = rowp[x4];
        pr[4 * x4] = v4.x;
        pr[4 * x4 + 1] = v4.y;
        pr[4 * x4 + 2] = v4.z;
        pr[4 * x4 + 3] = v4.w;
      }
      float q0 = 0.f, q1 = 0.f;
#pragma unroll
      for (int f = 0; f <= e; f += 2) {
        dev::ffma2(q0, q1, pr[f], pr[f + 1], bv[f], bv[f + 1]);
        dev::ffma2(dkd[f], dkd[f + 1], pr[f], pr[f + 1], av[e], av[e]);
      }
      dqd[e] = q0 + q1;
    }
#pragma unroll
    for (int e = 15; e >= 0; --e) {
      const int t = 16 * j + e;
      const long tg = (long)n * kC + t;
      const float dqd_e = dqd[e] * uu[e];
      const float dkd_e = dkd[e] * ww[e] * invGj;
      const float dqr = uu[e] * (Ej * xq[e] + offq_on * xqi[e]);
      const float dkr = ww[e] * (GAj * xk[e] + offk_on * xki[e]);
      run += (qv[e] * dqr - kv[e] * dkr) + (qv[e] * dqd_e - kv[e] * dkd_e);
      {
        // into the staging tiles (rows beyond T are clipped by the stores)
        const uint32_t e16 = (uint32_t)((cl >> 6) * 4096 + t * 64 + (cl & 63));
        const bf16 bq = __float2bfloat16_rn(dqr + dqd_e), bk = __float2bfloat16_rn(dkr + dkd_e);
        dev::st_shared_u16(sDq + 2u * e16, *reinterpret_cast<const uint16_t *>(&bq));
        dev::st_shared_u16(sDk + 2u * e16, *reinterpret_cast<const uint16_t *>(&bk));
        if (a.gate == GLA_GATE_VECTOR)
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(sDla + 4u * e16), "f"(run) : "memory");
        (void)tg;
      }
      if (a.gate == GLA_GATE_SCALAR) {
        float x = run;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) red[warp * 64 + t] = x;
      }
    }
  }
  dev::fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0 && ok) {
#pragma unroll
    for (int hc = 0; hc < kBwdKH / 64; ++hc) {
      dev::tma_store_3d(&tmDQ, smem + L::kSDq + hc * 8192, c0 + 64 * hc, n * kC, (int)bh);
      dev::tma_store_3d(&tmDK, smem + L::kSDk + hc * 8192, c0 + 64 * hc, n * kC, (int)bh);
      if (a.gate == GLA_GATE_VECTOR)
        dev::tma_store_3d(&tmDLA, smem + L::kSDla + hc * 16384, c0 + 64 * hc, n * kC, (int)bh);
    }
    dev::tma_store_commit();
  }
  if (a.gate == GLA_GATE_SCALAR) {
    if (tid < kC) {
      float ssum = 0.f;
#pragma unroll
      for (int w4 = 0; w4 < kBwdKH / 32; ++w4) ssum += red[w4 * 64 + tid];
      const long tg = (long)n * kC + tid;
      if (tg < a.T && ok) {
        if (kH == 1) a.dla[bh * a.T + tg] = ssum;
        else atomicAdd(a.dla + bh * a.T + tg, ssum);  // onto zero, two addends: exact and order-free
      }
    }
  }
  if (tid == 0) dev::tma_store_wait_all();  // the stores have read their tiles before the CTA ends
  dev::tc_fence_before();
  __syncthreads();
  if (warp == 0) dev::tmem_dealloc(tmem, kTmemCols);
}

template <int K>
int launch_bwd_main_k(const Problem &p, const BwdArgs &a, const CUtensorMap *maps, cudaStream_t st) {
  static DeviceSlots slots;
  const int smem = per_device(slots, [] {
    if (cudaFuncSetAttribute(k_bwd_main<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem) != cudaSuccess)
      return -1;
    return smem_for_tmem(k_bwd_main<K>, kBwdKH, BwdSmem::kBytes + 1024, 256);
  });
  if (smem < 0) return GLA_ERR_CUDA;
  GLA_LAUNCH(K_TC_BWD, st,
             if (launch_pdl(k_bwd_main<K>, dim3(K / kBwdKH, p.N, p.BH), dim3(kBwdKH), smem, st, a, maps[0], maps[1],
                            maps[2], maps[3], maps[4], maps[5], maps[6]) != cudaSuccess) return GLA_ERR_CUDA);
  return GLA_OK;
}

bool map3_bf16(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1);
// row-major staging tile -> tensor (no swizzle), bf16 or fp32 elements
bool map3_store(CUtensorMap *m, const void *base, bool fp32, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                uint32_t b1);

inline int launch_bwd_main(const Problem &p, const bf16 *q, const bf16 *k, const bf16 *v, const float *la,
                           const bf16 *dout, bf16 *dq, bf16 *dk, float *dla, const float *gam, const bf16 *hb,
                           const bf16 *dhb, unsigned *status, cudaStream_t st) {
  if (p.V % 64 != 0 || p.K % kBwdKH != 0) return GLA_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap maps[7];
  const uint64_t BH = (uint64_t)p.BH;
  bool ok = map3_bf16(&maps[0], v, p.V, p.T, BH, 64, 64) && map3_bf16(&maps[1], dout, p.V, p.T, BH, 64, 64) &&
            map3_bf16(&maps[2], q, p.K, p.T, BH, 64, 64) && map3_bf16(&maps[3], k, p.K, p.T, BH, 64, 64) &&
            map3_store(&maps[4], dq, false, p.K, p.T, BH, 64, 64) && map3_store(&maps[5], dk, false, p.K, p.T, BH, 64, 64);
  // dlog alpha through a tile store for vector gates (the map is unused otherwise)
  ok = ok && (p.gate == GLA_GATE_VECTOR ? map3_store(&maps[6], dla, true, p.K, p.T, BH, 64, 64)
                                        : map3_store(&maps[6], dq, false, p.K, p.T, BH, 64, 64));
  if (!ok) return GLA_ERR_CUDA;
  // with a scalar gate and two channel halves, dlog alpha is summed by atomic adds
  if (p.gate == GLA_GATE_SCALAR && p.K > kBwdKH)
    if (cudaMemsetAsync(dla, 0, (size_t)p.BH * p.T * sizeof(float), st) != cudaSuccess) return GLA_ERR_CUDA;
  BwdArgs a{p.T, p.N, p.V, p.gate, p.Tp, q, k, la, gam, hb, dhb, dq, dk, dla, status, 0, 0, 0u};
  {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    a.stagger0 = sms;  // the second CTA of each SM in the first wave
    a.stagger1 = 2 * sms;
    a.stagger_ns = kBwdStaggerNs;
  }
  if (p.K == 256) return launch_bwd_main_k<256>(p, a, maps, st);
  return launch_bwd_main_k<128>(p, a, maps, st);
}

}  // namespace tc
}  // namespace gla
