// tc_kernels.cuh -- bf16 tensor-core kernels of the chunkwise GLA path (sm_100a).
//
// Notation (one head): chunk size C = 64, sub-chunk c = 16, d_k = K, tile of
// d_v = BV.  B_t is the chunk-local inclusive cumulative log-gate, z_j = B at
// the last row before sub-chunk j (z_0 = 0, z_4 = B_63), Gam_j = e^{z_{j+1}-z_j}
// the decay of sub-chunk j, u_t = e^{B_t - z_{j(t)}} and w_t = e^{z_{j(t)+1} - B_t}
// (both in (0,1]).  Every rescaled operand is a product of such factors, so no
// factor exceeds 1 except the diagonal-block key factor 1/Gam_j (section 4.2 /
// Figure 3 of "Gated Linear Attention Transformers with Hardware-Efficient
// Training": secondary chunking with a reference point at each query sub-chunk).
#pragma once

#include "tc_common.cuh"

namespace gla {
namespace tc {

using bf16 = __nv_bfloat16;
constexpr int kC = 64;    // chunk
constexpr int kSub = 16;  // sub-chunk

// ============================================================================
// Prep: per (chunk, head).  Writes
//   qg[t]  = q_t (.) e^{B_t}              (bf16, inter-chunk query operand)
//   kg[t]  = k_t (.) e^{B_63 - B_t}       (bf16, state-update key operand)
//            (both written over the q / k tiles in shared memory, then TMA-stored)
//   gam    = e^{B_63}                     (fp32 per key channel)
//   PT[s][t] = causal intra-chunk score A[t][s] (bf16, transposed)
// The strictly-lower sub-chunk blocks of A come from three tcgen05 MMAs
// (M = 64 keys, N = 16 queries of sub-chunk j, reference point z_j); the four
// diagonal 16 x 16 blocks are summed in fp32 on CUDA cores.
// ============================================================================
struct PrepArgs {
  int T, N, gate;
  long Tp;
  const float *la;
  bf16 *qg, *kg, *PT;
  float *gam;
  unsigned *status;
};

template <int K>
struct PrepSmem {
  static constexpr int kRowsKw = 112;                  // key windows: rows [0,16) [16,48) [48,96) + pad
  static constexpr int kQ = 0;                         // q tile [64][K] bf16 (TMA)
  static constexpr int kK = kQ + 64 * K * 2;           // k tile [64][K] bf16 (TMA)
  static constexpr int kQh = kK + 64 * K * 2;          // Q-hat tile, 64 rows
  static constexpr int kKw = kQh + 64 * K * 2;         // key windows, 112 rows
  static constexpr int kAf = kKw + kRowsKw * K * 2;    // fp32 a_t = q_t u_t of one sub-chunk [16][K]
  static constexpr int kBf = kAf + 16 * K * 4;         // fp32 b_s = k_s e^{z_j - B_s} [16][K]
  static constexpr int kRed = kBf + 16 * K * 4;        // per-warp partial diagonal blocks [8][16][16]
  static constexpr int kPd = kRed + 8 * 256 * 4;       // fp32 diagonal blocks [64][16]
  static constexpr int kBar = kPd + 64 * 16 * 4;       // mbarriers + tmem slot
  static constexpr int kBytes = kBar + 64;
};

// fp32 [rows][K] tile with a 16-byte-chunk swizzle (bank-conflict-free for the
// diagonal-block access pattern: 4 rows 4 apart, or 8 rows 2 apart, per load).
template <int K>
__device__ __forceinline__ int f32_swz(int r, int c) {
  const int cc = c >> 2;
  const int sw = (r ^ (r >> 3)) & 7;
  return r * K + (((cc & ~7) | ((cc & 7) ^ sw)) << 2) + (c & 3);
}

template <int K>
__global__ void __launch_bounds__(256, 1)
    k_prep(PrepArgs a, const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
           const __grid_constant__ CUtensorMap tmqg, const __grid_constant__ CUtensorMap tmkg) {
  using L = PrepSmem<K>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sQ = dev::smem_u32(smem + L::kQ);
  const uint32_t sK = dev::smem_u32(smem + L::kK);
  const uint32_t sQh = dev::smem_u32(smem + L::kQh);
  const uint32_t sKw = dev::smem_u32(smem + L::kKw);
  float *Af = (float *)(smem + L::kAf);
  float *Bf = (float *)(smem + L::kBf);
  float *red = (float *)(smem + L::kRed);
  float *Pd = (float *)(smem + L::kPd);
  uint64_t *bar = (uint64_t *)(smem + L::kBar);  // [0] q/k loads, [1] MMA
  uint32_t *tslot = (uint32_t *)(smem + L::kBar + 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x;
  const long bh = blockIdx.y;

  if (tid == 0) {
    dev::mbar_init(&bar[0], 1);
    dev::mbar_init(&bar[1], 3);  // one arrival per MMA-issuing thread
    dev::fence_mbar_init();
    dev::prefetch_tmap(&tmq);
    dev::prefetch_tmap(&tmk);
  }
  dev::pdl_launch_dependents();
  dev::pdl_wait();
  if (warp == 0) dev::tmem_alloc(tslot, 64);
  if (tid == 0) {
    dev::mbar_arrive_expect_tx(&bar[0], (uint32_t)(2 * 64 * K * 2));
#pragma unroll
    for (int cb = 0; cb < K / 64; ++cb) {
      dev::tma_load_3d(smem + L::kQ + cb * 64 * 128, &tmq, cb * 64, n * kC, (int)bh, &bar[0]);
      dev::tma_load_3d(smem + L::kK + cb * 64 * 128, &tmk, cb * 64, n * kC, (int)bh, &bar[0]);
    }
  }
  __syncthreads();  // barriers initialised before anyone waits on them

  // ---- per key channel: chunk-local cumulative log-gate (all loads in flight) ----
  const int c = tid;
  float Bv[kC];
  float z[5], Gam[4], E[4], Gafter[4];
  if (tid < K) {
    float g[kC];
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      const long tg = (long)n * kC + t;
      g[t] = 0.f;
      if (tg < a.T) {
        if (a.gate == GLA_GATE_VECTOR) g[t] = __ldg(a.la + (bh * a.T + tg) * K + c);
        else if (a.gate == GLA_GATE_SCALAR) g[t] = __ldg(a.la + bh * a.T + tg);
      }
    }
    float acc = 0.f;
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      acc += g[t];
      Bv[t] = acc;
    }
    z[0] = 0.f;
    z[1] = Bv[15];
    z[2] = Bv[31];
    z[3] = Bv[47];
    z[4] = Bv[63];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      Gam[j] = __expf(z[j + 1] - z[j]);
      E[j] = __expf(z[j]);
    }
    if (Gam[0] < 1e-36f || Gam[1] < 1e-36f || Gam[2] < 1e-36f || Gam[3] < 1e-36f)
      atomicOr(a.status, (unsigned)ST_GATE_RANGE);
    Gafter[3] = 1.f;
    Gafter[2] = Gam[3];
    Gafter[1] = Gam[3] * Gam[2];
    Gafter[0] = Gam[3] * Gam[2] * Gam[1];
    a.gam[(bh * a.N + n) * K + c] = __expf(z[4]);
    // rows 96..111 of the window buffer are read by window 3 only for keys >= 48,
    // whose entries are discarded; keep them finite
    const bf16 zb = __float2bfloat16_rn(0.f);
    for (int r = 96; r < L::kRowsKw; ++r)
      dev::st_shared_u16(sKw + dev::sw128_off(L::kRowsKw, r, c), *reinterpret_cast<const uint16_t *>(&zb));
  }
  const bool ok_ld = dev::mbar_wait(&bar[0], 0, a.status);

  const int wrow[4] = {0, 0, 16, 48};  // window start row of query sub-chunk j (j >= 1)
#pragma unroll 1
  for (int j = 0; j < 4; ++j) {
    // ---- rescaled operands of sub-chunk j ----
    if (tid < K) {
      float Bc[16];
      dev::take16(Bv, j, Bc);
      const float zj = dev::sel4(j, z[0], z[1], z[2], z[3]);
      const float zj1 = dev::sel4(j, z[1], z[2], z[3], z[4]);
      const float Ej = dev::sel4(j, E[0], E[1], E[2], E[3]);
      const float Gj = dev::sel4(j, Gam[0], Gam[1], Gam[2], Gam[3]);
      const float GAj = dev::sel4(j, Gafter[0], Gafter[1], Gafter[2], Gafter[3]);
      const float invGj = 1.f / Gj;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int t = 16 * j + e;
        uint16_t qb, kb;
        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(qb) : "r"(sQ + dev::sw128_off(64, t, c)));
        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(kb) : "r"(sK + dev::sw128_off(64, t, c)));
        const float qf = ok_ld ? __bfloat162float(*reinterpret_cast<const bf16 *>(&qb)) : 0.f;
        const float kf = ok_ld ? __bfloat162float(*reinterpret_cast<const bf16 *>(&kb)) : 0.f;
        const float u = __expf(Bc[e] - zj);
        const float w = __expf(zj1 - Bc[e]);
        const float qh = qf * u;
        const float kw = kf * w;
        // qg and kg replace q and k in their tiles (same thread, same element),
        // which are then stored by TMA
        const bf16 qgb = __float2bfloat16_rn(qh * Ej), kgb = __float2bfloat16_rn(kw * GAj);
        dev::st_shared_u16(sQ + dev::sw128_off(64, t, c), *reinterpret_cast<const uint16_t *>(&qgb));
        dev::st_shared_u16(sK + dev::sw128_off(64, t, c), *reinterpret_cast<const uint16_t *>(&kgb));
        const bf16 qhb = __float2bfloat16_rn(qh);
        dev::st_shared_u16(sQh + dev::sw128_off(64, t, c), *reinterpret_cast<const uint16_t *>(&qhb));
        Af[f32_swz<K>(e, c)] = qh;
        Bf[f32_swz<K>(e, c)] = kw * invGj;
        // key operand for every later query sub-chunk jq: k_s e^{z_jq - B_s}
        float f = kw;
#pragma unroll
        for (int jq = 1; jq < 4; ++jq) {
          if (jq > j) {
            const bf16 b = __float2bfloat16_rn(f);
            dev::st_shared_u16(sKw + dev::sw128_off(L::kRowsKw, wrow[jq] + t, c), *reinterpret_cast<const uint16_t *>(&b));
            f *= Gam[jq];
          }
        }
      }
    }
    __syncthreads();
    // ---- diagonal block j in fp32: warp w sums its slice of key channels ----
    {
      constexpr int kCw = K / 8;
      const int tg = lane >> 3, sp = lane & 7;
      float acc[4][2] = {};
      if (2 * sp <= 4 * tg + 3) {
        const int c0 = warp * kCw;
#pragma unroll 4
        for (int cc = c0; cc < c0 + kCw; cc += 4) {
          float4 av[4], bv[2];
#pragma unroll
          for (int i = 0; i < 4; ++i) av[i] = *reinterpret_cast<const float4 *>(Af + f32_swz<K>(4 * tg + i, cc));
#pragma unroll
          for (int m = 0; m < 2; ++m) bv[m] = *reinterpret_cast<const float4 *>(Bf + f32_swz<K>(2 * sp + m, cc));
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < 2; ++m)
              acc[i][m] += av[i].x * bv[m].x + av[i].y * bv[m].y + av[i].z * bv[m].z + av[i].w * bv[m].w;
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < 2; ++m) red[warp * 256 + (4 * tg + i) * 16 + 2 * sp + m] = acc[i][m];
    }
    __syncthreads();
    {
      const int tl = tid >> 4, sl = tid & 15;
      float ssum = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) ssum += red[w8 * 256 + tl * 16 + sl];
      Pd[(16 * j + tl) * 16 + sl] = (sl <= tl) ? ssum : 0.f;
    }
  }
  dev::fence_proxy_async_smem();
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tslot;

  // ---- off-diagonal blocks on the tensor cores; qg, kg tiles out by TMA ------
  // query sub-chunk j (1..3) from lane 0 of warp j - 1 (a tcgen05.mma costs its
  // issuing thread tens of cycles; the three accumulators are independent)
  if (lane == 0 && warp < 3) {
    const int j = warp + 1;
    constexpr uint32_t idesc = dev::idesc_bf16(64, 16, false, false);
#pragma unroll 4
    for (int kk = 0; kk < K / 16; ++kk) {
      const uint64_t da = dev::desc_kmajor(sKw, L::kRowsKw, j == 1 ? 0 : (j == 2 ? 16 : 48), kk * 16);
      const uint64_t db = dev::desc_kmajor(sQh, 64, 16 * j, kk * 16);
      dev::umma_bf16(tmem + 16 * j, da, db, idesc, kk > 0 ? 1u : 0u);
    }
    dev::umma_commit(&bar[1]);
  }
  if (tid == 32 * 3) {
#pragma unroll
    for (int cb = 0; cb < K / 64; ++cb) {
      dev::tma_store_3d(&tmqg, smem + L::kQ + cb * 64 * 128, cb * 64, n * kC, (int)bh);
      dev::tma_store_3d(&tmkg, smem + L::kK + cb * 64 * 128, cb * 64, n * kC, (int)bh);
    }
    dev::tma_store_commit();
  }
  const bool ok = dev::mbar_wait(&bar[1], 0, a.status) && ok_ld;
  dev::tc_fence_after();

  // ---- assemble P^T rows (key s) and store: warps w and w+4 share the rows of
  // TMEM lane block w (columns t < 32 and t >= 32) -------------------------------
  {
    const int wb = warp & 3;
    const int s = 16 * wb + lane;  // valid for lane < 16
    const int js = wb;             // sub-chunk of key s
    const int t0 = (warp >> 2) * 32;
    float row[32];
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) dev::tmem_ld16(dev::tmem_addr(tmem, 32 * wb, t0 + 16 * cb), row + 16 * cb);
    dev::tmem_wait_ld();
    if (lane < 16) {
      bf16 *dst = a.PT + ((bh * a.N + n) * kC + s) * kC + t0;
#pragma unroll
      for (int t8 = 0; t8 < 4; ++t8) {
        float v8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int t = t0 + t8 * 8 + e;
          const int jt = t >> 4;
          float val = 0.f;
          if (jt > js) val = ok ? row[t8 * 8 + e] : 0.f;
          else if (jt == js && t >= s) val = Pd[t * 16 + (s - 16 * js)];
          v8[e] = val;
        }
        uint4 pk;
        pk.x = dev::pack_bf16(v8[0], v8[1]);
        pk.y = dev::pack_bf16(v8[2], v8[3]);
        pk.z = dev::pack_bf16(v8[4], v8[5]);
        pk.w = dev::pack_bf16(v8[6], v8[7]);
        *reinterpret_cast<uint4 *>(dst + t8 * 8) = pk;
      }
    }
  }
  if (tid == 32 * 3) dev::tma_store_wait_all();  // the qg / kg tile stores are complete
  dev::tc_fence_before();
  __syncthreads();
  if (warp == 0) dev::tmem_dealloc(tmem, 64);
}

// ============================================================================
// Arguments of the state walk (tc_walk.cuh): per (d_v tile, segment, head) the
// fp32 state tile is carried across the chunks of one segment.  Forward walks
// run S = diag(gam_n) S + kg_n^T V_n and, with outputs, O_n = qg_n S_{n-1} + A_n V_n;
// reverse (adjoint) walks run the chunks backwards with (qg, dO) in place of
// (kg, V): dS_{n-1} = diag(gam_n) dS_n + qg_n^T dO_n, dv_n = kg_n dS_n + A_n^T dO_n.
// ============================================================================
struct WalkArgs {
  int T, N, V, L;  // L = chunks per segment
  int P;           // segments per sequence (the grid covers segments seg0 .. seg0 + gridDim.y - 1)
  int seg0;
  int end_seg;     // -1: every segment writes end[BH][P][K/4][V][4]; s >= 0: only segment s writes end[BH][K][V]
  int reverse, do_out, state_mode;  // state_mode: 0 none, 1 bf16 chunk states, 2 fp32 chunk states
  int p_kmajor;                     // output intra term: 0 = P V (forward), 1 = P^T dO (reverse: dv)
  const float *gam;                 // [BH][N][K]
  const float *start;               // [BH][P][K][V] fp32 start states (materialised chunk states) or null
  const float *start_v;             // [BH][P][K/4][V][4] fp32 start states of the segments after the first
                                    // (before it, reverse) or null; the first starts from h0
  const float *h0;                  // initial state of the whole walk (h0, or dh_final in reverse) or null
  float *end;                       // state after the segment or null: end_seg < 0: [BH][P][K/4][V][4]
                                    // (segment contributions); else [BH][K][V] fp32
  float *gseg;                      // [BH][P][K] product of gam over the segment (written by d_v tile 0) or null
  float *h32;                       // [BH][N][K][V] fp32 states (state_mode 2)
  bf16 *hb;                         // bf16 states (state_mode 1), layout of state_chunk_off (tc_walk.cuh)
  bf16 *out;                        // [BH][T][V]
  unsigned *status;
  // layer epilogue fused into the output store (k_walkT<K, true> only): per-head
  // LayerNorm over d_v with weight / bias (null: ones / zeros) and epsilon, times
  // the Swish gate of r (read through its tensor map); y through its own map
  const float *ln_w, *ln_b;
  float eps;
};

}  // namespace tc
}  // namespace gla
