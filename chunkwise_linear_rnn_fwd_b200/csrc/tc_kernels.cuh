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
// Walk: per (d_v tile, segment, head); carries the fp32 state tile S (K x BV)
// in TMEM across the chunks of one segment.  Per chunk n (forward):
//     [state out]  h_n = S                       (bf16 via TMA, or fp32)
//     [output]     O_n = qg_n S_bf16 + A_n V_n   (tcgen05, M = 64)
//     S = diag(gam_n) S + kg_n^T V_n             (tcgen05, M = 128 per 128 key rows)
// Reverse (adjoint) walks run the chunks backwards with (qg, dO) in place of
// (kg, V): dS_{n-1} = diag(gam_n) dS_n + qg_n^T dO_n.
// ============================================================================
struct WalkArgs {
  int T, N, V, L;  // L = chunks per segment
  int P;           // segments per sequence (the grid covers segments seg0 .. seg0 + gridDim.y - 1)
  int seg0;
  int end_seg;     // -1: every segment writes end[BH][P][K][V]; s >= 0: only segment s writes end[BH][K][V]
  int reverse, do_out, state_mode;  // state_mode: 0 none, 1 bf16 (TMA store), 2 fp32
  int p_kmajor;                     // output intra term: 0 = P V (forward), 1 = P^T dO (reverse: dv)
  const float *gam;                 // [BH][N][K]
  const float *start;               // [BH][P][K][V] fp32 start states or null
  const float *delta;               // [BH][P][V/4][K] float4 segment contributions from a zero state (or null):
                                    // the start state is then composed in the kernel from h0 and the
                                    // contributions of the segments before this one (after it, reverse)
  const float *h0;                  // initial state of the whole walk (h0, or dh_final in reverse) or null
  float *end;                       // state after the segment or null: end_seg < 0: [BH][P][V/4][K] float4
                                    // (the delta layout); else [BH][K][V] fp32
  float *gseg;                      // [BH][P][K] product of gam over the segment (written by d_v tile 0) or null
  const float *gseg_in;             // the same products, read when composing start states
  float *h32;                       // [BH][N][K][V] fp32 states (state_mode 2)
  bf16 *hb;                         // [BH][N][K/128][V/8][128][8] bf16 states (state_mode 1)
  bf16 *out;                        // [BH][T][V]
  unsigned *status;
};

// Shared-memory layout of a walk CTA.  Output walks stage (kg, V, qg, P^T) once
// (two CTAs share an SM); state-only walks double-buffer (kg or qg, V or dO).
template <int K, int BV>
struct WalkSmem {
  static constexpr int kTileX = 64 * K * 2;   // kg or qg chunk tile
  static constexpr int kTileY = 64 * BV * 2;  // V or dO tile
  static constexpr int kTileQ = 64 * K * 2;   // qg for the output
  static constexpr int kTileP = 64 * 64 * 2;  // P^T
  __host__ __device__ static constexpr int stages(bool out) { return out ? 1 : 2; }
  __host__ __device__ static constexpr int stage_bytes(bool out) {
    return kTileX + kTileY + (out ? kTileQ + kTileP : 0);
  }
  __host__ __device__ static constexpr int sb_off(bool out) { return stages(out) * stage_bytes(out); }
  __host__ __device__ static constexpr int bar_off(bool out, bool sb) { return sb_off(out) + (sb ? K * BV * 2 : 0); }
  __host__ __device__ static constexpr int bytes(bool out, bool sb) { return bar_off(out, sb) + 64; }
};

template <int K, int BV>
__global__ void __launch_bounds__(K, 2)
    k_walk(WalkArgs a, const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
           const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmP) {
  using L = WalkSmem<K, BV>;
  constexpr int kThreads = K;
  constexpr int kMB = K / 128;         // 128-row blocks of the state
  constexpr int kColO = kMB * BV;      // TMEM column of the output accumulator
  constexpr int kTmemCols = (kColO + BV <= 256) ? 256 : 512;
  // The dynamic shared-memory window is allocated without alignment slack (two
  // CTAs must fit on one SM); its base is 1024-byte aligned when the kernel has
  // no static shared memory.  Checked: a misaligned base would break the
  // 128-byte swizzle, so the CTA reports it and does nothing.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  if ((dev::smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(a.status, (unsigned)ST_SMEM_ALIGN);
    return;
  }
  const bool need_sb = a.do_out != 0;
  const int nst = L::stages(a.do_out);
  const int kStage = L::stage_bytes(a.do_out);
  uint64_t *full = (uint64_t *)(smem + L::bar_off(a.do_out, need_sb));
  uint64_t *mma_bar = full + 2;
  uint32_t *tslot = (uint32_t *)(full + 3);
  uint8_t *sb_ptr = smem + L::sb_off(a.do_out);
  const uint32_t sSb = dev::smem_u32(sb_ptr);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vt = blockIdx.x, seg = blockIdx.y + a.seg0;
  const long bh = blockIdx.z;
  const int v0 = vt * BV;
  const int n_begin = seg * a.L;
  const int n_end = min(a.N, n_begin + a.L);
  const int nloc = n_end - n_begin;
  const int P = a.P;

  if (tid == 0) {
    dev::mbar_init(&full[0], 1);
    dev::mbar_init(&full[1], 1);
    dev::mbar_init(mma_bar, 1);
    dev::fence_mbar_init();
    dev::prefetch_tmap(&tmX);
    dev::prefetch_tmap(&tmY);
    if (a.do_out) {
      dev::prefetch_tmap(&tmQ);
      dev::prefetch_tmap(&tmP);
    }
  }
  dev::pdl_launch_dependents();
  dev::pdl_wait();
  if (warp == 0) dev::tmem_alloc(tslot, kTmemCols);
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tslot;

  auto chunk_of = [&](int i) { return a.reverse ? (n_end - 1 - i) : (n_begin + i); };
  auto stage_ptr = [&](int s) { return smem + s * kStage; };
  const uint32_t tx_bytes = (uint32_t)kStage;

  auto issue_loads = [&](int i) {
    const int s = i % nst;
    const int n = chunk_of(i);
    uint8_t *st = stage_ptr(s);
    dev::mbar_arrive_expect_tx(&full[s], tx_bytes);
#pragma unroll
    for (int cb = 0; cb < K / 64; ++cb) dev::tma_load_3d(st + cb * 64 * 128, &tmX, cb * 64, n * kC, (int)bh, &full[s]);
#pragma unroll
    for (int cb = 0; cb < BV / 64; ++cb)
      dev::tma_load_3d(st + L::kTileX + cb * 64 * 128, &tmY, v0 + cb * 64, n * kC, (int)bh, &full[s]);
    if (a.do_out) {
#pragma unroll
      for (int cb = 0; cb < K / 64; ++cb)
        dev::tma_load_3d(st + L::kTileX + L::kTileY + cb * 64 * 128, &tmQ, cb * 64, n * kC, (int)bh, &full[s]);
      dev::tma_load_3d(st + L::kTileX + L::kTileY + L::kTileQ, &tmP, 0, 0, (int)(bh * a.N + n), &full[s]);
    }
  };

  if (tid == 0)
    for (int i = 0; i < nst && i < nloc; ++i) issue_loads(i);

  // thread -> state row c; TMEM lane block of its warp
  const int mb = warp >> 2;
  const int c = tid;  // state row (key channel)
  const uint32_t tS = dev::tmem_addr(tmem, 32 * (warp & 3), mb * BV);
  const long KV = (long)K * a.V;

  // ---- initial state into TMEM --------------------------------------------
  // Composed segment start: S = h0; then for every earlier segment p (later, in
  // reverse) S = diag(gseg_p) S + delta_p -- the scan over segments, done per row.
  // Done in 16-column blocks so that the loads of up to four segments are in
  // flight together (the per-row chain is a sequence of dependent global loads).
  {
    const bool compose = (a.delta != nullptr);
    const float *src = nullptr;
    if (a.start) src = a.start + ((bh * P + seg) * K + c) * (long)a.V + v0;
    else if (a.h0 && (compose || seg == (a.reverse ? P - 1 : 0))) src = a.h0 + bh * KV + (long)c * a.V + v0;
    const int np = compose ? (a.reverse ? (P - 1 - seg) : seg) : 0;
    auto seg_of = [&](int i) { return a.reverse ? (P - 1 - i) : i; };
#pragma unroll 1
    for (int cb = 0; cb < BV / 16; ++cb) {
      float S[16];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float4 v4 =
            src ? __ldg(reinterpret_cast<const float4 *>(src + cb * 16) + x) : make_float4(0.f, 0.f, 0.f, 0.f);
        S[4 * x] = v4.x;
        S[4 * x + 1] = v4.y;
        S[4 * x + 2] = v4.z;
        S[4 * x + 3] = v4.w;
      }
      int i = 0;
#pragma unroll 1
      for (; i + 4 <= np; i += 4) {
        float gs[4];
        float4 d[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int p = seg_of(i + u);
          gs[u] = __ldg(a.gseg_in + (bh * P + p) * K + c);
          const float4 *d4 = reinterpret_cast<const float4 *>(a.delta) +
                             ((bh * P + p) * (a.V / 4) + v0 / 4 + cb * 4) * K + c;
#pragma unroll
          for (int x = 0; x < 4; ++x) d[u][x] = __ldg(d4 + (long)x * K);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            S[4 * x] = gs[u] * S[4 * x] + d[u][x].x;
            S[4 * x + 1] = gs[u] * S[4 * x + 1] + d[u][x].y;
            S[4 * x + 2] = gs[u] * S[4 * x + 2] + d[u][x].z;
            S[4 * x + 3] = gs[u] * S[4 * x + 3] + d[u][x].w;
          }
      }
      if (i < np) {  // 1 to 3 remaining segments, loads issued together
        float gs[3];
        float4 d[3][4];
#pragma unroll
        for (int u = 0; u < 3; ++u) {
          if (i + u < np) {
            const int p = seg_of(i + u);
            gs[u] = __ldg(a.gseg_in + (bh * P + p) * K + c);
            const float4 *d4 = reinterpret_cast<const float4 *>(a.delta) +
                               ((bh * P + p) * (a.V / 4) + v0 / 4 + cb * 4) * K + c;
#pragma unroll
            for (int x = 0; x < 4; ++x) d[u][x] = __ldg(d4 + (long)x * K);
          } else {
            gs[u] = 1.f;
#pragma unroll
            for (int x = 0; x < 4; ++x) d[u][x] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int u = 0; u < 3; ++u)
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            S[4 * x] = gs[u] * S[4 * x] + d[u][x].x;
            S[4 * x + 1] = gs[u] * S[4 * x + 1] + d[u][x].y;
            S[4 * x + 2] = gs[u] * S[4 * x + 2] + d[u][x].z;
            S[4 * x + 3] = gs[u] * S[4 * x + 3] + d[u][x].w;
          }
      }
      dev::tmem_st16(tS + cb * 16, S);
    }
    dev::tmem_wait_st();
  }

  bool ok = true;
  float gprod = 1.f;
  // Output accumulator: two TMEM buffers when the columns allow, so that chunk
  // i-1's output epilogue overlaps chunk i's MMAs.
  constexpr bool kDoubleO = (kColO + 2 * BV <= kTmemCols);
  auto o_col = [&](int i) { return (uint32_t)(kColO + (kDoubleO ? (i & 1) * BV : 0)); };
  // rows t of the chunk (M = 64 TMEM layout: lanes 32*sub + [0,16)), bf16 to out[t][v0 + ...]
  auto out_epilogue = [&](int i) {
    constexpr int kWarps = kThreads / 32;
    constexpr int kColsPerWarp = (kWarps >= 8) ? BV / 2 : BV;
    const int sub = warp & 3;
    const int col0 = (kWarps >= 8 && warp >= 4) ? BV / 2 : 0;
    const int t = 16 * sub + lane;
    const long tgl = (long)chunk_of(i) * kC + t;
#pragma unroll
    for (int cb = 0; cb < kColsPerWarp / 16; ++cb) {
      float v[16];
      dev::tmem_ld16(dev::tmem_addr(tmem, 32 * sub, o_col(i) + col0 + cb * 16), v);
      dev::tmem_wait_ld();
      if (lane < 16 && tgl < a.T && ok) {
        uint4 p0, p1;
        p0.x = dev::pack_bf16(v[0], v[1]);
        p0.y = dev::pack_bf16(v[2], v[3]);
        p0.z = dev::pack_bf16(v[4], v[5]);
        p0.w = dev::pack_bf16(v[6], v[7]);
        p1.x = dev::pack_bf16(v[8], v[9]);
        p1.y = dev::pack_bf16(v[10], v[11]);
        p1.z = dev::pack_bf16(v[12], v[13]);
        p1.w = dev::pack_bf16(v[14], v[15]);
        uint4 *dst = reinterpret_cast<uint4 *>(a.out + (bh * a.T + tgl) * (long)a.V + v0 + col0 + cb * 16);
        dst[0] = p0;
        dst[1] = p1;
      }
    }
  };
  float g_next = (nloc > 0) ? __ldg(a.gam + (bh * a.N + chunk_of(0)) * K + c) : 1.f;
  for (int i = 0; i < nloc; ++i) {
    const int s = i % nst;
    const int n = chunk_of(i);
    uint8_t *st = stage_ptr(s);
    const float g = g_next;
    if (i + 1 < nloc) g_next = __ldg(a.gam + (bh * a.N + chunk_of(i + 1)) * K + c);
    gprod *= g;

    // ---- S-pass: read S, publish bf16/fp32 copy, scale by gamma ---------------
    // (needs only the previous chunk's MMAs: it runs while this chunk's tiles load)
#pragma unroll
    for (int cb = 0; cb < BV / 32; ++cb) {
      float v[32];
      dev::tmem_ld32(tS + cb * 32, v);
      dev::tmem_wait_ld();
      if (a.do_out || a.state_mode == 1) {
        uint4 pk[4];
#pragma unroll
        for (int h = 0; h < 4; ++h)
          pk[h] = make_uint4(dev::pack_bf16(v[8 * h], v[8 * h + 1]), dev::pack_bf16(v[8 * h + 2], v[8 * h + 3]),
                             dev::pack_bf16(v[8 * h + 4], v[8 * h + 5]), dev::pack_bf16(v[8 * h + 6], v[8 * h + 7]));
        if (a.do_out) {
#pragma unroll
          for (int h = 0; h < 4; ++h)
            dev::st_shared_v4(sSb + dev::sw128_chunk(K, c, cb * 4 + h), pk[h].x, pk[h].y, pk[h].z, pk[h].w);
        }
        if (a.state_mode == 1) {
          // chunk state h_n in the [K/128][V/8][128][8] layout: a warp stores 512
          // contiguous bytes, and a 128-channel half of a 64-column tile is 16 KB
          uint4 *dst = reinterpret_cast<uint4 *>(a.hb) +
                       (((bh * a.N + n) * (K / 128) + (c >> 7)) * (a.V / 8) + (v0 + cb * 32) / 8) * 128 + (c & 127);
#pragma unroll
          for (int h = 0; h < 4; ++h) dst[h * 128] = pk[h];
        }
      }
      if (a.state_mode == 2) {
        float4 *dst = reinterpret_cast<float4 *>(a.h32 + ((bh * a.N + n) * K + c) * (long)a.V + v0 + cb * 32);
#pragma unroll
        for (int h = 0; h < 8; ++h) dst[h] = make_float4(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]);
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] *= g;
      dev::tmem_st16(tS + cb * 32, v);
      dev::tmem_st16(tS + cb * 32 + 16, v + 16);
    }
    dev::tmem_wait_st();
    dev::fence_proxy_async_smem();
    if (ok) ok = dev::mbar_wait(&full[s], (uint32_t)((i / nst) & 1), a.status);
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();

    // ---- MMA issue ---------------------------------------------------------
    if (tid == 0 && ok) {
      const uint32_t sX = dev::smem_u32(st);
      const uint32_t sY = sX + L::kTileX;
      const uint32_t sQ = sY + L::kTileY;
      const uint32_t sP = sQ + L::kTileQ;
      if (a.do_out) {
        const uint32_t tO = tmem + o_col(i);
        constexpr uint32_t id_qs = dev::idesc_bf16(64, BV, false, true);
#pragma unroll
        for (int kk = 0; kk < K / 16; ++kk)
          dev::umma_bf16(tO, dev::desc_kmajor(sQ, 64, 0, kk * 16), dev::desc_mnmajor(sSb, K, kk * 16, 0), id_qs,
                         kk > 0 ? 1u : 0u);
        if (!a.p_kmajor) {
          // O += A V with A[t][s] = P^T tile [s][t]: MN-major A
          constexpr uint32_t id_pv = dev::idesc_bf16(64, BV, true, true);
#pragma unroll
          for (int kk = 0; kk < kC / 16; ++kk)
            dev::umma_bf16(tO, dev::desc_mnmajor(sP, 64, kk * 16, 0), dev::desc_mnmajor(sY, 64, kk * 16, 0), id_pv,
                           1u);
        } else {
          // dv += A^T dO with A^T[s][t] = P^T tile [s][t]: K-major A
          constexpr uint32_t id_pt = dev::idesc_bf16(64, BV, false, true);
#pragma unroll
          for (int kk = 0; kk < kC / 16; ++kk)
            dev::umma_bf16(tO, dev::desc_kmajor(sP, 64, 0, kk * 16), dev::desc_mnmajor(sY, 64, kk * 16, 0), id_pt,
                           1u);
        }
      }
      constexpr uint32_t id_st = dev::idesc_bf16(128, BV, true, true);
#pragma unroll
      for (int m = 0; m < kMB; ++m)
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          dev::umma_bf16(tmem + m * BV, dev::desc_mnmajor(sX, 64, kk * 16, 128 * m),
                         dev::desc_mnmajor(sY, 64, kk * 16, 0), id_st, 1u);
      dev::umma_commit(mma_bar);
    }
    // the previous chunk's output is read out while this chunk's MMAs run
    if (a.do_out && kDoubleO && i > 0) out_epilogue(i - 1);
    if (ok) ok = dev::mbar_wait(mma_bar, i & 1, a.status);
    dev::tc_fence_after();
    if (tid == 0 && ok && i + nst < nloc) issue_loads(i + nst);
    if (a.do_out && !kDoubleO) out_epilogue(i);
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
  }
  if (a.do_out && kDoubleO && nloc > 0) {
    out_epilogue(nloc - 1);
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
  }

  // ---- final state of the segment ---------------------------------------------
  if (a.gseg && vt == 0) a.gseg[(bh * P + seg) * K + c] = gprod;
  if (a.end && (a.end_seg < 0 || a.end_seg == seg)) {
#pragma unroll
    for (int cb = 0; cb < BV / 16; ++cb) {
      float v[16];
      dev::tmem_ld16(tS + cb * 16, v);
      dev::tmem_wait_ld();
      if (a.end_seg < 0) {
        // segment contribution, float4-column layout (coalesced across the warp)
        float4 *d4 = reinterpret_cast<float4 *>(a.end) + ((bh * P + seg) * (a.V / 4) + v0 / 4 + cb * 4) * K + c;
#pragma unroll
        for (int x = 0; x < 4; ++x) d4[(long)x * K] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
      } else {
        float4 *d4 = reinterpret_cast<float4 *>(a.end + (bh * K + c) * (long)a.V + v0 + cb * 16);
#pragma unroll
        for (int x = 0; x < 4; ++x) d4[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
      }
    }
  }
  dev::tc_fence_before();
  __syncthreads();
  if (warp == 0) dev::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc
}  // namespace gla
