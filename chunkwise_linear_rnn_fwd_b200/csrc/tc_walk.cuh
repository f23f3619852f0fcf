// tc_walk.cuh -- the inter-chunk state walk of the bf16 tensor-core path (sm_100a).
//
// One CTA per (128-column tile of d_v, segment, head) carries the fp32 state of
// its tile across the chunks of one segment (section 3.3 / 4.2 of "Gated Linear
// Attention Transformers with Hardware-Efficient Training": the chunk-level
// recurrence S_n = diag(gam_n) S_{n-1} + kg_n^T V_n).  The state is kept
// transposed, S^T [v][c], in the registers of 256 threads: thread (v, h) holds
// row v of S^T for the key channels [h K/2, (h+1) K/2).  Per chunk n:
//
//   dS^T  = V_n^T kg_n                        tcgen05 M = 128 (v), N = K (c), K = 64 tokens
//   S^T  <- gam_n (.) S^T + dS^T               CUDA cores, fp32, in registers
//   O_n^T = S_{n-1}^T qg_n^T + V_n^T P_n^T     tcgen05 M = 128 (v), N = 64 (tokens);
//           S_{n-1}^T is the A operand straight from TMEM (bf16, written there by the
//           threads that hold it), so the state never passes through shared memory
//
// and the reverse (adjoint) walk runs the chunks backwards with (qg, dO) in place
// of (kg, V) and dv_n^T = dS^T kg_n^T + dO_n^T P_n.  Warp roles: warps 0-7 hold
// the state (and drain the output accumulator), warp 8 issues the TMA loads into
// two rings (the key-side tiles kg / qg; the value-side tile with the intra-chunk
// scores and the chunk's decay row), warp 9 issues the MMAs, warp 10 forms the
// segment's decay product from the staged decay rows.  Every wait is
// bounded (the status word records a timeout; the kernel then skips the dependent
// work and ends).
//
// k_walkT<K, true> is the forward output walk with the GLA layer's epilogue fused
// into its output store (section 4.4: per-head LayerNorm over d_v, then the Swish
// output gate r sigmoid(r)).  The walk_tiles CTAs of one (segment, head) form a
// thread-block cluster.  The state warps stage each chunk's bf16 output tile in
// shared memory (two buffers) and hand it to warps 10 and 11, which store it,
// take every token row's mean and squared deviations over the tile's 128 columns,
// exchange them with the other CTAs of the cluster through distributed shared
// memory, combine them over all d_v columns, and overwrite the tile with
// y = (w (o - mean) / sqrt(var + eps) + b) r sigmoid(r) for its second store.  The
// epilogue thus runs beside the state chain instead of on it.
#pragma once

#include "tc_kernels.cuh"

namespace gla {
namespace tc {

constexpr int kWalkBV = 128;       // d_v columns per walk CTA
constexpr int kWalkThreads = 384;  // two state warpgroups + one warpgroup for the TMA producer and MMA issuer
// Register budgets.  Launched with 384 threads, one CTA per SM, a thread gets 168
// registers (three warps share each of the SM's four 16K-register partitions);
// the state warpgroups then take 224 (their state rows alone hold K/2 = 128) and
// the producer/MMA warpgroup keeps 56: 256 x 224 + 128 x 56 = 64512 = 384 x 168.
constexpr int kWalkRegsLaunch = 168;
constexpr int kWalkRegsState = 224;
constexpr int kWalkRegsRole = 56;
static_assert(256 * kWalkRegsState + 128 * kWalkRegsRole <= kWalkThreads * kWalkRegsLaunch,
              "register budgets exceed the launch allocation");
// The fused-epilogue walk moves 8 registers per state thread to its epilogue warps.
constexpr int kWalkRegsStateEpi = 216;
constexpr int kWalkRegsRoleEpi = 72;
static_assert(256 * kWalkRegsStateEpi + 128 * kWalkRegsRoleEpi <= kWalkThreads * kWalkRegsLaunch,
              "register budgets exceed the launch allocation");

// EPI: the output walk with the layer epilogue fused into its output store (one
// ring slot fewer on each side, room for the gate tiles r and the row statistics).
template <int K, bool EPI = false>
struct WalkTSmem {
  static constexpr int kXSlot = 64 * K * 2;             // kg or qg chunk tile [64][K] bf16, SW128
  static constexpr int kYTile = 64 * kWalkBV * 2;       // V or dO tile [64][128] bf16, SW128
  static constexpr int kPTile = 64 * 64 * 2;            // P^T [64][64] bf16, SW128
  static constexpr int kYSlot = kYTile + kPTile + 1024;  // + the chunk's decay row gam [K] fp32
  static constexpr int NX = EPI ? ((K == 256) ? 3 : 6) : ((K == 256) ? 4 : 6);
  static constexpr int NY = EPI ? 2 : 3;
  static constexpr int kY0 = NX * kXSlot;
  static constexpr int kR0 = kY0 + NY * kYSlot;           // EPI: gate tiles r [2][64 t][128 v] bf16, SW128
  static constexpr int kRTile = 64 * kWalkBV * 2;
  static constexpr int kXch = kR0 + (EPI ? 2 * kRTile : 0);  // EPI: row statistics [4][4 ranks][64 t] float2
  static constexpr int kXchBuf = 4 * 64 * 8;
  static constexpr int kWB = kXch + (EPI ? 4 * kXchBuf : 0);   // EPI: LayerNorm weight and bias of the tile [2][128] fp32
  static constexpr int kOst = kWB + (EPI ? 1024 : 0);          // output staging, [8 warps][32 t][32 v] bf16
  static constexpr int kOstBuf = 8 * 32 * 32 * 2;              // (EPI: two, SW64, handed to the epilogue warps)
  static constexpr int kBar = kOst + (EPI ? 2 : 1) * kOstBuf;
  static constexpr int kBytes = kBar + 512;
  static_assert(K * 4 <= 1024, "decay row fits its slot");
};

// In-register transpose-and-add across a warp: v[e] on every lane in, out on
// lane l the sum over the warp's lanes of their v[l] (v is overwritten).  Five
// exchange rounds; in each, a lane keeps the half of its entries its partner
// drops and adds the partner's copy of them.
__device__ __forceinline__ float warp_transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int j = 0; j < w; ++j) {
      const float send = up ? v[j] : v[j + w];
      const float keep = up ? v[j + w] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}



// Byte offset of the 16-byte chunk (value column vg, key channels 8 c8 .. 8 c8 + 7)
// of a bf16 chunk state in the layout the backward reads: per chunk row, d_v tile
// of 64 columns and half of 128 key channels a contiguous 16 KB block
//   [BH*N][V/64][K/128][8 v-groups][16 c-groups][8 v][8 c],
// i.e. 8 x 8 core matrices (8 value columns x 16 bytes of channels) laid out
// channel-group-fastest.  It is the no-swizzle MN-major operand layout of the
// backward's MMAs (core matrices adjacent along the channels, 2 KB apart along
// the value columns), fetched with one bulk copy; a warp of the walk (32
// consecutive value columns) stores four full 128-byte lines per instruction.
template <int K>
__device__ __forceinline__ size_t state_chunk_off(long bhn, int V, int vg, int c8) {
  const int tile = vg >> 6, v8 = (vg >> 3) & 7, vr = vg & 7, half = c8 >> 4, cg = c8 & 15;
  return (((((size_t)bhn * (V / 64) + tile) * (K / 128) + half) * 8 + v8) * 16 + cg) * 128 + (size_t)(vr * 16);
}

template <int K, bool EPI>
__global__ void __launch_bounds__(kWalkThreads, 1)
    k_walkT(WalkArgs a, const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
            const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmP,
            const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmR,
            const __grid_constant__ CUtensorMap tmYo) {
  using L = WalkTSmem<K, EPI>;
  constexpr int BV = kWalkBV;
  constexpr int KH = K / 2;  // key channels per state thread
  constexpr int NX = L::NX, NY = L::NY;
  constexpr int kStateWarps = 8;
  constexpr int kTmemCols = 512;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(smem + L::kBar);
  uint64_t *xfull = bars;             // [NX]
  uint64_t *xempty = xfull + NX;      // [NX]
  uint64_t *yfull = xempty + NX;      // [NY]
  uint64_t *yempty = yfull + NY;      // [NY]  MMA commit + one arrival per state warp + warp 10
  uint64_t *dsfull = yempty + NY;     // [2]
  uint64_t *dsempty = dsfull + 2;     // [2]   one arrival per state warp
  uint64_t *afull = dsempty + 2;      // [1]   one arrival per state warp
  uint64_t *ofull = afull + 1;        // [2]
  uint64_t *oempty = ofull + 2;       // [2]   one arrival per state warp
  uint64_t *done = oempty + 2;        // [1]   the MMA thread's last commit
  uint64_t *rfull = done + 1;         // [2]   EPI: gate tile r of the chunk (one per epilogue warp)
  uint64_t *rempty = rfull + 2;       // [2]   (unused)
  uint64_t *xchf = rempty + 2;        // [4]   EPI: row statistics of a chunk from every CTA of the cluster
  uint64_t *ostaged = xchf + 4;       // [2]   EPI: one arrival per state warp (the chunk's output tile is staged)
  uint64_t *ofree = ostaged + 2;      // [2]   EPI: the epilogue warp is done with the staging tile
  uint32_t *tslot = (uint32_t *)(ofree + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vt = blockIdx.x, seg = blockIdx.y + a.seg0;
  const long bh = blockIdx.z;
  const int v0 = vt * BV;
  const int n_begin = seg * a.L;
  const int n_end = min(a.N, n_begin + a.L);
  const int nloc = max(0, n_end - n_begin);
  const int P = a.P;
  const bool out = a.do_out != 0;
  // dS buffers: two when the columns allow (every state-only walk; K = 128 with outputs)
  const int nds = (!out || 2 * K + K / 2 + 128 <= kTmemCols) ? 2 : 1;
  const uint32_t colA = (uint32_t)(nds * K);               // S^T (bf16) as the output MMA's A operand
  auto colO = [&](int b) { return colA + (uint32_t)(K / 2 + 64 * b); };  // O^T accumulators (64 columns each)

  if (tid == 0) {
    for (int i = 0; i < NX; ++i) {
      dev::mbar_init(&xfull[i], 1);
      dev::mbar_init(&xempty[i], 1);
    }
    for (int i = 0; i < NY; ++i) {
      dev::mbar_init(&yfull[i], 1);
      dev::mbar_init(&yempty[i], 1 + kStateWarps + (EPI ? 0 : 1));  // MMA commit, state warps, warp 10
    }
    for (int i = 0; i < 2; ++i) {
      dev::mbar_init(&dsfull[i], 1);
      dev::mbar_init(&dsempty[i], kStateWarps);
      dev::mbar_init(&ofull[i], 1);
      dev::mbar_init(&oempty[i], kStateWarps);
    }
    dev::mbar_init(afull, kStateWarps);
    dev::mbar_init(done, 1);
    if (EPI) {
      for (int i = 0; i < 2; ++i) {
        dev::mbar_init(&rfull[i], 1);
        dev::mbar_init(&ostaged[i], kStateWarps);
        dev::mbar_init(&ofree[i], 1);
      }
      for (int i = 0; i < 4; ++i) dev::mbar_init(&xchf[i], gridDim.x);  // the cluster spans grid x
      {
      }
    }
    dev::fence_mbar_init();
    dev::prefetch_tmap(&tmX);
    dev::prefetch_tmap(&tmY);
    if (out) {
      dev::prefetch_tmap(&tmQ);
      dev::prefetch_tmap(&tmP);
      dev::prefetch_tmap(&tmO);
    }
    if (EPI) {
      dev::prefetch_tmap(&tmR);
      dev::prefetch_tmap(&tmYo);
    }
  }
  dev::pdl_launch_dependents();
  dev::pdl_wait();
  if (warp == 0) dev::tmem_alloc(tslot, kTmemCols);
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  // EPI: the other CTAs of the cluster write into this CTA's shared memory; its
  // barriers are initialised before any of them may start
  if (EPI) dev::cluster_sync();
  const uint32_t tmem = *tslot;

  auto chunk_of = [&](int i) { return a.reverse ? (n_end - 1 - i) : (n_begin + i); };
  auto xslot = [&](int s) { return smem + s * L::kXSlot; };
  auto yslot = [&](int s) { return smem + L::kY0 + s * L::kYSlot; };

  if (warp >= kStateWarps) {
    dev::regs_dec<EPI ? kWalkRegsRoleEpi : kWalkRegsRole>();
    if (warp == kStateWarps) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      bool ok = true;
      int xi = 0, yi = 0;  // loads issued into each ring
      auto load_x = [&](const CUtensorMap *map, int n) {
        const int s = xi % NX;
        if (xi >= NX && ok) ok = dev::mbar_wait(&xempty[s], (uint32_t)(((xi / NX) - 1) & 1), a.status);
        if (!ok) return;
        dev::mbar_arrive_expect_tx(&xfull[s], (uint32_t)L::kXSlot);
#pragma unroll
        for (int cb = 0; cb < K / 64; ++cb)
          dev::tma_load_3d(xslot(s) + cb * 8192, map, cb * 64, n * kC, (int)bh, &xfull[s]);
        ++xi;
      };
      for (int i = 0; i < nloc && ok; ++i) {
        const int n = chunk_of(i);
        load_x(&tmX, n);
        const int sy = i % NY;
        if (i >= NY && ok) ok = dev::mbar_wait(&yempty[sy], (uint32_t)(((i / NY) - 1) & 1), a.status);
        if (ok) {
          ++yi;
          uint8_t *y = yslot(sy);
          dev::mbar_arrive_expect_tx(&yfull[sy], (uint32_t)(L::kYTile + (out ? L::kPTile : 0) + K * 4));
#pragma unroll
          for (int cb = 0; cb < BV / 64; ++cb)
            dev::tma_load_3d(y + cb * 8192, &tmY, v0 + cb * 64, n * kC, (int)bh, &yfull[sy]);
          if (out) dev::tma_load_3d(y + L::kYTile, &tmP, 0, 0, (int)(bh * a.N + n), &yfull[sy]);
          dev::bulk_load(y + L::kYTile + L::kPTile, a.gam + (bh * a.N + n) * K, (uint32_t)(K * 4), &yfull[sy]);
        }
        if (out) load_x(&tmQ, n);
      }
      // every load issued has landed before the CTA may end (the consumers normally
      // waited for them already; after a timeout nobody else does)
      for (int j = max(0, xi - NX); j < xi; ++j) (void)dev::mbar_wait(&xfull[j % NX], (uint32_t)((j / NX) & 1), a.status);
      for (int j = max(0, yi - NY); j < yi; ++j)
        (void)dev::mbar_wait(&yfull[j % NY], (uint32_t)((j / NY) & 1), a.status);
    }
    } else if (EPI && warp >= kStateWarps + 2) {
      // ============================ epilogue warps (EPI) ============================
      // Warp 10 + ew takes the chunks i with i % 2 == ew (staging buffer and gate
      // buffer ew); lane l the token rows l and l + 32 of the chunk's 128-column
      // output tile.  Per chunk: store the staged output, each row's mean and
      // squared deviations over the tile to every CTA of the cluster, their
      // combination over the d_v columns, y in place of o and its store.
      const int ew = warp - (kStateWarps + 2);
      float *sW = reinterpret_cast<float *>(smem + L::kWB);
      float *sB = sW + BV;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = 32 * ew + lane + 64 * u;
        sW[c] = a.ln_w ? __ldg(a.ln_w + v0 + c) : 1.f;
        sB[c] = a.ln_b ? __ldg(a.ln_b + v0 + c) : 0.f;
      }
      asm volatile("bar.sync 1, 64;" ::: "memory");  // both epilogue warps
      const uint32_t my_rank = dev::cluster_ctarank();
      const int ncta = (int)gridDim.x;
      const float inv_n = 1.f / (float)(BV * ncta);
      const dev::f2 half2 = dev::pk(0.5f, 0.5f);
      bool ok = true;
      uint8_t *stg = smem + L::kOst + ew * L::kOstBuf;
      uint8_t *rt = smem + L::kR0 + ew * L::kRTile;
      auto load_r = [&](int i) {
        dev::mbar_arrive_expect_tx(&rfull[ew], (uint32_t)L::kRTile);
#pragma unroll
        for (int cb = 0; cb < BV / 64; ++cb)
          dev::tma_load_3d(rt + cb * 8192, &tmR, v0 + cb * 64, chunk_of(i) * kC, (int)bh, &rfull[ew]);
      };
      if (lane == 0 && ew < nloc) load_r(ew);
      int last_r = ew;  // the last chunk whose gate tile this warp loaded
      // 16-byte unit j of block q of row 32 hr + lane (64-byte rows, 64-byte swizzle)
      auto oaddr = [&](int hr, int q, int j) {
        return dev::smem_u32(stg) + (uint32_t)((4 * hr + q) * 2048 + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4));
      };
      auto lds16 = [&](uint32_t addr) {
        uint4 u;
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(addr));
        return u;
      };
      for (int i = ew; i < nloc; i += 2) {
        const uint32_t par = (uint32_t)((i >> 1) & 1);
        if (ok) ok = dev::mbar_wait(&ostaged[ew], par, a.status);
        // the output tile: eight [32 t][32 v] blocks
        if (lane == 0 && ok) {
#pragma unroll
          for (int hr = 0; hr < 2; ++hr)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dev::tma_store_3d(&tmO, stg + (4 * hr + q) * 2048, v0 + 32 * q, chunk_of(i) * kC + 32 * hr, (int)bh);
          dev::tma_store_commit();
        }
        // row statistics in one pass, shifted by the row's first value: sums of
        // d = o - s and d^2 over the tile's 128 columns (both rows side by side, two
        // accumulators each, a block's eight 16-byte loads issued together)
        float mean[2], m2[2];
        {
          dev::f2 sh[2], sd[2][2], sq[2][2];
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const uint4 u = lds16(oaddr(hr, 0, 0));
            const float s0 = __uint_as_float(u.x << 16);
            sh[hr] = dev::pk(-s0, -s0);
            sd[hr][0] = sd[hr][1] = sq[hr][0] = sq[hr][1] = dev::pk(0.f, 0.f);
          }
#pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            uint4 u[2][4];
#pragma unroll
            for (int hr = 0; hr < 2; ++hr)
#pragma unroll
              for (int j = 0; j < 4; ++j) u[hr][j] = lds16(oaddr(hr, q, j));
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int hr = 0; hr < 2; ++hr) {
                const uint32_t w4[4] = {u[hr][j].x, u[hr][j].y, u[hr][j].z, u[hr][j].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const dev::f2 d = dev::add2(dev::bf16pair(w4[e]), sh[hr]);
                  sd[hr][e & 1] = dev::add2(sd[hr][e & 1], d);
                  sq[hr][e & 1] = dev::fma2(d, d, sq[hr][e & 1]);
                }
              }
          }
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            float s0, s1;
            dev::upk(sh[hr], s0, s1);
            const float sdv = dev::hsum(dev::add2(sd[hr][0], sd[hr][1]));
            mean[hr] = sdv * (1.f / (float)BV) - s0;
            m2[hr] = fmaxf(dev::hsum(dev::add2(sq[hr][0], sq[hr][1])) - sdv * sdv * (1.f / (float)BV), 0.f);
          }
        }
        // to slots [rank][t] of buffer i % 4 of every CTA, then one arrival per CTA
        const int xb4 = i & 3;
        const uint32_t slot = dev::smem_u32(smem + L::kXch + xb4 * L::kXchBuf) + (uint32_t)(((int)my_rank * 64 + lane) * 8);
        if (ok)
          for (int r = 0; r < ncta; ++r) {
            const uint32_t rs = dev::mapa(slot, (uint32_t)r);
            dev::st_cluster_f2(rs, mean[0], m2[0]);
            dev::st_cluster_f2(rs + 32 * 8, mean[1], m2[1]);
          }
        dev::fence_acq_rel_cluster();
        __syncwarp();
        if (lane < ncta && ok) dev::mbar_arrive_remote(dev::mapa(dev::smem_u32(&xchf[xb4]), (uint32_t)lane));
        if (ok) ok = dev::mbar_wait_cluster(&xchf[xb4], (uint32_t)((i >> 2) & 1), a.status);
        // Chan's combination of the ncta partials of BV columns each, per row
        dev::f2 nmu2[2], rs2[2];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const float2 *xb = reinterpret_cast<const float2 *>(smem + L::kXch + xb4 * L::kXchBuf) + 32 * hr + lane;
          float mu = 0.f;
          for (int r = 0; r < ncta; ++r) mu += xb[r * 64].x;
          mu *= 1.f / (float)ncta;
          float M2 = 0.f;
          for (int r = 0; r < ncta; ++r) {
            const float2 pr = xb[r * 64];
            const float d = pr.x - mu;
            M2 += fmaf((float)BV * d, d, pr.y);
          }
          const float rstd = rsqrtf(M2 * inv_n + a.eps);
          nmu2[hr] = dev::pk(-mu, -mu);
          rs2[hr] = dev::pk(rstd, rstd);
        }
        // y over o in the staging tile, once the output's stores have read it
        if (lane == 0) dev::tma_store_wait_read();
        __syncwarp();
        if (ok) ok = dev::mbar_wait(&rfull[ew], par, a.status);
        // columns 8 c16 .. 8 c16 + 7 of the tile per step; the next step's o and r
        // are loaded before this step's results are stored
        auto raddr = [&](int hr, int c16) {
          const int t = 32 * hr + lane;
          return dev::smem_u32(rt) + (uint32_t)((c16 >> 3) * 8192 + t * 128 + (((c16 & 7) ^ (t & 7)) << 4));
        };
        uint4 ou[2], ru[2];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          ou[hr] = lds16(oaddr(hr, 0, 0));
          ru[hr] = lds16(raddr(hr, 0));
        }
#pragma unroll 1
        for (int c16 = 0; c16 < 16; ++c16) {
          uint4 on[2], rn[2];
          const int cn = c16 < 15 ? c16 + 1 : c16;
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            on[hr] = lds16(oaddr(hr, cn >> 2, cn & 3));
            rn[hr] = lds16(raddr(hr, cn));
          }
          dev::f2 w2[4], b2[4];
          {
            const ulonglong2 w01 = *reinterpret_cast<const ulonglong2 *>(sW + 8 * c16);
            const ulonglong2 w23 = *reinterpret_cast<const ulonglong2 *>(sW + 8 * c16 + 4);
            const ulonglong2 b01 = *reinterpret_cast<const ulonglong2 *>(sB + 8 * c16);
            const ulonglong2 b23 = *reinterpret_cast<const ulonglong2 *>(sB + 8 * c16 + 4);
            w2[0] = w01.x, w2[1] = w01.y, w2[2] = w23.x, w2[3] = w23.y;
            b2[0] = b01.x, b2[1] = b01.y, b2[2] = b23.x, b2[3] = b23.y;
          }
          uint32_t pkd[2][4];
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const uint32_t xo[4] = {ou[hr].x, ou[hr].y, ou[hr].z, ou[hr].w};
            const uint32_t xr[4] = {ru[hr].x, ru[hr].y, ru[hr].z, ru[hr].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const dev::f2 nrm =
                  dev::fma2(dev::mul2(dev::add2(dev::bf16pair(xo[e]), nmu2[hr]), rs2[hr]), w2[e], b2[e]);
              const dev::f2 h = dev::mul2(dev::bf16pair(xr[e]), half2);
              float hl, hh2;
              dev::upk(h, hl, hh2);
              const dev::f2 g = dev::fma2(h, dev::pk(dev::tanh_approx(hl), dev::tanh_approx(hh2)), h);  // r sigmoid(r)
              float y0, y1;
              dev::upk(dev::mul2(nrm, g), y0, y1);
              pkd[hr][e] = dev::pack_bf16(y0, y1);
            }
          }
#pragma unroll
          for (int hr = 0; hr < 2; ++hr)
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(oaddr(hr, c16 >> 2, c16 & 3)), "r"(pkd[hr][0]),
                         "r"(pkd[hr][1]), "r"(pkd[hr][2]), "r"(pkd[hr][3])
                         : "memory");
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            ou[hr] = on[hr];
            ru[hr] = rn[hr];
          }
        }
        dev::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (ok) {
#pragma unroll
            for (int hr = 0; hr < 2; ++hr)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dev::tma_store_3d(&tmYo, stg + (4 * hr + q) * 2048, v0 + 32 * q, chunk_of(i) * kC + 32 * hr, (int)bh);
            dev::tma_store_commit();
          }
          // the next gate tile of this warp (every lane has read this one)
          if (i + 2 < nloc && ok) {
            load_r(i + 2);
            last_r = i + 2;
          }
          dev::tma_store_wait_read();  // the tile goes back to the state warps
          dev::mbar_arrive(&ofree[ew]);
        }
      }
      if (lane == 0) {
        dev::tma_store_wait_all();
        // the last gate tile load of this warp has landed before the CTA may end
        if (last_r < nloc) (void)dev::mbar_wait(&rfull[ew], (uint32_t)((last_r >> 1) & 1), a.status);
      }
    } else if (warp == kStateWarps + 2) {
      // the product of the segment's chunk decays per key channel (lane: channels
      // lane + 32 j), from the decay rows the producer stages with each chunk
      const bool want = a.gseg && vt == 0;
      float gp[K / 32];
#pragma unroll
      for (int j = 0; j < K / 32; ++j) gp[j] = 1.f;
      bool ok = true;
      for (int i = 0; i < nloc; ++i) {
        const int sy = i % NY;
        if (ok) ok = dev::mbar_wait(&yfull[sy], (uint32_t)((i / NY) & 1), a.status);
        if (want) {
          const float *g = reinterpret_cast<const float *>(yslot(sy) + L::kYTile + L::kPTile);
#pragma unroll
          for (int j = 0; j < K / 32; ++j) gp[j] *= g[lane + 32 * j];
        }
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&yempty[sy]);
      }
      if (want && ok) {
#pragma unroll
        for (int j = 0; j < K / 32; ++j) a.gseg[(bh * P + seg) * K + lane + 32 * j] = gp[j];
      }
    } else if (warp == kStateWarps + 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      bool ok = true;
      int xi = 0;
      constexpr uint32_t id_ds = dev::idesc_bf16(128, K, true, true);   // A = Y^T (MN), B = X (MN)
      constexpr uint32_t id_o = dev::idesc_bf16(128, 64, false, false);  // A = S^T (TMEM), B = Q (K-major)
      const uint32_t id_pv = a.p_kmajor ? dev::idesc_bf16(128, 64, true, false)  // B = P   (reverse)
                                        : dev::idesc_bf16(128, 64, true, true);  // B = P^T (forward)
      for (int i = 0; i < nloc && ok; ++i) {
        const int sx = xi % NX, sy = i % NY, d = i % nds;
        ok = dev::mbar_wait(&xfull[sx], (uint32_t)((xi / NX) & 1), a.status) &&
             dev::mbar_wait(&yfull[sy], (uint32_t)((i / NY) & 1), a.status);
        if (ok && i >= nds) ok = dev::mbar_wait(&dsempty[d], (uint32_t)(((i / nds) - 1) & 1), a.status);
        if (!ok) break;
        dev::tc_fence_after();
        const uint32_t sX = dev::smem_u32(xslot(sx)), sY = dev::smem_u32(yslot(sy));
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          dev::umma_bf16(tmem + (uint32_t)(d * K), dev::desc_mnmajor(sY, 64, kk * 16, 0),
                         dev::desc_mnmajor(sX, 64, kk * 16, 0), id_ds, kk > 0 ? 1u : 0u);
        dev::umma_commit(&dsfull[d]);
        dev::umma_commit(&xempty[sx]);
        ++xi;
        if (out) {
          const int sq = xi % NX;
          ok = dev::mbar_wait(&xfull[sq], (uint32_t)((xi / NX) & 1), a.status) &&
               dev::mbar_wait(afull, (uint32_t)(i & 1), a.status);
          if (ok && i >= 2) ok = dev::mbar_wait(&oempty[i & 1], (uint32_t)(((i >> 1) - 1) & 1), a.status);
          if (!ok) break;
          dev::tc_fence_after();
          const uint32_t sQ = dev::smem_u32(xslot(sq)), sP = sY + L::kYTile;
          const uint32_t tO = tmem + colO(i & 1);
#pragma unroll
          for (int kk = 0; kk < K / 16; ++kk)
            dev::umma_bf16_ts(tO, tmem + colA + (uint32_t)(kk * 8), dev::desc_kmajor(sQ, 64, 0, kk * 16), id_o,
                              kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kC / 16; ++kk)
            dev::umma_bf16(tO, dev::desc_mnmajor(sY, 64, kk * 16, 0),
                           a.p_kmajor ? dev::desc_kmajor(sP, 64, 0, kk * 16) : dev::desc_mnmajor(sP, 64, kk * 16, 0),
                           id_pv, 1u);
          dev::umma_commit(&ofull[i & 1]);
          dev::umma_commit(&xempty[sq]);
          ++xi;
        }
        dev::umma_commit(&yempty[sy]);
      }
      // all MMAs of this thread have completed before TMEM is released
      dev::umma_commit(done);
      (void)dev::mbar_wait(done, 0, a.status);
    }
    }
  } else {
    dev::regs_inc<EPI ? kWalkRegsStateEpi : kWalkRegsState>();
    // ============================ state threads ============================
    const int q4 = warp & 3, hh = warp >> 2;
    const int v = 32 * q4 + lane;  // TMEM lane = row of S^T
    const int c0 = hh * KH;
    const int vg = v0 + v;
    const bool vok = vg < a.V;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    const long KV = (long)K * a.V;
    float S[KH];

    // ---- start state: h0 for the first segment (the last, reverse), else the
    // segment's start state ([K/4][V] float4 groups of four channels: a warp reads
    // 512 contiguous bytes per group) or a materialised [K][V] chunk state
    {
      const bool first = seg == (a.reverse ? P - 1 : 0);
      if (a.start_v && !first) {
        const float4 *src = reinterpret_cast<const float4 *>(a.start_v) + ((bh * P + seg) * (K / 4) + c0 / 4) * a.V + vg;
#pragma unroll
        for (int j4 = 0; j4 < KH / 4; ++j4) {
          const float4 x = vok ? __ldg(src + (long)j4 * a.V) : make_float4(0.f, 0.f, 0.f, 0.f);
          S[4 * j4] = x.x;
          S[4 * j4 + 1] = x.y;
          S[4 * j4 + 2] = x.z;
          S[4 * j4 + 3] = x.w;
        }
      } else {
        const float *src = nullptr;
        if (a.start) src = a.start + (bh * P + seg) * KV;
        else if (a.h0 && first) src = a.h0 + bh * KV;
#pragma unroll
        for (int j = 0; j < KH; ++j) S[j] = (src && vok) ? __ldg(src + (long)(c0 + j) * a.V + vg) : 0.f;
      }
    }

    bool ok = true;
    // O_i^T (TMEM, lanes v, columns tokens) -> out[t][v]: this warp's [32 t][32 v]
    // block (tokens 32 hh .., columns 32 q4 ..) goes through a shared-memory tile to
    // one TMA store (the store clips rows beyond T and columns beyond V)
    uint8_t *ost = smem + L::kOst + warp * 2048;
    auto epilogue = [&](int i) {
      float o[32];
      dev::tmem_ld32(lane_base + colO(i & 1) + (uint32_t)(32 * hh), o);
      dev::tmem_wait_ld();
      dev::tc_fence_before();
      __syncwarp();
      if (EPI) {
        // the tile of chunk i - 2 went through the epilogue warps and its stores
        if (lane == 0) dev::mbar_arrive(&oempty[i & 1]);
        if (i >= 2 && ok) ok = dev::mbar_wait(&ofree[i & 1], (uint32_t)(((i >> 1) - 1) & 1), a.status);
        // block (q4, hh) of the chunk's staging tile, 64-byte rows with the 64-byte
        // swizzle (16-byte unit j of row e at unit j ^ ((e >> 1) & 3))
        const uint32_t blk = dev::smem_u32(smem + L::kOst + (i & 1) * L::kOstBuf) + (uint32_t)(warp * 2048);
        const uint32_t cb = (uint32_t)(lane * 2);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const bf16 b = __float2bfloat16_rn(o[e]);
          const uint32_t off = (uint32_t)(e * 64) + ((((cb >> 4) ^ (uint32_t)((e >> 1) & 3))) << 4) + (cb & 15u);
          dev::st_shared_u16(blk + off, *reinterpret_cast<const uint16_t *>(&b));
        }
        dev::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&ostaged[i & 1]);
        return;
      }
      if (lane == 0) {
        dev::mbar_arrive(&oempty[i & 1]);
        dev::tma_store_wait_read();  // this warp's previous store has read the tile
      }
      __syncwarp();
      const uint32_t so = dev::smem_u32(ost) + (uint32_t)(lane * 2);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const bf16 b = __float2bfloat16_rn(o[e]);
        dev::st_shared_u16(so + (uint32_t)(e * 64), *reinterpret_cast<const uint16_t *>(&b));
      }
      dev::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && ok) {
        dev::tma_store_3d(&tmO, ost, v0 + 32 * q4, chunk_of(i) * kC + 32 * hh, (int)bh);
        dev::tma_store_commit();
      }
    };
    // bf16 chunk state of this thread's row -> the backward's layout (4 x 16 bytes per 32 channels)
    uint8_t *hb = reinterpret_cast<uint8_t *>(a.hb);
    auto store_hb = [&](int n, int jb, const uint32_t *w) {
      const long bhn = bh * a.N + n;
#pragma unroll
      for (int x = 0; x < 4; ++x)
        *reinterpret_cast<uint4 *>(hb + state_chunk_off<K>(bhn, a.V, vg, c0 / 8 + 4 * jb + x)) =
            make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
    };
    const bool st_hb = a.state_mode == 1 && vok;

    for (int i = 0; i < nloc; ++i) {
      const int n = chunk_of(i);
      // ---- publish S_{i-1} as the A operand of O_i (the MMA warp waits on afull) ----
      if (out) {
        if (i >= 1) {
          if (ok) ok = dev::mbar_wait(&ofull[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1), a.status);
          dev::tc_fence_after();
        }
        uint32_t w[KH / 2];  // the bf16 row, kept for the chunk-state stores
#pragma unroll
        for (int jb = 0; jb < KH / 32; ++jb) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[16 * jb + e] = dev::pack_bf16(S[32 * jb + 2 * e], S[32 * jb + 2 * e + 1]);
          dev::tmem_st16u(lane_base + colA + (uint32_t)(c0 / 2 + 16 * jb), w + 16 * jb);
        }
        dev::tmem_wait_st();
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(afull);
        // S_{i-1} to the backward's layout from the same registers, after the MMA warp
        // has been released
        if (st_hb && ok) {
#pragma unroll
          for (int jb = 0; jb < KH / 32; ++jb) store_hb(n, jb, w + 16 * jb);
        }
      } else if (st_hb && ok) {
#pragma unroll
        for (int jb = 0; jb < KH / 32; ++jb) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = dev::pack_bf16(S[32 * jb + 2 * e], S[32 * jb + 2 * e + 1]);
          store_hb(n, jb, w);
        }
      }
      if (a.state_mode == 2 && vok && ok) {
        float *dst = a.h32 + (bh * a.N + n) * KV + vg;
#pragma unroll
        for (int j = 0; j < KH; ++j) dst[(long)(c0 + j) * a.V] = S[j];
      }
      // ---- S_i = gam_i (.) S_{i-1} + dS_i ----------------------------------------
      const int sy = i % NY, d = i % nds;
      if (ok) ok = dev::mbar_wait(&yfull[sy], (uint32_t)((i / NY) & 1), a.status);
      if (ok) ok = dev::mbar_wait(&dsfull[d], (uint32_t)((i / nds) & 1), a.status);
      dev::tc_fence_after();
      const float *g = reinterpret_cast<const float *>(yslot(sy) + L::kYTile + L::kPTile) + c0;
      // 64 columns of dS per TMEM round trip (two loads, one wait)
#pragma unroll
      for (int j = 0; j < KH / 64; ++j) {
        float dsv[64];
        dev::tmem_ld32(lane_base + (uint32_t)(d * K + c0 + 64 * j), dsv);
        dev::tmem_ld32(lane_base + (uint32_t)(d * K + c0 + 64 * j + 32), dsv + 32);
        dev::tmem_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 16; ++e4) {
          const float4 g4 = *reinterpret_cast<const float4 *>(g + 64 * j + 4 * e4);
          S[64 * j + 4 * e4 + 0] = g4.x * S[64 * j + 4 * e4 + 0] + dsv[4 * e4 + 0];
          S[64 * j + 4 * e4 + 1] = g4.y * S[64 * j + 4 * e4 + 1] + dsv[4 * e4 + 1];
          S[64 * j + 4 * e4 + 2] = g4.z * S[64 * j + 4 * e4 + 2] + dsv[4 * e4 + 2];
          S[64 * j + 4 * e4 + 3] = g4.w * S[64 * j + 4 * e4 + 3] + dsv[4 * e4 + 3];
        }
      }
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        dev::mbar_arrive(&dsempty[d]);
        dev::mbar_arrive(&yempty[sy]);
      }
      // ---- off the chain: S_{i-1} (still the A operand in TMEM) to the backward's
      // layout, then the previous chunk's output -------------------------------------
      if (out && i >= 1) epilogue(i - 1);
    }
    if (out && nloc > 0) {
      if (ok) ok = dev::mbar_wait(&ofull[(nloc - 1) & 1], (uint32_t)(((nloc - 1) >> 1) & 1), a.status);
      dev::tc_fence_after();
      epilogue(nloc - 1);
    }

    // ---- state after the segment ----------------------------------------------
    if (a.end && a.end_seg < 0 && vok && ok) {
      // segment contribution, [BH][P][K/4][V] float4 groups (a warp stores 512
      // contiguous bytes per group of four channels)
      float4 *dst = reinterpret_cast<float4 *>(a.end) + ((bh * P + seg) * (K / 4) + c0 / 4) * a.V + vg;
#pragma unroll
      for (int j4 = 0; j4 < KH / 4; ++j4)
        dst[(long)j4 * a.V] = make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
    }
    if (a.end && a.end_seg == seg && vok && ok) {
      // the walk's final state, [BH][K][V] (a warp stores 128 contiguous bytes per channel)
      float *dst = a.end + bh * KV + vg;
#pragma unroll
      for (int j = 0; j < KH; ++j) dst[(long)(c0 + j) * a.V] = S[j];
    }
  }

  if (warp < kStateWarps && lane == 0) dev::tma_store_wait_all();  // output stores complete
  dev::tc_fence_before();
  __syncthreads();
  // EPI: no CTA leaves while another may still read its statistics or write its buffers
  if (EPI) dev::cluster_sync();
  if (warp == 0) dev::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc
}  // namespace gla
