// tc_path.cu -- host orchestration of the bf16 tensor-core path (sm_100a).
//
// Forward (section 4.2 chunkwise form, section 3.3 Figure 1 variants):
//   prep                      qg, kg, gam, P^T per chunk (parallel over chunks)
//   FUSED, P segments:        walk(no output) over segments 0..P-2 from 0 -> delta_p,
//                             the fold of h0 and the delta_p into every segment's
//                             start state, walk(output) per segment from its start;
//                             the last segment writes h_final (P = 1: one walk from h0)
//   MATERIALIZED:             walk(fp32 chunk states) over whole sequences, then
//                             walk(output, one chunk per CTA) from those states.
// Backward: chunk states h_n (saved by the forward, or a forward walk), a reverse
// walk for the adjoints dh_n that also writes dv, then the per-chunk kernel (tc_bwd).
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "tc_bwd.cuh"
#include "tc_kernels.cuh"
#include "tc_path.h"
#include "tc_walk.cuh"

namespace gla {
namespace {

using tc::bf16;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  });
  return fn;
}

// 3-D bf16 tensor map: dims (d0 innermost, d1, d2), box (b0, b1, 1), 128-byte swizzle.
bool map3(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same without swizzle (row-major staging tiles, e.g. the walk's output blocks).
bool map3_plain(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same with the 64-byte swizzle (the fused epilogue's staging tiles: [32][32]
// boxes, 64-byte rows).
bool map3_sw64(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc::map3_bf16(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1) {
  return map3(m, base, d0, d1, d2, b0, b1);
}

bool tc::map3_store(CUtensorMap *m, const void *base, bool fp32, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                    uint32_t b1) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = fp32 ? 4 : 2;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// 1 if the current device is sm_100 (per device: 1 = yes, 2 = no).
int device_ok() {
  static DeviceSlots slots;
  return per_device(slots, [] {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return 2;
    return major == 10 ? 1 : 2;
  });
}

int sm_count() {
  static DeviceSlots slots;
  return per_device(slots, [] {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
  });
}

// d_v tiles of a walk (128 columns each; a last tile of 64 columns is padded by
// the TMA loads' zero fill and masked on store)
int walk_tiles(const Problem &p) { return (p.V + tc::kWalkBV - 1) / tc::kWalkBV; }

// Segment count for the FUSED forward: as many segments as one wave of walk
// CTAs (one per SM) can hold.
int segments_of(const Problem &p, int nvt) {
  if (p.variant == GLA_VARIANT_MATERIALIZED) return 1;
  int P = p.segments;
  if (P <= 0) {
    const long ctas = p.BH * nvt;
    P = (int)std::max<long>(1, (long)sm_count() / ctas);
  }
  P = std::min(P, p.N);
  const int L = (p.N + P - 1) / P;
  return (p.N + L - 1) / L;
}

struct TcWs {
  bf16 *qg, *kg, *PT;
  float *gam;
  float *delta;          // [BH][P][K/4][V][4] segment contributions from a zero state
  float *gseg;           // [BH][P][K] per-segment gate products
  float *starts;         // [BH][P][K/4][V][4] segment start states (folded from h0 and the contributions)
  float *h32;            // materialised fp32 chunk states [BH][N][K][V]
  // backward
  bf16 *hb, *dhb;        // bf16 chunk states and adjoints, tc::state_chunk_off layout
  float *ddelta;
  size_t bytes;
};

// Segment count of the backward walks (and of a forward that saves states):
// the FUSED choice for this descriptor whatever its forward variant.
int bwd_segments(const Problem &p, int nvt) {
  Problem pf = p;
  pf.variant = GLA_VARIANT_FUSED;
  return segments_of(pf, nvt);
}

// Workspace layout.  The forward layout is a prefix of the backward one up to
// gam; the backward layout (also used by a forward with GLA_FLAG_SAVE_STATES)
// keeps every offset independent of the forward variant: the MATERIALIZED
// fp32 states come last.
TcWs carve(const Problem &p, void *ws, bool bwd) {
  Carve cv(ws);
  TcWs w{};
  const int nvt = walk_tiles(p);
  w.qg = cv.take<bf16>((size_t)p.BH * p.Tp * p.K);
  w.kg = cv.take<bf16>((size_t)p.BH * p.Tp * p.K);
  w.PT = cv.take<bf16>((size_t)p.BH * p.N * tc::kC * tc::kC);
  w.gam = cv.take<float>((size_t)p.BH * p.N * p.K);
  if (!bwd) {
    const int P = segments_of(p, nvt);
    if (p.variant == GLA_VARIANT_MATERIALIZED) {
      w.h32 = cv.take<float>((size_t)p.BH * p.N * p.K * p.V);
    } else if (P > 1) {
      w.delta = cv.take<float>((size_t)p.BH * P * p.K * p.V);
      w.gseg = cv.take<float>((size_t)p.BH * P * p.K);
      w.starts = cv.take<float>((size_t)p.BH * P * p.K * p.V);
    }
  } else {
    const int P = bwd_segments(p, nvt);
    w.delta = cv.take<float>((size_t)p.BH * P * p.K * p.V);
    w.ddelta = cv.take<float>((size_t)p.BH * P * p.K * p.V);
    w.gseg = cv.take<float>((size_t)p.BH * P * p.K);
    w.starts = cv.take<float>((size_t)p.BH * P * p.K * p.V);
    w.hb = cv.take<bf16>((size_t)p.BH * p.N * p.K * p.V);
    w.dhb = cv.take<bf16>((size_t)p.BH * p.N * p.K * p.V);
    if (p.variant == GLA_VARIANT_MATERIALIZED && (p.flags & GLA_FLAG_SAVE_STATES))
      w.h32 = cv.take<float>((size_t)p.BH * p.N * p.K * p.V);
  }
  w.bytes = cv.bytes();
  return w;
}

template <int K>
int launch_prep(const Problem &p, const bf16 *q, const bf16 *k, const float *la, const TcWs &w, unsigned *status,
                cudaStream_t st) {
  tc::PrepArgs a{p.T, p.N, p.gate, p.Tp, la, w.qg, w.kg, w.PT, w.gam, status};
  CUtensorMap mq, mk, mqg, mkg;
  if (!map3(&mq, q, p.K, p.T, (uint64_t)p.BH, 64, 64) || !map3(&mk, k, p.K, p.T, (uint64_t)p.BH, 64, 64) ||
      !map3(&mqg, w.qg, p.K, p.Tp, (uint64_t)p.BH, 64, 64) || !map3(&mkg, w.kg, p.K, p.Tp, (uint64_t)p.BH, 64, 64))
    return GLA_ERR_CUDA;
  static DeviceSlots slots;
  const int smem = per_device(slots, [] {
    if (cudaFuncSetAttribute(tc::k_prep<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem) != cudaSuccess)
      return -1;
    return smem_for_tmem(tc::k_prep<K>, 256, tc::PrepSmem<K>::kBytes + 1024, 64);
  });
  if (smem < 0) return GLA_ERR_CUDA;
  GLA_LAUNCH(K_TC_PREP, st,
             if (launch_pdl(tc::k_prep<K>, dim3(p.N, p.BH), dim3(256), smem, st, a, mq, mk, mqg, mkg) != cudaSuccess)
                 return GLA_ERR_CUDA);
  return GLA_OK;
}

struct WalkMaps {
  CUtensorMap X, Y, Q, P, O;  // O: the output [BH][T][V] in [32 t][32 v] boxes (output walks)
  CUtensorMap R, Yo;          // fused epilogue: gate r (as Y) and the epilogue output y (as O)
};

template <int K, bool EPI>
int walk_smem_attr() {
  constexpr int smem = tc::WalkTSmem<K, EPI>::kBytes + 1024;
  static_assert(smem <= kMaxDynSmem, "walk shared memory");
  static DeviceSlots attr;  // the attribute belongs to the current device
  if (per_device(attr, [] {
        const cudaError_t e =
            cudaFuncSetAttribute(tc::k_walkT<K, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) note_cuda_error(e);
        return e == cudaSuccess ? 1 : -1;
      }) < 0)
    return -1;
  return smem;
}

// P here is the number of segments this launch covers (a.seg0 .. a.seg0 + P - 1).
template <int K>
int launch_walk(const Problem &p, const tc::WalkArgs &a, const WalkMaps &m, int P, cudaStream_t st) {
  const int smem = walk_smem_attr<K, false>();
  if (smem < 0) return GLA_ERR_CUDA;
  GLA_LAUNCH(K_TC_WALK, st,
             if (launch_pdl(tc::k_walkT<K, false>, dim3(walk_tiles(p), P, p.BH), dim3(tc::kWalkThreads), smem, st, a,
                            m.X, m.Y, m.Q, m.P, m.O, m.O, m.O) != cudaSuccess) return GLA_ERR_CUDA);
  return GLA_OK;
}

// The output walk with the fused layer epilogue: clusters of the walk_tiles(p)
// CTAs of one (segment, head), which exchange row statistics through DSMEM.
template <int K>
int launch_walk_epi(const Problem &p, const tc::WalkArgs &a, const WalkMaps &m, int P, cudaStream_t st) {
  const int smem = walk_smem_attr<K, true>();
  if (smem < 0) return GLA_ERR_CUDA;
  GLA_LAUNCH(K_TC_WALK_EPI, st,
             if (launch_pdl_cluster(tc::k_walkT<K, true>, dim3(walk_tiles(p), P, p.BH), dim3(tc::kWalkThreads), smem,
                                    st, (unsigned)walk_tiles(p), a, m.X, m.Y, m.Q, m.P, m.O, m.R,
                                    m.Yo) != cudaSuccess) return GLA_ERR_CUDA);
  return GLA_OK;
}

// Clusters of `nvt` fused-epilogue walk CTAs that fit on the device at once (0 on error).
template <int K>
int epi_max_clusters(int nvt) {
  static DeviceSlots slots[4];
  if (nvt < 1 || nvt > 4) return 0;
  return per_device(slots[nvt - 1], [nvt] {
    const int smem = walk_smem_attr<K, true>();
    if (smem < 0) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nvt, 1, 1);
    cfg.blockDim = dim3(tc::kWalkThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nvt;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tc::k_walkT<K, true>, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      return 0;
    }
    return n;
  });
}

int launch_walk_any(const Problem &p, const tc::WalkArgs &a, const WalkMaps &m, int P, cudaStream_t st) {
  if (P < 1 || P > 65535) return GLA_ERR_UNSUPPORTED_SHAPE;
  if (p.K == 256) return launch_walk<256>(p, a, m, P, st);
  if (p.K == 128) return launch_walk<128>(p, a, m, P, st);
  return GLA_ERR_UNSUPPORTED_SHAPE;
}

int launch_prep_any(const Problem &p, const bf16 *q, const bf16 *k, const float *la, const TcWs &w, unsigned *status,
                    cudaStream_t st) {
  if (p.K == 256) return launch_prep<256>(p, q, k, la, w, status, st);
  return launch_prep<128>(p, q, k, la, w, status, st);
}

#define TRY(x)                      \
  do {                              \
    const int _r = (x);             \
    if (_r != GLA_OK) return _r;    \
  } while (0)

}  // namespace

namespace {
// One thread waits, with the library's bounded wait, on an mbarrier that nothing
// will ever complete; the wait gives up after limit_ns and records ST_TIMEOUT.
__global__ void k_selftest_timeout(unsigned *status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  dev::mbar_init(&bar, 1);
  dev::fence_mbar_init();
  (void)dev::mbar_wait(&bar, 0, status, limit_ns);
}
}  // namespace

int selftest_timeout(unsigned *status, unsigned limit_us, cudaStream_t st) {
  k_selftest_timeout<<<1, 1, 0, st>>>(status, 1000ull * limit_us);
  return cudaGetLastError() == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

int tc_check(const Problem &p) {
  if (p.K != 128 && p.K != 256) return GLA_ERR_UNSUPPORTED_SHAPE;
  if (p.V % 64 != 0) return GLA_ERR_UNSUPPORTED_SHAPE;
  if (p.C != 64 || p.c != 16) return GLA_ERR_UNSUPPORTED_SHAPE;
  if (p.N > 65535) return GLA_ERR_UNSUPPORTED_SHAPE;  // chunk index is a grid y coordinate of the backward
  return GLA_OK;
}

size_t tc_workspace(const Problem &p, bool bwd) { return carve(p, nullptr, bwd).bytes; }

bool tc_epilogue_fusable(const Problem &p) {
  return tc_check(p) == GLA_OK && p.dtype == GLA_DTYPE_BF16 && p.V % tc::kWalkBV == 0 &&
         p.V / tc::kWalkBV <= 4 && p.variant != GLA_VARIANT_MATERIALIZED && !(p.flags & GLA_FLAG_REUSE_SEGMENTS);
}

namespace {
int tc_fwd_impl(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
                void *o, float *hT, void *ws, cudaStream_t st, const TcEpilogue *epi) {
  if (device_ok() != 1) return GLA_ERR_NO_DEVICE;
  const bool save = (p.flags & GLA_FLAG_SAVE_STATES) != 0;
  TcWs w = carve(p, ws, save);
  unsigned *status = (unsigned *)ws;
  if (!(p.flags & GLA_FLAG_REUSE_PREP)) TRY(launch_prep_any(p, (const bf16 *)q, (const bf16 *)k, la, w, status, st));

  const int nvt = walk_tiles(p);
  WalkMaps m;
  const uint64_t BH = (uint64_t)p.BH;
  bool okm = map3(&m.X, w.kg, p.K, p.Tp, BH, 64, 64) && map3(&m.Y, v, p.V, p.T, BH, 64, 64) &&
             map3(&m.Q, w.qg, p.K, p.Tp, BH, 64, 64) && map3(&m.P, w.PT, 64, 64, BH * p.N, 64, 64) &&
             map3_plain(&m.O, o, p.V, p.T, BH, 32, 32);
  if (epi)  // the fused epilogue stages o and y with the 64-byte swizzle
    okm = okm && map3(&m.R, epi->r, p.V, p.T, BH, 64, 64) && map3_sw64(&m.O, o, p.V, p.T, BH, 32, 32) &&
          map3_sw64(&m.Yo, epi->y, p.V, p.T, BH, 32, 32);
  if (!okm) return GLA_ERR_CUDA;

  tc::WalkArgs a{};
  a.T = p.T;
  a.N = p.N;
  a.V = p.V;
  a.gam = w.gam;
  a.out = (bf16 *)o;
  a.status = status;
  a.end_seg = -1;
  a.hb = save ? w.hb : nullptr;  // the output walk's bf16 chunk-entry states go to the backward's h_n

  if (p.variant == GLA_VARIANT_MATERIALIZED) {
    // pass 1: all chunk states in fp32 (sequential over chunks per (head, d_v tile))
    a.L = p.N;
    a.P = 1;
    a.state_mode = 2;
    a.h32 = w.h32;
    a.h0 = h0;
    a.end = hT;
    a.end_seg = 0;
    TRY(launch_walk_any(p, a, m, 1, st));
    // pass 2: every chunk's output in parallel from its materialised state
    tc::WalkArgs b = a;
    b.L = 1;
    b.P = p.N;
    b.state_mode = save ? 1 : 0;
    b.do_out = 1;
    b.start = w.h32;
    b.h0 = nullptr;
    b.end = nullptr;
    return launch_walk_any(p, b, m, p.N, st);
  }

  int P = save ? bwd_segments(p, nvt) : segments_of(p, nvt);
  if (epi) {
    // every cluster of the fused output walk resident at once: at most as many
    // segments per head as the device holds clusters (fewer than the workspace has room for)
    const int mc = p.K == 256 ? epi_max_clusters<256>(nvt) : epi_max_clusters<128>(nvt);
    if (mc < 1) return GLA_ERR_CUDA;
    if ((long)P * p.BH > mc) P = (int)std::max<long>(1, mc / p.BH);
    const int Lp = (p.N + P - 1) / P;
    P = (p.N + Lp - 1) / Lp;
    a.ln_w = epi->w;
    a.ln_b = epi->b;
    a.eps = epi->eps;
  }
  auto out_walk = [&](const tc::WalkArgs &wa, int nseg) {
    if (!epi) return launch_walk_any(p, wa, m, nseg, st);
    return p.K == 256 ? launch_walk_epi<256>(p, wa, m, nseg, st) : launch_walk_epi<128>(p, wa, m, nseg, st);
  };
  const int L = (p.N + P - 1) / P;
  a.L = L;
  a.P = P;
  a.do_out = 1;
  a.state_mode = save ? 1 : 0;
  a.end = hT;
  a.end_seg = P - 1;
  if (P == 1) {
    a.h0 = h0;
    return out_walk(a, 1);
  }
  // pre-pass: the contribution of segments 0 .. P-2 from a zero state (already in
  // the workspace after gla_fwd_state with GLA_FLAG_REUSE_SEGMENTS)
  if (!(p.flags & GLA_FLAG_REUSE_SEGMENTS)) {
    tc::WalkArgs pre = a;
    pre.do_out = 0;
    pre.state_mode = 0;
    pre.end = w.delta;
    pre.end_seg = -1;
    pre.gseg = w.gseg;
    TRY(launch_walk_any(p, pre, m, P - 1, st));
  }
  TRY(segment_starts(p.BH, p.K, p.V, P, 0, w.gseg, w.delta, h0, w.starts, st));
  a.start_v = w.starts;
  a.h0 = h0;
  return out_walk(a, P);
}
}  // namespace

int tc_fwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0, void *o,
           float *hT, void *ws, cudaStream_t st) {
  return tc_fwd_impl(p, q, k, v, la, h0, o, hT, ws, st, nullptr);
}

int tc_fwd_epilogue(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
                    void *o, float *hT, const TcEpilogue &epi, void *ws, cudaStream_t st) {
  if (!tc_epilogue_fusable(p)) return GLA_ERR_UNSUPPORTED_SHAPE;
  return tc_fwd_impl(p, q, k, v, la, h0, o, hT, ws, st, &epi);
}

int tc_bwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
           const void *dout, const float *dhT, void *dq, void *dk, void *dv, float *dla, float *dh0, void *ws,
           cudaStream_t st) {
  if (device_ok() != 1) return GLA_ERR_NO_DEVICE;
  TcWs w = carve(p, ws, true);
  unsigned *status = (unsigned *)ws;
  // qg, kg, P^T and gam sit at the same workspace offsets for gla_fwd and gla_bwd,
  // so a forward run on this workspace can hand them over
  if (!(p.flags & GLA_FLAG_REUSE_PREP)) TRY(launch_prep_any(p, (const bf16 *)q, (const bf16 *)k, la, w, status, st));
  const bool saved = (p.flags & GLA_FLAG_SAVE_STATES) != 0;
  const int nvt = walk_tiles(p);
  const int P = bwd_segments(p, nvt);
  const int L = (p.N + P - 1) / P;
  const uint64_t BH = (uint64_t)p.BH;

  // ---- chunk states h_n (bf16), recomputed ------------------------------------
  WalkMaps mf;
  bool okm = map3(&mf.X, w.kg, p.K, p.Tp, BH, 64, 64) && map3(&mf.Y, v, p.V, p.T, BH, 64, 64);
  mf.Q = mf.X;
  mf.P = mf.X;
  // ---- chunk adjoints dh_n (bf16) and dv = kg_n dh_n + P_n^T dO_n ------------------
  WalkMaps mr;
  okm = okm && map3(&mr.X, w.qg, p.K, p.Tp, BH, 64, 64) && map3(&mr.Y, dout, p.V, p.T, BH, 64, 64) &&
        map3(&mr.Q, w.kg, p.K, p.Tp, BH, 64, 64) && map3(&mr.P, w.PT, 64, 64, BH * p.N, 64, 64) &&
        map3_plain(&mr.O, dv, p.V, p.T, BH, 32, 32);
  mf.O = mf.X;
  if (!okm) return GLA_ERR_CUDA;

  tc::WalkArgs a{};
  a.T = p.T;
  a.N = p.N;
  a.V = p.V;
  a.L = L;
  a.P = P;
  a.gam = w.gam;
  a.status = status;
  a.end_seg = -1;
  if (!saved) {  // else the forward stored h_n in w.hb
    if (P > 1) {
      tc::WalkArgs pre = a;  // segments 0 .. P-2, forward
      pre.end = w.delta;
      pre.gseg = w.gseg;
      TRY(launch_walk_any(p, pre, mf, P - 1, st));
      TRY(segment_starts(p.BH, p.K, p.V, P, 0, w.gseg, w.delta, h0, w.starts, st));
      a.start_v = w.starts;
    }
    a.h0 = h0;
    a.state_mode = 1;
    a.hb = w.hb;
    TRY(launch_walk_any(p, a, mf, P, st));
  }

  tc::WalkArgs r{};
  r.T = p.T;
  r.N = p.N;
  r.V = p.V;
  r.L = L;
  r.P = P;
  r.reverse = 1;
  r.gam = w.gam;
  r.status = status;
  r.end = dh0;
  r.end_seg = 0;
  if (P > 1) {
    if (!(p.flags & GLA_FLAG_REUSE_SEGMENTS)) {  // else gla_bwd_state left them in the workspace
      tc::WalkArgs pre = r;  // segments 1 .. P-1, backward
      pre.end = w.ddelta;
      pre.end_seg = -1;
      pre.seg0 = 1;
      pre.gseg = w.gseg;
      TRY(launch_walk_any(p, pre, mr, P - 1, st));
    }
    TRY(segment_starts(p.BH, p.K, p.V, P, 1, w.gseg, w.ddelta, dhT, w.starts, st));
    r.start_v = w.starts;
  }
  r.h0 = dhT;
  r.state_mode = 1;
  r.hb = w.dhb;
  r.do_out = 1;
  r.p_kmajor = 1;
  r.out = (bf16 *)dv;
  TRY(launch_walk_any(p, r, mr, P, st));

  // ---- per-chunk gradients --------------------------------------------------------
  return tc::launch_bwd_main(p, (const bf16 *)q, (const bf16 *)k, (const bf16 *)v, la, (const bf16 *)dout,
                             (bf16 *)dq, (bf16 *)dk, dla, w.gam, w.hb, w.dhb, status, st);
}


// ---- sequence summaries (sequence parallelism) ----------------------------------
// Forward: the state after the whole sequence from h0 (zero if null), delta
// [BH][K][V], and the product of its gates, gamma [BH][K].  The walk runs without
// outputs over every segment in parallel from a zero state (the contributions stay
// in the workspace where gla_fwd with GLA_FLAG_REUSE_SEGMENTS finds them), then
// fold_segments composes them over h0.  Workspace layout and segment count are those
// of gla_fwd with the same flags (GLA_FLAG_SAVE_STATES: the backward layout).
int tc_fwd_state(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
                 float *delta, float *gamma, void *ws, cudaStream_t st) {
  if (device_ok() != 1) return GLA_ERR_NO_DEVICE;
  const bool save = (p.flags & GLA_FLAG_SAVE_STATES) != 0;
  Problem pf = p;
  pf.variant = GLA_VARIANT_FUSED;
  TcWs w = carve(pf, ws, save);
  unsigned *status = (unsigned *)ws;
  if (!(p.flags & GLA_FLAG_REUSE_PREP)) TRY(launch_prep_any(pf, (const bf16 *)q, (const bf16 *)k, la, w, status, st));
  const int nvt = walk_tiles(p);
  const int P = save ? bwd_segments(pf, nvt) : segments_of(pf, nvt);
  const uint64_t BH = (uint64_t)p.BH;
  WalkMaps m;
  if (!(map3(&m.X, w.kg, p.K, p.Tp, BH, 64, 64) && map3(&m.Y, v, p.V, p.T, BH, 64, 64))) return GLA_ERR_CUDA;
  m.Q = m.X;
  m.P = m.X;
  m.O = m.X;
  tc::WalkArgs a{};
  a.T = p.T;
  a.N = p.N;
  a.V = p.V;
  a.L = (p.N + P - 1) / P;
  a.P = P;
  a.gam = w.gam;
  a.status = status;
  if (P == 1) {  // one walk from h0 straight into delta; its gate product is gamma
    a.h0 = h0;
    a.end = delta;
    a.end_seg = 0;
    a.gseg = gamma;
    return launch_walk_any(pf, a, m, 1, st);
  }
  a.end = w.delta;
  a.end_seg = -1;
  a.gseg = w.gseg;
  TRY(launch_walk_any(pf, a, m, P, st));
  return fold_segments(p.BH, p.K, p.V, P, 0, w.gseg, w.delta, h0, delta, gamma, st);
}

// Reverse: the state adjoint before the first token from dh_final (zero if null),
// ddelta [BH][K][V] (what gla_bwd returns as dh0), and gamma as above (if not null).
// The reverse walk over qg and dO without dv, every segment from zero (left in the
// workspace for gla_bwd with GLA_FLAG_REUSE_SEGMENTS), folded over dh_final.
int tc_bwd_state(const Problem &p, const void *q, const void *k, const float *la, const void *dout,
                 const float *dhT, float *ddelta, float *gamma, void *ws, cudaStream_t st) {
  if (device_ok() != 1) return GLA_ERR_NO_DEVICE;
  TcWs w = carve(p, ws, true);
  unsigned *status = (unsigned *)ws;
  if (!(p.flags & GLA_FLAG_REUSE_PREP)) TRY(launch_prep_any(p, (const bf16 *)q, (const bf16 *)k, la, w, status, st));
  const int nvt = walk_tiles(p);
  const int P = bwd_segments(p, nvt);
  const uint64_t BH = (uint64_t)p.BH;
  WalkMaps m;
  if (!(map3(&m.X, w.qg, p.K, p.Tp, BH, 64, 64) && map3(&m.Y, dout, p.V, p.T, BH, 64, 64))) return GLA_ERR_CUDA;
  m.Q = m.X;
  m.P = m.X;
  m.O = m.X;
  tc::WalkArgs r{};
  r.T = p.T;
  r.N = p.N;
  r.V = p.V;
  r.L = (p.N + P - 1) / P;
  r.P = P;
  r.reverse = 1;
  r.gam = w.gam;
  r.status = status;
  if (P == 1) {
    r.h0 = dhT;
    r.end = ddelta;
    r.end_seg = 0;
    r.gseg = gamma;
    return launch_walk_any(p, r, m, 1, st);
  }
  r.end = w.ddelta;
  r.end_seg = -1;
  r.gseg = w.gseg;
  TRY(launch_walk_any(p, r, m, P, st));
  return fold_segments(p.BH, p.K, p.V, P, 1, w.gseg, w.ddelta, dhT, ddelta, gamma, st);
}

}  // namespace gla
