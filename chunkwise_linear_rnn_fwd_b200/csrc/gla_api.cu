// gla_api.cu -- the C ABI of include/gla.h: validation, workspace sizing,
// dispatch to the kernel paths, the device status word and launch timing.
#include <atomic>
#include <mutex>
#include <vector>

#include "internal.h"
#include "tc_path.h"

namespace gla {

const char *kernel_name(int id) {
  static const char *const names[] = {
      "f32_prep",     "f32_states",   "f32_scores",      "f32_out",    "f32_dstates",   "f32_dscores",
      "f32_dqk",      "f32_dv",       "f32_dg_out",      "tc_prep",    "tc_walk",       "tc_bwd",
      "status_clear", "decode",       "epilogue_fwd",    "epilogue_bwd", "epilogue_reduce", "state_scan",
      "fold_segments", "f32_dlog_beta", "segment_starts", "tc_walk_epi"};
  static_assert(sizeof(names) / sizeof(names[0]) == K_COUNT, "one name per KernelId");
  if (id < 0 || id >= K_COUNT) return "unknown";
  return names[id];
}

namespace {
std::atomic<int> g_last_cuda_error{0};
}  // namespace

void note_cuda_error(cudaError_t e) { g_last_cuda_error.store((int)e, std::memory_order_relaxed); }

// ------------------------------------------------------------------ timing
namespace {
struct TimedLaunch {
  int kid;
  cudaEvent_t a, b;
};
std::mutex g_tmu;
bool g_timing = false;
std::vector<TimedLaunch> g_open;      // launches since the last collect
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

void timing_begin(int kid, cudaStream_t s) {
  if (!g_timing) return;
  std::lock_guard<std::mutex> lk(g_tmu);
  TimedLaunch t{kid, take_event(), take_event()};
  cudaEventRecord(t.a, s);
  g_open.push_back(t);
}

void timing_end(int kid, cudaStream_t s) {
  if (!g_timing) return;
  std::lock_guard<std::mutex> lk(g_tmu);
  for (auto it = g_open.rbegin(); it != g_open.rend(); ++it) {
    if (it->kid == kid) {
      cudaEventRecord(it->b, s);
      return;
    }
  }
}

// ------------------------------------------------------------ validation
namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// The descriptor's limits common to both paths (on_tc picks the path).
int make_problem(const gla_desc *d, int chunk, Problem *p) {
  if (!d) return GLA_ERR_INVALID_ARG;
  if (d->B < 1 || d->H < 1 || d->T < 1 || d->dk < 1 || d->dv < 1) return GLA_ERR_INVALID_ARG;
  if (d->dtype != GLA_DTYPE_BF16 && d->dtype != GLA_DTYPE_FP32) return GLA_ERR_INVALID_ARG;
  if (d->gate != GLA_GATE_VECTOR && d->gate != GLA_GATE_SCALAR && d->gate != GLA_GATE_NONE)
    return GLA_ERR_INVALID_ARG;
  if (d->variant != GLA_VARIANT_AUTO && d->variant != GLA_VARIANT_FUSED && d->variant != GLA_VARIANT_MATERIALIZED)
    return GLA_ERR_INVALID_ARG;
  if (d->segments < 0) return GLA_ERR_INVALID_ARG;
  if (d->flags & ~(GLA_FLAG_REUSE_PREP | GLA_FLAG_SAVE_STATES | GLA_FLAG_REUSE_SEGMENTS)) return GLA_ERR_INVALID_ARG;
  const int sub = d->subchunk == 0 ? 16 : d->subchunk;
  if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return GLA_ERR_UNSUPPORTED_SHAPE;
  if (sub < 1 || chunk % sub != 0) return GLA_ERR_UNSUPPORTED_SHAPE;
  if (d->dk > 256) return GLA_ERR_UNSUPPORTED_SHAPE;
  if (d->dv > 4096) return GLA_ERR_UNSUPPORTED_SHAPE;
  if ((long)d->B * d->H > 65535) return GLA_ERR_UNSUPPORTED_SHAPE;
  p->B = d->B;
  p->H = d->H;
  p->T = d->T;
  p->K = d->dk;
  p->V = d->dv;
  p->dtype = d->dtype;
  p->gate = d->gate;
  p->C = chunk;
  p->c = sub;
  p->variant = d->variant;
  p->segments = d->segments;
  p->flags = d->flags;
  p->BH = (long)d->B * d->H;
  p->N = (d->T + chunk - 1) / chunk;
  p->Tp = (long)p->N * chunk;
  return GLA_OK;
}

// bf16 inputs run on the tensor-core path when it takes the shape (d_k 128 or 256,
// d_v a multiple of 64, chunk 64 with sub-chunk 16); every other shape, and fp32
// inputs, on the CUDA-core path (fp32 arithmetic, any element type)
bool on_tc(const Problem &p) { return p.dtype == GLA_DTYPE_BF16 && tc_check(p) == GLA_OK; }

size_t ws_bytes(const Problem &p, bool bwd) {
  if (on_tc(p)) return tc_workspace(p, bwd);
  return f32_workspace(p, bwd);
}

int check_ws(const gla_desc *d, const Problem &p, bool bwd) {
  const size_t need = ws_bytes(p, bwd);
  if (!d->workspace) return GLA_ERR_INVALID_ARG;
  if (((uintptr_t)d->workspace & 255u) != 0) return GLA_ERR_MISALIGNED;
  if (d->workspace_bytes < need) return GLA_ERR_WORKSPACE_TOO_SMALL;
  return GLA_OK;
}

int check_general_ws(const gla_desc *d, const Problem &p, bool bwd) {
  if (!d->workspace) return GLA_ERR_INVALID_ARG;
  if (((uintptr_t)d->workspace & 255u) != 0) return GLA_ERR_MISALIGNED;
  if (d->workspace_bytes < f32_general_workspace(p, bwd)) return GLA_ERR_WORKSPACE_TOO_SMALL;
  return GLA_OK;
}

int check_gate_ptr(const Problem &p, const void *la) {
  if (p.gate == GLA_GATE_NONE) return la ? GLA_ERR_INVALID_ARG : GLA_OK;
  if (!la) return GLA_ERR_INVALID_ARG;
  return aligned16(la) ? GLA_OK : GLA_ERR_MISALIGNED;
}

int check_opt(const void *x) { return (!x || aligned16(x)) ? GLA_OK : GLA_ERR_MISALIGNED; }
int check_req(const void *x) {
  if (!x) return GLA_ERR_INVALID_ARG;
  return aligned16(x) ? GLA_OK : GLA_ERR_MISALIGNED;
}

#define GLA_TRY(expr)            \
  do {                           \
    const int _r = (expr);       \
    if (_r != GLA_OK) return _r; \
  } while (0)

int clear_status(const gla_desc *d, cudaStream_t st) {
  if (cudaMemsetAsync(d->workspace, 0, kStatusBytes, st) != cudaSuccess) return GLA_ERR_CUDA;
  return GLA_OK;
}

}  // namespace
}  // namespace gla

using namespace gla;

extern "C" {

int gla_check(const gla_desc *desc, int chunk) {
  Problem p;
  return make_problem(desc, chunk, &p);
}

size_t gla_workspace_size(const gla_desc *desc, int chunk, int for_bwd) {
  Problem p;
  if (make_problem(desc, chunk, &p) != GLA_OK) return 0;
  return ws_bytes(p, for_bwd != 0);
}

int gla_fwd(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
            const float *h0, void *o, float *h_final, int chunk, void *stream) {
  Problem p;
  GLA_TRY(make_problem(desc, chunk, &p));
  GLA_TRY(check_req(q));
  GLA_TRY(check_req(k));
  GLA_TRY(check_req(v));
  GLA_TRY(check_req(o));
  GLA_TRY(check_gate_ptr(p, log_alpha));
  GLA_TRY(check_opt(h0));
  GLA_TRY(check_opt(h_final));
  // a forward that saves states for the backward writes into the backward's layout
  GLA_TRY(check_ws(desc, p, (p.flags & GLA_FLAG_SAVE_STATES) != 0));
  cudaStream_t st = (cudaStream_t)stream;
  GLA_TRY(clear_status(desc, st));
  if (on_tc(p)) return tc_fwd(p, q, k, v, log_alpha, h0, o, h_final, desc->workspace, st);
  return f32_fwd(p, q, k, v, log_alpha, nullptr, h0, o, h_final, desc->workspace, st);
}

int gla_bwd(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
            const float *h0, const void *do_, const float *dh_final, void *dq, void *dk, void *dv,
            float *dlog_alpha, float *dh0, int chunk, void *stream) {
  Problem p;
  GLA_TRY(make_problem(desc, chunk, &p));
  GLA_TRY(check_req(q));
  GLA_TRY(check_req(k));
  GLA_TRY(check_req(v));
  GLA_TRY(check_req(do_));
  GLA_TRY(check_req(dq));
  GLA_TRY(check_req(dk));
  GLA_TRY(check_req(dv));
  GLA_TRY(check_gate_ptr(p, log_alpha));
  if (p.gate == GLA_GATE_NONE) {
    if (dlog_alpha) return GLA_ERR_INVALID_ARG;
  } else {
    GLA_TRY(check_req(dlog_alpha));
  }
  GLA_TRY(check_opt(h0));
  GLA_TRY(check_opt(dh_final));
  GLA_TRY(check_opt(dh0));
  GLA_TRY(check_ws(desc, p, true));
  cudaStream_t st = (cudaStream_t)stream;
  GLA_TRY(clear_status(desc, st));
  if (on_tc(p))
    return tc_bwd(p, q, k, v, log_alpha, h0, do_, dh_final, dq, dk, dv, dlog_alpha, dh0, desc->workspace, st);
  return f32_bwd(p, q, k, v, log_alpha, nullptr, h0, do_, dh_final, dq, dk, dv, dlog_alpha, nullptr, dh0,
                 desc->workspace, st);
}

size_t gla_general_workspace_size(const gla_desc *desc, int chunk, int for_bwd) {
  Problem p;
  if (make_problem(desc, chunk, &p) != GLA_OK) return 0;
  return f32_general_workspace(p, for_bwd != 0);
}

int gla_fwd_general(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *log_beta, const float *h0, void *o, float *h_final, int chunk, void *stream) {
  Problem p;
  GLA_TRY(make_problem(desc, chunk, &p));
  GLA_TRY(check_req(q));
  GLA_TRY(check_req(k));
  GLA_TRY(check_req(v));
  GLA_TRY(check_req(o));
  GLA_TRY(check_gate_ptr(p, log_alpha));
  GLA_TRY(check_req(log_beta));
  GLA_TRY(check_opt(h0));
  GLA_TRY(check_opt(h_final));
  GLA_TRY(check_general_ws(desc, p, false));
  cudaStream_t st = (cudaStream_t)stream;
  GLA_TRY(clear_status(desc, st));
  return f32_fwd(p, q, k, v, log_alpha, log_beta, h0, o, h_final, desc->workspace, st);
}

int gla_bwd_general(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *log_beta, const float *h0, const void *do_, const float *dh_final, void *dq,
                    void *dk, void *dv, float *dlog_alpha, float *dlog_beta, float *dh0, int chunk, void *stream) {
  Problem p;
  GLA_TRY(make_problem(desc, chunk, &p));
  GLA_TRY(check_req(q));
  GLA_TRY(check_req(k));
  GLA_TRY(check_req(v));
  GLA_TRY(check_req(do_));
  GLA_TRY(check_req(dq));
  GLA_TRY(check_req(dk));
  GLA_TRY(check_req(dv));
  GLA_TRY(check_gate_ptr(p, log_alpha));
  if (p.gate == GLA_GATE_NONE) {
    if (dlog_alpha) return GLA_ERR_INVALID_ARG;
  } else {
    GLA_TRY(check_req(dlog_alpha));
  }
  GLA_TRY(check_req(log_beta));
  GLA_TRY(check_req(dlog_beta));
  GLA_TRY(check_opt(h0));
  GLA_TRY(check_opt(dh_final));
  GLA_TRY(check_opt(dh0));
  GLA_TRY(check_general_ws(desc, p, true));
  cudaStream_t st = (cudaStream_t)stream;
  GLA_TRY(clear_status(desc, st));
  return f32_bwd(p, q, k, v, log_alpha, log_beta, h0, do_, dh_final, dq, dk, dv, dlog_alpha, dlog_beta, dh0,
                 desc->workspace, st);
}

int gla_fwd_state(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *h0, float *delta, float *gamma, int chunk, void *stream) {
  Problem p;
  GLA_TRY(make_problem(desc, chunk, &p));
  if (!on_tc(p)) return GLA_ERR_UNSUPPORTED_SHAPE;  // the summaries exist on the tensor-core path
  GLA_TRY(check_req(q));
  GLA_TRY(check_req(k));
  GLA_TRY(check_req(v));
  GLA_TRY(check_gate_ptr(p, log_alpha));
  GLA_TRY(check_opt(h0));
  GLA_TRY(check_req(delta));
  GLA_TRY(check_req(gamma));
  // with GLA_FLAG_SAVE_STATES the summary uses the backward's (larger) layout
  GLA_TRY(check_ws(desc, p, (p.flags & GLA_FLAG_SAVE_STATES) != 0));
  cudaStream_t st = (cudaStream_t)stream;
  GLA_TRY(clear_status(desc, st));
  return tc_fwd_state(p, q, k, v, log_alpha, h0, delta, gamma, desc->workspace, st);
}

int gla_bwd_state(const gla_desc *desc, const void *q, const void *k, const float *log_alpha, const void *do_,
                  const float *dh_final, float *ddelta, float *gamma, int chunk, void *stream) {
  Problem p;
  GLA_TRY(make_problem(desc, chunk, &p));
  if (!on_tc(p)) return GLA_ERR_UNSUPPORTED_SHAPE;  // the summaries exist on the tensor-core path
  GLA_TRY(check_req(q));
  GLA_TRY(check_req(k));
  GLA_TRY(check_gate_ptr(p, log_alpha));
  GLA_TRY(check_req(do_));
  GLA_TRY(check_opt(dh_final));
  GLA_TRY(check_req(ddelta));
  GLA_TRY(check_opt(gamma));
  GLA_TRY(check_ws(desc, p, true));
  cudaStream_t st = (cudaStream_t)stream;
  GLA_TRY(clear_status(desc, st));
  return tc_bwd_state(p, q, k, log_alpha, do_, dh_final, ddelta, gamma, desc->workspace, st);
}

int gla_state_scan(const gla_desc *desc, int nseg, int seg, int reverse, const float *gammas, const float *deltas,
                   const float *init, float *out, void *stream) {
  if (!desc || desc->B < 1 || desc->H < 1 || desc->dk < 1 || desc->dv < 1) return GLA_ERR_INVALID_ARG;
  if (desc->dv % 4 != 0) return GLA_ERR_UNSUPPORTED_SHAPE;
  if (nseg < 1 || seg < 0 || seg >= nseg || (reverse != 0 && reverse != 1)) return GLA_ERR_INVALID_ARG;
  const bool empty = reverse ? seg == nseg - 1 : seg == 0;  // no piece to fold: out = init
  if (!empty) {
    GLA_TRY(check_req(gammas));
    GLA_TRY(check_req(deltas));
  }
  GLA_TRY(check_opt(init));
  GLA_TRY(check_req(out));
  return gla::state_scan((long)desc->B * desc->H, desc->dk, desc->dv, nseg, seg, reverse, gammas, deltas, init, out,
                         (cudaStream_t)stream);
}

int gla_poll_status(const gla_desc *desc, void *stream) {
  if (!desc || !desc->workspace) return GLA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, desc->workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GLA_ERR_CUDA;
  if (cudaMemsetAsync(desc->workspace, 0, sizeof(word), st) != cudaSuccess) return GLA_ERR_CUDA;
  if (word & (ST_TIMEOUT | ST_SMEM_ALIGN)) return GLA_ERR_TIMEOUT;
  if (word & ST_GATE_RANGE) return GLA_ERR_GATE_RANGE;
  return GLA_OK;
}

const char *gla_status_string(int code) {
  switch (code) {
    case GLA_OK: return "ok";
    case GLA_ERR_INVALID_ARG: return "invalid argument";
    case GLA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape, chunk or dtype combination";
    case GLA_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned (workspace: 256-byte)";
    case GLA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case GLA_ERR_CUDA: return "CUDA runtime error";
    case GLA_ERR_TIMEOUT: return "device-side bounded wait timed out";
    case GLA_ERR_GATE_RANGE: return "gate decay too strong for the bf16 sub-chunk rescaling";
    case GLA_ERR_NO_DEVICE: return "no sm_100 device for the bf16 tensor-core path";
    default: return "unknown status";
  }
}

int gla_timing_enable(int on) {
  std::lock_guard<std::mutex> lk(g_tmu);
  g_timing = on != 0;
  return GLA_OK;
}

int gla_timing_collect(int max, int *kernel_ids, float *ms) {
  std::lock_guard<std::mutex> lk(g_tmu);
  int n = 0;
  for (auto &t : g_open) {
    if (n < max) {
      float e = -1.f;
      if (cudaEventSynchronize(t.b) == cudaSuccess) cudaEventElapsedTime(&e, t.a, t.b);
      if (kernel_ids) kernel_ids[n] = t.kid;
      if (ms) ms[n] = e;
      ++n;
    }
    g_event_pool.push_back(t.a);
    g_event_pool.push_back(t.b);
  }
  g_open.clear();
  return n;
}

const char *gla_kernel_name(int kernel_id) { return gla::kernel_name(kernel_id); }

int gla_decode_step(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                    float *state, void *o, void *stream) {
  if (!desc) return GLA_ERR_INVALID_ARG;
  if (desc->B < 1 || desc->H < 1 || desc->T != 1 || desc->dk < 1 || desc->dv < 1) return GLA_ERR_INVALID_ARG;
  if (desc->dtype != GLA_DTYPE_BF16 && desc->dtype != GLA_DTYPE_FP32) return GLA_ERR_INVALID_ARG;
  if (desc->gate != GLA_GATE_VECTOR && desc->gate != GLA_GATE_SCALAR && desc->gate != GLA_GATE_NONE)
    return GLA_ERR_INVALID_ARG;
  if (desc->dk > 4096 || desc->dv % 4 != 0 || (long)desc->B * desc->H > 65535) return GLA_ERR_UNSUPPORTED_SHAPE;
  GLA_TRY(check_req(q));
  GLA_TRY(check_req(k));
  GLA_TRY(check_req(v));
  GLA_TRY(check_req(o));
  GLA_TRY(check_req(state));
  if (desc->gate == GLA_GATE_NONE) {
    if (log_alpha) return GLA_ERR_INVALID_ARG;
  } else {
    GLA_TRY(check_req(log_alpha));
  }
  return decode_step(desc, q, k, v, log_alpha, state, o, (cudaStream_t)stream);
}

namespace {
int check_epilogue_desc(const gla_desc *d) {
  if (!d) return GLA_ERR_INVALID_ARG;
  if (d->B < 1 || d->H < 1 || d->T < 1 || d->dv < 1) return GLA_ERR_INVALID_ARG;
  if (d->dtype != GLA_DTYPE_BF16 && d->dtype != GLA_DTYPE_FP32) return GLA_ERR_INVALID_ARG;
  if (d->dv % 8 != 0 || d->dv > 1024 || (long)d->B * d->H * d->T > (1L << 40)) return GLA_ERR_UNSUPPORTED_SHAPE;
  return GLA_OK;
}
int check_eps(float eps) { return (eps > 0.f && eps < 1.f) ? GLA_OK : GLA_ERR_INVALID_ARG; }
// the epilogue's workspace: the status word always, the dw / db partial sums when asked
int check_epilogue_ws(const gla_desc *d, bool partials) {
  if (!d->workspace) return GLA_ERR_INVALID_ARG;
  if (((uintptr_t)d->workspace & 255u) != 0) return GLA_ERR_MISALIGNED;
  if (d->workspace_bytes < (partials ? gla::epilogue_workspace(d) : kStatusBytes)) return GLA_ERR_WORKSPACE_TOO_SMALL;
  return GLA_OK;
}
}  // namespace

size_t gla_epilogue_workspace_size(const gla_desc *desc) {
  if (check_epilogue_desc(desc) != GLA_OK) return 0;
  return gla::epilogue_workspace(desc);
}

int gla_epilogue_fwd(const gla_desc *desc, const void *o, const void *r, const float *w, const float *b, float eps,
                     void *y, void *stream) {
  GLA_TRY(check_epilogue_desc(desc));
  GLA_TRY(check_eps(eps));
  GLA_TRY(check_req(o));
  GLA_TRY(check_req(r));
  GLA_TRY(check_req(y));
  GLA_TRY(check_opt(w));
  GLA_TRY(check_opt(b));
  GLA_TRY(check_epilogue_ws(desc, false));
  return gla::epilogue_fwd(desc, o, r, w, b, eps, y, (cudaStream_t)stream);
}

int gla_fwd_epilogue(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                     const float *h0, const void *r, const float *w, const float *b, float eps, void *o, void *y,
                     float *h_final, int chunk, void *stream) {
  Problem p;
  GLA_TRY(make_problem(desc, chunk, &p));
  if (p.flags & GLA_FLAG_REUSE_SEGMENTS) return GLA_ERR_INVALID_ARG;
  GLA_TRY(check_req(q));
  GLA_TRY(check_req(k));
  GLA_TRY(check_req(v));
  GLA_TRY(check_req(o));
  GLA_TRY(check_req(r));
  GLA_TRY(check_req(y));
  GLA_TRY(check_gate_ptr(p, log_alpha));
  GLA_TRY(check_opt(h0));
  GLA_TRY(check_opt(h_final));
  GLA_TRY(check_opt(w));
  GLA_TRY(check_opt(b));
  GLA_TRY(check_eps(eps));
  GLA_TRY(check_ws(desc, p, (p.flags & GLA_FLAG_SAVE_STATES) != 0));
  const bool fused = tc_epilogue_fusable(p);
  if (!fused) GLA_TRY(check_epilogue_desc(desc));
  cudaStream_t st = (cudaStream_t)stream;
  GLA_TRY(clear_status(desc, st));
  if (fused) {
    const TcEpilogue epi{r, w, b, eps, y};
    return tc_fwd_epilogue(p, q, k, v, log_alpha, h0, o, h_final, epi, desc->workspace, st);
  }
  // two passes: the forward, then the epilogue over its bf16 / fp32 output (the
  // second pass keeps the status word, so a device error of either stays reported)
  const int rf = on_tc(p) ? tc_fwd(p, q, k, v, log_alpha, h0, o, h_final, desc->workspace, st)
                                           : f32_fwd(p, q, k, v, log_alpha, nullptr, h0, o, h_final, desc->workspace, st);
  if (rf != GLA_OK) return rf;
  return gla::epilogue_fwd(desc, o, r, w, b, eps, y, st, false);
}

int gla_epilogue_bwd(const gla_desc *desc, const void *o, const void *r, const float *w, const float *b, float eps,
                     const void *dy, void *do_, void *dr, float *dw, float *db, void *stream) {
  GLA_TRY(check_epilogue_desc(desc));
  GLA_TRY(check_eps(eps));
  GLA_TRY(check_req(o));
  GLA_TRY(check_req(r));
  GLA_TRY(check_req(dy));
  GLA_TRY(check_req(do_));
  GLA_TRY(check_req(dr));
  GLA_TRY(check_opt(w));
  GLA_TRY(check_opt(b));
  GLA_TRY(check_opt(dw));
  GLA_TRY(check_opt(db));
  GLA_TRY(check_epilogue_ws(desc, dw || db));
  return gla::epilogue_bwd(desc, o, r, w, b, eps, dy, do_, dr, dw, db, (cudaStream_t)stream);
}

int gla_selftest_timeout(void *status_word, unsigned limit_us, void *stream) {
  if (!status_word || limit_us < 1 || limit_us > 1000000) return GLA_ERR_INVALID_ARG;
  if (((uintptr_t)status_word & 3u) != 0) return GLA_ERR_MISALIGNED;
  return gla::selftest_timeout((unsigned *)status_word, limit_us, (cudaStream_t)stream);
}

const char *gla_last_cuda_error(void) {
  const int e = gla::g_last_cuda_error.load(std::memory_order_relaxed);
  return e == 0 ? "no error" : cudaGetErrorString((cudaError_t)e);
}

const char *gla_build_info(void) {
  return "gla-b200: sm_100a; bf16 path tcgen05/TMEM/TMA; fp32 path CUDA cores";
}

}  // extern "C"
