// internal.h -- host-side internals shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/gla.h"

namespace gla {

// Kernel ids reported by gla_timing_collect / gla_kernel_name.
enum KernelId : int {
  K_F32_PREP = 0,
  K_F32_STATES,
  K_F32_SCORES,
  K_F32_OUT,
  K_F32_DSTATES,
  K_F32_DSCORES,
  K_F32_DQK,
  K_F32_DV,
  K_F32_DG_SCALAR,
  K_TC_PREP,
  K_TC_WALK,
  K_TC_BWD,
  K_STATUS_CLEAR,
  K_DECODE,
  K_EPI_FWD,
  K_EPI_BWD,
  K_EPI_REDUCE,
  K_STATE_SCAN,
  K_FOLD_SEGMENTS,
  K_F32_DLB,
  K_SEG_STARTS,
  K_TC_WALK_EPI,
  K_COUNT
};

const char *kernel_name(int id);

// The most recent CUDA runtime error that made a call return GLA_ERR_CUDA
// (gla_last_cuda_error reports its text).
void note_cuda_error(cudaError_t e);

// Launch bracketing for gla_timing_* (no-ops unless enabled).
void timing_begin(int kid, cudaStream_t s);
void timing_end(int kid, cudaStream_t s);

// Everything a launcher needs about one call.
struct Problem {
  int B, H, T, K, V;
  int dtype, gate, C, c, variant, segments, flags;
  long BH;     // B*H
  int N;       // chunks per sequence
  long Tp;     // N*C (padded tokens per head)
};

// Status word bits written by kernels into the workspace header.
enum StatusBits : unsigned { ST_TIMEOUT = 1u, ST_GATE_RANGE = 2u, ST_SMEM_ALIGN = 4u };

constexpr size_t kStatusBytes = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// A bump allocator over the caller's workspace.
struct Carve {
  char *base;
  size_t off;
  explicit Carve(void *b) : base((char *)b), off(kStatusBytes) {}
  template <typename T>
  T *take(size_t count) {
    off = align_up(off, 1024);
    T *p = base ? (T *)(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
  size_t bytes() const { return align_up(off, 1024); }
};

// fp32 CUDA-core path (any element type; exact pairwise log-space intra-chunk math)
// lb / dlb: log beta and its gradient of the general gate (null: beta == 1)
size_t f32_workspace(const Problem &p, bool bwd);
size_t f32_general_workspace(const Problem &p, bool bwd);
int f32_fwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *lb,
            const float *h0, void *o, float *hT, void *ws, cudaStream_t st);
int f32_bwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *lb,
            const float *h0, const void *dout, const float *dhT, void *dq, void *dk, void *dv, float *dla,
            float *dlb, float *dh0, void *ws, cudaStream_t st);

// recurrent decode step (CUDA cores); arguments validated by the caller
int decode_step(const gla_desc *d, const void *q, const void *k, const void *v, const float *la, float *state,
                void *o, cudaStream_t st);

// layer epilogue (CUDA cores); arguments validated by the caller
size_t epilogue_workspace(const gla_desc *d);
// sequence parallelism (seqpar.cu)
int fold_segments(long BH, int K, int V, int P, int reverse, const float *gseg, const float *delta, const float *h0,
                  float *out, float *gamma, cudaStream_t st);
int state_scan(long BH, int K, int V, int nseg, int seg, int reverse, const float *gammas, const float *deltas,
               const float *init, float *out, cudaStream_t st);
// start states of a walk's segments from their contributions (tc path)
int segment_starts(long BH, int K, int V, int P, int reverse, const float *gseg, const float *delta, const float *h0,
                   float *starts, cudaStream_t st);
// clear_status = false: keep the status word (a second pass after a forward in the same call)
int epilogue_fwd(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
                 void *y, cudaStream_t st, bool clear_status = true);
int epilogue_bwd(const gla_desc *d, const void *o, const void *r, const float *w, const float *b, float eps,
                 const void *dy, void *dout, void *dr, float *dw, float *db, cudaStream_t st);

}  // namespace gla

#define GLA_LAUNCH(kid, stream, launch_expr)         \
  do {                                               \
    gla::timing_begin((kid), (stream));              \
    launch_expr;                                     \
    gla::timing_end((kid), (stream));                \
    const cudaError_t _le = cudaGetLastError();      \
    if (_le != cudaSuccess) {                        \
      gla::note_cuda_error(_le);                     \
      return GLA_ERR_CUDA;                           \
    }                                                \
  } while (0)
