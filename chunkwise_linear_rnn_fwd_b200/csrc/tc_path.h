// tc_path.h -- bf16 tensor-core (tcgen05 / TMEM / TMA) path, sm_100a.
#pragma once
#include "internal.h"

namespace gla {
int tc_check(const Problem &p);
int selftest_timeout(unsigned *status, unsigned limit_us, cudaStream_t st);
size_t tc_workspace(const Problem &p, bool bwd);
int tc_fwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
           void *o, float *hT, void *ws, cudaStream_t st);
// The layer epilogue fused into the forward's output store: y = LayerNorm(o) w + b
// times r sigmoid(r), written beside o (tc_fwd_epilogue).
struct TcEpilogue {
  const void *r;
  const float *w, *b;
  float eps;
  void *y;
};
// bf16, a tensor-core shape, d_v a multiple of 128 up to 512, the fused variant,
// no reuse of segment contributions
bool tc_epilogue_fusable(const Problem &p);
int tc_fwd_epilogue(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
                    void *o, float *hT, const TcEpilogue &epi, void *ws, cudaStream_t st);
int tc_bwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
           const void *dout, const float *dhT, void *dq, void *dk, void *dv, float *dla, float *dh0, void *ws,
           cudaStream_t st);
int tc_fwd_state(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
                 float *delta, float *gamma, void *ws, cudaStream_t st);
int tc_bwd_state(const Problem &p, const void *q, const void *k, const float *la, const void *dout,
                 const float *dhT, float *ddelta, float *gamma, void *ws, cudaStream_t st);
}  // namespace gla
