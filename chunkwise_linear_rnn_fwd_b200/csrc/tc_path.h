// tc_path.h -- bf16 tensor-core (tcgen05 / TMEM / TMA) path, sm_100a.
#pragma once
#include "internal.h"

namespace gla {
int tc_check(const Problem &p);
int selftest_timeout(unsigned *status, unsigned limit_us, cudaStream_t st);
size_t tc_workspace(const Problem &p, bool bwd);
int tc_fwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
           void *o, float *hT, void *ws, cudaStream_t st);
int tc_bwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
           const void *dout, const float *dhT, void *dq, void *dk, void *dv, float *dla, float *dh0, void *ws,
           cudaStream_t st);
int tc_fwd_state(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
                 float *delta, float *gamma, void *ws, cudaStream_t st);
int tc_bwd_state(const Problem &p, const void *q, const void *k, const float *la, const void *dout,
                 const float *dhT, float *ddelta, float *gamma, void *ws, cudaStream_t st);
}  // namespace gla
