// tc_path.cu -- bf16 path entry points (temporary: CUDA-core kernels).
#include "tc_path.h"

namespace gla {
int tc_check(const Problem &p) { (void)p; return GLA_OK; }
size_t tc_workspace(const Problem &p, bool bwd) { return f32_workspace(p, bwd); }
int tc_fwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
           void *o, float *hT, void *ws, cudaStream_t st) {
  return f32_fwd(p, q, k, v, la, h0, o, hT, ws, st);
}
int tc_bwd(const Problem &p, const void *q, const void *k, const void *v, const float *la, const float *h0,
           const void *dout, const float *dhT, void *dq, void *dk, void *dv, float *dla, float *dh0, void *ws,
           cudaStream_t st) {
  return f32_bwd(p, q, k, v, la, h0, dout, dhT, dq, dk, dv, dla, dh0, ws, st);
}
}  // namespace gla
