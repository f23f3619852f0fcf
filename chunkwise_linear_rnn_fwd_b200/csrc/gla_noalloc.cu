// gla_noalloc.cu -- gla_fwd for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: a program whose device
// memory is entirely owned by another allocator (a fixed arena reserved up
// front), or a plain C caller with no device-memory management of its own.
// gla_fwd_noalloc serves them: it runs exactly the gla_fwd path, but its
// scratch is g_scratch below, a fixed-size array in the library's own device
// memory.  It calls no cudaMalloc / cudaFree and no allocating library routine.
//
// Rules that come with a single shared array:
//   * every call shares g_scratch and it keeps the last call's contents; the
//     only part that must start at zero (the 256-byte status word) is cleared
//     by every call, everything else is written before it is read;
//   * calls that overlap on the GPU (other streams, other host threads) race
//     on g_scratch and must be serialised by the caller;
//   * the first call on a device resolves the array's device address with
//     cudaGetSymbolAddress (once per device, with that device current); make
//     that first call before any stream capture;
//   * the status word at the start of g_scratch (a bounded wait that ran out, a
//     gate beyond the bf16 range) is read and cleared by
//     gla_poll_status_noalloc, the counterpart of gla_poll_status.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)GLA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// In host code this name is only a stand-in for the device array; the kernels
// receive the address obtained from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

int scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GLA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return GLA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GLA_OK;
}

}  // namespace

extern "C" int gla_fwd_noalloc(const gla_desc *desc, const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *h0, void *o, float *h_final, int chunk,
                               void *stream) {
  if (!desc) return GLA_ERR_INVALID_ARG;
  // Nothing but an earlier no-allocation forward writes g_scratch, and that call's
  // intermediates are not a promise to the next one: a flag that would make this
  // call read them instead of computing them is refused.
  if (desc->flags & (GLA_FLAG_REUSE_PREP | GLA_FLAG_REUSE_SEGMENTS)) return GLA_ERR_INVALID_ARG;
  gla_desc d = *desc;
  d.workspace = nullptr;
  d.workspace_bytes = 0;
  const size_t need = gla_workspace_size(&d, chunk, (d.flags & GLA_FLAG_SAVE_STATES) ? 1 : 0);
  if (need == 0) return gla_check(&d, chunk);
  if (need > kScratchBytes) return GLA_ERR_WORKSPACE_TOO_SMALL;
  void *scratch = nullptr;
  const int r = scratch_address(&scratch);
  if (r != GLA_OK) return r;
  d.workspace = scratch;
  d.workspace_bytes = kScratchBytes;
  return gla_fwd(&d, q, k, v, log_alpha, h0, o, h_final, chunk, stream);
}

// Counterpart of gla_poll_status for the no-allocation forward: the status word
// sits at the start of g_scratch, which a caller cannot name.
extern "C" int gla_poll_status_noalloc(void *stream) {
  void *scratch = nullptr;
  const int r = scratch_address(&scratch);
  if (r != GLA_OK) return r;
  gla_desc d{};
  d.workspace = scratch;
  d.workspace_bytes = kScratchBytes;
  return gla_poll_status(&d, stream);
}
