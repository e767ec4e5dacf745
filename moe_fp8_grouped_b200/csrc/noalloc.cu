// noalloc.cu -- gmm_fwd_noalloc: the forward gmm for callers that cannot
// allocate device memory.  Its scratch (status word, group plan, lhs codes and
// scales) is a fixed array of device memory that belongs to this file, not a
// caller-provided workspace.  The arithmetic is gmm_fwd's: this file only
// finds the array's device address and passes it as the workspace.
#include <mutex>

#include "internal.h"

namespace {

// 32 MiB: enough for the forward scratch of M x K up to about 30 M elements
// (for example 4096 x 7168).  Every device that loads this file's module holds
// the array until the process exits.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;

static __device__ __align__(256) unsigned char g_fwd_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_fwd_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
gmm_status scratch_on_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GMM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GMM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return GMM_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GMM_OK;
}

}  // namespace

extern "C" gmm_status gmm_fwd_noalloc(gmm_operand lhs, gmm_operand rhs, int transpose_rhs,
                                      const int32_t *group_sizes, int32_t G, int64_t M, int64_t K, int64_t N,
                                      void *out, gmm_dtype out_dtype, void *stream) {
  const size_t need = gmm_workspace_bytes(GMM_OP_FWD, M, K, N, G);
  if (need == 0)  // invalid sizes: gmm_fwd reports which check failed, before any launch
    return gmm_fwd(lhs, rhs, transpose_rhs, group_sizes, G, M, K, N, out, out_dtype, nullptr, 0, stream);
  if (need > kNoAllocScratchBytes) return GMM_ERR_WORKSPACE;
  void *ws = nullptr;
  const gmm_status s = scratch_on_current_device(&ws);
  if (s != GMM_OK) return s;
  return gmm_fwd(lhs, rhs, transpose_rhs, group_sizes, G, M, K, N, out, out_dtype, ws, kNoAllocScratchBytes,
                 stream);
}
