// noalloc.cu -- gmm_fwd_noalloc: the forward gmm for callers that cannot
// allocate device memory.  Its scratch (status word, group plan, lhs codes and
// scales) is a fixed array of device memory that belongs to this file, not a
// caller-provided workspace.  The arithmetic is gmm_fwd's: this file only
// finds the array's device address and passes it as the workspace.
#include <map>
#include <mutex>

#include "internal.h"

namespace {

// 32 MiB: enough for the forward scratch of M x K up to about 30 M elements
// (for example 4096 x 7168).  Every context that loads this file's module
// holds the array until the context is destroyed or the process exits.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;

static __device__ __align__(256) unsigned char g_fwd_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct CtxFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const CtxFns &ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return f;
}

std::mutex g_mu;
// device address of g_fwd_scratch per CUDA context, keyed by the context's
// unique ID (never reused within a process, unlike the handle or the device
// ordinal: a reset device or a second context on the same device gets its own
// lookup)
std::map<unsigned long long, void *> g_scratch_ptr;

// Device address of g_fwd_scratch in the context current to this thread.  In
// host code the array's name is only a host-side stand-in, so the address is
// looked up once per context (with that context current) and cached.
gmm_status scratch_in_current_context(void **out) {
  const CtxFns &f = ctx_fns();
  if (!f.get_current || !f.get_id) return GMM_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS) return GMM_ERR_CUDA;
  void *p = nullptr;
  if (!ctx) {
    // no context current yet: the runtime binds the current device's primary
    // context on its first call that needs one (this lookup)
    if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return GMM_ERR_CUDA;
    if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return GMM_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return GMM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_scratch_ptr.find(id);
  if (it == g_scratch_ptr.end()) {
    if (!p && (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr)) return GMM_ERR_CUDA;
    it = g_scratch_ptr.emplace(id, p).first;
  }
  *out = it->second;
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
  const gmm_status s = scratch_in_current_context(&ws);
  if (s != GMM_OK) return s;
  return gmm_fwd(lhs, rhs, transpose_rhs, group_sizes, G, M, K, N, out, out_dtype, ws, kNoAllocScratchBytes,
                 stream);
}

extern "C" gmm_status gmm_fwd_noalloc_status(uint32_t *bits_out, void *stream) {
  void *ws = nullptr;
  const gmm_status s = scratch_in_current_context(&ws);
  if (s != GMM_OK) return s;
  return gmm_read_device_status(ws, bits_out, stream);
}
