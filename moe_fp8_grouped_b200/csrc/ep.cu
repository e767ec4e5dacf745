// ep.cu -- row movement around the grouped matmul when experts are spread
// over ranks (expert parallelism): the permute that sorts routed token rows
// by expert before the exchange, and the unpermute that brings expert
// outputs back to their tokens and sums them with the routing weights
// ("add static LHS scaling support for GMM v2 FWD", maxtext PR #4735,
// rebase commit text: activations are quantized before the expert-parallel
// exchange and ragged sort so that E4M3 rows move instead of bf16, and
// permute / unpermute handle the quantized array; "FP8 Megablox for batch
// split", maxtext PR #3770, Description item 3: group_offset selects the
// local experts of a ragged dot).  The exchange itself is NCCL all-to-all,
// issued by the caller between these kernels.
#include <cuda_bf16.h>

#include <climits>

#include "internal.h"

namespace gmm {

// dst[i] = src[idx[i]] for rows of row_bytes (a multiple of 16); an index
// outside [0, src_rows) gives a row of zeros.  One CTA per row, grid-stride.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4 *__restrict__ src, const int32_t *__restrict__ idx,
                                                          int64_t nrows, int64_t row_vec, int64_t src_rows,
                                                          uint4 *__restrict__ dst) {
  for (int64_t i = blockIdx.x; i < nrows; i += gridDim.x) {
    const int64_t r = idx[i];
    const bool ok = r >= 0 && r < src_rows;
    const uint4 *s = src + (ok ? r : 0) * row_vec;
    uint4 *d = dst + i * row_vec;
    for (int64_t v = threadIdx.x; v < row_vec; v += blockDim.x) d[v] = ok ? s[v] : make_uint4(0, 0, 0, 0);
  }
}

// dst[i] = bf16(fl32(src[idx[i]]) * scale[i]) for bf16 rows of n8 * 8 values
// (an index outside [0, src_rows) gives zeros).  One CTA per row, grid-stride.
__global__ void __launch_bounds__(256) gather_scale_rows_kernel(const __nv_bfloat16 *__restrict__ src,
                                                                const int32_t *__restrict__ idx,
                                                                const float *__restrict__ scale, int64_t nrows,
                                                                int64_t n8, int64_t src_rows,
                                                                __nv_bfloat16 *__restrict__ dst) {
  for (int64_t i = blockIdx.x; i < nrows; i += gridDim.x) {
    const int64_t r = idx[i];
    const bool ok = r >= 0 && r < src_rows;
    const float f = scale[i];
    const uint4 *s = reinterpret_cast<const uint4 *>(src + (ok ? r : 0) * n8 * 8);
    uint4 *d = reinterpret_cast<uint4 *>(dst + i * n8 * 8);
    for (int64_t v = threadIdx.x; v < n8; v += blockDim.x) {
      uint4 o = make_uint4(0, 0, 0, 0);
      if (ok) {
        const uint4 a = s[v];
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&a);
        __nv_bfloat162 *q = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = __bfloat1622float2(h[e]);
          q[e] = __floats2bfloat162_rn(__fmul_rn(x.x, f), __fmul_rn(x.y, f));
        }
      }
      d[v] = o;
    }
  }
}

// y[t, :] = sum_j weight[t, j] * rows[slot[t, j], :] (fp32, j in order; a
// slot outside [0, nrows) contributes nothing).  One CTA per token, 8
// columns per thread step.
__global__ void __launch_bounds__(256) combine_rows_kernel(const __nv_bfloat16 *__restrict__ rows,
                                                           const int32_t *__restrict__ slot,
                                                           const float *__restrict__ weight, int64_t T, int k,
                                                           int64_t nrows, int64_t N, void *y, int y_f32) {
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    for (int64_t c = static_cast<int64_t>(threadIdx.x) * 8; c < N; c += static_cast<int64_t>(blockDim.x) * 8) {
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int j = 0; j < k; ++j) {
        const int64_t r = slot[t * k + j];
        if (r < 0 || r >= nrows) continue;
        const float wgt = weight[t * k + j];
        const uint4 v = *reinterpret_cast<const uint4 *>(rows + r * N + c);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h[e]);
          acc[2 * e] = __fmaf_rn(wgt, f.x, acc[2 * e]);
          acc[2 * e + 1] = __fmaf_rn(wgt, f.y, acc[2 * e + 1]);
        }
      }
      if (y_f32) {
        float4 *d = reinterpret_cast<float4 *>(static_cast<float *>(y) + t * N + c);
        d[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        d[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      } else {
        uint4 o;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
        *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(y) + t * N + c) = o;
      }
    }
  }
}

// Regrouping of the rows that arrive from an all-to-all: they come in source
// rank order, then expert order within each source (block (p, e) holds
// cnt[p * El + e] rows); the gmm wants them grouped by local expert, then by
// source rank.  For arrival row i of block (p, e):
//   pos = D[e, p] + (i - A[p, e]),  perm[pos] = i,  inv[i] = pos,
// A the arrival offsets (prefix over (p, e) order), D the grouped offsets
// (prefix over (e, p) order).  Every CTA builds A and D in shared memory
// (warp 0 scans A, warp 1 scans D), then its threads take one arrival row
// each.  CTA 0 also writes gsz[e] = sum_p cnt[p * El + e].  A row whose pos
// falls outside [0, total) (counts that do not sum to total) is skipped.
constexpr int kMaxEpBlocks = 1024;  // P * El

__device__ __forceinline__ void warp_scan_blocks(const int64_t *cnt, int n, int P, int El, bool by_expert, int *out,
                                                 int lane) {
  // entry j of the scan order: (p, e) = (j / El, j % El) for arrival order,
  // (j % P, j / P) for grouped order; out[p * El + e] = exclusive prefix
  const int per = (n + 31) / 32;
  const int j0 = min(lane * per, n), j1 = min(j0 + per, n);
  auto cnt_at = [&](int j) -> int {
    const int p = by_expert ? j % P : j / El, e = by_expert ? j / P : j % El;
    return static_cast<int>(cnt[p * El + e]);
  };
  int sum = 0;
  for (int j = j0; j < j1; ++j) sum += cnt_at(j);
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  int run = incl - sum;
  for (int j = j0; j < j1; ++j) {
    const int p = by_expert ? j % P : j / El, e = by_expert ? j / P : j % El;
    out[p * El + e] = run;
    run += cnt_at(j);
  }
}

__global__ void __launch_bounds__(256) ep_local_order_kernel(const int64_t *__restrict__ cnt, int P, int El,
                                                             int total, int32_t *__restrict__ perm,
                                                             int32_t *__restrict__ inv, int32_t *__restrict__ gsz) {
  __shared__ int sA[kMaxEpBlocks], sD[kMaxEpBlocks];
  const int n = P * El;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) warp_scan_blocks(cnt, n, P, El, false, sA, lane);
  if (warp == 1) warp_scan_blocks(cnt, n, P, El, true, sD, lane);
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e < El; e += blockDim.x) {
      int64_t t = 0;
      for (int p = 0; p < P; ++p) t += cnt[p * El + e];
      gsz[e] = static_cast<int32_t>(t);
    }
  __syncthreads();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    // the last block b with A[b] <= i (A is non-decreasing; that block is non-empty)
    int lo = 0, hi = n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sA[mid] <= i) lo = mid;
      else hi = mid - 1;
    }
    const int pos = sD[lo] + (i - sA[lo]);
    if (pos < 0 || pos >= total) continue;
    perm[pos] = i;
    inv[i] = pos;
  }
}

static unsigned grid_for(int64_t n) {
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  return static_cast<unsigned>(n < cap ? (n > 0 ? n : 1) : cap);
}

}  // namespace gmm

using namespace gmm;

extern "C" {

gmm_status gmm_gather_rows(const void *src, const int32_t *idx, int64_t nrows, int64_t row_bytes, int64_t src_rows,
                           void *dst, void *stream) {
  if (nrows < 0 || row_bytes <= 0 || src_rows < 0) return GMM_ERR_INVALID_ARG;
  if (nrows == 0) return GMM_OK;
  if (!src || !idx || !dst) return GMM_ERR_INVALID_ARG;
  if (row_bytes % 16) return GMM_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) return GMM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gather_rows_kernel<<<grid_for(nrows), 256, 0, st>>>(static_cast<const uint4 *>(src), idx, nrows, row_bytes / 16,
                                                      src_rows, static_cast<uint4 *>(dst));
  return cudaGetLastError() == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
}

gmm_status gmm_gather_scale_rows(const void *src_bf16, const int32_t *idx, const float *scale, int64_t nrows,
                                 int64_t ncols, int64_t src_rows, void *dst_bf16, void *stream) {
  if (nrows < 0 || ncols <= 0 || src_rows < 0) return GMM_ERR_INVALID_ARG;
  if (nrows == 0) return GMM_OK;
  if (!src_bf16 || !idx || !scale || !dst_bf16) return GMM_ERR_INVALID_ARG;
  if (ncols % 8) return GMM_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(src_bf16) | reinterpret_cast<uintptr_t>(dst_bf16)) & 15u) return GMM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gather_scale_rows_kernel<<<grid_for(nrows), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(src_bf16), idx, scale,
                                                            nrows, ncols / 8, src_rows,
                                                            static_cast<__nv_bfloat16 *>(dst_bf16));
  return cudaGetLastError() == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
}

gmm_status gmm_ep_local_order(const int64_t *recv_counts, int32_t P, int32_t El, int64_t total, int32_t *perm,
                              int32_t *inv, int32_t *group_sizes, void *stream) {
  if (P <= 0 || El <= 0 || total < 0) return GMM_ERR_INVALID_ARG;
  if (static_cast<int64_t>(P) * El > kMaxEpBlocks || total > INT32_MAX) return GMM_ERR_UNSUPPORTED;
  if (!recv_counts || !group_sizes || (total > 0 && (!perm || !inv))) return GMM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t blocks = (total + 255) / 256;
  const unsigned grid = static_cast<unsigned>(blocks < 1 ? 1 : (blocks < num_sms() * 4 ? blocks : num_sms() * 4));
  ep_local_order_kernel<<<grid, 256, 0, st>>>(recv_counts, P, El, static_cast<int>(total), perm, inv, group_sizes);
  return cudaGetLastError() == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
}

gmm_status gmm_combine_rows(const void *rows_bf16, int64_t nrows, const int32_t *slot, const float *weight, int64_t T,
                            int32_t k, int64_t N, void *y, gmm_dtype y_dtype, void *stream) {
  if (T < 0 || k <= 0 || N <= 0 || nrows < 0) return GMM_ERR_INVALID_ARG;
  if (y_dtype != GMM_BF16 && y_dtype != GMM_F32) return GMM_ERR_INVALID_ARG;
  if (T == 0) return GMM_OK;
  if (!slot || !weight || !y || (nrows > 0 && !rows_bf16)) return GMM_ERR_INVALID_ARG;
  if (N % 8) return GMM_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(rows_bf16) | reinterpret_cast<uintptr_t>(y)) & 15u) return GMM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  combine_rows_kernel<<<grid_for(T), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(rows_bf16), slot, weight, T, k,
                                                   nrows, N, y, y_dtype == GMM_F32);
  return cudaGetLastError() == cudaSuccess ? GMM_OK : GMM_ERR_CUDA;
}

}  // extern "C"
