// plan_quant.cu -- the group plan and the E4M3 quantizers.
//
// Quantization follows "add static LHS scaling support for GMM v2 FWD"
// (maxtext PR #4735), review threads on the LhsRef docstring (lhs arrives
// unquantized, qvalue = clip(lhs / scale)) and on inner_kernel (inverse scale
// 0 where the scale is 0; lhs * inverse cast to the fp8 dtype): inv =
// fl32(1/s), code = E4M3 round-to-nearest-even of fl32(x * inv), saturated to
// +-448.  Every fp32 step is an explicit _rn intrinsic so that no FMA is
// contracted and the codes are bit-identical to a plain IEEE evaluation.
#include <cuda_bf16.h>
#include <cfloat>

#include "internal.h"
#include "ptx.cuh"

namespace gmm {

// ------------------------------------------------------------------ plan

// One warp.  Lane l owns groups [l*per, (l+1)*per).  Negative sizes count as
// 0; group g spans rows [min(P_g, M), min(P_g + s_g, M)) with P the prefix of
// the non-negative sizes.  tpre is the prefix of ceil(rows / 128).
__global__ void plan_kernel(const int32_t *__restrict__ sizes, int G, int64_t M, int *__restrict__ offs,
                            int *__restrict__ tpre, uint32_t *__restrict__ status) {
  const int lane = threadIdx.x;
  const int per = (G + 31) / 32;
  const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
  long long local = 0;
  int bad = 0;
  for (int g = g0; g < g1; ++g) {
    int s = sizes[g];
    if (s < 0) bad = 1;
    local += s < 0 ? 0 : s;
  }
  long long incl = local;
  for (int d = 1; d < 32; d <<= 1) {
    long long v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  long long run = incl - local;  // exclusive prefix of this lane's first group
  const long long total = __shfl_sync(0xffffffffu, incl, 31);
  int tiles_local = 0;
  for (int g = g0; g < g1; ++g) {
    int s = sizes[g] < 0 ? 0 : sizes[g];
    long long a = run < M ? run : M, b = run + s < M ? run + s : M;
    tiles_local += static_cast<int>((b - a + kBlk - 1) / kBlk);
    run += s;
  }
  int tincl = tiles_local;
  for (int d = 1; d < 32; d <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, tincl, d);
    if (lane >= d) tincl += v;
  }
  int trun = tincl - tiles_local;
  run = incl - local;
  for (int g = g0; g < g1; ++g) {
    int s = sizes[g] < 0 ? 0 : sizes[g];
    long long a = run < M ? run : M, b = run + s < M ? run + s : M;
    offs[g] = static_cast<int>(a);
    tpre[g] = trun;
    trun += static_cast<int>((b - a + kBlk - 1) / kBlk);
    run += s;
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 31) {
    offs[G] = static_cast<int>(total < M ? total : M);
    tpre[G] = tincl;
  }
  if (lane == 0) *status = (bad || total > M) ? GMM_DEV_GROUP_SIZES : 0u;
}

cudaError_t launch_plan(const int32_t *sizes, int G, int64_t M, int *offs, int *tpre, uint32_t *status,
                        cudaStream_t st) {
  plan_kernel<<<1, 32, 0, st>>>(sizes, G, M, offs, tpre, status);
  return cudaGetLastError();
}

// --------------------------------------------------------------- helpers

__device__ __forceinline__ bool static_scale_ok(float s) { return isfinite(s) && s > FLT_MIN; }

// Dynamic scale of a block: s = fl32(amax / 448), inv = fl32(1 / s), both 0
// when s is 0 or when 1/s overflows.
__device__ __forceinline__ void dyn_scale(float amax, float &s, float &inv) {
  s = __fdiv_rn(amax, 448.0f);
  inv = (s == 0.0f) ? 0.0f : __fdiv_rn(1.0f, s);
  if (isinf(inv)) {
    s = 0.0f;
    inv = 0.0f;
  }
}

__device__ __forceinline__ int group_of_row(const int *s_offs, int G, int64_t r) {
  // first index i in [0, G] with offs[i] > r, minus one
  int lo = 0, hi = G + 1;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (s_offs[mid] > r) hi = mid;
    else lo = mid + 1;
  }
  int g = lo - 1;
  return (g >= 0 && g < G && r < s_offs[g + 1]) ? g : -1;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&v)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// ------------------------------------------------------ rows (axis 1)

// A warp takes whole rows.  Within a row it covers 256 consecutive values
// per segment (each half-warp one block of 128, each lane 8 values = 16
// bytes) and kSegs segments per step, all loads issued first.
constexpr int kSegs = 4;

template <bool kDynamic, bool kColMult>
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                         int64_t cols, const float *__restrict__ static_scale,
                                                         const float *__restrict__ col_scale,
                                                         const int *__restrict__ offs, int G,
                                                         uint8_t *__restrict__ codes, float *__restrict__ scales,
                                                         uint32_t *__restrict__ status) {
  __shared__ int s_offs[kMaxGroups + 1];
  if constexpr (kColMult) {
    for (int i = threadIdx.x; i <= G; i += blockDim.x) s_offs[i] = offs[i];
    __syncthreads();
  }
  float inv_static = 0.0f;
  if constexpr (!kDynamic) {
    const float s = *static_scale;
    const bool ok = static_scale_ok(s);
    inv_static = ok ? __fdiv_rn(1.0f, s) : 0.0f;
    if (!ok && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, GMM_DEV_SCALE);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, hl = lane & 15;
  const int segs_per_row = static_cast<int>((cols + 255) / 256);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + warp; r < rows; r += nwarps) {
    const __nv_bfloat16 *xr = x + r * cols;
    uint8_t *cr = codes + r * cols;
    const float *csr = nullptr;
    bool row_in_group = true;
    if constexpr (kColMult) {
      const int g = group_of_row(s_offs, G, r);
      row_in_group = g >= 0;
      csr = col_scale + static_cast<int64_t>(g < 0 ? 0 : g) * cols;
    }
    for (int sb = 0; sb < segs_per_row; sb += kSegs) {
      uint4 raw[kSegs];
      float4 cs[kSegs][2];
      int cb[kSegs];
      bool valid[kSegs];
#pragma unroll
      for (int u = 0; u < kSegs; ++u) {
        cb[u] = (sb + u) * 256 + half * 128;
        valid[u] = sb + u < segs_per_row && cb[u] < cols;
        raw[u] = valid[u] ? __ldg(reinterpret_cast<const uint4 *>(xr + cb[u] + hl * 8)) : make_uint4(0, 0, 0, 0);
        if constexpr (kColMult) {
          if (valid[u] && row_in_group) {
            const float4 *c = reinterpret_cast<const float4 *>(csr + cb[u] + hl * 8);
            cs[u][0] = __ldg(c);
            cs[u][1] = __ldg(c + 1);
          } else {
            cs[u][0] = cs[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kSegs; ++u) {
        if (sb + u >= segs_per_row) break;  // warp-uniform
        float v[8];
        bf16x8_to_f32(raw[u], v);
        if constexpr (kColMult) {
          // t = fl32(dout * s_r[g(m), n]); rows in no group give t = +0
          v[0] = __fmul_rn(v[0], cs[u][0].x); v[1] = __fmul_rn(v[1], cs[u][0].y);
          v[2] = __fmul_rn(v[2], cs[u][0].z); v[3] = __fmul_rn(v[3], cs[u][0].w);
          v[4] = __fmul_rn(v[4], cs[u][1].x); v[5] = __fmul_rn(v[5], cs[u][1].y);
          v[6] = __fmul_rn(v[6], cs[u][1].z); v[7] = __fmul_rn(v[7], cs[u][1].w);
          if (!row_in_group) {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.0f;
          }
        }
        float s = 0.0f, inv;
        if constexpr (kDynamic) {
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
          for (int d = 8; d >= 1; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
          dyn_scale(amax, s, inv);
        } else {
          inv = inv_static;
        }
        if (valid[u]) {
          uint2 out;
          out.x = static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv))) |
                  (static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv))) << 16);
          out.y = static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(v[4], inv), __fmul_rn(v[5], inv))) |
                  (static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(v[6], inv), __fmul_rn(v[7], inv))) << 16);
          *reinterpret_cast<uint2 *>(cr + cb[u] + hl * 8) = out;
          if (kDynamic && hl == 0) scales[static_cast<int64_t>(cb[u] / kBlk) * rows + r] = s;
        }
      }
    }
  }
}

cudaError_t launch_quant_rows(const void *x, int64_t rows, int64_t cols, bool dynamic, const float *static_scale,
                              const float *col_scale, const int *offs, int G, uint8_t *codes, float *scales,
                              uint32_t *status, cudaStream_t st) {
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  if (dynamic && col_scale)
    quant_rows_kernel<true, true><<<blocks, 256, 0, st>>>(xb, rows, cols, static_scale, col_scale, offs, G, codes,
                                                          scales, status);
  else if (dynamic)
    quant_rows_kernel<true, false><<<blocks, 256, 0, st>>>(xb, rows, cols, static_scale, col_scale, offs, G,
                                                           codes, scales, status);
  else if (col_scale)
    quant_rows_kernel<false, true><<<blocks, 256, 0, st>>>(xb, rows, cols, static_scale, col_scale, offs, G,
                                                           codes, scales, status);
  else
    quant_rows_kernel<false, false><<<blocks, 256, 0, st>>>(xb, rows, cols, static_scale, col_scale, offs, G,
                                                            codes, scales, status);
  return cudaGetLastError();
}

// ---------------------------------------------------- chunks (axis 0)

// 32 code bytes: one 256-bit store when dst is 32-byte aligned, else two
// 128-bit stores (dst is always 16-byte aligned here).
__device__ __forceinline__ void store_codes32(uint8_t *dst, const uint32_t (&w)[8], bool v8) {
  if (v8) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
  } else {
    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}


// One CTA of 128 threads per (128-column slice, chunk).  The chunk's rows (at
// most 128, the rest zero) are staged in shared memory with cp.async; threads
// t and t + 64 own the adjacent columns 2t and 2t+1, each for one half of the
// rows: the halves' absmax (on packed bf16 pairs, exact) meet in shared
// memory, and each thread writes its 64 rows of both columns' code lines in
// the chunk-major transposed layout [chunk][column][128], so a CTA writes one
// contiguous block.  The 34 KB tile keeps six CTAs per SM, so loads of some
// overlap the work of others.
constexpr int kChunkCols = 128;
constexpr int kChunkPairs = kChunkCols / 2;  // column pairs per slice
constexpr int kChunkThreads = 2 * kChunkPairs;
constexpr int kChunkPitch = kChunkCols + 8;  // bf16 per staged row (16-byte aligned rows)
constexpr size_t kChunkSmem = static_cast<size_t>(kBlk) * kChunkPitch * sizeof(__nv_bfloat16);

__device__ __forceinline__ void cp_async_16_zfill(void *dst_smem, const void *src, bool in_range) {
  // src-size 0 writes 16 zero bytes without reading
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst_smem)), "l"(src),
               "r"(in_range ? 16 : 0)
               : "memory");
}

// Chunk j (over all groups, in group order): first row r0 and row count nr;
// false when j is past the last chunk.
__device__ __forceinline__ bool find_chunk(int j, const int *offs, const int *tpre, int G, int &r0, int &nr) {
  if (j >= tpre[G]) return false;
  int lo = 0, hi = G + 1;  // first i with tpre[i] > j
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (tpre[mid] > j) hi = mid;
    else lo = mid + 1;
  }
  const int g = lo - 1;
  r0 = offs[g] + kBlk * (j - tpre[g]);
  nr = min(r0 + kBlk, offs[g + 1]) - r0;
  return true;
}

template <bool kDynamic, bool kCopy>
__global__ void __launch_bounds__(kChunkThreads) quant_chunks_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t rows, int64_t cols, const float *__restrict__ static_scale,
    const int *__restrict__ offs, const int *__restrict__ tpre, int G, void *codes_t, float *__restrict__ scales,
    uint32_t *__restrict__ status) {
  extern __shared__ __align__(16) uint8_t qsm[];
  __nv_bfloat16 *tile = reinterpret_cast<__nv_bfloat16 *>(qsm);  // [128][kChunkPitch]
  __shared__ int s_info[3];
  __shared__ __nv_bfloat162 s_am[2][kChunkPairs];
  const int j = blockIdx.y;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kChunkCols;
  if (threadIdx.x == 0) s_info[0] = find_chunk(j, offs, tpre, G, s_info[1], s_info[2]) ? 1 : 0;
  __syncthreads();
  if (!s_info[0]) return;
  const int r0 = s_info[1], nr = s_info[2];
  // 128 rows x 16 sixteen-byte pieces, all in flight; rows past the chunk and
  // columns past the matrix are zero-filled
  for (int i = threadIdx.x; i < kBlk * (kChunkCols / 8); i += kChunkThreads) {
    const int rr = i / (kChunkCols / 8), cc = (i % (kChunkCols / 8)) * 8;
    const bool in = rr < nr && c0 + cc < cols;
    const __nv_bfloat16 *src = in ? x + static_cast<int64_t>(r0 + rr) * cols + c0 + cc : x;
    cp_async_16_zfill(tile + rr * kChunkPitch + cc, src, in);
  }
  cp_async_wait_all();
  __syncthreads();
  const int cp = threadIdx.x % kChunkPairs, rh = threadIdx.x / kChunkPairs;  // column pair, row half
  const int col = 2 * cp;                                                     // and col + 1
  const int rbeg = rh * (kBlk / 2);
  const bool active = c0 + col < cols;  // both columns are in or out (cols is even)
  const __nv_bfloat162 *t2 = reinterpret_cast<const __nv_bfloat162 *>(tile);
  constexpr int kPitch2 = kChunkPitch / 2;  // bf16 pairs per staged row
  const int64_t line = (static_cast<int64_t>(j) * cols + c0 + col) * kBlk;  // element offset of column col's line
  if constexpr (kCopy) {
    // bf16 family: transposed bf16 copy, no scale
    if (!active) return;
    const uint32_t *t32 = reinterpret_cast<const uint32_t *>(tile);
    uint16_t *dst0 = static_cast<uint16_t *>(codes_t) + line + rbeg;
    uint16_t *dst1 = dst0 + kBlk;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t w0[4], w1[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t a = t32[(rbeg + q * 8 + 2 * e) * kPitch2 + cp];
        const uint32_t b = t32[(rbeg + q * 8 + 2 * e + 1) * kPitch2 + cp];
        w0[e] = (a & 0xFFFFu) | (b << 16);
        w1[e] = (a >> 16) | (b & 0xFFFF0000u);
      }
      *reinterpret_cast<uint4 *>(dst0 + q * 8) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
      *reinterpret_cast<uint4 *>(dst1 + q * 8) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
    }
  } else {
    float s0, s1, inv0, inv1;
    if constexpr (kDynamic) {
      __nv_bfloat162 m2 = __float2bfloat162_rn(0.0f);
#pragma unroll 16
      for (int r = rbeg; r < rbeg + kBlk / 2; ++r) m2 = __hmax2(m2, __habs2(t2[r * kPitch2 + cp]));
      s_am[rh][cp] = m2;
      __syncthreads();
      const float2 am = __bfloat1622float2(__hmax2(s_am[0][cp], s_am[1][cp]));
      dyn_scale(am.x, s0, inv0);
      dyn_scale(am.y, s1, inv1);
    } else {
      float s = *static_scale;
      const bool ok = static_scale_ok(s);
      const float inv = ok ? __fdiv_rn(1.0f, s) : 0.0f;
      if (!ok) s = 0.0f;
      if (!ok && j == 0 && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, GMM_DEV_SCALE);
      s0 = s1 = s;
      inv0 = inv1 = inv;
    }
    if (!active) return;
    const float2 inv = make_float2(inv0, inv1);
    uint8_t *dst0 = static_cast<uint8_t *>(codes_t) + line + rbeg;
    uint8_t *dst1 = dst0 + kBlk;
    const bool v8 = (reinterpret_cast<uintptr_t>(codes_t) & 31u) == 0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t w0[8], w1[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int r = rbeg + q * 32 + e * 4;
        float2 f[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __fmul2_rn(__bfloat1622float2(t2[(r + i) * kPitch2 + cp]), inv);
        w0[e] = static_cast<uint32_t>(cvt_e4m3x2(f[0].x, f[1].x)) |
                (static_cast<uint32_t>(cvt_e4m3x2(f[2].x, f[3].x)) << 16);
        w1[e] = static_cast<uint32_t>(cvt_e4m3x2(f[0].y, f[1].y)) |
                (static_cast<uint32_t>(cvt_e4m3x2(f[2].y, f[3].y)) << 16);
      }
      store_codes32(dst0 + q * 32, w0, v8);
      store_codes32(dst1 + q * 32, w1, v8);
    }
    if (rh == 0)
      *reinterpret_cast<float2 *>(scales + static_cast<int64_t>(j) * cols + c0 + col) = make_float2(s0, s1);
  }
}

template <bool kDynamic, bool kCopy>
static cudaError_t launch_chunks_inst(dim3 grid, cudaStream_t st, const __nv_bfloat16 *xb, int64_t rows,
                                      int64_t cols, const float *static_scale, const int *offs, const int *tpre,
                                      int G, void *codes_t, float *scales, uint32_t *status) {
  auto kern = quant_chunks_kernel<kDynamic, kCopy>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kChunkSmem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kChunkThreads, kChunkSmem, st>>>(xb, rows, cols, static_scale, offs, tpre, G, codes_t, scales, status);
  return cudaGetLastError();
}

cudaError_t launch_quant_chunks(const void *x, int64_t rows, int64_t cols, bool dynamic, const float *static_scale,
                                const int *offs, const int *tpre, int G, int64_t capacity, void *codes_t,
                                float *scales, bool bf16_copy, uint32_t *status, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((cols + kChunkCols - 1) / kChunkCols), static_cast<unsigned>(capacity));
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  if (bf16_copy)
    return launch_chunks_inst<false, true>(grid, st, xb, rows, cols, static_scale, offs, tpre, G, codes_t, scales,
                                           status);
  if (dynamic)
    return launch_chunks_inst<true, false>(grid, st, xb, rows, cols, static_scale, offs, tpre, G, codes_t, scales,
                                           status);
  return launch_chunks_inst<false, false>(grid, st, xb, rows, cols, static_scale, offs, tpre, G, codes_t, scales,
                                          status);
}

// Backward dout from one read: the tgmm chunk operand and the dlhs row
// operand.  One CTA per (chunk, 128-column slice) stages the chunk's rows
// (zero-filled past the chunk) by cp.async, then two warp roles work on the
// tile at once:
//   warps 0-1, the columns: thread t holds columns 2t, 2t+1; the absmax over
//     the chunk's rows is taken on packed bf16 pairs (exact: a max of bf16
//     values), then each column's 128 codes form one code line;
//   warps 2-5, the rows: a warp takes 8 rows per step, lane = row (lane & 7)
//     and 32 columns (lane >> 3), so a quarter-warp reads 8 rows at one bank
//     offset each (row pitch 68 words) and the block scale is computed once
//     per 32 elements; t = fl32(dout * s_r[g, n]) when kFold, absmax over the
//     128-column block by two shuffles, codes and the block scale exactly as
//     quant_rows_kernel computes them.
// Packed f32x2 multiplies and 32-byte stores keep the instruction count low
// enough for the kernel to stream at memory speed.  The small tile (34 KB)
// keeps six CTAs per SM, so loads of some overlap the arithmetic of others.
constexpr int kDoutCols = 128;
constexpr int kDoutPitch = kDoutCols + 8;                 // bf16 per staged row (16-byte aligned rows)
constexpr int kDoutColThreads = kDoutCols / 2;            // two columns per thread
constexpr int kDoutRowWarps = 4;
constexpr int kDoutThreads = kDoutColThreads + 32 * kDoutRowWarps;
constexpr int kDoutRowsPerStep = 8;                       // rows per row-warp step (lane & 7)
constexpr int kDoutLaneCols = kDoutCols / 4;              // columns per row lane (lane >> 3)

// column scale s_r[g, c0 + c] staged at c + 4 (c / 32): the four 32-column
// groups start in different banks
__device__ __forceinline__ int cs_slot(int c) { return c + ((c >> 5) << 2); }

template <bool kFold>
__global__ void __launch_bounds__(kDoutThreads, 6) quant_dout_both_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t rows, int64_t cols, const float *__restrict__ col_scale,
    const int *__restrict__ offs, const int *__restrict__ tpre, int G, uint8_t *__restrict__ codes_t,
    float *__restrict__ scales_t, uint8_t *__restrict__ codes_r, float *__restrict__ scales_r) {
  __shared__ __align__(16) __nv_bfloat16 tile[kBlk * kDoutPitch];
  __shared__ __align__(16) float s_cs[kDoutCols + 16];
  __shared__ int s_info[4];
  const int j = blockIdx.y;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kDoutCols;  // cols is a multiple of 128
  if (threadIdx.x == 0) {
    s_info[0] = find_chunk(j, offs, tpre, G, s_info[1], s_info[2]) ? 1 : 0;
    if (s_info[0]) {  // the chunk's group
      int lo = 0, hi = G + 1;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (tpre[mid] > j) hi = mid;
        else lo = mid + 1;
      }
      s_info[3] = lo - 1;
    }
  }
  __syncthreads();
  if (!s_info[0]) return;
  const int r0 = s_info[1], nr = s_info[2], g = s_info[3];
  for (int i = threadIdx.x; i < kBlk * (kDoutCols / 8); i += kDoutThreads) {
    const int rr = i / (kDoutCols / 8), cc = (i % (kDoutCols / 8)) * 8;
    const bool in = rr < nr;
    const __nv_bfloat16 *src = in ? x + static_cast<int64_t>(r0 + rr) * cols + c0 + cc : x;
    cp_async_16_zfill(tile + rr * kDoutPitch + cc, src, in);
  }
  if constexpr (kFold) {
    for (int c = threadIdx.x; c < kDoutCols; c += kDoutThreads)
      s_cs[cs_slot(c)] = __ldg(col_scale + static_cast<int64_t>(g) * cols + c0 + c);
  }
  cp_async_wait_all();
  __syncthreads();
  if (threadIdx.x >= kDoutColThreads) {
    // ---- rows: the dlhs operand
    const int lane = threadIdx.x & 31, warp = (threadIdx.x - kDoutColThreads) >> 5;
    const int rl = lane & (kDoutRowsPerStep - 1), cl = (lane >> 3) * kDoutLaneCols;
    const bool v8 = (reinterpret_cast<uintptr_t>(codes_r) & 31u) == 0;
    for (int rb = kDoutRowsPerStep * warp; rb < nr; rb += kDoutRowsPerStep * kDoutRowWarps) {
      const int r = rb + rl;  // < 128; rows past the chunk hold zeros and are not stored
      float2 v[16];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(tile + r * kDoutPitch + cl + 8 * k);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) v[4 * k + e] = __bfloat1622float2(h[e]);
      }
      if constexpr (kFold) {
        const float4 *c4 = reinterpret_cast<const float4 *>(s_cs + cs_slot(cl));
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 c = c4[k];
          v[2 * k] = __fmul2_rn(v[2 * k], make_float2(c.x, c.y));
          v[2 * k + 1] = __fmul2_rn(v[2 * k + 1], make_float2(c.z, c.w));
        }
      }
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(v[i].x), fabsf(v[i].y)));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 8));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
      float sc, inv;
      dyn_scale(amax, sc, inv);
      if (r < nr) {
        const float2 inv2 = make_float2(inv, inv);
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 a = __fmul2_rn(v[2 * i], inv2), b = __fmul2_rn(v[2 * i + 1], inv2);
          w[i] = static_cast<uint32_t>(cvt_e4m3x2(a.x, a.y)) | (static_cast<uint32_t>(cvt_e4m3x2(b.x, b.y)) << 16);
        }
        const int64_t m = r0 + r;
        store_codes32(codes_r + m * cols + c0 + cl, w, v8);
        if (cl == 0) scales_r[(c0 / kBlk) * rows + m] = sc;
      }
    }
    return;
  }
  // ---- columns: the tgmm operand (quant_chunks_kernel, dynamic rule)
  const int t = threadIdx.x;  // columns 2t, 2t + 1
  const __nv_bfloat162 *t2 = reinterpret_cast<const __nv_bfloat162 *>(tile);
  constexpr int kPitch2 = kDoutPitch / 2;  // bf16 pairs per staged row
  __nv_bfloat162 m2 = __float2bfloat162_rn(0.0f);
#pragma unroll 16
  for (int r = 0; r < kBlk; ++r) m2 = __hmax2(m2, __habs2(t2[r * kPitch2 + t]));
  const float2 am = __bfloat1622float2(m2);
  float s0, s1, inv0, inv1;
  dyn_scale(am.x, s0, inv0);
  dyn_scale(am.y, s1, inv1);
  const float2 inv = make_float2(inv0, inv1);
  uint8_t *dst0 = codes_t + (static_cast<int64_t>(j) * cols + c0 + 2 * t) * kBlk;
  uint8_t *dst1 = dst0 + kBlk;
  const bool v8 = (reinterpret_cast<uintptr_t>(codes_t) & 31u) == 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w0[8], w1[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int r = q * 32 + e * 4;
      float2 f[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) f[i] = __fmul2_rn(__bfloat1622float2(t2[(r + i) * kPitch2 + t]), inv);
      w0[e] = static_cast<uint32_t>(cvt_e4m3x2(f[0].x, f[1].x)) |
              (static_cast<uint32_t>(cvt_e4m3x2(f[2].x, f[3].x)) << 16);
      w1[e] = static_cast<uint32_t>(cvt_e4m3x2(f[0].y, f[1].y)) |
              (static_cast<uint32_t>(cvt_e4m3x2(f[2].y, f[3].y)) << 16);
    }
    store_codes32(dst0 + q * 32, w0, v8);
    store_codes32(dst1 + q * 32, w1, v8);
  }
  *reinterpret_cast<float2 *>(scales_t + static_cast<int64_t>(j) * cols + c0 + 2 * t) = make_float2(s0, s1);
}

cudaError_t launch_quant_dout_both(const void *x, int64_t rows, int64_t cols, const float *col_scale, const int *offs,
                                   const int *tpre, int G, int64_t capacity, void *codes_t, float *scales_t,
                                   uint8_t *codes_r, float *scales_r, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(cols / kDoutCols), static_cast<unsigned>(capacity));
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  auto kern = col_scale ? quant_dout_both_kernel<true> : quant_dout_both_kernel<false>;
  kern<<<grid, kDoutThreads, 0, st>>>(xb, rows, cols, col_scale, offs, tpre, G, static_cast<uint8_t *>(codes_t),
                                      scales_t, codes_r, scales_r);
  return cudaGetLastError();
}

// Already-quantized E4M3 lhs (static rule): its codes laid out as the chunk
// quantizer lays out the codes it makes (transposed, padded, zero pad rows),
// bytes copied unchanged.  64 threads per (128-column slice, chunk), one
// column pair each.
constexpr int kCodePitch = kChunkCols + 16;  // bytes per staged row (16-byte aligned rows)
constexpr int kCodeThreads = kChunkPairs;     // one column pair per thread

__global__ void __launch_bounds__(kCodeThreads) chunk_codes_kernel(const uint8_t *__restrict__ x, int64_t cols,
                                                                    const int *__restrict__ offs,
                                                                    const int *__restrict__ tpre, int G,
                                                                    uint8_t *__restrict__ codes_t) {
  __shared__ __align__(16) uint8_t tile[kBlk * kCodePitch];
  __shared__ int s_info[3];
  const int j = blockIdx.y;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kChunkCols;
  if (threadIdx.x == 0) s_info[0] = find_chunk(j, offs, tpre, G, s_info[1], s_info[2]) ? 1 : 0;
  __syncthreads();
  if (!s_info[0]) return;
  const int r0 = s_info[1], nr = s_info[2];
  for (int i = threadIdx.x; i < kBlk * (kChunkCols / 16); i += kCodeThreads) {
    const int rr = i / (kChunkCols / 16), cc = (i % (kChunkCols / 16)) * 16;
    const bool in = rr < nr && c0 + cc < cols;
    const uint8_t *src = in ? x + static_cast<int64_t>(r0 + rr) * cols + c0 + cc : x;
    cp_async_16_zfill(tile + rr * kCodePitch + cc, src, in);
  }
  cp_async_wait_all();
  __syncthreads();
  const int col = 2 * threadIdx.x;  // and col + 1
  if (c0 + col >= cols) return;     // cols is a multiple of 128: both columns are in or out
  uint8_t *dst0 = codes_t + (static_cast<int64_t>(j) * cols + c0 + col) * kBlk;
  uint8_t *dst1 = dst0 + kBlk;
  auto pair = [&](int r) -> uint32_t { return *reinterpret_cast<const uint16_t *>(tile + r * kCodePitch + col); };
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t w0[4], w1[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = q * 16 + e * 4;
      const uint32_t a = pair(r), b = pair(r + 1), c = pair(r + 2), d = pair(r + 3);
      w0[e] = (a & 0xFFu) | ((b & 0xFFu) << 8) | ((c & 0xFFu) << 16) | ((d & 0xFFu) << 24);
      w1[e] = (a >> 8) | ((b >> 8) << 8) | ((c >> 8) << 16) | ((d >> 8) << 24);
    }
    *reinterpret_cast<uint4 *>(dst0 + q * 16) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
    *reinterpret_cast<uint4 *>(dst1 + q * 16) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
  }
}

cudaError_t launch_chunk_codes(const uint8_t *codes, int64_t rows, int64_t cols, const int *offs, const int *tpre,
                               int G, int64_t capacity, uint8_t *codes_t, cudaStream_t st) {
  (void)rows;  // rows past the plan are never read
  dim3 grid(static_cast<unsigned>((cols + kChunkCols - 1) / kChunkCols), static_cast<unsigned>(capacity));
  chunk_codes_kernel<<<grid, kCodeThreads, 0, st>>>(codes, cols, offs, tpre, G, codes_t);
  return cudaGetLastError();
}

// ------------------------------------------------------------ rhs (K7)

// Column absmax of W[g, :, n] into amax_bits (fp32 bit patterns of values
// >= 0 order like unsigned integers, so atomicMax on the bits is a max).
__global__ void __launch_bounds__(256) rhs_amax_kernel(const __nv_bfloat16 *__restrict__ w, int64_t K, int64_t N,
                                                       unsigned int *__restrict__ amax_bits) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int g = blockIdx.z;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * 128;
  if (n >= N) return;
  float m = 0.0f;
  const int64_t k1 = min(k0 + 128, K);
  for (int64_t k = k0; k < k1; ++k) m = fmaxf(m, fabsf(__bfloat162float(w[(g * K + k) * N + n])));
  atomicMax(amax_bits + static_cast<int64_t>(g) * N + n, __float_as_uint(m));
}

// 128 x 128 tiles of W[g] (rows k, columns n): codes written row-wise
// ([G, K, N]) or column-wise ([G, N, K]).
template <bool kTranspose>
__global__ void __launch_bounds__(256) rhs_codes_kernel(const __nv_bfloat16 *__restrict__ w, int64_t K, int64_t N,
                                                        const unsigned int *__restrict__ amax_bits,
                                                        uint8_t *__restrict__ codes) {
  __shared__ __align__(16) __nv_bfloat16 tile[kBlk][kBlk + 8];
  __shared__ float s_inv[kBlk];
  const int g = blockIdx.z;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kBlk, k0 = static_cast<int64_t>(blockIdx.y) * kBlk;
  for (int i = threadIdx.x; i < kBlk * 16; i += 256) {
    const int rr = i >> 4, cc = (i & 15) * 8;
    *reinterpret_cast<uint4 *>(&tile[rr][cc]) =
        __ldg(reinterpret_cast<const uint4 *>(w + (g * K + k0 + rr) * N + n0 + cc));
  }
  if (threadIdx.x < kBlk) {
    float s, inv;
    dyn_scale(__uint_as_float(amax_bits[static_cast<int64_t>(g) * N + n0 + threadIdx.x]), s, inv);
    s_inv[threadIdx.x] = inv;
  }
  __syncthreads();
  const int t = threadIdx.x & 127, h = threadIdx.x >> 7;
  if constexpr (!kTranspose) {
    // thread (row t, half h): 64 columns of row k0 + t
    uint8_t *dst = codes + (g * K + k0 + t) * N + n0 + 64 * h;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t wv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 64 * h + q * 16 + e * 4;
        const float a0 = __fmul_rn(__bfloat162float(tile[t][c]), s_inv[c]);
        const float a1 = __fmul_rn(__bfloat162float(tile[t][c + 1]), s_inv[c + 1]);
        const float a2 = __fmul_rn(__bfloat162float(tile[t][c + 2]), s_inv[c + 2]);
        const float a3 = __fmul_rn(__bfloat162float(tile[t][c + 3]), s_inv[c + 3]);
        wv[e] = static_cast<uint32_t>(cvt_e4m3x2(a0, a1)) | (static_cast<uint32_t>(cvt_e4m3x2(a2, a3)) << 16);
      }
      *reinterpret_cast<uint4 *>(dst + q * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
  } else {
    // thread (column t, half h): 64 rows of column n0 + t
    const float inv = s_inv[t];
    uint8_t *dst = codes + (g * N + n0 + t) * K + k0 + 64 * h;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t wv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = 64 * h + q * 16 + e * 4;
        const float a0 = __fmul_rn(__bfloat162float(tile[r][t]), inv);
        const float a1 = __fmul_rn(__bfloat162float(tile[r + 1][t]), inv);
        const float a2 = __fmul_rn(__bfloat162float(tile[r + 2][t]), inv);
        const float a3 = __fmul_rn(__bfloat162float(tile[r + 3][t]), inv);
        wv[e] = static_cast<uint32_t>(cvt_e4m3x2(a0, a1)) | (static_cast<uint32_t>(cvt_e4m3x2(a2, a3)) << 16);
      }
      *reinterpret_cast<uint4 *>(dst + q * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
  }
}

// amax -> scale, in place.
__global__ void rhs_scale_kernel(float *__restrict__ scales, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n) return;
  float s, inv;
  dyn_scale(scales[i], s, inv);
  scales[i] = s;
}

cudaError_t launch_quant_rhs(const void *w, int G, int64_t K, int64_t N, bool transpose_out, uint8_t *codes,
                             float *scales, cudaStream_t st) {
  const __nv_bfloat16 *wb = static_cast<const __nv_bfloat16 *>(w);
  cudaError_t e = cudaMemsetAsync(scales, 0, sizeof(float) * G * N, st);
  if (e != cudaSuccess) return e;
  rhs_amax_kernel<<<dim3(static_cast<unsigned>((N + 255) / 256), static_cast<unsigned>((K + 127) / 128), G), 256,
                    0, st>>>(wb, K, N, reinterpret_cast<unsigned int *>(scales));
  dim3 grid(static_cast<unsigned>(N / kBlk), static_cast<unsigned>(K / kBlk), G);
  if (transpose_out)
    rhs_codes_kernel<true><<<grid, 256, 0, st>>>(wb, K, N, reinterpret_cast<unsigned int *>(scales), codes);
  else
    rhs_codes_kernel<false><<<grid, 256, 0, st>>>(wb, K, N, reinterpret_cast<unsigned int *>(scales), codes);
  const int64_t n = static_cast<int64_t>(G) * N;
  rhs_scale_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(scales, n);
  return cudaGetLastError();
}

// Block-wise weight scales: one scale per 128-block of W[g] along K (kAxis 0,
// scales [G, K/128, N]) or along N (kAxis 1, scales [G, N/128, K]).  One CTA
// per 128 x 128 tile (rows k, columns n); a tile holds exactly one block per
// column (axis 0) or per row (axis 1).  Codes keep W's layout [G, K, N].
template <int kAxis>
__global__ void __launch_bounds__(256) rhs_blocks_kernel(const __nv_bfloat16 *__restrict__ w, int64_t K, int64_t N,
                                                         uint8_t *__restrict__ codes, float *__restrict__ scales) {
  __shared__ __align__(16) __nv_bfloat16 tile[kBlk][kBlk + 8];
  __shared__ float s_inv[kBlk];
  const int g = blockIdx.z;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kBlk, k0 = static_cast<int64_t>(blockIdx.y) * kBlk;
  for (int i = threadIdx.x; i < kBlk * 16; i += 256) {
    const int rr = i >> 4, cc = (i & 15) * 8;
    *reinterpret_cast<uint4 *>(&tile[rr][cc]) =
        __ldg(reinterpret_cast<const uint4 *>(w + (g * K + k0 + rr) * N + n0 + cc));
  }
  __syncthreads();
  if (threadIdx.x < kBlk) {
    const int t = threadIdx.x;
    float m = 0.0f;
    if constexpr (kAxis == 0) {
      for (int r = 0; r < kBlk; ++r) m = fmaxf(m, fabsf(__bfloat162float(tile[r][t])));  // column t
    } else {
      for (int c = 0; c < kBlk; ++c) m = fmaxf(m, fabsf(__bfloat162float(tile[t][c])));  // row t
    }
    float sc, inv;
    dyn_scale(m, sc, inv);
    s_inv[t] = inv;
    if constexpr (kAxis == 0)
      scales[(static_cast<int64_t>(g) * (K / kBlk) + blockIdx.y) * N + n0 + t] = sc;
    else
      scales[(static_cast<int64_t>(g) * (N / kBlk) + blockIdx.x) * K + k0 + t] = sc;
  }
  __syncthreads();
  // thread (row t, half h): 64 columns of row k0 + t
  const int t = threadIdx.x & 127, h = threadIdx.x >> 7;
  uint8_t *dst = codes + (g * K + k0 + t) * N + n0 + 64 * h;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t wv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = 64 * h + q * 16 + e * 4;
      float a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        a[i] = __fmul_rn(__bfloat162float(tile[t][c + i]), kAxis == 0 ? s_inv[c + i] : s_inv[t]);
      wv[e] = static_cast<uint32_t>(cvt_e4m3x2(a[0], a[1])) | (static_cast<uint32_t>(cvt_e4m3x2(a[2], a[3])) << 16);
    }
    *reinterpret_cast<uint4 *>(dst + q * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }
}

cudaError_t launch_quant_rhs_blocks(const void *w, int G, int64_t K, int64_t N, int axis, uint8_t *codes,
                                    float *scales, cudaStream_t st) {
  const __nv_bfloat16 *wb = static_cast<const __nv_bfloat16 *>(w);
  dim3 grid(static_cast<unsigned>(N / kBlk), static_cast<unsigned>(K / kBlk), G);
  if (axis == 0)
    rhs_blocks_kernel<0><<<grid, 256, 0, st>>>(wb, K, N, codes, scales);
  else
    rhs_blocks_kernel<1><<<grid, 256, 0, st>>>(wb, K, N, codes, scales);
  return cudaGetLastError();
}

// -------------------------------------------------- bounded-wait self-test

// Waits on a barrier that nothing arrives on; the bounded wait gives up after
// limit_ns and records GMM_DEV_TIMEOUT.
__global__ void timeout_selftest_kernel(uint32_t *status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtl ctl{limit_ns, &abort_flag, status};
    mbar_wait(&bar, 0, ctl);  // phase 0 never completes
  }
}

cudaError_t launch_timeout_selftest(uint32_t *status, uint64_t limit_ns, cudaStream_t st) {
  timeout_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace gmm
