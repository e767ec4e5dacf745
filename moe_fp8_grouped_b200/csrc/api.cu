// api.cu -- the extern "C" entry points declared in include/gmm_fp8.h:
// argument validation, workspace carving, TMA tensor maps and launches.
// Nothing here allocates device memory; every buffer is the caller's.
#include <climits>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace gmm {

static uint64_t g_wait_limit_ns = kDefaultWaitLimitNs;
static int g_cta_pairs = GMM_TILES_AUTO;
// The automatic choice (measured on every workload, same box, 20-step runs):
// CTA pairs for the E4M3 tgmm (2-5 % faster: half of the lhs chunk per SM)
// and for the static E4M3 row passes when the groups average two row tiles
// or more (Mixtral forward 1.54 -> 1.45 ms, EP-merged 0.068 -> 0.060 ms);
// one-CTA tiles for the promoted row passes (pairs 8-60 % slower) and for the
// bf16 family.

// 256-row tiles over a CTA pair for the row passes when the groups average at
// least two such tiles (a group's last pair tile is half empty when its
// 128-row tile count is odd); for the tgmm when its rows do too and its dout
// columns split into 256-wide pair tiles.
static bool use_pairs(bool tgmm, int64_t M, int64_t N, int32_t G, int elem, bool promoted) {
  if (g_cta_pairs == GMM_TILES_ONE_CTA) return false;
  if (tgmm && N % 256) return false;
  if (g_cta_pairs == GMM_TILES_CTA_PAIRS || g_cta_pairs == GMM_TILES_CTA_PAIRS_NARROW) return true;
  if (elem != 1) return false;
  return tgmm || (!promoted && M >= 256 * static_cast<int64_t>(G));
}

// 128-column pair tiles (four TMEM accumulator buffers) for the promoted E4M3
// passes whose B operand is K-major
static constexpr bool kAutoNarrow = false;

static int tile_cols(bool pairs, bool promote_fp8, bool b_k_major, bool swiglu) {
  if (!pairs || !promote_fp8 || !b_k_major || swiglu) return 256;
  return (g_cta_pairs == GMM_TILES_CTA_PAIRS_NARROW || (kAutoNarrow && g_cta_pairs == GMM_TILES_AUTO)) ? 128 : 256;
}
static thread_local int32_t g_launches = 0;

// ------------------------------------------------------------ profiling

struct ProfRec {
  const char *name;
  cudaEvent_t a, b;
};
static std::mutex g_prof_mu;
static bool g_prof_on = false;
static std::vector<ProfRec> g_prof;
static std::vector<cudaEvent_t> g_event_pool;

static cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Runs one launch; when profiling is on, brackets it with events on `st`.
template <class F>
static cudaError_t prof(const char *name, cudaStream_t st, F &&launch) {
  if (!g_prof_on) return launch();
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ProfRec r{name, pool_event(), pool_event()};
  cudaEventRecord(r.a, st);
  cudaError_t e = launch();
  cudaEventRecord(r.b, st);
  g_prof.push_back(r);
  return e;
}

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int64_t chunk_capacity(int64_t rows, int32_t G) { return (rows + kBlk - 1) / kBlk + G; }

WsLayout ws_layout(gmm_op op, int64_t M, int64_t K, int64_t N, int32_t G) {
  WsLayout L{};
  size_t o = sizeof(WsHeader);
  L.plan_offs = o;
  o += align256(sizeof(int) * (G + 1));
  L.plan_tpre = o;
  o += align256(sizeof(int) * (G + 1));
  if (op == GMM_OP_FWD || op == GMM_OP_DLHS) {
    const int64_t C = (op == GMM_OP_FWD) ? K : N;  // contraction of the row operand
    L.codes_a = o;
    o += align256(static_cast<size_t>(M) * C);
    L.scales_a = o;
    o += align256(sizeof(float) * static_cast<size_t>(M) * (C / kBlk));
    L.codes_b = L.scales_b = 0;
    L.codes_r = L.scales_r = 0;
  } else {
    L.codes_r = L.scales_r = 0;
    // transposed, chunk-padded operands; sized for 2-byte elements so that the
    // bf16 family fits as well
    const int64_t cap = chunk_capacity(M, G);
    L.codes_a = o;
    o += align256(static_cast<size_t>(K) * kBlk * cap * 2);
    L.codes_b = o;
    o += align256(static_cast<size_t>(N) * kBlk * cap * 2);
    L.scales_a = o;
    o += align256(sizeof(float) * static_cast<size_t>(cap) * K);
    L.scales_b = o;
    o += align256(sizeof(float) * static_cast<size_t>(cap) * N);
    if (op == GMM_OP_BWD) {  // + the dlhs row operand of dout
      L.codes_r = o;
      o += align256(static_cast<size_t>(M) * N);
      L.scales_r = o;
      o += align256(sizeof(float) * static_cast<size_t>(M) * (N / kBlk));
    }
  }
  L.total = o;
  return L;
}

// ----------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major 2-D tensor [outer, inner] with a row pitch in bytes; box
// [box_outer, box_inner] with the 128-byte swizzle (box_inner * elem = 128).
static bool make_map(CUtensorMap *m, const void *base, int elem, uint64_t inner, uint64_t outer,
                     uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, elem == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output map for TMA stores: row-major [outer, inner] of f32 or bf16, no
// swizzle, box [box_outer, box_inner].
static bool make_out_map(CUtensorMap *m, const void *base, bool f32, uint64_t inner, uint64_t outer,
                         uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t esz = f32 ? 4 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * esz};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------ validation

static bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static gmm_status check_sizes(int64_t M, int64_t K, int64_t N, int32_t G) {
  if (M <= 0 || K <= 0 || N <= 0 || G <= 0) return GMM_ERR_SHAPE;
  if (K % kBlk || N % kBlk) return GMM_ERR_SHAPE;
  if (G > kMaxGroups) return GMM_ERR_UNSUPPORTED;
  // 32-bit tile coordinates and row indices
  if (M > (1 << 24) || K > (1 << 20) || N > (1 << 20) || static_cast<int64_t>(G) * (K > N ? K : N) > INT_MAX)
    return GMM_ERR_UNSUPPORTED;
  // the chunk quantizers index chunks by gridDim.y: ceil(M / 128) + G chunks at most
  if ((M + kBlk - 1) / kBlk + G > 65535) return GMM_ERR_UNSUPPORTED;
  return GMM_OK;
}

static gmm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GMM_OK : GMM_ERR_CUDA; }

// Launch size of a row pass (forward, dlhs) over `cols` output columns: one CTA
// per SM at most; for pairs the number of pair items (the launch caps it)
static int row_pass_grid(bool pairs, int64_t M, int64_t cols, int32_t G, int tn = 256) {
  const int64_t rows = pairs ? 256 : 128;
  const int64_t items = ((M + rows - 1) / rows + G) * ((cols + tn - 1) / tn);
  if (pairs) return static_cast<int>(items < INT_MAX ? items : INT_MAX);
  return static_cast<int>(items < num_sms() ? items : num_sms());
}

struct WsPtrs {
  uint32_t *status;
  int *offs, *tpre;
  uint8_t *codes_a, *codes_b, *codes_r;
  float *scales_a, *scales_b, *scales_r;
};

static WsPtrs carve(void *ws, const WsLayout &L) {
  uint8_t *w = static_cast<uint8_t *>(ws);
  WsPtrs P;
  P.status = reinterpret_cast<uint32_t *>(w);
  P.offs = reinterpret_cast<int *>(w + L.plan_offs);
  P.tpre = reinterpret_cast<int *>(w + L.plan_tpre);
  P.codes_a = w + L.codes_a;
  P.codes_b = L.codes_b ? w + L.codes_b : nullptr;
  P.scales_a = reinterpret_cast<float *>(w + L.scales_a);
  P.scales_b = L.scales_b ? reinterpret_cast<float *>(w + L.scales_b) : nullptr;
  P.codes_r = L.codes_r ? w + L.codes_r : nullptr;
  P.scales_r = L.scales_r ? reinterpret_cast<float *>(w + L.scales_r) : nullptr;
  return P;
}

// quantized (fp8) or bf16-family operand pair; returns the element size
static gmm_status classify(const gmm_operand &x, const gmm_operand &w, bool w_is_rhs, int *elem) {
  if (!x.data || !w.data) return GMM_ERR_INVALID_ARG;
  if (x.rule == GMM_Q_NONE) {
    if (x.dtype != GMM_BF16 || w.dtype != GMM_BF16) return GMM_ERR_INVALID_ARG;
    if (!w_is_rhs && w.rule != GMM_Q_NONE) return GMM_ERR_INVALID_ARG;
    *elem = 2;
    return GMM_OK;
  }
  if (x.rule != GMM_Q_STATIC && x.rule != GMM_Q_DYNAMIC) return GMM_ERR_INVALID_ARG;
  if (x.dtype == GMM_E4M3) {
    // pre-quantized lhs: its scales come with it (the forward takes either
    // rule, the tgmm the static one only)
    if (!x.scale || (!w_is_rhs && x.rule != GMM_Q_STATIC)) return GMM_ERR_INVALID_ARG;
  } else if (x.dtype != GMM_BF16) {
    return GMM_ERR_INVALID_ARG;
  }
  if (x.rule == GMM_Q_STATIC && !x.scale) return GMM_ERR_INVALID_ARG;  // a present rule must be applied
  if (w_is_rhs) {
    // rule NONE: per-channel scales [G, N]; DYNAMIC: block-wise scales
    if (w.dtype != GMM_E4M3 || !w.scale) return GMM_ERR_INVALID_ARG;
    if (w.rule != GMM_Q_NONE && w.rule != GMM_Q_DYNAMIC) return GMM_ERR_INVALID_ARG;
  } else {
    if (w.dtype != GMM_BF16 || w.rule != GMM_Q_DYNAMIC) return GMM_ERR_INVALID_ARG;
  }
  *elem = 1;
  return GMM_OK;
}

}  // namespace gmm

using namespace gmm;

extern "C" {

size_t gmm_workspace_bytes(gmm_op op, int64_t M, int64_t K, int64_t N, int32_t G) {
  if (check_sizes(M, K, N, G) != GMM_OK) return 0;
  if (op != GMM_OP_FWD && op != GMM_OP_DLHS && op != GMM_OP_DRHS && op != GMM_OP_BWD) return 0;
  return ws_layout(op, M, K, N, G).total;
}

int64_t gmm_chunk_capacity(int64_t rows, int32_t G) { return chunk_capacity(rows, G); }

const char *gmm_status_string(gmm_status s) {
  switch (s) {
    case GMM_OK: return "ok";
    case GMM_ERR_INVALID_ARG: return "invalid argument";
    case GMM_ERR_SHAPE: return "invalid shape (sizes must be positive, K and N multiples of 128)";
    case GMM_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case GMM_ERR_SCALE: return "static scale not finite or not above FLT_MIN";
    case GMM_ERR_UNSUPPORTED: return "unsupported size or option combination";
    case GMM_ERR_CUDA: return "CUDA runtime error";
    case GMM_ERR_GROUP_SIZES: return "group_sizes negative or summing past M";
    case GMM_ERR_TIMEOUT: return "a device wait timed out";
    case GMM_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int32_t gmm_last_launch_count(void) { return g_launches; }

void gmm_set_wait_limit_ns(uint64_t limit_ns) { g_wait_limit_ns = limit_ns ? limit_ns : kDefaultWaitLimitNs; }

gmm_status gmm_set_tiles(int32_t mode) {
  if (mode != GMM_TILES_AUTO && mode != GMM_TILES_ONE_CTA && mode != GMM_TILES_CTA_PAIRS &&
      mode != GMM_TILES_CTA_PAIRS_NARROW)
    return GMM_ERR_INVALID_ARG;
  g_cta_pairs = mode;
  return GMM_OK;
}

gmm_status gmm_quantize_rhs(const void *w_bf16, int32_t G, int64_t K, int64_t N, int transpose_out,
                            uint8_t *codes, float *scales, void *stream) {
  g_launches = 0;
  if (!w_bf16 || !codes || !scales) return GMM_ERR_INVALID_ARG;
  gmm_status s = check_sizes(1, K, N, G);
  if (s != GMM_OK) return s;
  if (!al16(w_bf16) || !al16(codes) || !al16(scales)) return GMM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = cuda_status(prof("quant_rhs", st, [&] {
    return launch_quant_rhs(w_bf16, G, K, N, transpose_out != 0, codes, scales, st);
  }));
  if (s == GMM_OK) g_launches = 3;
  return s;
}

gmm_status gmm_quantize_rhs_blocks(const void *w_bf16, int32_t G, int64_t K, int64_t N, int axis, uint8_t *codes,
                                   float *scales, void *stream) {
  g_launches = 0;
  if (!w_bf16 || !codes || !scales || (axis != 0 && axis != 1)) return GMM_ERR_INVALID_ARG;
  gmm_status s = check_sizes(1, K, N, G);
  if (s != GMM_OK) return s;
  if (!al16(w_bf16) || !al16(codes) || !al16(scales)) return GMM_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = cuda_status(prof("quant_rhs_blocks", st, [&] {
    return launch_quant_rhs_blocks(w_bf16, G, K, N, axis, codes, scales, st);
  }));
  if (s == GMM_OK) g_launches = 1;
  return s;
}

gmm_status gmm_quantize(const void *x_bf16, int64_t rows, int64_t cols, gmm_qrule rule, int axis,
                        const float *static_scale, const int32_t *group_sizes, int32_t G, const float *col_scale,
                        uint8_t *codes, float *scales, void *ws, size_t ws_bytes, void *stream) {
  g_launches = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!x_bf16 || !codes) return GMM_ERR_INVALID_ARG;
  if (rule != GMM_Q_STATIC && rule != GMM_Q_DYNAMIC) return GMM_ERR_INVALID_ARG;
  if (rule == GMM_Q_STATIC && !static_scale) return GMM_ERR_INVALID_ARG;
  if (rule == GMM_Q_DYNAMIC && !scales) return GMM_ERR_INVALID_ARG;
  if (axis != 0 && axis != 1) return GMM_ERR_INVALID_ARG;
  if ((axis == 0 || col_scale) && !group_sizes) return GMM_ERR_INVALID_ARG;
  if (axis == 0 && !scales) return GMM_ERR_INVALID_ARG;
  if (col_scale && rule != GMM_Q_DYNAMIC) return GMM_ERR_INVALID_ARG;
  const int32_t Gq = group_sizes ? G : 1;
  gmm_status s = check_sizes(rows, cols, cols, Gq);
  if (s != GMM_OK) return s;
  if (!al16(x_bf16) || !al16(codes) || (scales && !al16(scales)) || (col_scale && !al16(col_scale)))
    return GMM_ERR_ALIGNMENT;
  // the plan and status live in the first part of any pass's workspace
  const WsLayout L = ws_layout(GMM_OP_FWD, 1, kBlk, kBlk, Gq);
  if (!ws || ws_bytes < L.codes_a) return GMM_ERR_WORKSPACE;
  WsPtrs P = carve(ws, L);
  int n = 0;
  if (group_sizes) {
    s = cuda_status(prof("plan", st, [&] { return launch_plan(group_sizes, Gq, rows, P.offs, P.tpre, P.status, st); }));
    ++n;
  } else {
    s = cuda_status(cudaMemsetAsync(P.status, 0, sizeof(uint32_t), st));
  }
  if (s != GMM_OK) return s;
  const bool dyn = rule == GMM_Q_DYNAMIC;
  if (axis == 1)
    s = cuda_status(prof("quant_rows", st, [&] {
      return launch_quant_rows(x_bf16, rows, cols, dyn, dyn ? nullptr : static_scale, col_scale, P.offs, Gq, codes,
                               scales, P.status, st);
    }));
  else
    s = cuda_status(prof("quant_chunks", st, [&] {
      return launch_quant_chunks(x_bf16, rows, cols, dyn, dyn ? nullptr : static_scale, P.offs, P.tpre, Gq,
                                 chunk_capacity(rows, Gq), codes, scales, false, P.status, st);
    }));
  if (s == GMM_OK) g_launches = n + 1;
  return s;
}

}  // extern "C"

// Forward pass shared by gmm_fwd (F == 0), gmm_fwd_swiglu (F = N / 2) and
// gmm_fwd_keep_lhs (codes_out != NULL: the lhs codes and dynamic scales are
// written to the caller's buffers instead of the workspace).
static gmm_status fwd_impl(gmm_operand lhs, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes, int32_t G,
                           int64_t M, int64_t K, int64_t N, void *out, gmm_dtype out_dtype, void *ws, size_t ws_bytes,
                           void *stream, int64_t F, uint8_t *codes_out = nullptr, float *scales_out = nullptr) {
  g_launches = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gmm_status s = check_sizes(M, K, N, G);
  if (s != GMM_OK) return s;
  if (F && N != 2 * F) return GMM_ERR_SHAPE;
  if (!group_sizes || !out) return GMM_ERR_INVALID_ARG;
  if (out_dtype != GMM_BF16 && out_dtype != GMM_F32) return GMM_ERR_INVALID_ARG;
  int elem = 0;
  if ((s = classify(lhs, rhs, true, &elem)) != GMM_OK) return s;
  if (!al16(lhs.data) || !al16(rhs.data) || !al16(out) || !al16(ws) || (rhs.scale && !al16(rhs.scale)))
    return GMM_ERR_ALIGNMENT;
  const WsLayout L = ws_layout(GMM_OP_FWD, M, K, N, G);
  if (!ws || ws_bytes < L.total) return GMM_ERR_WORKSPACE;
  WsPtrs P = carve(ws, L);
  if ((s = cuda_status(prof("plan", st, [&] { return launch_plan(group_sizes, G, M, P.offs, P.tpre, P.status, st); }))) != GMM_OK) return s;
  int n = 1;
  const bool dyn = lhs.rule == GMM_Q_DYNAMIC;
  const bool preq = lhs.dtype == GMM_E4M3;  // codes and scales supplied by the caller
  const bool blk = elem == 1 && rhs.rule == GMM_Q_DYNAMIC;  // block-wise rhs scales [G, K/128, N]
  if (blk && transpose_rhs) return GMM_ERR_UNSUPPORTED;
  const void *A = lhs.data;
  uint8_t *codes = codes_out ? codes_out : P.codes_a;
  float *qscales = (codes_out && dyn) ? scales_out : P.scales_a;
  if (elem == 1 && !preq) {
    s = cuda_status(prof("quant_rows", st, [&] {
      return launch_quant_rows(lhs.data, M, K, dyn, dyn ? nullptr : lhs.scale, nullptr, P.offs, G, codes, qscales,
                               P.status, st);
    }));
    if (s != GMM_OK) return s;
    ++n;
    A = codes;
  }
  const bool bmn = transpose_rhs == 0;  // [G, K, N]: N contiguous = MN-major B
  const uint32_t bke = 128 / elem;
  const bool pairs = use_pairs(false, M, N, G, elem, dyn || blk);
  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, A, elem, K, M, K * elem, bke, 128)) return GMM_ERR_CUDA;
  // SwiGLU tiles take the gate rows and the up rows of a K-major rhs as two
  // 128-row boxes
  const int tn = tile_cols(pairs, elem == 1 && (dyn || blk), !bmn, F != 0);
  const bool okB = bmn ? make_map(&tmB, rhs.data, elem, N, static_cast<uint64_t>(G) * K, N * elem, bke, bke)
                       : make_map(&tmB, rhs.data, elem, K, static_cast<uint64_t>(G) * N, K * elem, bke,
                                  pairs ? tn / 2 : (F ? 128 : 256));
  if (!okB) return GMM_ERR_CUDA;
  GemmParams p{};
  p.G = G;
  p.M = static_cast<int>(M);
  p.ncols = static_cast<int>(N);
  p.swiglu_f = static_cast<int>(F);
  p.kblocks = static_cast<int>(K / bke);
  p.b_group_rows = static_cast<int>(bmn ? K : N);
  p.offs = P.offs;
  p.tpre = P.tpre;
  p.row_scale = (elem == 1 && dyn) ? (preq ? lhs.scale : qscales) : nullptr;
  p.row_scale_ld = M;
  p.col_scale = (elem == 1 && !blk) ? rhs.scale : nullptr;
  p.colblk_scale = blk ? rhs.scale : nullptr;
  p.colblk_ld = N;
  p.static_scale = (elem == 1 && !dyn) ? lhs.scale : nullptr;
  p.out = out;
  p.out_f32 = out_dtype == GMM_F32;
  p.ld_out = F ? F : N;
  p.status = P.status;
  p.wait_limit_ns = g_wait_limit_ns;
  // per-block promotion for dynamic lhs scales or block-wise rhs scales
  const GemmConfig cfg{blk ? MODE_ROWS_BLK : MODE_ROWS, elem, bmn, elem == 1 && (dyn || blk), pairs,
                       blk ? 256 : tn};
  const int grid = row_pass_grid(pairs, M, N, G, cfg.tile_n);
  if ((s = cuda_status(prof(F ? "gemm_fwd_swiglu" : "gemm_fwd", st,
                            [&] { return launch_gemm(cfg, tmA, tmB, tmA, p, grid, st); }))) != GMM_OK)
    return s;
  g_launches = n + 1;
  return GMM_OK;
}

extern "C" {

gmm_status gmm_fwd(gmm_operand lhs, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes, int32_t G,
                   int64_t M, int64_t K, int64_t N, void *out, gmm_dtype out_dtype, void *ws, size_t ws_bytes,
                   void *stream) {
  return fwd_impl(lhs, rhs, transpose_rhs, group_sizes, G, M, K, N, out, out_dtype, ws, ws_bytes, stream, 0);
}

gmm_status gmm_fwd_keep_lhs(gmm_operand lhs, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes,
                            int32_t G, int64_t M, int64_t K, int64_t N, void *out, gmm_dtype out_dtype, void *ws,
                            size_t ws_bytes, uint8_t *lhs_codes, float *lhs_scales, void *stream) {
  g_launches = 0;
  if (!lhs_codes || lhs.dtype != GMM_BF16 || (lhs.rule != GMM_Q_STATIC && lhs.rule != GMM_Q_DYNAMIC))
    return GMM_ERR_INVALID_ARG;
  if (lhs.rule == GMM_Q_DYNAMIC && !lhs_scales) return GMM_ERR_INVALID_ARG;
  if (!al16(lhs_codes) || (lhs_scales && !al16(lhs_scales))) return GMM_ERR_ALIGNMENT;
  return fwd_impl(lhs, rhs, transpose_rhs, group_sizes, G, M, K, N, out, out_dtype, ws, ws_bytes, stream, 0,
                  lhs_codes, lhs_scales);
}

gmm_status gmm_fwd_swiglu(gmm_operand lhs, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes,
                          int32_t G, int64_t M, int64_t K, int64_t N, void *out, gmm_dtype out_dtype, void *ws,
                          size_t ws_bytes, void *stream) {
  g_launches = 0;
  if (N <= 0 || N % (2 * kBlk)) return GMM_ERR_SHAPE;
  return fwd_impl(lhs, rhs, transpose_rhs, group_sizes, G, M, K, N, out, out_dtype, ws, ws_bytes, stream, N / 2);
}

}  // extern "C"

// dlhs GEMM on the row operand A [M, N]: E4M3 codes with block scales
// A_scales [N/128, M] (elem 1) or bf16 dout (elem 2).  blk: block-wise rhs
// scales [G, N/128, K] (A then carries no rhs scale).
static gmm_status run_dlhs_gemm(const void *A, const float *A_scales, int elem, const gmm_operand &rhs,
                                int transpose_rhs, bool blk, const WsPtrs &P, int32_t G, int64_t M, int64_t K,
                                int64_t N, void *dlhs, gmm_dtype out_dtype, cudaStream_t st) {
  const bool bmn = transpose_rhs != 0;  // [G, N, K]: K contiguous = MN-major B for dlhs
  const uint32_t bke = 128 / elem;
  const bool pairs = use_pairs(false, M, K, G, elem, elem == 1);
  const int tn = tile_cols(pairs, elem == 1, !bmn, false);
  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, A, elem, N, M, N * elem, bke, 128)) return GMM_ERR_CUDA;
  const bool okB = bmn ? make_map(&tmB, rhs.data, elem, K, static_cast<uint64_t>(G) * N, K * elem, bke, bke)
                       : make_map(&tmB, rhs.data, elem, N, static_cast<uint64_t>(G) * K, N * elem, bke,
                                  pairs ? tn / 2 : 256);
  if (!okB) return GMM_ERR_CUDA;
  GemmParams p{};
  p.G = G;
  p.M = static_cast<int>(M);
  p.ncols = static_cast<int>(K);
  p.kblocks = static_cast<int>(N / bke);
  p.b_group_rows = static_cast<int>(bmn ? N : K);
  p.offs = P.offs;
  p.tpre = P.tpre;
  p.row_scale = elem == 1 ? A_scales : nullptr;
  p.row_scale_ld = M;
  p.col_scale = nullptr;
  p.colblk_scale = blk ? rhs.scale : nullptr;
  p.colblk_ld = K;
  p.static_scale = nullptr;
  p.out = dlhs;
  p.out_f32 = out_dtype == GMM_F32;
  p.ld_out = K;
  p.status = P.status;
  p.wait_limit_ns = g_wait_limit_ns;
  const GemmConfig cfg{blk ? MODE_ROWS_BLK : MODE_ROWS, elem, bmn, elem == 1, pairs, tn};
  const int grid = row_pass_grid(pairs, M, K, G, tn);
  return cuda_status(prof("gemm_dlhs", st, [&] { return launch_gemm(cfg, tmA, tmB, tmA, p, grid, st); }));
}

// tgmm GEMM on the chunk-major operands in the workspace (codes_a: lhs,
// codes_b: dout; scales_a / scales_b their chunk scales).
static gmm_status run_drhs_gemm(int elem, bool dyn, const float *static_scale, int64_t cap, const WsPtrs &P,
                                int32_t G, int64_t M, int64_t K, int64_t N, void *drhs, gmm_dtype out_dtype,
                                cudaStream_t st) {
  const uint32_t bke = 128 / elem;
  // tile rows = dout columns n (A = dout^T chunks), tile columns = lhs columns
  // k (B = lhs^T chunks); the epilogue writes dW[g, k, n].  The chunk-major
  // operands [chunk][column][128] are 2-D tensors of 128-element lines: chunk
  // j's line of column c is row j * C + c, so every box is one contiguous block.
  const bool pairs = use_pairs(true, M, N, G, elem, elem == 1);
  const int tn = tile_cols(pairs, elem == 1, true, false);
  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, P.codes_b, elem, kBlk, static_cast<uint64_t>(cap) * N, kBlk * elem, bke, 128))
    return GMM_ERR_CUDA;
  if (!make_map(&tmB, P.codes_a, elem, kBlk, static_cast<uint64_t>(cap) * K, kBlk * elem, bke, pairs ? tn / 2 : 256))
    return GMM_ERR_CUDA;
  CUtensorMap tmOut;  // dW as [G*K, N]: each epilogue warp stores 32 k-rows x 32 n
  if (!make_out_map(&tmOut, drhs, out_dtype == GMM_F32, N, static_cast<uint64_t>(G) * K, 32, 32))
    return GMM_ERR_CUDA;
  GemmParams p{};
  p.G = G;
  p.M = static_cast<int>(M);
  p.ncols = static_cast<int>(K);
  p.rtiles = static_cast<int>(N / kBlk);
  p.stages_per_chunk = elem;
  p.offs = P.offs;
  p.tpre = P.tpre;
  // fp8: dout chunk scales per tile row; lhs chunk scales per tile column
  // (dynamic rule) or the static scale; the bf16 family has no scales
  p.row_scale = elem == 1 ? P.scales_b : nullptr;
  p.row_scale_ld = N;
  p.colblk_scale = (elem == 1 && dyn) ? P.scales_a : nullptr;
  p.colblk_ld = K;
  p.static_scale = (elem == 1 && !dyn) ? static_scale : nullptr;
  // groups averaging under 512 rows: row tiles fastest (see GemmParams)
  p.tg_rows_fastest = M < 512 * static_cast<int64_t>(G) ? 1 : 0;
  p.out = drhs;
  p.out_f32 = out_dtype == GMM_F32;
  p.ld_out = N;
  p.status = P.status;
  p.wait_limit_ns = g_wait_limit_ns;
  const GemmConfig cfg{MODE_TGMM, elem, false, elem == 1, pairs, tn};
  const int64_t items = static_cast<int64_t>(G) * (N / (pairs ? 2 * kBlk : kBlk)) * ((K + tn - 1) / tn);
  const int grid = pairs ? static_cast<int>(items < INT_MAX ? items : INT_MAX)
                         : static_cast<int>(items < num_sms() ? items : num_sms());
  return cuda_status(prof("gemm_drhs", st, [&] { return launch_gemm(cfg, tmA, tmB, tmOut, p, grid, st); }));
}

// The tgmm lhs operand into the workspace: quantized per chunk, re-laid out
// when the caller gives the forward's static codes, or copied (bf16 family).
static gmm_status prepare_tgmm_lhs(const gmm_operand &lhs, int elem, int64_t cap, const WsPtrs &P, int32_t G,
                                   int64_t M, int64_t K, cudaStream_t st) {
  const bool dyn = lhs.rule == GMM_Q_DYNAMIC;
  if (lhs.dtype == GMM_E4M3)  // static codes given: re-laid out only
    return cuda_status(prof("chunk_codes", st, [&] {
      return launch_chunk_codes(static_cast<const uint8_t *>(lhs.data), M, K, P.offs, P.tpre, G, cap, P.codes_a, st);
    }));
  return cuda_status(prof("quant_chunks", st, [&] {
    return launch_quant_chunks(lhs.data, M, K, dyn, (elem == 1 && !dyn) ? lhs.scale : nullptr, P.offs, P.tpre, G, cap,
                               P.codes_a, P.scales_a, elem == 2, P.status, st);
  }));
}

// dlhs argument checks shared by gmm_dlhs and gmm_backward
static gmm_status check_dlhs(const gmm_operand &dout, const gmm_operand &rhs, int transpose_rhs, int *elem) {
  gmm_status s = classify(dout, rhs, true, elem);
  if (s != GMM_OK) return s;
  if (*elem == 1 && dout.rule != GMM_Q_DYNAMIC) return GMM_ERR_INVALID_ARG;  // gradients: dynamic blocks
  if (dout.dtype != GMM_BF16) return GMM_ERR_INVALID_ARG;                    // the rhs scale is folded in
  if (*elem == 1 && rhs.rule == GMM_Q_DYNAMIC && transpose_rhs) return GMM_ERR_UNSUPPORTED;
  return GMM_OK;
}

extern "C" {

gmm_status gmm_dlhs(gmm_operand dout, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes, int32_t G,
                    int64_t M, int64_t K, int64_t N, void *dlhs, gmm_dtype out_dtype, void *ws, size_t ws_bytes,
                    void *stream) {
  g_launches = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gmm_status s = check_sizes(M, K, N, G);
  if (s != GMM_OK) return s;
  if (!group_sizes || !dlhs) return GMM_ERR_INVALID_ARG;
  if (out_dtype != GMM_BF16 && out_dtype != GMM_F32) return GMM_ERR_INVALID_ARG;
  int elem = 0;
  if ((s = check_dlhs(dout, rhs, transpose_rhs, &elem)) != GMM_OK) return s;
  if (!al16(dout.data) || !al16(rhs.data) || !al16(dlhs) || !al16(ws) || (rhs.scale && !al16(rhs.scale)))
    return GMM_ERR_ALIGNMENT;
  const WsLayout L = ws_layout(GMM_OP_DLHS, M, K, N, G);
  if (!ws || ws_bytes < L.total) return GMM_ERR_WORKSPACE;
  WsPtrs P = carve(ws, L);
  if ((s = cuda_status(prof("plan", st, [&] { return launch_plan(group_sizes, G, M, P.offs, P.tpre, P.status, st); }))) != GMM_OK) return s;
  int n = 1;
  const void *A = dout.data;
  // block-wise rhs scales along n ([G, N/128, K]): they vary along k as well,
  // so dout is quantized on its own and both scales are applied per block
  const bool blk = elem == 1 && rhs.rule == GMM_Q_DYNAMIC;
  if (elem == 1) {
    // per-channel rhs: t = fl32(dout * s_r[g(m), n]); dynamic 128-blocks along n
    s = cuda_status(prof("quant_rows", st, [&] {
      return launch_quant_rows(dout.data, M, N, true, nullptr, blk ? nullptr : rhs.scale, P.offs, G, P.codes_a,
                               P.scales_a, P.status, st);
    }));
    if (s != GMM_OK) return s;
    ++n;
    A = P.codes_a;
  }
  if ((s = run_dlhs_gemm(A, P.scales_a, elem, rhs, transpose_rhs, blk, P, G, M, K, N, dlhs, out_dtype, st)) != GMM_OK)
    return s;
  g_launches = n + 1;
  return GMM_OK;
}

gmm_status tgmm_drhs(gmm_operand lhs, gmm_operand dout, const int32_t *group_sizes, int32_t G, int64_t M,
                     int64_t K, int64_t N, void *drhs, gmm_dtype out_dtype, void *ws, size_t ws_bytes,
                     void *stream) {
  g_launches = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gmm_status s = check_sizes(M, K, N, G);
  if (s != GMM_OK) return s;
  if (!group_sizes || !drhs) return GMM_ERR_INVALID_ARG;
  if (out_dtype != GMM_BF16 && out_dtype != GMM_F32) return GMM_ERR_INVALID_ARG;
  int elem = 0;
  if ((s = classify(lhs, dout, false, &elem)) != GMM_OK) return s;
  if (!al16(lhs.data) || !al16(dout.data) || !al16(drhs) || !al16(ws)) return GMM_ERR_ALIGNMENT;
  const WsLayout L = ws_layout(GMM_OP_DRHS, M, K, N, G);
  if (!ws || ws_bytes < L.total) return GMM_ERR_WORKSPACE;
  WsPtrs P = carve(ws, L);
  if ((s = cuda_status(prof("plan", st, [&] { return launch_plan(group_sizes, G, M, P.offs, P.tpre, P.status, st); }))) != GMM_OK) return s;
  const int64_t cap = chunk_capacity(M, G);
  if ((s = prepare_tgmm_lhs(lhs, elem, cap, P, G, M, K, st)) != GMM_OK) return s;
  s = cuda_status(prof("quant_chunks", st, [&] {
    return launch_quant_chunks(dout.data, M, N, true, nullptr, P.offs, P.tpre, G, cap, P.codes_b, P.scales_b,
                               elem == 2, P.status, st);
  }));
  if (s != GMM_OK) return s;
  if ((s = run_drhs_gemm(elem, lhs.rule == GMM_Q_DYNAMIC, lhs.scale, cap, P, G, M, K, N, drhs, out_dtype, st)) !=
      GMM_OK)
    return s;
  g_launches = 4;
  return GMM_OK;
}

gmm_status gmm_backward(gmm_operand lhs, gmm_operand dout, gmm_operand rhs, int transpose_rhs,
                        const int32_t *group_sizes, int32_t G, int64_t M, int64_t K, int64_t N, void *dlhs,
                        gmm_dtype dlhs_dtype, void *drhs, gmm_dtype drhs_dtype, void *ws, size_t ws_bytes,
                        void *stream) {
  g_launches = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gmm_status s = check_sizes(M, K, N, G);
  if (s != GMM_OK) return s;
  if (!group_sizes || !dlhs || !drhs) return GMM_ERR_INVALID_ARG;
  if ((dlhs_dtype != GMM_BF16 && dlhs_dtype != GMM_F32) || (drhs_dtype != GMM_BF16 && drhs_dtype != GMM_F32))
    return GMM_ERR_INVALID_ARG;
  int elem = 0, elem_t = 0;
  if ((s = check_dlhs(dout, rhs, transpose_rhs, &elem)) != GMM_OK) return s;
  if ((s = classify(lhs, dout, false, &elem_t)) != GMM_OK) return s;
  if (elem != elem_t) return GMM_ERR_INVALID_ARG;  // both passes in the same family
  if (!al16(lhs.data) || !al16(dout.data) || !al16(rhs.data) || !al16(dlhs) || !al16(drhs) || !al16(ws) ||
      (rhs.scale && !al16(rhs.scale)))
    return GMM_ERR_ALIGNMENT;
  const WsLayout L = ws_layout(GMM_OP_BWD, M, K, N, G);
  if (!ws || ws_bytes < L.total) return GMM_ERR_WORKSPACE;
  WsPtrs P = carve(ws, L);
  if ((s = cuda_status(prof("plan", st, [&] { return launch_plan(group_sizes, G, M, P.offs, P.tpre, P.status, st); }))) != GMM_OK) return s;
  const int64_t cap = chunk_capacity(M, G);
  if ((s = prepare_tgmm_lhs(lhs, elem, cap, P, G, M, K, st)) != GMM_OK) return s;
  const bool blk = elem == 1 && rhs.rule == GMM_Q_DYNAMIC;
  const void *A = dout.data;
  if (elem == 1) {
    // one read of dout gives both operands: dlhs row blocks (per-channel rhs
    // scale folded in) and the tgmm chunk columns
    s = cuda_status(prof("quant_dout", st, [&] {
      return launch_quant_dout_both(dout.data, M, N, blk ? nullptr : rhs.scale, P.offs, P.tpre, G, cap, P.codes_b,
                                    P.scales_b, P.codes_r, P.scales_r, st);
    }));
    A = P.codes_r;
  } else {
    s = cuda_status(prof("quant_chunks", st, [&] {
      return launch_quant_chunks(dout.data, M, N, true, nullptr, P.offs, P.tpre, G, cap, P.codes_b, P.scales_b, true,
                                 P.status, st);
    }));
  }
  if (s != GMM_OK) return s;
  if ((s = run_dlhs_gemm(A, P.scales_r, elem, rhs, transpose_rhs, blk, P, G, M, K, N, dlhs, dlhs_dtype, st)) !=
      GMM_OK)
    return s;
  if ((s = run_drhs_gemm(elem, lhs.rule == GMM_Q_DYNAMIC, lhs.scale, cap, P, G, M, K, N, drhs, drhs_dtype, st)) !=
      GMM_OK)
    return s;
  g_launches = 5;
  return GMM_OK;
}

gmm_status gmm_read_device_status(const void *ws, uint32_t *bits_out, void *stream) {
  if (!ws) return GMM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t bits = 0;
  if (cudaMemcpyAsync(&bits, ws, sizeof(bits), cudaMemcpyDeviceToHost, st) != cudaSuccess) return GMM_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GMM_ERR_CUDA;
  if (bits_out) *bits_out = bits;
  if (bits & GMM_DEV_TIMEOUT) return GMM_ERR_TIMEOUT;
  if (bits & GMM_DEV_SCALE) return GMM_ERR_SCALE;
  if (bits & GMM_DEV_GROUP_SIZES) return GMM_ERR_GROUP_SIZES;
  return GMM_OK;
}

gmm_status gmm_selftest_timeout(void *ws, uint64_t limit_ns, void *stream) {
  g_launches = 0;
  if (!ws) return GMM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *status = static_cast<uint32_t *>(ws);
  gmm_status s = cuda_status(cudaMemsetAsync(status, 0, sizeof(uint32_t), st));
  if (s != GMM_OK) return s;
  s = cuda_status(launch_timeout_selftest(status, limit_ns, st));
  if (s == GMM_OK) g_launches = 1;
  return s;
}

void gmm_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
}

int32_t gmm_profile_collect(gmm_profile_entry *entries, int32_t max_entries) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  // names point at string literals of this library, so they stay valid
  std::map<std::string, std::pair<const char *, std::pair<int32_t, double>>> agg;
  for (ProfRec &r : g_prof) {
    float ms = 0.0f;
    cudaEventSynchronize(r.b);
    cudaEventElapsedTime(&ms, r.a, r.b);
    auto &x = agg[r.name];
    x.first = r.name;
    x.second.first += 1;
    x.second.second += ms;
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof.clear();
  int32_t n = 0;
  for (auto &kv : agg) {
    if (n >= max_entries) break;
    entries[n].name = kv.second.first;
    entries[n].launches = kv.second.second.first;
    entries[n].total_ms = kv.second.second.second;
    ++n;
  }
  return n;
}

}  // extern "C"
