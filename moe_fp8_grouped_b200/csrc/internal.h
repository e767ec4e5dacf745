// internal.h -- declarations shared by the C-ABI layer (api.cu) and the
// kernels (plan_quant.cu, gemm_tc.cu).  Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "gmm_fp8.h"

namespace gmm {

constexpr int kBlk = 128;         // quantization block / chunk length
constexpr int kMaxGroups = 1024;  // groups handled per call
constexpr uint64_t kDefaultWaitLimitNs = 4000000000ull;

// Workspace: a 256-byte header (status word), the group plan, then the
// quantized operands of the pass.
struct WsHeader {
  uint32_t status;  // GMM_DEV_* bits of the last call
  uint32_t pad[63];
};

struct WsLayout {
  size_t plan_offs;    // int32 [G + 1] row offsets (clamped)
  size_t plan_tpre;    // int32 [G + 1] prefix of 128-row tiles / chunks per group
  size_t codes_a;      // operand A codes
  size_t codes_b;      // operand B codes (tgmm only)
  size_t scales_a;     // fp32 scales of A
  size_t scales_b;     // fp32 scales of B (tgmm only)
  size_t codes_r;      // dlhs row codes of dout (fused backward only)
  size_t scales_r;     // their block scales [N/128, M]
  size_t total;
};

WsLayout ws_layout(gmm_op op, int64_t M, int64_t K, int64_t N, int32_t G);

// Group plan: validates group_sizes, writes clamped offsets and the tile
// prefix, and resets the status word to the group-size verdict.
cudaError_t launch_plan(const int32_t *sizes, int G, int64_t M, int *offs, int *tpre, uint32_t *status,
                        cudaStream_t st);

// Row quantizer (axis 1).  static_scale != NULL selects the static rule;
// col_scale != NULL folds col_scale[g(m), n] in (needs offs).
cudaError_t launch_quant_rows(const void *x, int64_t rows, int64_t cols, bool dynamic, const float *static_scale,
                              const float *col_scale, const int *offs, int G, uint8_t *codes, float *scales,
                              uint32_t *status, cudaStream_t st);

// Chunk quantizer (axis 0, tgmm operand), transposed + padded codes.
// bf16_copy: write the bf16 values instead of codes (bf16 family packing).
cudaError_t launch_quant_chunks(const void *x, int64_t rows, int64_t cols, bool dynamic, const float *static_scale,
                                const int *offs, const int *tpre, int G, int64_t capacity, void *codes_t,
                                float *scales, bool bf16_copy, uint32_t *status, cudaStream_t st);

// Backward dout, both quantized layouts from one read: the tgmm chunk operand
// (as launch_quant_chunks, dynamic) and the dlhs row operand (as
// launch_quant_rows, dynamic, col_scale folded in when not NULL).  Rows in no
// group are left unwritten in the row operand (no GEMM tile keeps them).
cudaError_t launch_quant_dout_both(const void *x, int64_t rows, int64_t cols, const float *col_scale, const int *offs,
                                   const int *tpre, int G, int64_t capacity, void *codes_t, float *scales_t,
                                   uint8_t *codes_r, float *scales_r, cudaStream_t st);

// Already-quantized E4M3 rows [rows, cols] into the chunk layout of
// launch_quant_chunks (codes only).
cudaError_t launch_chunk_codes(const uint8_t *codes, int64_t rows, int64_t cols, const int *offs, const int *tpre,
                               int G, int64_t capacity, uint8_t *codes_t, cudaStream_t st);

cudaError_t launch_quant_rhs(const void *w, int G, int64_t K, int64_t N, bool transpose_out, uint8_t *codes,
                             float *scales, cudaStream_t st);

// Block-wise weight quantizer: axis 0 scales [G, K/128, N], axis 1 [G, N/128, K].
cudaError_t launch_quant_rhs_blocks(const void *w, int G, int64_t K, int64_t N, int axis, uint8_t *codes,
                                    float *scales, cudaStream_t st);

cudaError_t launch_timeout_selftest(uint32_t *status, uint64_t limit_ns, cudaStream_t st);

// MODE_ROWS_BLK: MODE_ROWS whose rhs has block-wise scales (a column scale per
// contraction block, applied per TMEM unit); a separate instantiation so that
// the per-channel kernels carry none of its code.
enum GemmMode { MODE_ROWS = 0, MODE_TGMM = 1, MODE_ROWS_BLK = 2 };

// Tile space of one GEMM launch.  MODE_ROWS (forward, dlhs): tile rows are
// 128-row slices of one group's rows, tile columns the output columns.
// MODE_TGMM (drhs): tile rows are 128 dout columns n, tile columns 256 lhs
// columns k, the contraction runs over the group's 128-row chunks, and the
// result is written transposed into dW[g, k, n].
struct GemmParams {
  int G;
  int M;               // rows of the row operand (MODE_ROWS) / of x (MODE_TGMM)
  int ncols;           // tile-space columns: N (forward), K (dlhs, tgmm)
  int kblocks;         // MODE_ROWS: contraction stages (128 bytes of operand row each)
  int rtiles;          // MODE_TGMM: 128-row tiles (N / 128)
  int b_group_rows;    // MODE_ROWS: rows per group in B's 2-D view
  int stages_per_chunk;// MODE_TGMM: stages per 128-row chunk (1 fp8, 2 bf16)
  const int *offs;     // [G + 1]
  const int *tpre;     // [G + 1]
  const float *row_scale;     // MODE_ROWS: [kblocks][M]; MODE_TGMM: dout chunk scales [chunk][N]
  int64_t row_scale_ld;
  const float *colblk_scale;  // per-unit column scales.  MODE_TGMM, dynamic x: lhs chunk
                              // scales [chunk][K]; MODE_ROWS: block-wise rhs scales
                              // [G][kblocks][ncols] (then col_scale is NULL)
  int64_t colblk_ld;
  const float *col_scale;     // MODE_ROWS: [G][ncols] final per-column scale, or NULL
  const float *static_scale;  // device scalar multiplied in at the end, or NULL
  void *out;
  int out_f32;
  int64_t ld_out;             // MODE_ROWS: output row pitch; MODE_TGMM: N
  int swiglu_f;               // MODE_ROWS forward: F > 0 fuses SwiGLU over the merged
                              // columns [0, F) gate | [F, 2F) up and writes [M, F];
                              // 0 writes the plain product
  int tg_rows_fastest;        // MODE_TGMM item order within a group: 1 = row tiles (dout
                              // columns) fastest, each lhs column tile reused by
                              // consecutive items; 0 = column tiles fastest
  uint32_t *status;
  uint64_t wait_limit_ns;
};

struct GemmConfig {
  int mode;         // GemmMode
  int elem_bytes;   // 1: E4M3 (kind::f8f6f4), 2: BF16 (kind::f16)
  bool b_mn_major;  // B operand MN-major in shared memory
  bool promote;     // one TMEM unit per contraction block, promoted in registers
  bool cta_pairs;   // 256-row tiles over a cluster of two CTAs (M = 256 MMAs);
                    // the B tensor map's K-major box is then tile_n / 2 rows
  int tile_n;       // tile columns: 256, or 128 (CTA pairs, promoted E4M3,
                    // K-major B: four TMEM accumulator buffers)
};

int num_sms();

// tmOut: the output as a TMA tensor (MODE_TGMM: dW [G*K, N], box 32 x 32);
// unused by MODE_ROWS.  grid: CTAs (one-CTA tiles) or items (pairs; the
// launch caps it at the pairs that fit on the GPU at once).
cudaError_t launch_gemm(const GemmConfig &cfg, const CUtensorMap &tmA, const CUtensorMap &tmB,
                        const CUtensorMap &tmOut, const GemmParams &p, int grid, cudaStream_t st);

// The CTA-pair kernels (gemm_pair.cu); launch_gemm dispatches to them.
cudaError_t launch_gemm_pair(const GemmConfig &cfg, const CUtensorMap &tmA, const CUtensorMap &tmB,
                             const CUtensorMap &tmOut, const GemmParams &p, int items, cudaStream_t st);

}  // namespace gmm
