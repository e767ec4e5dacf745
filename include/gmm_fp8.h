/*
 * gmm_fp8.h -- C-ABI of the B200 (sm_100a) FP8 grouped matmul library
 * (libgmm_fp8.so): forward gmm, backward gmm wrt lhs (dlhs) and the transposed
 * gmm wrt rhs (tgmm drhs) of Mixture-of-Experts expert MLPs.
 *
 * The operations (sources named by page title and section):
 *   forward   out[m, :] = lhs[m, :] @ rhs[g(m)], rows sorted by expert and
 *             partitioned by group_sizes ("FP8 Megablox for batch split",
 *             maxtext PR #3770, Description; "Support quantization for
 *             tokamax gmm v2", maxtext PR #4451, Description).
 *   dlhs      dlhs[m, :] = dout[m, :] @ rhs[g(m)]^T, a gmm against the same
 *             rhs with the transpose flag flipped (PR #4451, review thread on
 *             ops.py).
 *   drhs      dW[g] = lhs[rows of g]^T @ dout[rows of g], the transposed gmm
 *             ("drhs_tgmm2", PR #4451, Description).
 * FP8 recipe: lhs arrives unquantized and is quantized inside the call as
 * clip(lhs / scale) to E4M3 with a static per-tensor [1, 1] scale or a dynamic
 * per-block absmax scale, and results are multiplied back by the scales
 * ("add static LHS scaling support for GMM v2 FWD", maxtext PR #4735, review
 * threads on the LhsRef docstring and on inner_kernel).  rhs arrives already
 * quantized with a per-channel scale of shape [G, N] (PR #3770 Description:
 * weights quantized manually; PR #4451 review thread: a 2-D scale is per
 * channel).  Gradients are quantized too (PR #3770 Description).
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers of the current CUDA device unless a
 *    comment says otherwise.  The caller owns every buffer; the library never
 *    allocates or frees device memory.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous on it; no call synchronizes except gmm_read_device_status.
 *  - Matrices are row-major and dense (leading dimension = number of columns).
 *  - Errors that the host can see (null pointers, bad sizes, misalignment,
 *    a rule with no scale, a too-small workspace) return before anything is
 *    launched.  Errors that only the device can see (bad group_sizes, an
 *    unusable static scale, a wait that timed out) set bits in a status word
 *    inside `ws`; read them with gmm_read_device_status.  Kernels clamp every
 *    index, so bad group_sizes never cause an out-of-bounds access.
 *  - Scales are fp32.  E4M3 codes are bytes (OCP E4M3: bias 7, no infinities,
 *    largest finite 448).  Quantization: inv = fl32(1/s) (0 where s = 0),
 *    code = E4M3 round-to-nearest-even of fl32(x * inv) saturated to +-448.
 *    A dynamic scale is fl32(amax / 448) over a block of 128 values along the
 *    contraction axis; a scale whose inverse overflows counts as 0.
 *  - Shapes: K and N multiples of 128, all sizes positive, G <= 1024;
 *    M <= 2^24 with ceil(M / 128) + G <= 65535, K and N <= 2^20 (larger
 *    requests return GMM_ERR_UNSUPPORTED).
 */
#ifndef GMM_FP8_H
#define GMM_FP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GMM_OK = 0,
  GMM_ERR_INVALID_ARG = 1, /* null pointer, unknown enum, rule/dtype mismatch */
  GMM_ERR_SHAPE = 2,       /* a size <= 0, or K/N not a multiple of 128 */
  GMM_ERR_ALIGNMENT = 3,   /* a pointer not 16-byte aligned (TMA needs it) */
  GMM_ERR_SCALE = 4,       /* device: static scale not finite or <= FLT_MIN */
  GMM_ERR_UNSUPPORTED = 5, /* a valid request this build does not implement */
  GMM_ERR_CUDA = 6,        /* a CUDA runtime call failed */
  GMM_ERR_GROUP_SIZES = 7, /* device: a negative size or sum(group_sizes) > M */
  GMM_ERR_TIMEOUT = 8,     /* device: a pipeline wait exceeded its time limit */
  GMM_ERR_WORKSPACE = 9    /* ws is NULL or smaller than gmm_workspace_bytes */
} gmm_status;

typedef enum {
  GMM_Q_NONE = 0,   /* no quantization: bf16 operands (the bf16 family) */
  GMM_Q_STATIC = 1, /* per-tensor [1, 1] scale given by the caller */
  GMM_Q_DYNAMIC = 2 /* per-block absmax scale, blocks of 128 along the contraction axis */
} gmm_qrule;

typedef enum { GMM_BF16 = 0, GMM_F32 = 1, GMM_E4M3 = 2 } gmm_dtype;

typedef enum { GMM_OP_FWD = 0, GMM_OP_DLHS = 1, GMM_OP_DRHS = 2, GMM_OP_BWD = 3 } gmm_op;

/* Device status bits (gmm_read_device_status, `bits_out`). */
#define GMM_DEV_GROUP_SIZES 1u
#define GMM_DEV_SCALE 2u
#define GMM_DEV_TIMEOUT 4u

/*
 * An operand with its optional scale, after the pages' LhsRef / WeightsRef
 * (PR #4735, review thread on the should_use_external_scale comment): the
 * direction of the scale follows from the dtype.  An E4M3 operand is already
 * quantized and `scale` dequantizes it (rhs: [G, N]).  A bf16 operand with
 * rule STATIC is quantized inside the call with `scale` ([1, 1], one float);
 * with rule DYNAMIC the call computes the scales itself (`scale` unused);
 * with rule NONE it is used as bf16 (bf16 family; rhs must be bf16 too).
 */
typedef struct {
  const void *data;
  gmm_dtype dtype;
  const float *scale;
  gmm_qrule rule;
} gmm_operand;

/* Bytes of workspace that gmm_fwd (op FWD), gmm_dlhs (DLHS), tgmm_drhs (DRHS)
 * or gmm_backward (BWD) needs for these sizes; also enough for gmm_quantize
 * with the same operand.  Returns 0 for invalid sizes. */
size_t gmm_workspace_bytes(gmm_op op, int64_t M, int64_t K, int64_t N, int32_t G);

/* Number of 128-row chunks a tgmm operand of `rows` rows and G groups can
 * occupy at most: ceil(rows / 128) + G.  Sizes the axis-0 outputs below. */
int64_t gmm_chunk_capacity(int64_t rows, int32_t G);

/*
 * Weight quantization (done once per weight update, outside the timed passes;
 * PR #3770 Description: weights are quantized manually outside the kernel).
 * w_bf16: [G, K, N] bf16.  scales: [G, N] fp32, s[g, n] = fl32(max_k |w| / 448).
 * codes: E4M3 [G, K, N] when transpose_out == 0, else [G, N, K].
 */
gmm_status gmm_quantize_rhs(const void *w_bf16, int32_t G, int64_t K, int64_t N, int transpose_out,
                            uint8_t *codes, float *scales, void *stream);

/*
 * Weight quantization with block-wise scales ("Support quantization for
 * tokamax gmm v2", maxtext PR #4451, review thread on the rhs scale: a 2-D
 * scale is per channel, a 3-D scale block-wise).  w_bf16: [G, K, N].  codes:
 * [G, K, N] E4M3.  One scale per block of 128 weights along
 *   axis 0: K (the forward's contraction): scales [G, K/128, N];
 *   axis 1: N (the contraction of dlhs):    scales [G, N/128, K].
 * Each block: s = fl32(amax / 448), code = e4m3_rn(fl32(w * fl32(1 / s)))
 * (0 for an all-zero block).  Pass the codes to gmm_fwd (axis 0) or gmm_dlhs
 * (axis 1) as an E4M3 rhs with rule GMM_Q_DYNAMIC.  Runs once per weight
 * update, outside the passes.
 */
gmm_status gmm_quantize_rhs_blocks(const void *w_bf16, int32_t G, int64_t K, int64_t N, int axis, uint8_t *codes,
                                   float *scales, void *stream);

/*
 * Activation / gradient quantization, the step each pass runs first.  x_bf16
 * is [rows, cols] bf16.
 * axis == 1: blocks of 128 along each row (the forward lhs, the dlhs dout).
 *   codes [rows, cols]; scales [cols/128, rows] (block-major) for DYNAMIC,
 *   unused for STATIC.  With col_scale != NULL ([G, cols]) the quantized
 *   value is fl32(x[m, n] * col_scale[g(m), n]) and rows in no group are 0
 *   (this folds the rhs scale into dout for dlhs); group_sizes is then needed.
 * axis == 0: the tgmm operand.  Each group's rows are cut into 128-row chunks
 *   starting at the group's first row; chunk j (over all groups, in group
 *   order) gets one scale per column.  codes are stored transposed,
 *   chunk-major and padded: [gmm_chunk_capacity(rows, G), cols, 128], the
 *   128 codes of chunk j and column c contiguous (its rows in order, pad rows
 *   0).  scales [gmm_chunk_capacity, cols] (written for STATIC too, all equal
 *   to the static scale).
 * rule: STATIC (static_scale = device pointer to one float) or DYNAMIC.
 * ws: workspace of at least gmm_workspace_bytes(...) for the pass that
 * consumes this operand.
 */
gmm_status gmm_quantize(const void *x_bf16, int64_t rows, int64_t cols, gmm_qrule rule, int axis,
                        const float *static_scale, const int32_t *group_sizes, int32_t G,
                        const float *col_scale, uint8_t *codes, float *scales, void *ws, size_t ws_bytes,
                        void *stream);

/*
 * Forward gmm.  lhs: bf16 [M, K] with rule STATIC / DYNAMIC (or NONE for the
 * bf16 family), quantized inside the call; or E4M3 codes [M, K] already
 * quantized by the caller ("add static LHS scaling support for GMM v2 FWD",
 * maxtext PR #4735, rebase commit text: activations quantized before the
 * expert-parallel all-gather arrive as a pre-quantized array whose scale is
 * re-applied after the matmul), with lhs.scale the static scale (rule STATIC,
 * one float) or the block scales [K/128, M] (rule DYNAMIC, the layout
 * gmm_quantize writes for axis 1); the quantize step is then skipped.  rhs: E4M3 codes with scales [G, N] (or bf16 for the bf16
 * family), [G, K, N] when transpose_rhs == 0, [G, N, K] when 1.  rhs.rule
 * NONE: per-channel scales [G, N]; rhs.rule DYNAMIC: block-wise scales
 * [G, K/128, N] from gmm_quantize_rhs_blocks axis 0 (transpose_rhs 0 only;
 * else GMM_ERR_UNSUPPORTED), applied per 128-block of K:
 *   out[m, n] = sum_b s_l[m, b] * s_r[g, b, n] * sum_{k in b} q_l[m, k] * q_r[g, k, n]
 * group_sizes: device int32 [G]; rows are sorted by group.
 * out: [M, N] of out_dtype (BF16 or F32):
 *   out[m, n] = s_r[g, n] * sum_b s_l[m, b] * sum_{k in b} q_l[m, k] * q_r[g, k, n]
 * Rows outside every group are written as 0.
 */
gmm_status gmm_fwd(gmm_operand lhs, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes, int32_t G,
                   int64_t M, int64_t K, int64_t N, void *out, gmm_dtype out_dtype, void *ws, size_t ws_bytes,
                   void *stream);

/*
 * gmm_fwd that also hands its lhs quantization back to the caller
 * ("add static LHS scaling support for GMM v2 FWD", maxtext PR #4735, rebase
 * commit text: activations quantized once and the quantized array passed on).
 * lhs must be bf16 with rule STATIC or DYNAMIC.  lhs_codes: device E4M3
 * [M, K], written with the codes the forward multiplies (rows in no group
 * included, as gmm_quantize axis 1 writes them); lhs_scales: device float
 * [K/128, M] for DYNAMIC (unused and may be NULL for STATIC).  The codes are
 * made in these buffers instead of the workspace, so the call costs the same
 * as gmm_fwd.  With the static rule the codes are tgmm_drhs's / gmm_backward's
 * lhs operand as they are (a pre-quantized lhs), which then skips its
 * quantization of lhs.  Every other argument, result and error is gmm_fwd's;
 * a NULL lhs_codes (or NULL lhs_scales with DYNAMIC) is GMM_ERR_INVALID_ARG.
 */
gmm_status gmm_fwd_keep_lhs(gmm_operand lhs, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes,
                            int32_t G, int64_t M, int64_t K, int64_t N, void *out, gmm_dtype out_dtype, void *ws,
                            size_t ws_bytes, uint8_t *lhs_codes, float *lhs_scales, void *stream);

/*
 * Forward gmm of the merged gate|up weights with the SwiGLU activation fused
 * into its epilogue ("FP8 Megablox for batch split", maxtext PR #3770,
 * Description (2): W0 and W1 are concatenated so that one gmm call covers
 * both projections; SwiGLU is the activation they feed).  rhs is the merged
 * buffer W = [W0 | W1] along N, exactly as for the merged gmm_fwd call, with
 * N = 2F and F a multiple of 128.  Every other argument is gmm_fwd's.
 * out: [M, F] of out_dtype:
 *   out[m, j] = silu(h[m, j]) * h[m, F + j],  silu(z) = z / (1 + exp(-z)),
 * where h = gmm_fwd(lhs, rhs) is the merged product, computed in fp32 and
 * never written to memory.  Rows outside every group are 0.  N not a multiple
 * of 256 returns GMM_ERR_SHAPE.  Workspace: gmm_workspace_bytes(GMM_OP_FWD,
 * M, K, N, G) with the merged N.
 */
gmm_status gmm_fwd_swiglu(gmm_operand lhs, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes,
                          int32_t G, int64_t M, int64_t K, int64_t N, void *out, gmm_dtype out_dtype, void *ws,
                          size_t ws_bytes, void *stream);

/*
 * Forward gmm without a workspace argument, for callers that cannot allocate
 * device memory: code under a runtime or framework that owns all device
 * memory (a caching allocator or a fixed memory plan that reserved it at
 * start-up and forbids allocations afterwards), where a cudaMalloc would fail
 * or break the plan, and latency-bound callers that cannot afford the device
 * synchronization cudaMalloc and cudaFree imply.  The pages have no
 * counterpart; it is a convenience of this library.
 * Arguments and results are gmm_fwd's, minus ws and ws_bytes.  The scratch
 * lives in one 32 MiB array of device memory inside the library, which each
 * CUDA context holds until it is destroyed or the process exits.  With lazy
 * module loading (the CUDA default) the array is committed on the first call
 * in a context; with eager loading, when the library loads.  A call whose
 * gmm_workspace_bytes(GMM_OP_FWD, M, K, N, G) exceeds 32 MiB returns
 * GMM_ERR_WORKSPACE before anything runs.  No cudaMalloc, cudaFree or other
 * allocating routine is called.  The first call in a context (of this entry
 * point or of gmm_fwd_noalloc_status) looks up the array's device address:
 * make it at start-up, before any stream capture, so that the 32 MiB are
 * committed while memory is still free.  All calls share the array, which
 * keeps the last call's contents (each call rewrites all it reads): calls
 * whose kernels overlap on the GPU (concurrent streams) race, so serialize
 * them.  Device-detected errors clamp or zero as in gmm_fwd; read them with
 * gmm_fwd_noalloc_status.
 */
gmm_status gmm_fwd_noalloc(gmm_operand lhs, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes,
                           int32_t G, int64_t M, int64_t K, int64_t N, void *out, gmm_dtype out_dtype,
                           void *stream);

/*
 * Device status of the last gmm_fwd_noalloc call in the current context (the
 * GMM_DEV_* bits of its scratch array's status word), as
 * gmm_read_device_status does for a workspace: synchronizes `stream`, writes
 * the bits to *bits_out (if not NULL) and returns GMM_ERR_TIMEOUT,
 * GMM_ERR_SCALE or GMM_ERR_GROUP_SIZES when the matching bit is set, else
 * GMM_OK.  Read it after the call whose status it should report and before
 * the next one.  The pages have no counterpart.  Allocates nothing.
 */
gmm_status gmm_fwd_noalloc_status(uint32_t *bits_out, void *stream);

/*
 * Backward gmm wrt lhs.  dout: bf16 [M, N], always quantized with DYNAMIC
 * 128-blocks along N after folding the rhs column scale in (dout.rule must be
 * DYNAMIC, or NONE for the bf16 family).  rhs: the same buffer and layout as
 * for gmm_fwd with the same transpose_rhs.  dlhs: [M, K] of out_dtype:
 *   dlhs[m, k] = sum_b s_t[m, b] * sum_{n in b} q_t[m, n] * q_r[g, k, n],
 *   q_t, s_t = quantize(fl32(dout[m, n] * s_r[g, n]))
 * With block-wise weights (rhs.rule DYNAMIC: codes [G, K, N] and scales
 * [G, N/128, K] from gmm_quantize_rhs_blocks axis 1; transpose_rhs 0 only)
 * dout is quantized on its own and
 *   dlhs[m, k] = sum_b s_d[m, b] * s_r[g, b, k] * sum_{n in b} q_d[m, n] * q_r[g, k, n]
 */
gmm_status gmm_dlhs(gmm_operand dout, gmm_operand rhs, int transpose_rhs, const int32_t *group_sizes, int32_t G,
                    int64_t M, int64_t K, int64_t N, void *dlhs, gmm_dtype out_dtype, void *ws, size_t ws_bytes,
                    void *stream);

/*
 * Transposed gmm (weight gradient).  lhs: bf16 [M, K] with rule STATIC (the
 * forward's static scale, giving the forward's codes) or DYNAMIC; dout: bf16
 * [M, N], rule DYNAMIC (or both NONE for the bf16 family).  Both are
 * quantized per 128-row chunk of each group (axis 0 above).  With the static
 * rule lhs may instead be the E4M3 codes [M, K] the forward used (from
 * gmm_quantize, axis 1, or passed to gmm_fwd pre-quantized) with lhs.scale
 * the same static scale: the codes are only re-laid out, not quantized again
 * ("add static LHS scaling support for GMM v2 FWD", maxtext PR #4735, rebase
 * commit text: activations quantized once, ahead of the pass that uses them).
 * A pre-quantized lhs with rule DYNAMIC returns GMM_ERR_INVALID_ARG (its
 * blocks run along K, the tgmm's along rows).
 * drhs: [G, K, N] of out_dtype (F32 or BF16):
 *   dW[g, k, n] = sum_c s_x[c, k] * s_d[c, n] * sum_{m in chunk c} q_x[m, k] * q_d[m, n]
 * Empty groups get dW[g] = 0.
 */
gmm_status tgmm_drhs(gmm_operand lhs, gmm_operand dout, const int32_t *group_sizes, int32_t G, int64_t M,
                     int64_t K, int64_t N, void *drhs, gmm_dtype out_dtype, void *ws, size_t ws_bytes,
                     void *stream);

/*
 * Both backward passes in one call: gmm_dlhs(dout, rhs) and tgmm_drhs(lhs,
 * dout) with the arguments and results of those two calls, except that dout
 * is read once: one kernel quantizes it into both operands (the dlhs row
 * blocks, with the per-channel rhs scale folded in, and the tgmm chunk
 * columns), which bit for bit equal what the two calls quantize.  The pages
 * run dlhs and drhs as two kernels of the same backward ("Support
 * quantization for tokamax gmm v2", maxtext PR #4451, Description); sharing
 * the read of their common operand is a choice of this library.  lhs and
 * dout are in the same family as for the separate calls (fp8: dout rule
 * DYNAMIC; bf16 family: both NONE, rhs bf16).  Workspace:
 * gmm_workspace_bytes(GMM_OP_BWD, M, K, N, G).  dlhs [M, K] of dlhs_dtype,
 * drhs [G, K, N] of drhs_dtype.
 */
gmm_status gmm_backward(gmm_operand lhs, gmm_operand dout, gmm_operand rhs, int transpose_rhs,
                        const int32_t *group_sizes, int32_t G, int64_t M, int64_t K, int64_t N, void *dlhs,
                        gmm_dtype dlhs_dtype, void *drhs, gmm_dtype drhs_dtype, void *ws, size_t ws_bytes,
                        void *stream);

/*
 * Row movement for expert parallelism, the steps either side of the NCCL
 * all-to-all that carries routed token rows to the rank holding their expert
 * ("add static LHS scaling support for GMM v2 FWD", maxtext PR #4735, rebase
 * commit text: activations quantized before the expert-parallel exchange and
 * ragged sort, so E4M3 rows move instead of bf16; permute / unpermute).
 *
 * gmm_gather_rows: dst[i, :] = src[idx[i], :] for i < nrows, rows of
 * row_bytes bytes (a multiple of 16; E4M3 codes or bf16).  src has src_rows
 * rows; an index outside [0, src_rows) writes a row of zeros.  idx: device
 * int32 [nrows].  src and dst 16-byte aligned, not overlapping.  Returns
 * GMM_ERR_SHAPE for row_bytes % 16, GMM_ERR_ALIGNMENT, GMM_ERR_INVALID_ARG for
 * negative sizes or NULL pointers (nrows == 0 is a no-op).
 */
gmm_status gmm_gather_rows(const void *src, const int32_t *idx, int64_t nrows, int64_t row_bytes, int64_t src_rows,
                           void *dst, void *stream);

/*
 * gmm_gather_scale_rows: the routed gradient rows of the expert-parallel
 * backward, dst[i, :] = bf16(fl32(src[idx[i], :]) * scale[i]) (one
 * round-to-nearest-even multiply per value, then the bf16 rounding); bf16
 * rows of ncols values (a multiple of 8); idx device int32 [nrows], scale
 * device float [nrows]; an index outside [0, src_rows) writes zeros.  Errors
 * as for gmm_gather_rows.
 */
gmm_status gmm_gather_scale_rows(const void *src_bf16, const int32_t *idx, const float *scale, int64_t nrows,
                                 int64_t ncols, int64_t src_rows, void *dst_bf16, void *stream);

/*
 * gmm_ep_local_order: regrouping of the rows an expert-parallel all-to-all
 * delivers.  recv_counts: device int64 [P, El], the rows each source rank p
 * sent for each local expert e; they arrive in source order, then expert
 * order within a source ("FP8 Megablox for batch split", maxtext PR #3770,
 * Description item 3: a rank's experts as a group_offset slice of the ragged
 * dot).  Writes, on the device, perm [total] (perm[j] = arrival index of the
 * j-th row once grouped by local expert, then by source rank), inv [total]
 * (its inverse: the grouped position of each arrival row) and group_sizes
 * [El] (rows per local expert).  total = sum of recv_counts, known on the
 * host (it is the receive size the exchange needed).  No host
 * synchronization.  P * El > 1024 or total > INT32_MAX returns
 * GMM_ERR_UNSUPPORTED; counts that do not sum to total leave the rows they
 * would misplace unwritten.
 */
gmm_status gmm_ep_local_order(const int64_t *recv_counts, int32_t P, int32_t El, int64_t total, int32_t *perm,
                              int32_t *inv, int32_t *group_sizes, void *stream);

/*
 * gmm_combine_rows: the weighted sum that returns expert outputs to their
 * tokens (the unpermute of the MoE combine):
 *   y[t, :] = sum_{j < k} weight[t, j] * rows[slot[t, j], :]
 * rows: bf16 [nrows, N] (gmm_fwd outputs in the order they came back from
 * the exchange); slot: device int32 [T, k], the row of token t's j-th expert
 * choice (outside [0, nrows): no contribution); weight: device float [T, k].
 * Accumulated in fp32 in the order j = 0 .. k-1 (deterministic); y: [T, N]
 * of y_dtype (BF16 or F32).  N must be a multiple of 8; rows and y 16-byte
 * aligned.
 */
gmm_status gmm_combine_rows(const void *rows_bf16, int64_t nrows, const int32_t *slot, const float *weight, int64_t T,
                            int32_t k, int64_t N, void *y, gmm_dtype y_dtype, void *stream);

/*
 * Synchronizes `stream`, then reads the device status word that the last call
 * using `ws` left.  *bits_out (may be NULL) receives the raw GMM_DEV_* bits.
 * Returns GMM_OK, or the most severe device error: TIMEOUT, SCALE,
 * GROUP_SIZES.  ws is a device pointer.
 */
gmm_status gmm_read_device_status(const void *ws, uint32_t *bits_out, void *stream);

/*
 * Self-test of the bounded waits: launches one block that waits on a barrier
 * nothing ever arrives on, with a limit of `limit_ns` nanoseconds; the wait
 * gives up, sets GMM_DEV_TIMEOUT in ws's status word and the kernel returns.
 * Read the result with gmm_read_device_status.
 */
gmm_status gmm_selftest_timeout(void *ws, uint64_t limit_ns, void *stream);

/* Time limit of every pipeline wait in the kernels (default 4e9 ns). */
void gmm_set_wait_limit_ns(uint64_t limit_ns);

/*
 * GEMM tile choice for the calls that follow (process-wide; a tuning and
 * testing knob: every tile gives the same results bit for bit, each output
 * being accumulated over the same contraction steps in the same order).
 *   GMM_TILES_AUTO          (default) the tile this library measured fastest
 *                           for the call's shape and pass: CTA pairs for the
 *                           E4M3 tgmm and for static E4M3 row passes whose
 *                           groups average two 128-row tiles or more (M >=
 *                           256 G), one-CTA tiles otherwise;
 *   GMM_TILES_ONE_CTA       128 x 256 tiles on one CTA;
 *   GMM_TILES_CTA_PAIRS     256 x 256 tiles over a pair of CTAs (a two-CTA
 *                           cluster sharing each M = 256 tensor-core MMA;
 *                           the tgmm keeps one-CTA tiles when N is not a
 *                           multiple of 256);
 *   GMM_TILES_CTA_PAIRS_NARROW  CTA pairs, and the promoted E4M3 passes whose
 *                           weights or tgmm operand are K-major (dlhs with
 *                           transpose_rhs 0, per channel or block-wise, the
 *                           dynamic forward with transpose_rhs 1, the tgmm)
 *                           on 256 x 128 tiles: four 128-column
 *                           tensor-memory accumulators per SM instead of two
 *                           of 256.
 * Any other value returns GMM_ERR_INVALID_ARG.  Not part of the pages: how a
 * tile maps onto the B200's SMs is this library's choice.
 */
enum { GMM_TILES_AUTO = 0, GMM_TILES_ONE_CTA = 1, GMM_TILES_CTA_PAIRS = 2, GMM_TILES_CTA_PAIRS_NARROW = 3 };
gmm_status gmm_set_tiles(int32_t mode);

/* Static text for a status code. */
const char *gmm_status_string(gmm_status s);

/* Number of kernels the last successful call on this host thread launched. */
int32_t gmm_last_launch_count(void);

/* Per-kernel timing for benchmarks.  While enabled, every kernel the library
 * launches is bracketed by two CUDA events recorded on its stream (events
 * come from a host-side pool; no device memory is allocated).  name is one of
 * "plan", "quant_rows", "quant_chunks", "quant_rhs", "gemm_fwd", "gemm_dlhs",
 * "gemm_drhs". */
typedef struct {
  const char *name;
  int32_t launches;
  double total_ms;
} gmm_profile_entry;

void gmm_profile_enable(int on);

/* Synchronizes on the recorded events, aggregates them per kernel name into
 * entries (at most max_entries), clears the record and returns the number of
 * entries written. */
int32_t gmm_profile_collect(gmm_profile_entry *entries, int32_t max_entries);

#ifdef __cplusplus
}
#endif

#endif /* GMM_FP8_H */
