// gemm_tc.cu -- persistent, warp-specialized grouped GEMM on the sm_100a
// tensor cores (tcgen05), shared by the three passes:
//
//   forward gmm   tile rows = lhs rows of one group, contraction K, columns N
//                 ("FP8 Megablox for batch split", maxtext PR #3770,
//                 Description; "Support quantization for tokamax gmm v2",
//                 maxtext PR #4451, Description)
//   dlhs gmm      tile rows = dout rows, contraction N, columns K: the same
//                 rhs read with the other major-ness (PR #4451, review thread
//                 on ops.py: transpose_rhs flipped)
//   tgmm drhs     tile rows = dout columns n, columns = lhs columns k,
//                 contraction = the 128-row chunks of one group, written
//                 transposed into dW[g, k, n] ("drhs_tgmm2", PR #4451,
//                 Description).  With rows = n the dout chunk scale is one
//                 number per accumulator row, like the row scale of dlhs.
//
// CTA layout (384 threads, one CTA per SM):
//   warp 0     TMA producer: A tile 128 x 128 B, B tile 256 x 128 B per stage,
//              4 stages in shared memory (128-byte swizzle)
//   warp 1     TMEM allocator + MMA issuer: tcgen05.mma M=128 N=256, four
//              32-byte K steps per stage, fp32 accumulators in TMEM, two
//              256-column accumulator buffers
//   warp 2     scale loader: row / column scales of each TMEM unit into a
//              shared-memory ring ahead of the epilogue
//   warp 3     second MMA issuer (promoted kernels and static E4M3 row
//              passes; idle in the bf16 family, giving its registers to the
//              epilogue)
//
// One thread cannot issue tcgen05.mma fast enough to keep the tensor core
// busy once it also waits on the pipeline barriers (measured: ~2.2-3.3
// PFLOP/s from one issuing thread, ~4.3 from two or three).  In the promoted
// kernels every 128-long block is its own TMEM unit and units alternate
// between the two accumulator buffers, so warp 1 issues the even units
// (buffer 0) and warp 3 the odd ones (buffer 1): each unit is still
// accumulated by one thread in contraction order, so the results do not
// depend on the split.  Each issuer waits for its buffer to be released
// before it waits for the unit's stage: units are released in order, so by
// then every earlier use of that stage has completed and the stage barrier's
// phase parity is unambiguous, whatever the stage count.  The static E4M3
// row passes split each tile instead (see two_issuers below).
//   warps 4-11 epilogue: tcgen05.ld, scale, store.  Warp w reads TMEM lanes
//              32 (w % 4) .. +31 (rows) and column half (w - 4) / 4.
//
// Promoted row tiles of at most 64 rows (small groups) run M = 64 MMAs: they
// read half of the A stage from shared memory, which the weight stream of the
// memory-bound shapes competes for (the static kernels keep M = 128: the
// extra index arithmetic cost their epilogue more than it saved).  An M = 64 accumulator puts tile row r in
// TMEM lane 32 (r / 16) + r % 16 and leaves lanes 16 .. 31 of each 32-lane
// quarter untouched, so in those tiles only the first 16 lanes of each
// epilogue warp hold rows.
//
// Scaling ("add static LHS scaling support for GMM v2 FWD", maxtext PR
// #4735, review thread on the LhsRef docstring: the result is multiplied back
// by the scale):
//   promote == false  one TMEM unit per tile; out = acc * s * col_scale
//   promote == true   one TMEM unit per 128-long contraction block; the
//                     epilogue accumulates acc += unit * row_scale (* the
//                     block's column scale for dynamic-lhs tgmm) in registers.
//
// The same GEMM on tiles shared by a pair of CTAs (tcgen05 cta_group::2) is
// gemm_pair.cu; launch_gemm dispatches to it for GemmConfig::cta_pairs.
//
// SwiGLU (forward only, p.swiglu_f = F > 0): the rhs holds the gate and up
// weights side by side, W = [W0 | W1] along N = 2F ("FP8 Megablox for batch
// split", maxtext PR #3770, Description (2): the merged gating gmm).  A tile
// takes 128 gate columns and the same 128 up columns (two B boxes), so one
// thread holds matching gate and up results and writes silu(gate) * up into
// out[M, F]; the 2F-wide product never reaches memory.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace gmm {

constexpr int kBM = 128, kBN = 256;
constexpr int kStages = 4;
constexpr int kAStage = kBM * 128;  // bytes
constexpr int kBStage = kBN * 128;
constexpr int kThreads = 384;     // 3 warpgroups: control, 2 x epilogue
constexpr int kEpiWarp0 = 4;      // first epilogue warp
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 256;
constexpr int kTmemCols = 512;
constexpr int kScaleSlots = 8;    // ring of per-unit scale slots (scale loader -> epilogue)
constexpr int kNumBars = 32;      // mbarriers reserved in shared memory
// Two MMA issuers (warps 1 and 3): the promoted kernels (one TMEM unit per
// 128-long block, units alternating between the two buffers) and the static
// E4M3 row passes (each tile's blocks split between the buffers, even blocks
// in buffer 0, odd ones in buffer 1; the epilogue adds the two partial sums).
// The bf16 family keeps one issuer and one accumulator per tile (its dlhs
// measured slower split: the tile-end wait for both buffers is not paid back).
template <int kElem, bool kPromote, int kMode>
constexpr bool two_issuers() { return kPromote || (kElem == 1 && kMode != MODE_TGMM); }

// Register split (setmaxnreg): the control warpgroup gives registers to the
// two epilogue warpgroups.  Sum must not exceed the launch allocation
// (registers per thread at launch x 384); launch_inst checks it.
// Kernels whose epilogue holds a thread's 128 accumulators in registers get
// the larger epilogue share (the static row passes keep a little more for
// their producer's SwiGLU box logic: fewer spills measured with 56 / 224 than
// with 40 / 232).
template <int kElem, bool kPromote, int kMode>
constexpr int regs_ctl() { return kPromote ? 40 : (two_issuers<kElem, kPromote, kMode>() ? 56 : 72); }
template <int kElem, bool kPromote, int kMode>
constexpr int regs_epi() { return kPromote ? 232 : (two_issuers<kElem, kPromote, kMode>() ? 224 : 216); }

// tgmm keeps 3 pipeline stages and uses the freed shared memory to stage its
// output for TMA stores (one 4 KB block per epilogue warp)
template <int kMode>
constexpr int stages_of() { return kMode == MODE_TGMM ? 3 : kStages; }
constexpr int kStageOut = 4096;  // bytes of one output staging buffer (tgmm); two per epilogue warp

// scale ring slots: tgmm keeps 4 to make room for its output staging
template <int kMode>
constexpr int ring_of() { return kMode == MODE_TGMM ? 4 : kScaleSlots; }

template <int kMode>
constexpr size_t gemm_smem_bytes() {
  return 1024                                    // alignment slack
         + static_cast<size_t>(stages_of<kMode>()) * (kAStage + kBStage)
         + kNumBars * 8                          // mbarriers
         + 16                                    // tmem slot, abort flags
         + ring_of<kMode>() * (kBN + kBM) * sizeof(float)  // scale ring
         + 2 * (kMaxGroups + 1) * sizeof(int)    // plan copy
         + (kMode == MODE_TGMM ? 128 + kEpiWarps * 2 * kStageOut : 0);  // + alignment slack
}

// One work item: tile row index rt (MODE_ROWS: rows r0 .. rend of group g;
// MODE_TGMM: dout columns 128 rt ..), tile column index ct, and the number of
// contraction stages.
struct Item {
  int g, rt, ct, nblocks, r0, rend;
};

// Column of the (2-D view of the) rhs held by tile column c (0 .. 255) of
// column tile ct: plain tiles are 256 consecutive columns; SwiGLU tiles are
// gate columns 128 ct .. 128 ct + 127, then up columns F + 128 ct ..
__device__ __forceinline__ int tile_col_n(int ct, int c, int F) {
  return F ? (c < 128 ? 128 * ct + c : F + 128 * ct + (c - 128)) : kBN * ct + c;
}

// x * sigmoid(x); -0 for large negative x, where exp(-x) overflows
__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }

template <int kMode>
__device__ __forceinline__ Item decode_item(int w, const GemmParams &p, const int *s_offs, const int *s_tpre,
                                            int tn) {
  Item t;
  if constexpr (kMode != MODE_TGMM) {
    // items of group g: (tpre[g+1] - tpre[g]) row tiles x tn column tiles,
    // row tiles fastest
    int lo = 0, hi = p.G + 1;  // first i with tpre[i] * tn > w
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if (s_tpre[mid] * tn > w) hi = mid;
      else lo = mid + 1;
    }
    const int g = lo - 1;
    const int mt_g = s_tpre[g + 1] - s_tpre[g];
    const int local = w - s_tpre[g] * tn;
    t.g = g;
    t.rt = local % mt_g;
    t.ct = local / mt_g;
    t.r0 = s_offs[g] + kBM * t.rt;
    t.rend = min(s_offs[g + 1], t.r0 + kBM);
    t.nblocks = p.kblocks;
  } else {
    // items of group g: rtiles row tiles x tn column tiles; column tiles
    // fastest (the group's dout chunk columns are reused by consecutive
    // items), or row tiles fastest (its lhs chunk columns are: for small
    // groups, whose many items would otherwise space the reuses of a lhs
    // tile further apart than the dW stream lets it stay in L2)
    const int per_g = p.rtiles * tn;
    const int g = w / per_g, local = w % per_g;
    t.g = g;
    t.rt = p.tg_rows_fastest ? local % p.rtiles : local / tn;
    t.ct = p.tg_rows_fastest ? local / p.rtiles : local % tn;
    t.r0 = 0;
    t.rend = 0;
    t.nblocks = (s_tpre[g + 1] - s_tpre[g]) * p.stages_per_chunk;
  }
  return t;
}

__device__ __forceinline__ void st_v8(void *dst, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                      uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(a0), "r"(a1), "r"(a2),
               "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&b);
}

// Stores 32 consecutive outputs of one row.  v8: the destination is 32-byte
// aligned, so each instruction writes one full 32-byte sector.
__device__ __forceinline__ void store_row32(void *out, int64_t off_elems, const float (&v)[32], int out_f32,
                                            bool v8) {
  if (out_f32) {
    float *dst = static_cast<float *>(out) + off_elems;
    if (v8) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        st_v8(dst + 8 * i, __float_as_uint(v[8 * i]), __float_as_uint(v[8 * i + 1]), __float_as_uint(v[8 * i + 2]),
              __float_as_uint(v[8 * i + 3]), __float_as_uint(v[8 * i + 4]), __float_as_uint(v[8 * i + 5]),
              __float_as_uint(v[8 * i + 6]), __float_as_uint(v[8 * i + 7]));
    } else {
      float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
      for (int i = 0; i < 8; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  } else {
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(out) + off_elems;
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    if (v8) {
      st_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
      st_v8(dst + 16, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
    } else {
      uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
      for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
  }
}

// Stores 32 outputs of one tile row that are one column of the output
// (dW[g, k0 + j, n] for j < 32, stride `pitch` elements).  The 32 lanes of a
// warp hold 32 consecutive n, so each instruction writes 128 (f32) or 64
// (bf16) contiguous bytes.
__device__ __forceinline__ void store_col32(void *out, int64_t off_elems, int64_t pitch, const float (&v)[32],
                                            int out_f32) {
  if (out_f32) {
    float *dst = static_cast<float *>(out) + off_elems;
#pragma unroll
    for (int j = 0; j < 32; ++j) dst[j * pitch] = v[j];
  } else {
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(out) + off_elems;
#pragma unroll
    for (int j = 0; j < 32; ++j) dst[j * pitch] = __float2bfloat16_rn(v[j]);
  }
}

template <int kElem, bool kBMN, bool kPromote, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    gmm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  constexpr bool kF16 = (kElem == 2);
  constexpr bool kTg = (kMode == MODE_TGMM);
  constexpr int kBKe = 128 / kElem;                 // contraction elements per stage
  constexpr int kMmaK = 32 / kElem;                 // contraction elements per MMA
  constexpr int kBBoxes = kBMN ? 2 * kElem : 1;     // TMA boxes per B stage
  constexpr int kBBoxBytes = kBStage / kBBoxes;
  constexpr uint32_t kIdesc = instr_desc(kF16, kBMN);
  constexpr uint32_t kIdesc64 = instr_desc(kF16, kBMN, 64);  // row tiles of <= 64 rows
  constexpr int kSt = stages_of<kMode>();
  constexpr bool kTwo = two_issuers<kElem, kPromote, kMode>();
  constexpr bool kSplit = kTwo && !kPromote;  // static row pass: a tile's blocks split between the buffers
  static_assert(!kSplit || kSt % 2 == 0, "split tiles: each stage serves one issuer");
  constexpr int kRing = ring_of<kMode>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + kSt * kAStage;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + kSt * kBStage);
  uint64_t *full = bars;                    // [kSt] TMA -> MMA
  uint64_t *empty = bars + kSt;         // [kSt] MMA -> TMA
  uint64_t *tfull = bars + 2 * kSt;     // [2] MMA -> epilogue
  uint64_t *tempty = tfull + 2;             // [2] epilogue -> MMA
  uint64_t *drain = tempty + 2;             // MMA completion at exit
  uint64_t *sfull = drain + 1;              // [kRing] scale loader -> epilogue
  uint64_t *sempty = sfull + kRing;   // [kRing] epilogue -> scale loader
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *no_abort = reinterpret_cast<volatile int *>(tmem_slot + 2);
  float *s_scol = reinterpret_cast<float *>(tmem_slot + 4);  // [kRing][256] column scales per unit
  float *s_srow = s_scol + kRing * kBN;                // [kRing][128] row scales per unit
  int *s_offs = reinterpret_cast<int *>(s_srow + kRing * kBM);
  int *s_tpre = s_offs + (kMaxGroups + 1);
  // tgmm output staging, 128-byte aligned (TMA store sources must be aligned)
  uint8_t *s_stage_out =
      reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(s_tpre + (kMaxGroups + 1)) + 127) & ~uintptr_t(127));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Which scales each TMEM unit carries (the same decision in every role):
  //   column scales: forward s_r[g, n] (every unit of a tile, applied at the
  //                  end); block-wise rhs scales s_r[g, b, n] (one set per
  //                  unit, applied per unit); tgmm with a dynamic lhs rule:
  //                  s_x[chunk, k] (per unit)
  //   row scales:    promoted row-ragged passes with a dynamic row operand
  //                  (s_l / s_t per 128-block); tgmm: s_d[chunk, n]
  constexpr bool kBlkScales = (kMode == MODE_ROWS_BLK);
  const bool need_col = kTg ? (kPromote && p.colblk_scale != nullptr) : (kBlkScales || p.col_scale != nullptr);
  // block-wise rhs with a static lhs has no row scales (s is applied at the end)
  const bool need_row = kPromote && (!kBlkScales || p.row_scale != nullptr);
  const bool unit_col = kBlkScales || (kTg && kPromote && p.colblk_scale != nullptr);  // column scales per unit
  const bool use_ring = need_col || need_row;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSt; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiWarps);
    }
    mbar_init(drain, kTwo ? 2 : 1);  // one commit per MMA issuer
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sfull[i], 32);
      mbar_init(&sempty[i], kEpiWarps);
    }
    *abort_flag = 0;
    *no_abort = 0;  // never raised: the exit drains ignore aborts
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i <= p.G; i += kThreads) {
    s_offs[i] = p.offs[i];
    s_tpre[i] = p.tpre[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const int tn = (p.ncols + kBN - 1) / kBN;
  const int total = kTg ? p.G * p.rtiles * tn : s_tpre[p.G] * tn;
  const WaitCtl ctl{p.wait_limit_ns, abort_flag, p.status};
  const WaitCtl ctl_drain{p.wait_limit_ns, no_abort, p.status};

  if (warp < 4) {
    setmaxnreg_dec<regs_ctl<kElem, kPromote, kMode>()>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------- TMA producer
      int it = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
        const Item t = decode_item<kMode>(w, p, s_offs, s_tpre, tn);
        for (int b = 0; b < t.nblocks; ++b, ++it) {
          const int s = it % kSt;
          if (!mbar_wait(&empty[s], ((it / kSt) & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kAStage + kBStage);
          int ax, ay, bx, by;
          if constexpr (!kTg) {
            ax = b * kBKe;
            ay = t.r0;
            if (kBMN) {
              bx = t.ct * kBN;
              by = t.g * p.b_group_rows + b * kBKe;
            } else {
              bx = b * kBKe;
              by = t.g * p.b_group_rows + t.ct * kBN;
            }
          } else {
            // chunk jj of the group (stages_per_chunk stages each) in the
            // chunk-major operands: line rows jj * N + n and jj * K + k
            const int jj = s_tpre[t.g] + b / p.stages_per_chunk;
            ax = (b % p.stages_per_chunk) * kBKe;
            ay = jj * (p.rtiles * kBM) + t.rt * kBM;  // dout columns n
            bx = ax;
            by = jj * p.ncols + t.ct * kBN;           // lhs columns k (rows past K belong to the
                                                      // next chunk: their columns are never stored)
          }
          tma_load_2d(sA + s * kAStage, &tmA, ax, ay, &full[s]);
          if constexpr (kBMN) {
            // boxes of 128 bytes along n (columns of W[g] in [K, N])
#pragma unroll
            for (int h = 0; h < kBBoxes; ++h)
              tma_load_2d(sB + s * kBStage + h * kBBoxBytes, &tmB, tile_col_n(t.ct, h * kBKe, p.swiglu_f), by,
                          &full[s]);
          } else if (!kTg && p.swiglu_f) {
            // two boxes of 128 rows (n) of W[g] in [N, K]: gate rows, up rows
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tma_load_2d(sB + s * kBStage + h * (kBStage / 2), &tmB, bx,
                          t.g * p.b_group_rows + tile_col_n(t.ct, h * 128, p.swiglu_f), &full[s]);
          } else {
            tma_load_2d(sB + s * kBStage, &tmB, bx, by, &full[s]);
          }
        }
      }
      // let every issued copy land before the CTA can exit
      for (int i = (it > kSt ? it - kSt : 0); i < it; ++i)
        mbar_wait(&full[i % kSt], (i / kSt) & 1, ctl_drain);
    } else if (warp == 1 || (kTwo && warp == 3)) {
      // ---------------------------------------------------- MMA issuer(s)
      // two issuers: warp 1 fills buffer 0 (the even units, or the even blocks
      // of a split tile), warp 3 buffer 1
      const int par = warp == 3 ? 1 : 0;
      if (lane == 0) {
        int it = 0, u = 0;
        int nuse = 0;  // split tiles: uses of this issuer's buffer
        bool ok = true;
        auto issue = [&](int s, uint32_t d, uint32_t idesc, bool first) {
          const uint32_t a0 = smem_u32(sA + s * kAStage), b0 = smem_u32(sB + s * kBStage);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = smem_desc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bdesc = kBMN ? smem_desc_sw128(b0 + kk * kMmaK * 128, kBBoxBytes, 1024)
                                        : smem_desc_sw128(b0 + kk * 32, 16, 1024);
            tc_mma<kF16>(d, adesc, bdesc, idesc, (first && kk == 0) ? 0u : 1u);
          }
          tc_commit(&empty[s]);
        };
        for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
          const Item t = decode_item<kMode>(w, p, s_offs, s_tpre, tn);
          const uint32_t idesc = (kPromote && !kTg && t.rend - t.r0 <= 64) ? kIdesc64 : kIdesc;
          if constexpr (kSplit) {
            // blocks b = par, par + 2, .. of the tile into buffer par.  Every
            // tile of a row pass has the same block count, so either no tile
            // uses buffer 1 (one block) or every tile uses both: an issuer's
            // buffer release then always follows the previous tile's MMAs,
            // which keeps its stage waits unambiguous
            const bool mine = t.nblocks > par;
            if (mine) {
              if (!mbar_wait(&tempty[par], (nuse & 1) ^ 1, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            for (int b = 0; b < t.nblocks; ++b, ++it) {
              if ((b & 1) != par) continue;
              const int s = it % kSt;
              if (!mbar_wait(&full[s], (it / kSt) & 1, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue(s, tbase + par * kBN, idesc, b == par);
            }
            if (!ok) break;
            if (mine) {
              tc_commit(&tfull[par]);
              ++nuse;
            }
            continue;
          }
          uint32_t buf = 0;
          for (int b = 0; b < t.nblocks; ++b, ++it) {
            const bool unit_start = kPromote || b == 0;
            if (kPromote && (u & 1) != par) {  // the other issuer's unit
              ++u;
              continue;
            }
            if (unit_start) {
              buf = u & 1;
              if (!mbar_wait(&tempty[buf], ((u >> 1) & 1) ^ 1, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const int s = it % kSt;
            if (!mbar_wait(&full[s], (it / kSt) & 1, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue(s, tbase + buf * kBN, idesc, unit_start);
            if (kPromote || b == t.nblocks - 1) {
              tc_commit(&tfull[buf]);
              ++u;
            }
          }
        }
        tc_commit(drain);
        mbar_wait(drain, 0, ctl_drain);
      }
      __syncwarp();
    } else if (warp == 2 && use_ring) {
      // --------------------------------------------------- scale loader
      // Fills one ring slot per TMEM unit, in the order the epilogue consumes
      // them, so that no global-memory latency sits on the epilogue's path.
      int v = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
        const Item t = decode_item<kMode>(w, p, s_offs, s_tpre, tn);
        const int units = kPromote ? t.nblocks : (t.nblocks > 0 ? 1 : 0);
        const int64_t ch0 = kTg ? s_tpre[t.g] : 0;
        for (int j = 0; j < units; ++j, ++v) {
          const int slot = v % kRing;
          bool got = true;
          if (lane == 0) got = mbar_wait(&sempty[slot], ((v / kRing) & 1) ^ 1, ctl);
          if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
            ok = false;
            break;
          }
          // cp.async straight into the slot: the loader never waits for the
          // data, the slot's barrier completes when all 32 lanes' copies land
          if (need_col) {
            // 8 columns per lane (never straddling a gate / up boundary);
            // columns >= ncols are never read
            const int n = kTg ? t.ct * kBN + 8 * lane : tile_col_n(t.ct, 8 * lane, p.swiglu_f);
            if (n < p.ncols) {
              const float *src =
                  kTg ? p.colblk_scale + (ch0 + j) * p.colblk_ld + n
                      : (kBlkScales ? p.colblk_scale + (static_cast<int64_t>(t.g) * p.kblocks + j) * p.colblk_ld + n
                              : p.col_scale + static_cast<int64_t>(t.g) * p.ncols + n);
              float *dst = s_scol + slot * kBN + 8 * lane;
              cp_async_16(dst, src);
              cp_async_16(dst + 4, src + 4);
            }
          }
          if (need_row) {
            float *dst = s_srow + slot * kBM + 4 * lane;
            if constexpr (kTg) {
              cp_async_16(dst, p.row_scale + (ch0 + j) * p.row_scale_ld + t.rt * kBM + 4 * lane);
            } else {
              const float *src = p.row_scale + static_cast<int64_t>(j) * p.row_scale_ld;
              const int64_t last = p.M - 1;
              const int64_t r0 = t.r0 + 4 * lane;
#pragma unroll
              for (int e = 0; e < 4; ++e) cp_async_4(dst + e, src + min(r0 + e, last));
            }
          }
          cp_async_mbar_arrive(&sfull[slot]);
        }
      }
      cp_async_wait_all();  // no copy in flight when the warp leaves
    }
  } else {
    setmaxnreg_inc<regs_epi<kElem, kPromote, kMode>()>();
    // ---------------------------------------------------------- epilogue
    const int et = threadIdx.x - kEpiWarp0 * 32;  // 0 .. 255
    const int q = warp & 3, h = (warp - kEpiWarp0) >> 2;
    const int row = q * 32 + lane;
    const uint32_t tl = tbase + (static_cast<uint32_t>(q * 32) << 16);  // the warp's TMEM lanes
    const bool sw = !kTg && p.swiglu_f > 0;
    // tile column of the thread's 32-column chunk c (0 .. 3): the column half h
    // of the tile, or for SwiGLU gate columns 64 h .. (c = 0, 1) and the
    // matching up columns 128 + 64 h .. (c = 2, 3)
    auto colt = [&](int c) -> int { return sw ? ((c & 2) ? 128 : 0) + h * 64 + (c & 1) * 32 : h * 128 + c * 32; };
    float s_eff = 1.0f;
    if (p.static_scale) {
      const float v = *p.static_scale;
      s_eff = (isfinite(v) && v > 1.17549435e-38f) ? v : 0.0f;
      // reported here too for operands quantized before the call
      if (s_eff == 0.0f && blockIdx.x == 0 && et == 0) atomicOr(p.status, GMM_DEV_SCALE);
    }
    const bool out_v8 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
    const uint64_t evict_first = kTg ? l2_policy_evict_first() : 0;  // dW is written once: keep operands in L2
    int nstore = 0;                                                     // tgmm stores issued by this warp
    int u = 0;  // TMEM units consumed
    int n0 = 0, n1 = 0;  // split tiles: uses of buffers 0 and 1 consumed
    int v = 0;  // scale slots consumed
    bool ok = true;
    // waits for TMEM unit u (and its scale slot); the decision is uniform
    // within the warp.  Warps decide on their own: one that stops raises the
    // abort flag, which ends every other warp's next wait, and no barrier
    // among the epilogue warps is ever entered after that point.
    auto wait_unit = [&](uint32_t buf, int slot) -> bool {
      bool got = mbar_wait(&tfull[buf], (u >> 1) & 1, ctl);
      if (got && use_ring) got = mbar_wait(&sfull[slot], (v / kRing) & 1, ctl);
      return __all_sync(0xffffffffu, got);
    };
    auto release_slot = [&](int slot) {
      if (use_ring) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[slot]);
        ++v;
      }
    };
    for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
      const Item t = decode_item<kMode>(w, p, s_offs, s_tpre, tn);
      const int col0 = t.ct * kBN + h * 128;
      int64_t orow;
      bool row_ok;
      int trow = row;  // the tile row held by this thread's TMEM lane
      if constexpr (!kTg) {
        const bool m64 = kPromote && t.rend - t.r0 <= 64;  // M = 64 accumulator layout
        if (m64) trow = q * 16 + (lane & 15);
        orow = t.r0 + trow;
        row_ok = (!m64 || lane < 16) && orow < t.rend;
      } else {
        orow = static_cast<int64_t>(t.rt) * kBM + row;  // n
        row_ok = true;
      }
      // writes 32 tile columns starting at tile column col (a multiple of 32)
      auto emit = [&](int col, const float(&o)[32]) {
        if constexpr (!kTg) {
          store_row32(p.out, orow * p.ld_out + col, o, p.out_f32, out_v8);
        } else {
          // the warp's 32 x 32 block of dW[g, col .. col+31, n0 .. n0+31]:
          // staged row-major (row k, 32 consecutive n) and written by one
          // TMA store; the buffer is reused once the previous store read it
          uint8_t *stg = s_stage_out + ((warp - kEpiWarp0) * 2 + (nstore & 1)) * kStageOut;
          ++nstore;
          if (lane == 0) bulk_wait_read1();  // the store issued from this buffer two stores ago has read it
          __syncwarp();
          if (p.out_f32) {
            float *sf = reinterpret_cast<float *>(stg);
#pragma unroll
            for (int j = 0; j < 32; ++j) sf[j * 32 + lane] = o[j];
          } else {
            __nv_bfloat16 *sb = reinterpret_cast<__nv_bfloat16 *>(stg);
#pragma unroll
            for (int j = 0; j < 32; ++j) sb[j * 32 + lane] = __float2bfloat16_rn(o[j]);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d_hint(&tmOut, t.rt * kBM + q * 32, t.g * p.ncols + col, stg, evict_first);
            bulk_commit();
          }
        }
      };
      if (t.nblocks == 0) {  // empty group in tgmm: dW tile = 0
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (col0 + c * 32 < p.ncols) emit(col0 + c * 32, z);
        continue;
      }
      if constexpr (kPromote) {
        float2 acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
        int slot = 0;
        for (int b = 0; b < t.nblocks; ++b) {
          const uint32_t buf = u & 1;
          slot = v % kRing;
          if (!wait_unit(buf, slot)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float rs = need_row ? s_srow[slot * kBM + trow] : 1.0f;
          const float2 rs2 = make_float2(rs, rs);
          const float *cs = s_scol + slot * kBN;
#pragma unroll
          for (int cp = 0; cp < 2; ++cp) {
            // chunks 2 cp, 2 cp + 1 (compile-time accumulator indices)
            // colt(2 cp + 1) = colt(2 cp) + 32: one 64-column load
            uint32_t va[32], vb[32];
            tmem_ld64(tl + buf * kBN + colt(2 * cp), va, vb);
            tmem_wait_ld();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const uint32_t *vv = half ? vb : va;
              const int c = 2 * cp + half;
              if (!unit_col) {
                // one scale per accumulator row
#pragma unroll
                for (int i = 0; i < 16; ++i)
                  acc[c * 16 + i] = __ffma2_rn(make_float2(__uint_as_float(vv[2 * i]), __uint_as_float(vv[2 * i + 1])),
                                               rs2, acc[c * 16 + i]);
              } else if (kBlkScales && !need_row) {
                // block-wise rhs scales with a static lhs (s applied at the
                // end): the column scale multiplies the unit directly; a loop
                // of its own, so that no row-scale product is formed
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float4 c4 = *reinterpret_cast<const float4 *>(cs + colt(c) + 4 * i);
                  acc[c * 16 + 2 * i] = __ffma2_rn(
                      make_float2(__uint_as_float(vv[4 * i]), __uint_as_float(vv[4 * i + 1])),
                      make_float2(c4.x, c4.y), acc[c * 16 + 2 * i]);
                  acc[c * 16 + 2 * i + 1] = __ffma2_rn(
                      make_float2(__uint_as_float(vv[4 * i + 2]), __uint_as_float(vv[4 * i + 3])),
                      make_float2(c4.z, c4.w), acc[c * 16 + 2 * i + 1]);
                }
              } else {
                // tgmm with a dynamic lhs rule (lhs chunk scale along the
                // columns k) or block-wise rhs scales (along the columns n)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float4 c4 = *reinterpret_cast<const float4 *>(cs + colt(c) + 4 * i);
                  // without row scales (static lhs: s is applied at the end)
                  // the column scale multiplies the unit directly
                  const bool rowmul = kTg || need_row;  // tgmm always has dout chunk scales
                  const float2 c01 = rowmul ? __fmul2_rn(make_float2(c4.x, c4.y), rs2) : make_float2(c4.x, c4.y);
                  const float2 c23 = rowmul ? __fmul2_rn(make_float2(c4.z, c4.w), rs2) : make_float2(c4.z, c4.w);
                  acc[c * 16 + 2 * i] = __ffma2_rn(
                      make_float2(__uint_as_float(vv[4 * i]), __uint_as_float(vv[4 * i + 1])), c01,
                      acc[c * 16 + 2 * i]);
                  acc[c * 16 + 2 * i + 1] = __ffma2_rn(
                      make_float2(__uint_as_float(vv[4 * i + 2]), __uint_as_float(vv[4 * i + 3])), c23,
                      acc[c * 16 + 2 * i + 1]);
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          ++u;
          if (b + 1 < t.nblocks) release_slot(slot);  // the last slot is read again below
        }
        if (!ok) break;
        if (row_ok) {
          // per-channel rhs column scale (in every unit's slot); static lhs: s
          const float fin = ((kTg || kBlkScales) && p.static_scale) ? s_eff : 1.0f;
          const bool colmul = !kTg && p.col_scale != nullptr;
          const float *cf = s_scol + slot * kBN;
          if (sw) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const float *fg = cf + colt(c), *fu = cf + colt(c + 2);
              float o[32];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 a = acc[c * 16 + i], b2 = acc[(c + 2) * 16 + i];
                const float g0 = (colmul ? a.x * fg[2 * i] : a.x) * fin;
                const float g1 = (colmul ? a.y * fg[2 * i + 1] : a.y) * fin;
                const float u0 = (colmul ? b2.x * fu[2 * i] : b2.x) * fin;
                const float u1 = (colmul ? b2.y * fu[2 * i + 1] : b2.y) * fin;
                o[2 * i] = silu(g0) * u0;
                o[2 * i + 1] = silu(g1) * u1;
              }
              emit(t.ct * 128 + h * 64 + c * 32, o);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int col = t.ct * kBN + colt(c);
              if (col >= p.ncols) continue;
              float o[32];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float2 a = acc[c * 16 + i];
                if (colmul) {
                  a.x *= cf[colt(c) + 2 * i];
                  a.y *= cf[colt(c) + 2 * i + 1];
                }
                o[2 * i] = a.x * fin;
                o[2 * i + 1] = a.y * fin;
              }
              emit(col, o);
            }
          }
        }
        release_slot(slot);
      } else if constexpr (kSplit) {
        // partial sums of the even blocks (buffer 0) and the odd ones (buffer
        // 1): both into registers, the buffers released, then scale and store
        const bool two = t.nblocks > 1;
        const int slot = v % kRing;
        bool got = mbar_wait(&tfull[0], n0 & 1, ctl);
        if (got && two) got = mbar_wait(&tfull[1], n1 & 1, ctl);
        if (got && use_ring) got = mbar_wait(&sfull[slot], (v / kRing) & 1, ctl);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float2 acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
        for (int bi = 0; bi < (two ? 2 : 1); ++bi) {
#pragma unroll
          for (int cp = 0; cp < 2; ++cp) {
            // chunks 2 cp, 2 cp + 1: colt(2 cp + 1) = colt(2 cp) + 32
            uint32_t va[32], vb[32];
            tmem_ld64(tl + bi * kBN + colt(2 * cp), va, vb);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              acc[2 * cp * 16 + i] =
                  __fadd2_rn(acc[2 * cp * 16 + i], make_float2(__uint_as_float(va[2 * i]), __uint_as_float(va[2 * i + 1])));
              acc[(2 * cp + 1) * 16 + i] = __fadd2_rn(
                  acc[(2 * cp + 1) * 16 + i], make_float2(__uint_as_float(vb[2 * i]), __uint_as_float(vb[2 * i + 1])));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tempty[0]);
          if (two) mbar_arrive(&tempty[1]);
        }
        ++n0;
        if (two) ++n1;
        if (row_ok) {
          const float s0 = p.static_scale ? s_eff : 1.0f;
          const float *cf = s_scol + slot * kBN;
          if (sw) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const float *fg = cf + colt(c), *fu = cf + colt(c + 2);
              float o[32];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 a = acc[c * 16 + i], b2 = acc[(c + 2) * 16 + i];
                const float gs0 = need_col ? fg[2 * i] : 1.0f, gs1 = need_col ? fg[2 * i + 1] : 1.0f;
                const float us0 = need_col ? fu[2 * i] : 1.0f, us1 = need_col ? fu[2 * i + 1] : 1.0f;
                o[2 * i] = silu(a.x * s0 * gs0) * (b2.x * s0 * us0);
                o[2 * i + 1] = silu(a.y * s0 * gs1) * (b2.y * s0 * us1);
              }
              emit(t.ct * 128 + h * 64 + c * 32, o);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int col = t.ct * kBN + colt(c);
              if (col >= p.ncols) continue;
              float o[32];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 a = acc[c * 16 + i];
                o[2 * i] = a.x * s0 * (need_col ? cf[colt(c) + 2 * i] : 1.0f);
                o[2 * i + 1] = a.y * s0 * (need_col ? cf[colt(c) + 2 * i + 1] : 1.0f);
              }
              emit(col, o);
            }
          }
        }
        release_slot(slot);
      } else {
        const uint32_t buf = u & 1;
        const int slot = v % kRing;
        if (!wait_unit(buf, slot)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float s0 = p.static_scale ? s_eff : 1.0f;
        const float *cf = s_scol + slot * kBN;
#pragma unroll
        for (int cp = 0; cp < 2; ++cp) {
          const int ca = sw ? cp : 2 * cp, cb = sw ? cp + 2 : 2 * cp + 1;
          uint32_t va[32], vb[32];
          tmem_ld32(tl + buf * kBN + colt(ca), va);
          tmem_ld32(tl + buf * kBN + colt(cb), vb);
          tmem_wait_ld();
          if (sw) {
            if (row_ok) {
              const float *fg = cf + colt(ca), *fu = cf + colt(cb);
              float o[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float gs = need_col ? fg[i] : 1.0f, us = need_col ? fu[i] : 1.0f;
                o[i] = silu(__uint_as_float(va[i]) * s0 * gs) * (__uint_as_float(vb[i]) * s0 * us);
              }
              emit(t.ct * 128 + h * 64 + cp * 32, o);
            }
            continue;
          }
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t *vv = half ? vb : va;
            const int c = half ? cb : ca;
            const int col = t.ct * kBN + colt(c);
            if (!row_ok || col >= p.ncols) continue;
            float o[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float cs1 = need_col ? cf[colt(c) + i] : 1.0f;
              o[i] = __uint_as_float(vv[i]) * s0 * cs1;
            }
            emit(col, o);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        ++u;
        release_slot(slot);
      }
    }
    if constexpr (kTg) {
      if (lane == 0) bulk_wait0();  // every dW store of this warp has landed
      __syncwarp();
    }
    // rows outside every group are zero (row-ragged passes only)
    if constexpr (!kTg) {
      const int esz = p.out_f32 ? 4 : 2;
      const int64_t tail0 = s_offs[p.G];
      const int64_t out_w = sw ? p.swiglu_f : p.ncols;           // output columns
      const int64_t cpr = out_w * esz / 16;                      // 16-byte chunks per row
      const int64_t n = (static_cast<int64_t>(p.M) - tail0) * cpr;
      for (int64_t i = static_cast<int64_t>(blockIdx.x) * kEpiThreads + et; i < n;
           i += static_cast<int64_t>(gridDim.x) * kEpiThreads) {
        const int64_t r = tail0 + i / cpr, c = i % cpr;
        *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.out) + (r * p.ld_out) * esz + c * 16) =
            make_uint4(0, 0, 0, 0);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

static int g_num_sms = 0;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

template <int kElem, bool kBMN, bool kPromote, int kMode>
static cudaError_t launch_inst(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                               const GemmParams &p, int grid, cudaStream_t st) {
  auto kern = gmm_tc_kernel<kElem, kBMN, kPromote, kMode>;
  const size_t smem = gemm_smem_bytes<kMode>();
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc waits for registers the CTA owns: never launch a split that
  // does not fit the launch allocation
  if (attr.numRegs * kThreads < regs_ctl<kElem, kPromote, kMode>() * 128 + regs_epi<kElem, kPromote, kMode>() * 256)
    return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(tmA, tmB, tmOut, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmConfig &cfg, const CUtensorMap &tmA, const CUtensorMap &tmB,
                        const CUtensorMap &tmOut, const GemmParams &p, int grid, cudaStream_t st) {
  if (cfg.cta_pairs) return launch_gemm_pair(cfg, tmA, tmB, tmOut, p, grid, st);
  if (cfg.tile_n != 256) return cudaErrorInvalidValue;
  if (cfg.mode == MODE_TGMM) {
    if (cfg.b_mn_major) return cudaErrorInvalidValue;
    if (cfg.elem_bytes == 1 && cfg.promote) return launch_inst<1, false, true, MODE_TGMM>(tmA, tmB, tmOut, p, grid, st);
    if (cfg.elem_bytes == 2 && !cfg.promote) return launch_inst<2, false, false, MODE_TGMM>(tmA, tmB, tmOut, p, grid, st);
    return cudaErrorInvalidValue;
  }
  if (cfg.mode == MODE_ROWS_BLK) {  // block-wise rhs scales: promoted fp8 only
    if (cfg.elem_bytes != 1 || !cfg.promote) return cudaErrorInvalidValue;
    return cfg.b_mn_major ? launch_inst<1, true, true, MODE_ROWS_BLK>(tmA, tmB, tmOut, p, grid, st)
                          : launch_inst<1, false, true, MODE_ROWS_BLK>(tmA, tmB, tmOut, p, grid, st);
  }
  if (cfg.elem_bytes == 1) {
    if (cfg.b_mn_major)
      return cfg.promote ? launch_inst<1, true, true, MODE_ROWS>(tmA, tmB, tmOut, p, grid, st)
                         : launch_inst<1, true, false, MODE_ROWS>(tmA, tmB, tmOut, p, grid, st);
    return cfg.promote ? launch_inst<1, false, true, MODE_ROWS>(tmA, tmB, tmOut, p, grid, st)
                       : launch_inst<1, false, false, MODE_ROWS>(tmA, tmB, tmOut, p, grid, st);
  }
  if (cfg.promote) return cudaErrorInvalidValue;
  return cfg.b_mn_major ? launch_inst<2, true, false, MODE_ROWS>(tmA, tmB, tmOut, p, grid, st)
                        : launch_inst<2, false, false, MODE_ROWS>(tmA, tmB, tmOut, p, grid, st);
}

}  // namespace gmm
