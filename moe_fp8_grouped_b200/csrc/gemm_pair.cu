// gemm_pair.cu -- the grouped GEMM of gemm_tc.cu on tiles shared by a pair
// of CTAs (a two-CTA cluster issuing tcgen05 cta_group::2 MMAs of M = 256):
// the same three passes, the same roles per warp and the same scaling, with
// each CTA holding 128 rows of every item's A tile and half of its B tile in
// its own shared memory and its 128 rows of the accumulator in its own
// tensor memory.  Rank 0 of the pair issues the MMAs (from two threads, as
// in gemm_tc.cu, for the static E4M3 row tiles and the promoted 256-column
// tiles); the loads of both CTAs complete on rank 0's full barriers; rank 0
// commits to both CTAs' barriers; the epilogue warps of both CTAs release
// accumulators on rank 0's barriers.  Tile width kTN = 256, or 128 for the
// promoted E4M3 passes with a K-major B operand (four accumulator buffers
// instead of two).  The automatic tile choice takes these tiles for the E4M3
// tgmm and the static E4M3 row passes with large groups.
//
// Passes and sources as in gemm_tc.cu: forward gmm ("FP8 Megablox for batch
// split", maxtext PR #3770, Description; "Support quantization for tokamax
// gmm v2", maxtext PR #4451, Description), dlhs gmm (PR #4451, review thread
// on ops.py: transpose_rhs flipped), tgmm drhs (PR #4451, Description:
// "drhs_tgmm2"), scales multiplied back ("add static LHS scaling support for
// GMM v2 FWD", maxtext PR #4735, review thread on the LhsRef docstring),
// SwiGLU of the merged gate|up call (PR #3770, Description (2)).
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace gmm {
namespace pair {

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
constexpr int kNumBars = 48;      // mbarriers reserved in shared memory
// Register split (setmaxnreg): the control warpgroup gives registers to the
// two epilogue warpgroups.  Sum must not exceed the launch allocation
// (registers per thread at launch x 384); launch_inst checks it.
// The promote variants keep 128 accumulators per thread and get the larger
// epilogue share.
template <bool kPromote>
constexpr int regs_ctl() { return kPromote ? 40 : 72; }
template <bool kPromote>
constexpr int regs_epi() { return kPromote ? 232 : 216; }

// Pipeline stages.  One CTA: A 16 KB + B 32 KB per stage, 4 stages (tgmm: 3,
// the freed shared memory stages its output for TMA stores, one 4 KB block
// per epilogue warp).  A CTA pair (kCta = 2): each CTA holds its 128 rows of A
// and half of B: 16 KB + 16 KB with 256-column tiles, 6 stages (tgmm: 4);
// 16 KB + 8 KB with 128-column tiles (kTN = 128), 8 stages (tgmm: 5).
template <int kCta, int kMode, int kTN = 256>
constexpr int stages_of() {
  return kCta == 2 ? (kTN == 128 ? (kMode == MODE_TGMM ? 5 : 8) : (kMode == MODE_TGMM ? 4 : 6))
                   : (kMode == MODE_TGMM ? 3 : kStages);
}
constexpr int kStageOut = 4096;  // bytes of one output staging buffer (tgmm); two per epilogue warp

// scale ring slots: tgmm keeps 4 to make room for its output staging
template <int kMode>
constexpr int ring_of() { return kMode == MODE_TGMM ? 4 : kScaleSlots; }

// int arrays [kMaxGroups + 1] in shared memory: group offsets, 128-row tile
// prefix and the prefix of pair tiles
template <int kCta, int kMode>
constexpr int plan_arrays() { return (kCta == 2 || kMode != MODE_TGMM) ? 3 : 2; }

template <int kCta, int kMode, int kTN = 256>
constexpr size_t gemm_smem_bytes() {
  return 1024                                    // alignment slack
         + static_cast<size_t>(stages_of<kCta, kMode, kTN>()) * (kAStage + (kTN * 128) / kCta)
         + kNumBars * 8                          // mbarriers
         + 16                                    // tmem slot, abort flags
         + ring_of<kMode>() * (kBN + kBM) * sizeof(float)  // scale ring
         + plan_arrays<kCta, kMode>() * (kMaxGroups + 1) * sizeof(int)  // plan copy, item prefix
         + (kMode == MODE_TGMM ? 128 + kEpiWarps * 2 * kStageOut : 0);  // + alignment slack
}
static_assert(gemm_smem_bytes<2, MODE_ROWS>() <= 232448, "pair-tile shared memory");
static_assert(gemm_smem_bytes<2, MODE_TGMM>() <= 232448, "pair-tile tgmm shared memory");
static_assert(gemm_smem_bytes<1, MODE_ROWS>() <= 232448, "shared memory");
static_assert(gemm_smem_bytes<1, MODE_TGMM>() <= 232448, "tgmm shared memory");
static_assert(gemm_smem_bytes<1, MODE_ROWS>() == gemm_smem_bytes<1, MODE_ROWS_BLK>(), "row-pass shared memory");
static_assert(gemm_smem_bytes<2, MODE_ROWS, 128>() <= 232448, "narrow pair-tile shared memory");
static_assert(gemm_smem_bytes<2, MODE_TGMM, 128>() <= 232448, "narrow pair-tile tgmm shared memory");

// One work item: tile row index rt (MODE_ROWS: rows r0 .. rend of group g;
// MODE_TGMM: dout columns 128 rt ..), tile column index ct, and the number of
// contraction stages.
struct Item {
  int g, rt, ct, nblocks, r0, rend;
};

// Column of the (2-D view of the) rhs held by tile column c (0 .. tn - 1) of
// column tile ct: plain tiles are tn (256 or 128) consecutive columns; SwiGLU
// tiles (256 wide) are gate columns 128 ct .. 128 ct + 127, then up columns
// F + 128 ct ..
__device__ __forceinline__ int tile_col_n(int ct, int c, int F, int tn = kBN) {
  return F ? (c < 128 ? 128 * ct + c : F + 128 * ct + (c - 128)) : tn * ct + c;
}

// x * sigmoid(x); -0 for large negative x, where exp(-x) overflows
__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }

// A CTA pair (kCta = 2) takes one item of twice the rows: rank r of the pair
// holds tile rows 128 r .. 128 r + 127 of it.
template <int kMode, int kCta>
__device__ __forceinline__ Item decode_item(int w, const GemmParams &p, const int *s_offs, const int *s_tpre,
                                            const int *s_ppre, int tn, int rank) {
  Item t;
  if constexpr (kMode != MODE_TGMM) {
    // items of group g: (pre[g+1] - pre[g]) row tiles (128 rows, or 256 for a
    // pair) x tn column tiles, row tiles fastest
    const int *pre = kCta == 2 ? s_ppre : s_tpre;
    int lo = 0, hi = p.G + 1;  // first i with pre[i] * tn > w
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if (pre[mid] * tn > w) hi = mid;
      else lo = mid + 1;
    }
    const int g = lo - 1;
    const int mt_g = pre[g + 1] - pre[g];
    const int local = w - pre[g] * tn;
    t.g = g;
    t.rt = local % mt_g;
    t.ct = local / mt_g;
    t.r0 = s_offs[g] + kCta * kBM * t.rt + kBM * rank;
    t.rend = min(s_offs[g + 1], t.r0 + kBM);  // at or before r0: the pair's second half is past the group
    t.nblocks = p.kblocks;
  } else {
    // items of group g: rtiles / kCta row tiles x tn column tiles; column
    // tiles fastest (the group's dout chunk columns are reused by consecutive
    // items), or row tiles fastest (its lhs chunk columns are: for small
    // groups, whose many items would otherwise space the reuses of a lhs
    // tile further apart than the dW stream lets it stay in L2); pairs need
    // an even rtiles
    const int rtp = p.rtiles / kCta;
    const int per_g = rtp * tn;
    const int g = w / per_g, local = w % per_g;
    t.g = g;
    t.rt = (p.tg_rows_fastest ? local % rtp : local / tn) * kCta + rank;
    t.ct = p.tg_rows_fastest ? local / rtp : local % tn;
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

// kCta = 2: the kernel runs as clusters of two CTAs (a pair) that share each
// M = 256 MMA (tcgen05 cta_group::2): rank r holds rows 128 r .. of every
// item's A tile and columns 128 r .. 128 r + 127 of its B tile, and receives
// its 128 rows of the accumulator.  Rank 0 issues the MMAs.  Halving B per SM
// halves the shared-memory traffic per MMA (TMA writes plus tensor-core
// reads), which bounds the one-CTA tile.
// kTN: tile columns, 256, or 128 for CTA pairs in the promoted passes with a
// K-major B (four 128-column TMEM buffers instead of two of 256: the MMA can
// run three units ahead of the epilogue).
template <int kElem, bool kBMN, bool kPromote, int kMode, int kTN>
__global__ void __launch_bounds__(kThreads, 1)
    gmm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  constexpr int kCta = 2;
  constexpr bool kF16 = (kElem == 2);
  constexpr bool kTg = (kMode == MODE_TGMM);
  constexpr bool kPair = (kCta == 2);
  constexpr int kBKe = 128 / kElem;                 // contraction elements per stage
  constexpr int kMmaK = 32 / kElem;                 // contraction elements per MMA
  static_assert(kTN == 256 || (kTN == 128 && kPair && kPromote && !kBMN), "128-column tiles: pairs, promoted, K-major B");
  constexpr int kBS = (kTN * 128) / kCta;           // bytes of B per CTA per stage
  constexpr int kBBoxes = kBMN ? (2 / kCta) * kElem : 1;  // TMA boxes per B stage (128-byte wide if MN-major)
  constexpr int kBBoxBytes = kBS / kBBoxes;
  constexpr uint32_t kIdesc = instr_desc_mn(kF16, false, kBMN, kTN, kPair ? 256u : 128u);
  constexpr int kSt = stages_of<kCta, kMode, kTN>();
  constexpr int kNB = kTmemCols / kTN;              // TMEM accumulator buffers
  constexpr int kCh = kTN / 64;                     // 32-column chunks per epilogue thread
  constexpr int kRing = ring_of<kMode>();
  // static E4M3 row tiles accumulate their even and odd blocks in the two
  // TMEM buffers, as the one-CTA kernel does (bit-identical results)
  constexpr bool kSplit = !kPromote && !kTg && kElem == 1;
  static_assert(!kSplit || stages_of<kCta, kMode, kTN>() % 2 == 0, "split tiles: each stage serves one issuer");
  // two MMA issuers: split static tiles, and promoted 256-column tiles (units
  // alternate between the two TMEM buffers; each issuer waits for its buffer's
  // release before the unit's stage, so the stage parities stay unambiguous)
  constexpr bool kTwo = kSplit || (kPromote && kTN == 256);
  constexpr uint32_t kStageTx = kCta * (kAStage + kBS);  // bytes completing one stage (both CTAs)

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + kSt * kAStage;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + kSt * kBS);
  uint64_t *full = bars;                    // [kSt] TMA -> MMA
  uint64_t *empty = bars + kSt;         // [kSt] MMA -> TMA
  uint64_t *tfull = bars + 2 * kSt;     // [kNB] MMA -> epilogue
  uint64_t *tempty = tfull + kNB;           // [kNB] epilogue -> MMA
  uint64_t *drain = tempty + kNB;           // MMA completion at exit
  uint64_t *sfull = drain + 1;              // [kRing] scale loader -> epilogue
  uint64_t *sempty = sfull + kRing;   // [kRing] epilogue -> scale loader
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *no_abort = reinterpret_cast<volatile int *>(tmem_slot + 2);
  float *s_scol = reinterpret_cast<float *>(tmem_slot + 4);  // [kRing][256] column scales per unit
  float *s_srow = s_scol + kRing * kBN;                // [kRing][128] row scales per unit
  int *s_offs = reinterpret_cast<int *>(s_srow + kRing * kBM);
  int *s_tpre = s_offs + (kMaxGroups + 1);
  // prefix of 256-row pair tiles per group (row passes)
  int *s_ppre = s_tpre + (kMaxGroups + 1);
  // tgmm output staging, 128-byte aligned (TMA store sources must be aligned)
  uint8_t *s_stage_out = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(s_offs + plan_arrays<kCta, kMode>() * (kMaxGroups + 1)) + 127) & ~uintptr_t(127));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = kPair ? static_cast<int>(cluster_ctarank()) : 0;
  const bool leader = rank == 0;
  // items: one per CTA, or one per pair (consecutive blockIdx.x form a cluster)
  const int w0 = kPair ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int wstep = kPair ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);

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
    for (int i = 0; i < kNB; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kCta * kEpiWarps);  // a pair: the epilogue warps of both CTAs arrive on rank 0's
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
  if constexpr (kPair) {
    // the other CTA's barriers are used (remote arrivals, byte counts,
    // multicast commits) only after both CTAs initialized theirs
    cluster_sync();
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish();
    }
  }
  for (int i = threadIdx.x; i <= p.G; i += kThreads) {
    s_offs[i] = p.offs[i];
    s_tpre[i] = p.tpre[i];
  }
  const int tn = (p.ncols + kTN - 1) / kTN;
  if constexpr (!kTg) {
    __syncthreads();
    if (warp == 2) {
      // pair tiles per group: ceil(row tiles / 2) (x tn column tiles where
      // decoded).  Lane l scans groups
      // [l * per, (l + 1) * per), then the lane totals are scanned across the warp
      auto items_of = [&](int g) -> int { return (s_tpre[g + 1] - s_tpre[g] + 1) >> 1; };
      const int per = (p.G + 31) / 32;
      const int g0 = min(lane * per, p.G), g1 = min(g0 + per, p.G);
      int sum = 0;
      for (int g = g0; g < g1; ++g) sum += items_of(g);
      int incl = sum;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
      }
      int run = incl - sum;
      for (int g = g0; g < g1; ++g) {
        s_ppre[g] = run;
        run += items_of(g);
      }
      if (lane == 31) s_ppre[p.G] = incl;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const int total = kTg ? p.G * (p.rtiles / kCta) * tn : s_ppre[p.G] * tn;
  // rank 0's barriers as shared::cluster addresses (a pair's shared barriers)
  const uint32_t full0_cl = kPair ? mapa_shared(smem_u32(full), 0) : 0;
  const uint32_t tempty0_cl = kPair ? mapa_shared(smem_u32(tempty), 0) : 0;
  const WaitCtl ctl{p.wait_limit_ns, abort_flag, p.status};
  const WaitCtl ctl_drain{p.wait_limit_ns, no_abort, p.status};

  if (warp < 4) {
    setmaxnreg_dec<regs_ctl<kPromote>()>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------- TMA producer
      int it = 0;
      bool ok = true;
      // a pair's loads complete on rank 0's full barrier, which rank 0 arms
      // with both CTAs' bytes
      auto load = [&](void *dst, const CUtensorMap *map, int x, int y, int s) {
        if constexpr (kPair) tma_load_2d_pair(dst, map, x, y, full0_cl + 8u * s);
        else tma_load_2d(dst, map, x, y, &full[s]);
      };
      for (int w = w0; ok && w < total; w += wstep) {
        const Item t = decode_item<kMode, kCta>(w, p, s_offs, s_tpre, s_ppre, tn, rank);
        for (int b = 0; b < t.nblocks; ++b, ++it) {
          const int s = it % kSt;
          if (!mbar_wait(&empty[s], ((it / kSt) & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], kStageTx);
          int ax, ay, bx, by;
          if constexpr (!kTg) {
            ax = b * kBKe;
            ay = t.r0;
            if (kBMN) {
              bx = t.ct * kTN;
              by = t.g * p.b_group_rows + b * kBKe;
            } else {
              bx = b * kBKe;
              by = t.g * p.b_group_rows + t.ct * kTN + (kTN / kCta) * rank;
            }
          } else {
            // chunk jj of the group (stages_per_chunk stages each) in the
            // chunk-major operands: line rows jj * N + n and jj * K + k
            const int jj = s_tpre[t.g] + b / p.stages_per_chunk;
            ax = (b % p.stages_per_chunk) * kBKe;
            ay = jj * (p.rtiles * kBM) + t.rt * kBM;  // dout columns n
            bx = ax;
            by = jj * p.ncols + t.ct * kTN + (kTN / kCta) * rank;  // lhs columns k (rows past K belong
                                                      // to the next chunk: their columns are never stored)
          }
          load(sA + s * kAStage, &tmA, ax, ay, s);
          if constexpr (kBMN) {
            // boxes of 128 bytes along n (columns of W[g] in [K, N]); a pair
            // CTA takes tile columns 128 rank ..
#pragma unroll
            for (int h = 0; h < kBBoxes; ++h)
              load(sB + s * kBS + h * kBBoxBytes, &tmB,
                   tile_col_n(t.ct, (kTN / kCta) * rank + h * kBKe, p.swiglu_f, kTN), by, s);
          } else if (!kTg && p.swiglu_f) {
            // boxes of 128 rows (n) of W[g] in [N, K]: gate rows, up rows (a
            // pair CTA loads one of them)
#pragma unroll
            for (int h = 0; h < 2 / kCta; ++h)
              load(sB + s * kBS + h * (kBStage / 2), &tmB, bx,
                   t.g * p.b_group_rows + tile_col_n(t.ct, (h + rank) * 128, p.swiglu_f), s);
          } else {
            load(sB + s * kBS, &tmB, bx, by, s);
          }
        }
      }
      // let every issued copy land before the CTA can exit.  A pair's copies
      // complete on rank 0's barriers, so rank 0 waits for both CTAs' copies;
      // rank 1 leaves only after the closing cluster barrier, which rank 0
      // reaches after this wait.
      if (leader)
        for (int i = (it > kSt ? it - kSt : 0); i < it; ++i)
          mbar_wait(&full[i % kSt], (i / kSt) & 1, ctl_drain);
    } else if (warp == 1 || (kTwo && warp == 3)) {
      // ---------------------------------------------------- MMA issuer(s)
      // two issuers (both in the leader CTA): warp 1 fills buffer 0 (even
      // blocks of a split static tile, or even units), warp 3 buffer 1
      const int par = warp == 3 ? 1 : 0;
      if (lane == 0 && leader) {
        int it = 0, u = 0;
        bool ok = true;
        int nuse = 0;  // split tiles: tiles this issuer accumulated into its buffer
        for (int w = w0; ok && w < total; w += wstep) {
          const Item t = decode_item<kMode, kCta>(w, p, s_offs, s_tpre, s_ppre, tn, rank);
          if constexpr (kSplit) {
            // the same accumulation as the one-CTA static row tiles: even
            // blocks into buffer 0, odd ones into buffer 1, summed by the
            // epilogue
            // (every tile of a row pass has the same block count: see gemm_tc.cu)
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
              const uint32_t a0 = smem_u32(sA + s * kAStage), b0 = smem_u32(sB + s * kBS);
              const uint32_t d = tbase + par * kTN;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t adesc = smem_desc_sw128(a0 + kk * 32, 16, 1024);
                const uint64_t bdesc = kBMN ? smem_desc_sw128(b0 + kk * kMmaK * 128, kBBoxBytes, 1024)
                                            : smem_desc_sw128(b0 + kk * 32, 16, 1024);
                if constexpr (kPair) tc_mma_pair<kF16>(d, adesc, bdesc, kIdesc, (b == par && kk == 0) ? 0u : 1u);
                else tc_mma<kF16>(d, adesc, bdesc, kIdesc, (b == par && kk == 0) ? 0u : 1u);
              }
              if constexpr (kPair) tc_commit_pair_both(&empty[s], 0x3);
              else tc_commit(&empty[s]);
            }
            if (!ok) break;
            if (mine) {
              if constexpr (kPair) tc_commit_pair_both(&tfull[par], 0x3);
              else tc_commit(&tfull[par]);
              ++nuse;
            }
            continue;
          }
          uint32_t buf = 0;
          for (int b = 0; b < t.nblocks; ++b, ++it) {
            const bool unit_start = kPromote || b == 0;
            if (kTwo && (u & 1) != par) {  // the other issuer's unit
              ++u;
              continue;
            }
            if (unit_start) {
              buf = u % kNB;
              if (!mbar_wait(&tempty[buf], ((u / kNB) & 1) ^ 1, ctl)) {
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
            const uint32_t a0 = smem_u32(sA + s * kAStage), b0 = smem_u32(sB + s * kBS);
            const uint32_t d = tbase + buf * kTN;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t adesc = smem_desc_sw128(a0 + kk * 32, 16, 1024);
              const uint64_t bdesc = kBMN ? smem_desc_sw128(b0 + kk * kMmaK * 128, kBBoxBytes, 1024)
                                          : smem_desc_sw128(b0 + kk * 32, 16, 1024);
              // a pair's descriptors name rank 0's shared memory; the tensor
              // core reads the same offsets in rank 1 for its half
              if constexpr (kPair) tc_mma_pair<kF16>(d, adesc, bdesc, kIdesc, (unit_start && kk == 0) ? 0u : 1u);
              else tc_mma<kF16>(d, adesc, bdesc, kIdesc, (unit_start && kk == 0) ? 0u : 1u);
            }
            // stage s free again / TMEM unit ready: in both CTAs of a pair
            if constexpr (kPair) tc_commit_pair_both(&empty[s], 0x3);
            else tc_commit(&empty[s]);
            if (kPromote || b == t.nblocks - 1) {
              if constexpr (kPair) tc_commit_pair_both(&tfull[buf], 0x3);
              else tc_commit(&tfull[buf]);
              ++u;
            }
          }
        }
        if constexpr (kPair) tc_commit_pair_local(drain);
        else tc_commit(drain);
        mbar_wait(drain, 0, ctl_drain);
      }
      __syncwarp();
    } else if (warp == 2 && use_ring) {
      // --------------------------------------------------- scale loader
      // Fills one ring slot per TMEM unit, in the order the epilogue consumes
      // them, so that no global-memory latency sits on the epilogue's path.
      int v = 0;
      bool ok = true;
      for (int w = w0; ok && w < total; w += wstep) {
        const Item t = decode_item<kMode, kCta>(w, p, s_offs, s_tpre, s_ppre, tn, rank);
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
            // kTN / 32 columns per lane (never straddling a gate / up
            // boundary); columns >= ncols are never read
            constexpr int kCpl = kTN / 32;
            const int n = kTg ? t.ct * kTN + kCpl * lane : tile_col_n(t.ct, kCpl * lane, p.swiglu_f, kTN);
            if (n < p.ncols) {
              const float *src =
                  kTg ? p.colblk_scale + (ch0 + j) * p.colblk_ld + n
                      : (kBlkScales ? p.colblk_scale + (static_cast<int64_t>(t.g) * p.kblocks + j) * p.colblk_ld + n
                              : p.col_scale + static_cast<int64_t>(t.g) * p.ncols + n);
              float *dst = s_scol + slot * kBN + kCpl * lane;
#pragma unroll
              for (int e = 0; e < kCpl; e += 4) cp_async_16(dst + e, src + e);
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
    setmaxnreg_inc<regs_epi<kPromote>()>();
    // ---------------------------------------------------------- epilogue
    const int et = threadIdx.x - kEpiWarp0 * 32;  // 0 .. 255
    const int q = warp & 3, h = (warp - kEpiWarp0) >> 2;
    const int row = q * 32 + lane;
    const uint32_t tl = tbase + (static_cast<uint32_t>(q * 32) << 16);  // the warp's TMEM lanes
    const bool sw = !kTg && p.swiglu_f > 0;
    // tile column of the thread's 32-column chunk c (0 .. 3): the column half h
    // of the tile, or for SwiGLU gate columns 64 h .. (c = 0, 1) and the
    // matching up columns 128 + 64 h .. (c = 2, 3)
    auto colt = [&](int c) -> int {
      return sw ? ((c & 2) ? 128 : 0) + h * 64 + (c & 1) * 32 : h * (kTN / 2) + c * 32;
    };
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
      bool got = mbar_wait(&tfull[buf], (u / kNB) & 1, ctl);
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
    // TMEM unit consumed: a pair's epilogue warps arrive on rank 0's barrier
    auto release_unit = [&](uint32_t buf) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair) mbar_arrive_cluster(tempty0_cl + 8u * buf);
        else mbar_arrive(&tempty[buf]);
      }
    };
    for (int w = w0; ok && w < total; w += wstep) {
      const Item t = decode_item<kMode, kCta>(w, p, s_offs, s_tpre, s_ppre, tn, rank);
      const int col0 = t.ct * kTN + h * (kTN / 2);
      int64_t orow;
      bool row_ok;
      if constexpr (!kTg) {
        orow = t.r0 + row;
        row_ok = orow < t.rend;
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
        for (int c = 0; c < kCh; ++c)
          if (col0 + c * 32 < p.ncols) emit(col0 + c * 32, z);
        continue;
      }
      if constexpr (kPromote) {
        float2 acc[kCh * 16];
#pragma unroll
        for (int i = 0; i < kCh * 16; ++i) acc[i] = make_float2(0.0f, 0.0f);
        int slot = 0;
        for (int b = 0; b < t.nblocks; ++b) {
          const uint32_t buf = u % kNB;
          slot = v % kRing;
          if (!wait_unit(buf, slot)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float rs = need_row ? s_srow[slot * kBM + row] : 1.0f;
          const float2 rs2 = make_float2(rs, rs);
          const float *cs = s_scol + slot * kBN;
#pragma unroll
          for (int cp = 0; cp < kCh / 2; ++cp) {
            // chunks 2 cp, 2 cp + 1 (compile-time accumulator indices)
            // colt(2 cp + 1) = colt(2 cp) + 32: one 64-column load
            uint32_t va[32], vb[32];
            tmem_ld64(tl + buf * kTN + colt(2 * cp), va, vb);
            tmem_wait_ld();
            // 128-column tiles: the unit is in registers now; hand its TMEM
            // buffer back before the promotion math
            if constexpr (kCh == 2) release_unit(buf);
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
          if constexpr (kCh != 2) release_unit(buf);
          ++u;
          if (b + 1 < t.nblocks) release_slot(slot);  // the last slot is read again below
        }
        if (!ok) break;
        if (row_ok) {
          // per-channel rhs column scale (in every unit's slot); static lhs: s
          const float fin = ((kTg || kBlkScales) && p.static_scale) ? s_eff : 1.0f;
          const bool colmul = !kTg && p.col_scale != nullptr;
          const float *cf = s_scol + slot * kBN;
          if (kTN == 256 && sw) {  // SwiGLU tiles are 256 wide (128 gate + 128 up columns)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const float *fg = cf + colt(c), *fu = cf + colt(c + 2);
              float o[32];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 a = acc[c * 16 + i], b2 = acc[((c + 2) % kCh) * 16 + i];
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
            for (int c = 0; c < kCh; ++c) {
              const int col = t.ct * kTN + colt(c);
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
        static_assert(kTN == 256, "one pair of units per tile: 256-column tiles");
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
            uint32_t va[32], vb[32];
            tmem_ld64(tl + bi * kTN + colt(2 * cp), va, vb);
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
        release_unit(0);
        if (two) release_unit(1);
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
              const int col = t.ct * kTN + colt(c);
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
        static_assert(kPromote || kTN == 256, "one unit per tile: 256-column tiles");
        const uint32_t buf = u % kNB;
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
          tmem_ld32(tl + buf * kTN + colt(ca), va);
          tmem_ld32(tl + buf * kTN + colt(cb), vb);
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
            const int col = t.ct * kTN + colt(c);
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
        release_unit(buf);
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
  // a pair: neither CTA frees its tensor memory or leaves while the other may
  // still read its shared memory (MMAs) or count bytes on its barriers (loads)
  if constexpr (kPair) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tbase, kTmemCols);
    else tmem_dealloc(tbase, kTmemCols);
  }
}

template <int kElem, bool kBMN, bool kPromote, int kMode, int kTN = 256>
static cudaError_t launch_inst(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                               const GemmParams &p, int items, cudaStream_t st) {
  auto kern = gmm_pair_kernel<kElem, kBMN, kPromote, kMode, kTN>;
  const size_t smem = gemm_smem_bytes<2, kMode, kTN>();
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc waits for registers the CTA owns: never launch a split that
  // does not fit the launch allocation
  if (attr.numRegs * kThreads < regs_ctl<kPromote>() * 128 + regs_epi<kPromote>() * 256)
    return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // clusters of two CTAs; as many pairs as can be resident at once (a
  // persistent grid), never more than there are items
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  static int max_pairs = 0;  // per instantiation
  if (max_pairs == 0) {
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = num_sms() / 2;
    max_pairs = n;
  }
  const int pairs = items < max_pairs ? items : max_pairs;
  if (pairs <= 0) return cudaErrorInvalidConfiguration;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmOut, p);
}

}  // namespace pair

cudaError_t launch_gemm_pair(const GemmConfig &cfg, const CUtensorMap &tmA, const CUtensorMap &tmB,
                             const CUtensorMap &tmOut, const GemmParams &p, int items, cudaStream_t st) {
  using namespace pair;
  if (cfg.tile_n == 128) {  // four 128-column TMEM buffers: promoted E4M3, K-major B
    if (cfg.elem_bytes != 1 || !cfg.promote || cfg.b_mn_major || p.swiglu_f) return cudaErrorInvalidValue;
    if (cfg.mode == MODE_ROWS) return launch_inst<1, false, true, MODE_ROWS, 128>(tmA, tmB, tmOut, p, items, st);
    if (cfg.mode == MODE_TGMM) return launch_inst<1, false, true, MODE_TGMM, 128>(tmA, tmB, tmOut, p, items, st);
    if (cfg.mode == MODE_ROWS_BLK)
      return launch_inst<1, false, true, MODE_ROWS_BLK, 128>(tmA, tmB, tmOut, p, items, st);
    return cudaErrorInvalidValue;
  }
  if (cfg.tile_n != 256) return cudaErrorInvalidValue;
  if (cfg.mode == MODE_TGMM) {
    if (cfg.b_mn_major) return cudaErrorInvalidValue;
    if (cfg.elem_bytes == 1 && cfg.promote) return launch_inst<1, false, true, MODE_TGMM>(tmA, tmB, tmOut, p, items, st);
    if (cfg.elem_bytes == 2 && !cfg.promote)
      return launch_inst<2, false, false, MODE_TGMM>(tmA, tmB, tmOut, p, items, st);
    return cudaErrorInvalidValue;
  }
  if (cfg.mode == MODE_ROWS_BLK) {  // block-wise rhs scales: promoted fp8 only
    if (cfg.elem_bytes != 1 || !cfg.promote) return cudaErrorInvalidValue;
    return cfg.b_mn_major ? launch_inst<1, true, true, MODE_ROWS_BLK>(tmA, tmB, tmOut, p, items, st)
                          : launch_inst<1, false, true, MODE_ROWS_BLK>(tmA, tmB, tmOut, p, items, st);
  }
  if (cfg.elem_bytes == 1) {
    if (cfg.b_mn_major)
      return cfg.promote ? launch_inst<1, true, true, MODE_ROWS>(tmA, tmB, tmOut, p, items, st)
                         : launch_inst<1, true, false, MODE_ROWS>(tmA, tmB, tmOut, p, items, st);
    return cfg.promote ? launch_inst<1, false, true, MODE_ROWS>(tmA, tmB, tmOut, p, items, st)
                       : launch_inst<1, false, false, MODE_ROWS>(tmA, tmB, tmOut, p, items, st);
  }
  if (cfg.promote) return cudaErrorInvalidValue;
  return cfg.b_mn_major ? launch_inst<2, true, false, MODE_ROWS>(tmA, tmB, tmOut, p, items, st)
                        : launch_inst<2, false, false, MODE_ROWS>(tmA, tmB, tmOut, p, items, st);
}

}  // namespace gmm
