/*
 * oracle.c -- plain CPU reference for the FP8 grouped matmul that runs MoE
 * expert MLPs: forward gmm, backward gmm wrt lhs (dlhs) and the transposed
 * gmm wrt rhs (tgmm drhs), plus the quantizers they use.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py load this file.  The CUDA library never links,
 * loads or calls it, and it shares no code, header or table with the CUDA
 * path.
 *
 * Style: explicit loops, no blocking or fusion.  Quantization arithmetic is
 * single-precision, one IEEE round-to-nearest-even operation per C operator
 * (built with -ffp-contract=off so no FMA is formed).  Products of decoded
 * FP8 codes are accumulated in fp64.
 *
 * Sources (page title, section):
 *  - "FP8 Megablox for batch split" (maxtext PR #3770), Description: gmm
 *    forward and backward run FP8 recipes; weights quantized manually
 *    outside the kernel; activations and gradients quantized; W0 and W1
 *    concatenated so one call covers gate and up.
 *  - "Support quantization for tokamax gmm v2" (maxtext PR #4451),
 *    Description and review thread on ops.py: fwd gmm, dlhs gmm (same rhs with
 *    the transpose flag flipped), drhs tgmm; per-channel rhs scale when the
 *    scale is 2-D.
 *  - "add static LHS scaling support for GMM v2 FWD" (maxtext PR #4735),
 *    review threads on the LhsRef docstring (the kernel gets lhs unquantized,
 *    quantizes it as clip(lhs / scale), multiplies the result back by scale;
 *    per-tensor [1,1] scale) and on inner_kernel (dynamic block scale with
 *    inverse = 0 where the scale is 0, multiply, cast to the fp8 dtype).
 *  - OCP 8-bit floating point specification (E4M3 encoding): bias 7, three
 *    mantissa bits, no infinities, S.1111.111 is NaN, largest finite 448.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - the fp8 format is E4M3 and clip means saturate to +-448;
 *  - lhs / scale is computed as lhs * fl32(1/scale) (the inner_kernel form);
 *  - a dynamic scale is fl32(amax / 448) over a block of 128 values along the
 *    contraction axis; a scale whose inverse overflows is treated as 0;
 *  - gradients are always quantized with dynamic blocks; in dlhs the rhs
 *    column scale is folded into dout before quantizing; in tgmm the blocks
 *    are 128 rows long and start at each group's first row;
 *  - rows outside every group produce zero rows; negative group sizes count
 *    as 0 and the groups are clamped so that they end by row M.
 *
 * Parity status: every function here is pinned by tests/test_oracle_*.py
 * (format definition, closed forms, library matmul and autograd special
 * cases, merged/separate identity).  The quantization conventions listed
 * above are readings, not facts the pages fix.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define GMO_Q_NONE 0
#define GMO_Q_STATIC 1
#define GMO_Q_DYNAMIC 2

#define GMO_FLAG_GROUP_SIZES 1
#define GMO_FLAG_SCALE 2

#define BLK 128 /* quantization block length along the contraction axis */

int gmo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---------------------------------------------------------------- formats */

/* Value of an E4M3 code, straight from the format definition. */
double gmo_e4m3_decode(uint8_t c) {
  int sign = c >> 7;
  int e = (c >> 3) & 0xF;
  int m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9); /* subnormal: (m/8) * 2^(1-7) */
  else
    v = ldexp(8.0 + m, e - 10); /* (1 + m/8) * 2^(e-7) */
  return sign ? -v : v;
}

/* Clip to [-448, 448], then round to the nearest E4M3 value with ties going
 * to the even mantissa.  The sign of zero is kept. */
uint8_t gmo_e4m3_encode(double v) {
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs(v);
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2); /* a = f * 2^e2 with f in [0.5, 1) */
  int E = e2 - 1; /* floor(log2(a)) */
  if (E < -6) E = -6; /* below 2^-6 the spacing stays 2^-9 */
  double q = ldexp(a, 3 - E); /* a in units of the spacing 2^(E-3), exact */
  double fl = floor(q);
  double frac = q - fl;
  double r;
  if (frac > 0.5)
    r = fl + 1.0;
  else if (frac < 0.5)
    r = fl;
  else
    r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  if (E == -6 && r < 8.0) return sign | (uint8_t)r; /* subnormal or zero */
  if (r == 16.0) { /* carried into the next binade */
    r = 8.0;
    E += 1;
  }
  return sign | (uint8_t)(((E + 7) << 3) | ((int)r - 8));
}

float gmo_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ------------------------------------------------------------------ scales */

/* Dynamic scale of a block with absolute maximum amax: s = amax / 448 and
 * inv = 1 / s, with inv = 0 where s == 0; a scale so small that 1/s
 * overflows is treated as 0 too. */
static void dyn_scale(float amax, float *s_out, float *inv_out) {
  float s = amax / 448.0f;
  float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
  if (isinf(inv)) {
    s = 0.0f;
    inv = 0.0f;
  }
  *s_out = s;
  *inv_out = inv;
}

/* A static per-tensor scale is usable when it is finite and above FLT_MIN;
 * its inverse is then finite too. */
int gmo_static_scale_ok(float s) { return isfinite(s) && s > FLT_MIN; }

/* -------------------------------------------------------------------- plan */

/* Row offsets of the groups.  Negative sizes count as 0 and each group is
 * clamped to the rows that remain below M.  offs has G+1 entries; flags gets
 * GMO_FLAG_GROUP_SIZES when anything had to be clamped. */
void gmo_plan(const int32_t *sizes, int32_t G, int64_t M, int64_t *offs, int32_t *flags) {
  int64_t run = 0;
  int bad = 0;
  for (int32_t g = 0; g < G; ++g) {
    int64_t s = sizes[g];
    if (s < 0) {
      bad = 1;
      s = 0;
    }
    offs[g] = run < M ? run : M; /* the group ends at offs[g+1], also clamped */
    run += s;
  }
  offs[G] = run < M ? run : M;
  if (run > M) bad = 1;
  if (flags) *flags = bad ? GMO_FLAG_GROUP_SIZES : 0;
}

static int32_t group_of_row(const int64_t *offs, int32_t G, int64_t m) {
  for (int32_t g = 0; g < G; ++g)
    if (m >= offs[g] && m < offs[g + 1]) return g;
  return -1;
}

/* ---------------------------------------------------------------- quantize */

/* Quantize a row-major bf16 matrix [rows, cols] in blocks of 128 values
 * along each row.  Dynamic: one scale per (row, block).  Static: the given
 * per-tensor scale for every block.  scales is [rows][cols/128]. */
void gmo_quantize_rows(const uint16_t *x, int64_t rows, int64_t cols, int32_t rule, float s_static,
                       uint8_t *codes, float *scales, int32_t *flags) {
  int64_t nb = cols / BLK;
  int static_ok = gmo_static_scale_ok(s_static);
  if (flags) *flags = (rule == GMO_Q_STATIC && !static_ok) ? GMO_FLAG_SCALE : 0;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const uint16_t *xb = x + r * cols + b * BLK;
      float s, inv;
      if (rule == GMO_Q_STATIC) {
        s = static_ok ? s_static : 0.0f;
        inv = static_ok ? 1.0f / s_static : 0.0f;
      } else {
        float amax = 0.0f;
        for (int i = 0; i < BLK; ++i) {
          float a = fabsf(gmo_bf16_to_f32(xb[i]));
          if (a > amax) amax = a;
        }
        dyn_scale(amax, &s, &inv);
      }
      scales[r * nb + b] = s;
      for (int i = 0; i < BLK; ++i) {
        float t = gmo_bf16_to_f32(xb[i]) * inv;
        codes[r * cols + b * BLK + i] = gmo_e4m3_encode((double)t);
      }
    }
  }
}

/* The dlhs operand: t[m,n] = fl32(dout[m,n] * s_r[g(m), n]), quantized with
 * dynamic 128-blocks along n.  Rows outside every group get t = 0. */
void gmo_quantize_rows_scaled(const uint16_t *dout, int64_t M, int64_t N, const float *sr,
                              const int32_t *sizes, int32_t G, uint8_t *codes, float *scales) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
  int64_t nb = N / BLK;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    int32_t g = group_of_row(offs, G, m);
    for (int64_t b = 0; b < nb; ++b) {
      float t[BLK];
      float amax = 0.0f;
      for (int i = 0; i < BLK; ++i) {
        int64_t n = b * BLK + i;
        t[i] = (g < 0) ? 0.0f : gmo_bf16_to_f32(dout[m * N + n]) * sr[(int64_t)g * N + n];
        float a = fabsf(t[i]);
        if (a > amax) amax = a;
      }
      float s, inv;
      dyn_scale(amax, &s, &inv);
      scales[m * nb + b] = s;
      for (int i = 0; i < BLK; ++i) codes[m * N + b * BLK + i] = gmo_e4m3_encode((double)(t[i] * inv));
    }
  }
  free(offs);
}

/* Weights W[g, k, n] (bf16): one scale per (g, n), the absolute maximum over
 * k divided by 448 (per-channel rhs scale of shape [G, N]). */
void gmo_quantize_rhs(const uint16_t *w, int32_t G, int64_t K, int64_t N, uint8_t *codes, float *scales) {
#pragma omp parallel for schedule(static)
  for (int64_t gn = 0; gn < (int64_t)G * N; ++gn) {
    int64_t g = gn / N, n = gn % N;
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(gmo_bf16_to_f32(w[(g * K + k) * N + n]));
      if (a > amax) amax = a;
    }
    float s, inv;
    dyn_scale(amax, &s, &inv);
    scales[g * N + n] = s;
    for (int64_t k = 0; k < K; ++k) {
      float t = gmo_bf16_to_f32(w[(g * K + k) * N + n]) * inv;
      codes[(g * K + k) * N + n] = gmo_e4m3_encode((double)t);
    }
  }
}

/* Number of 128-row chunks over all groups. */
int64_t gmo_num_chunks(const int32_t *sizes, int32_t G, int64_t M) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
  int64_t n = 0;
  for (int32_t g = 0; g < G; ++g) n += (offs[g + 1] - offs[g] + BLK - 1) / BLK;
  free(offs);
  return n;
}

/* tgmm operand quantization: each group's rows are cut into chunks of 128
 * rows starting at the group's first row; every column of every chunk gets
 * one scale (dynamic) or the static scale.  codes keep x's layout [M, C];
 * rows outside every group get code 0.  scales is [num_chunks][C] with the
 * chunks in group order. */
void gmo_quantize_chunks(const uint16_t *x, int64_t M, int64_t C, int32_t rule, float s_static,
                         const int32_t *sizes, int32_t G, uint8_t *codes, float *scales) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
  int static_ok = gmo_static_scale_ok(s_static);
  memset(codes, 0, (size_t)(M * C));
  int64_t chunk0 = 0;
  for (int32_t g = 0; g < G; ++g) {
    int64_t r0 = offs[g], r1 = offs[g + 1];
    int64_t nch = (r1 - r0 + BLK - 1) / BLK;
#pragma omp parallel for schedule(static)
    for (int64_t cj = 0; cj < nch * C; ++cj) {
      int64_t c = cj / C, j = cj % C;
      int64_t a0 = r0 + c * BLK, a1 = a0 + BLK < r1 ? a0 + BLK : r1;
      float s, inv;
      if (rule == GMO_Q_STATIC) {
        s = static_ok ? s_static : 0.0f;
        inv = static_ok ? 1.0f / s_static : 0.0f;
      } else {
        float amax = 0.0f;
        for (int64_t m = a0; m < a1; ++m) {
          float a = fabsf(gmo_bf16_to_f32(x[m * C + j]));
          if (a > amax) amax = a;
        }
        dyn_scale(amax, &s, &inv);
      }
      scales[(chunk0 + c) * C + j] = s;
      for (int64_t m = a0; m < a1; ++m) {
        float t = gmo_bf16_to_f32(x[m * C + j]) * inv;
        codes[m * C + j] = gmo_e4m3_encode((double)t);
      }
    }
    chunk0 += nch;
  }
  free(offs);
}

/* ------------------------------------------------------------- the passes */

static void decode_table(double *tab) {
  for (int c = 0; c < 256; ++c) tab[c] = gmo_e4m3_decode((uint8_t)c);
}

/* Forward gmm on selected rows:
 *   out[m, n] = s_r[g, n] * sum_b s_l[m, b] * sum_{k in block b} dec(q_l[m,k]) * dec(q_r[g,k,n])
 * with g the group of row m (rows in no group give 0).  absum holds the same
 * sum over |terms| (the tolerance scale).  rhs codes are [G, K, N]; rows is a
 * list of nrows row indices, out and absum are [nrows][N]. */
void gmo_gmm_fwd(const uint16_t *lhs, int32_t rule, float s_static, const uint8_t *qr, const float *sr,
                 const int32_t *sizes, int32_t G, int64_t M, int64_t K, int64_t N, const int64_t *rows,
                 int64_t nrows, double *out, double *absum) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
  double tab[256];
  decode_table(tab);
  int64_t nb = K / BLK;
#pragma omp parallel
  {
    uint8_t *ql = (uint8_t *)malloc((size_t)K);
    float *sl = (float *)malloc(sizeof(float) * nb);
    double *blk = (double *)malloc(sizeof(double) * N);
    double *bab = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
      int64_t m = rows[i];
      double *o = out + i * N, *a = absum + i * N;
      for (int64_t n = 0; n < N; ++n) o[n] = a[n] = 0.0;
      int32_t g = group_of_row(offs, G, m);
      if (g < 0) continue;
      gmo_quantize_rows(lhs + m * K, 1, K, rule, s_static, ql, sl, NULL);
      for (int64_t b = 0; b < nb; ++b) {
        for (int64_t n = 0; n < N; ++n) blk[n] = bab[n] = 0.0;
        for (int64_t k = b * BLK; k < (b + 1) * BLK; ++k) {
          double x = tab[ql[k]];
          const uint8_t *wrow = qr + ((int64_t)g * K + k) * N;
          for (int64_t n = 0; n < N; ++n) {
            double p = x * tab[wrow[n]];
            blk[n] += p;
            bab[n] += fabs(p);
          }
        }
        for (int64_t n = 0; n < N; ++n) {
          o[n] += (double)sl[b] * blk[n];
          a[n] += (double)sl[b] * bab[n];
        }
      }
      for (int64_t n = 0; n < N; ++n) {
        o[n] *= (double)sr[(int64_t)g * N + n];
        a[n] *= (double)sr[(int64_t)g * N + n];
      }
    }
    free(ql);
    free(sl);
    free(blk);
    free(bab);
  }
  free(offs);
}

/* Backward gmm wrt lhs on selected rows:
 *   t[m, n] = fl32(dout[m, n] * s_r[g, n]), quantized in 128-blocks along n
 *   dlhs[m, k] = sum_b s_t[m, b] * sum_{n in block b} dec(q_t[m,n]) * dec(q_r[g,k,n])
 * i.e. a gmm against the same rhs codes with the roles of K and N swapped. */
void gmo_gmm_dlhs(const uint16_t *dout, const uint8_t *qr, const float *sr, const int32_t *sizes, int32_t G,
                  int64_t M, int64_t K, int64_t N, const int64_t *rows, int64_t nrows, double *out,
                  double *absum) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
  double tab[256];
  decode_table(tab);
  int64_t nb = N / BLK;
#pragma omp parallel
  {
    float *t = (float *)malloc(sizeof(float) * N);
    uint8_t *qt = (uint8_t *)malloc((size_t)N);
    float *st = (float *)malloc(sizeof(float) * nb);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
      int64_t m = rows[i];
      double *o = out + i * K, *a = absum + i * K;
      for (int64_t k = 0; k < K; ++k) o[k] = a[k] = 0.0;
      int32_t g = group_of_row(offs, G, m);
      if (g < 0) continue;
      for (int64_t b = 0; b < nb; ++b) {
        float amax = 0.0f;
        for (int64_t n = b * BLK; n < (b + 1) * BLK; ++n) {
          t[n] = gmo_bf16_to_f32(dout[m * N + n]) * sr[(int64_t)g * N + n];
          if (fabsf(t[n]) > amax) amax = fabsf(t[n]);
        }
        float s, inv;
        dyn_scale(amax, &s, &inv);
        st[b] = s;
        for (int64_t n = b * BLK; n < (b + 1) * BLK; ++n) qt[n] = gmo_e4m3_encode((double)(t[n] * inv));
      }
      for (int64_t k = 0; k < K; ++k) {
        const uint8_t *wrow = qr + ((int64_t)g * K + k) * N;
        for (int64_t b = 0; b < nb; ++b) {
          double sum = 0.0, sab = 0.0;
          for (int64_t n = b * BLK; n < (b + 1) * BLK; ++n) {
            double p = tab[qt[n]] * tab[wrow[n]];
            sum += p;
            sab += fabs(p);
          }
          o[k] += (double)st[b] * sum;
          a[k] += (double)st[b] * sab;
        }
      }
    }
    free(t);
    free(qt);
    free(st);
  }
  free(offs);
}

/* ------------------------------------------------ block-wise rhs scales */

/* Weights with one scale per 128-block along one axis of W[g] ("Support
 * quantization for tokamax gmm v2", maxtext PR #4451, review thread on the
 * rhs scale: a 2-D scale is per channel, a 3-D scale block-wise):
 *   axis 0: blocks of 128 k for each column n, scales [G, K/128, N] -- block-
 *           wise along the forward's contraction;
 *   axis 1: blocks of 128 n for each row k, scales [G, N/128, K] -- block-
 *           wise along the contraction of dlhs.
 * codes keep W's layout [G, K, N].  Each block: s = fl32(amax / 448),
 * inv = fl32(1 / s) (0 when s is 0 or the inverse overflows), code =
 * e4m3(fl32(w * inv)).  K and N are multiples of 128. */
void gmo_quantize_rhs_blocks(const uint16_t *w, int32_t G, int64_t K, int64_t N, int32_t axis, uint8_t *codes,
                             float *scales) {
  const int64_t kb_n = K / BLK, nb_n = N / BLK;
#pragma omp parallel for schedule(static)
  for (int32_t g = 0; g < G; ++g) {
    const uint16_t *wg = w + (int64_t)g * K * N;
    uint8_t *cg = codes + (int64_t)g * K * N;
    if (axis == 0) {
      for (int64_t kb = 0; kb < kb_n; ++kb)
        for (int64_t n = 0; n < N; ++n) {
          float amax = 0.0f;
          for (int64_t k = kb * BLK; k < (kb + 1) * BLK; ++k) {
            float v = fabsf(gmo_bf16_to_f32(wg[k * N + n]));
            if (v > amax) amax = v;
          }
          float sc, inv;
          dyn_scale(amax, &sc, &inv);
          scales[((int64_t)g * kb_n + kb) * N + n] = sc;
          for (int64_t k = kb * BLK; k < (kb + 1) * BLK; ++k)
            cg[k * N + n] = gmo_e4m3_encode((double)(gmo_bf16_to_f32(wg[k * N + n]) * inv));
        }
    } else {
      for (int64_t k = 0; k < K; ++k)
        for (int64_t nb = 0; nb < nb_n; ++nb) {
          float amax = 0.0f;
          for (int64_t n = nb * BLK; n < (nb + 1) * BLK; ++n) {
            float v = fabsf(gmo_bf16_to_f32(wg[k * N + n]));
            if (v > amax) amax = v;
          }
          float sc, inv;
          dyn_scale(amax, &sc, &inv);
          scales[((int64_t)g * nb_n + nb) * K + k] = sc;
          for (int64_t n = nb * BLK; n < (nb + 1) * BLK; ++n)
            cg[k * N + n] = gmo_e4m3_encode((double)(gmo_bf16_to_f32(wg[k * N + n]) * inv));
        }
    }
  }
}

/* Forward gmm with block-wise rhs scales s_r[g, b, n] ([G, K/128, N]) on
 * selected rows:
 *   out[m, n] = sum_b s_l[m, b] * s_r[g, b, n] * sum_{k in b} dec(q_l[m,k]) * dec(q_r[g,k,n])
 * with s_l[m, b] = s for the static rule.  Rows outside every group are 0. */
void gmo_gmm_fwd_blockwise(const uint16_t *lhs, int32_t rule, float s_static, const uint8_t *qr, const float *srb,
                           const int32_t *sizes, int32_t G, int64_t M, int64_t K, int64_t N, const int64_t *rows,
                           int64_t nrows, double *out, double *absum) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
  double tab[256];
  decode_table(tab);
  int64_t nb = K / BLK;
#pragma omp parallel
  {
    uint8_t *ql = (uint8_t *)malloc((size_t)K);
    float *sl = (float *)malloc(sizeof(float) * nb);
    double *blk = (double *)malloc(sizeof(double) * N);
    double *bab = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
      int64_t m = rows[i];
      double *o = out + i * N, *a = absum + i * N;
      for (int64_t n = 0; n < N; ++n) o[n] = a[n] = 0.0;
      int32_t g = group_of_row(offs, G, m);
      if (g < 0) continue;
      gmo_quantize_rows(lhs + m * K, 1, K, rule, s_static, ql, sl, NULL);
      for (int64_t b = 0; b < nb; ++b) {
        for (int64_t n = 0; n < N; ++n) blk[n] = bab[n] = 0.0;
        for (int64_t k = b * BLK; k < (b + 1) * BLK; ++k) {
          double x = tab[ql[k]];
          const uint8_t *wrow = qr + ((int64_t)g * K + k) * N;
          for (int64_t n = 0; n < N; ++n) {
            double p = x * tab[wrow[n]];
            blk[n] += p;
            bab[n] += fabs(p);
          }
        }
        const float *sb = srb + ((int64_t)g * nb + b) * N;
        for (int64_t n = 0; n < N; ++n) {
          o[n] += (double)sl[b] * (double)sb[n] * blk[n];
          a[n] += (double)sl[b] * (double)sb[n] * bab[n];
        }
      }
    }
    free(ql);
    free(sl);
    free(blk);
    free(bab);
  }
  free(offs);
}

/* dlhs with block-wise rhs scales along n, s_r[g, b, k] ([G, N/128, K]), on
 * selected rows.  dout is quantized on its own (dynamic 128-blocks along n;
 * no rhs scale is folded in, since it now varies along k too):
 *   dlhs[m, k] = sum_b s_d[m, b] * s_r[g, b, k] * sum_{n in b} dec(q_d[m,n]) * dec(q_r[g,k,n]) */
void gmo_gmm_dlhs_blockwise(const uint16_t *dout, const uint8_t *qr, const float *srb, const int32_t *sizes,
                            int32_t G, int64_t M, int64_t K, int64_t N, const int64_t *rows, int64_t nrows,
                            double *out, double *absum) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
  double tab[256];
  decode_table(tab);
  int64_t nb = N / BLK;
#pragma omp parallel
  {
    uint8_t *qd = (uint8_t *)malloc((size_t)N);
    float *sd = (float *)malloc(sizeof(float) * nb);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
      int64_t m = rows[i];
      double *o = out + i * K, *a = absum + i * K;
      for (int64_t k = 0; k < K; ++k) o[k] = a[k] = 0.0;
      int32_t g = group_of_row(offs, G, m);
      if (g < 0) continue;
      gmo_quantize_rows(dout + m * N, 1, N, GMO_Q_DYNAMIC, 0.0f, qd, sd, NULL);
      for (int64_t k = 0; k < K; ++k) {
        const uint8_t *wrow = qr + ((int64_t)g * K + k) * N;
        for (int64_t b = 0; b < nb; ++b) {
          double sum = 0.0, sab = 0.0;
          for (int64_t n = b * BLK; n < (b + 1) * BLK; ++n) {
            double p = tab[qd[n]] * tab[wrow[n]];
            sum += p;
            sab += fabs(p);
          }
          double f = (double)sd[b] * (double)srb[((int64_t)g * nb + b) * K + k];
          o[k] += f * sum;
          a[k] += f * sab;
        }
      }
    }
    free(qd);
    free(sd);
  }
  free(offs);
}

/* Transposed gmm (weight gradient) on selected (g, k) rows of dW:
 *   dW[g, k, n] = sum_c s_x[c, k] * s_d[c, n] * sum_{m in chunk c} dec(q_x[m,k]) * dec(q_d[m,n])
 * over the 128-row chunks c of group g; an empty group gives dW[g] = 0.
 * sel holds indices g*K + k; out and absum are [nsel][N]. */
void gmo_tgmm_drhs(const uint16_t *x, int32_t rule, float s_static, const uint16_t *dout, const int32_t *sizes,
                   int32_t G, int64_t M, int64_t K, int64_t N, const int64_t *sel, int64_t nsel, double *out,
                   double *absum) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
  int64_t nch_all = gmo_num_chunks(sizes, G, M);
  int64_t *chunk0 = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  chunk0[0] = 0;
  for (int32_t g = 0; g < G; ++g) chunk0[g + 1] = chunk0[g] + (offs[g + 1] - offs[g] + BLK - 1) / BLK;
  uint8_t *qx = (uint8_t *)malloc((size_t)(M * K));
  uint8_t *qd = (uint8_t *)malloc((size_t)(M * N));
  float *sx = (float *)malloc(sizeof(float) * (nch_all * K + 1));
  float *sd = (float *)malloc(sizeof(float) * (nch_all * N + 1));
  gmo_quantize_chunks(x, M, K, rule, s_static, sizes, G, qx, sx);
  gmo_quantize_chunks(dout, M, N, GMO_Q_DYNAMIC, 0.0f, sizes, G, qd, sd);
  double tab[256];
  decode_table(tab);
#pragma omp parallel
  {
    double *blk = (double *)malloc(sizeof(double) * N);
    double *bab = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < nsel; ++i) {
      int64_t g = sel[i] / K, k = sel[i] % K;
      double *o = out + i * N, *a = absum + i * N;
      for (int64_t n = 0; n < N; ++n) o[n] = a[n] = 0.0;
      int64_t r0 = offs[g], r1 = offs[g + 1];
      for (int64_t c = 0; r0 + c * BLK < r1; ++c) {
        int64_t a0 = r0 + c * BLK, a1 = a0 + BLK < r1 ? a0 + BLK : r1;
        for (int64_t n = 0; n < N; ++n) blk[n] = bab[n] = 0.0;
        for (int64_t m = a0; m < a1; ++m) {
          double xv = tab[qx[m * K + k]];
          const uint8_t *drow = qd + m * N;
          for (int64_t n = 0; n < N; ++n) {
            double p = xv * tab[drow[n]];
            blk[n] += p;
            bab[n] += fabs(p);
          }
        }
        double sxk = (double)sx[(chunk0[g] + c) * K + k];
        const float *sdc = sd + (chunk0[g] + c) * N;
        for (int64_t n = 0; n < N; ++n) {
          o[n] += sxk * (double)sdc[n] * blk[n];
          a[n] += sxk * (double)sdc[n] * bab[n];
        }
      }
    }
    free(blk);
    free(bab);
  }
  free(qx);
  free(qd);
  free(sx);
  free(sd);
  free(chunk0);
  free(offs);
}

/* ------------------------------------------------ bf16 family (no quant) */

/* out[m, n] = sum_k lhs[m,k] * W[g,k,n] with bf16 operands, fp64 sums. */
void gmo_gmm_fwd_bf16(const uint16_t *lhs, const uint16_t *w, const int32_t *sizes, int32_t G, int64_t M,
                      int64_t K, int64_t N, const int64_t *rows, int64_t nrows, double *out, double *absum) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t m = rows[i];
    double *o = out + i * N, *a = absum + i * N;
    for (int64_t n = 0; n < N; ++n) o[n] = a[n] = 0.0;
    int32_t g = group_of_row(offs, G, m);
    if (g < 0) continue;
    for (int64_t k = 0; k < K; ++k) {
      double xv = gmo_bf16_to_f32(lhs[m * K + k]);
      const uint16_t *wrow = w + ((int64_t)g * K + k) * N;
      for (int64_t n = 0; n < N; ++n) {
        double p = xv * gmo_bf16_to_f32(wrow[n]);
        o[n] += p;
        a[n] += fabs(p);
      }
    }
  }
  free(offs);
}

/* dlhs[m, k] = sum_n dout[m,n] * W[g,k,n] with bf16 operands. */
void gmo_gmm_dlhs_bf16(const uint16_t *dout, const uint16_t *w, const int32_t *sizes, int32_t G, int64_t M,
                       int64_t K, int64_t N, const int64_t *rows, int64_t nrows, double *out, double *absum) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t m = rows[i];
    double *o = out + i * K, *a = absum + i * K;
    for (int64_t k = 0; k < K; ++k) o[k] = a[k] = 0.0;
    int32_t g = group_of_row(offs, G, m);
    if (g < 0) continue;
    for (int64_t k = 0; k < K; ++k) {
      const uint16_t *wrow = w + ((int64_t)g * K + k) * N;
      double sum = 0.0, sab = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        double p = (double)gmo_bf16_to_f32(dout[m * N + n]) * gmo_bf16_to_f32(wrow[n]);
        sum += p;
        sab += fabs(p);
      }
      o[k] = sum;
      a[k] = sab;
    }
  }
  free(offs);
}

/* dW[g, k, n] = sum_{m in group g} x[m,k] * dout[m,n] with bf16 operands. */
void gmo_tgmm_drhs_bf16(const uint16_t *x, const uint16_t *dout, const int32_t *sizes, int32_t G, int64_t M,
                        int64_t K, int64_t N, const int64_t *sel, int64_t nsel, double *out, double *absum) {
  int64_t *offs = (int64_t *)malloc(sizeof(int64_t) * (G + 1));
  gmo_plan(sizes, G, M, offs, NULL);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nsel; ++i) {
    int64_t g = sel[i] / K, k = sel[i] % K;
    double *o = out + i * N, *a = absum + i * N;
    for (int64_t n = 0; n < N; ++n) o[n] = a[n] = 0.0;
    for (int64_t m = offs[g]; m < offs[g + 1]; ++m) {
      double xv = gmo_bf16_to_f32(x[m * K + k]);
      for (int64_t n = 0; n < N; ++n) {
        double p = xv * gmo_bf16_to_f32(dout[m * N + n]);
        o[n] += p;
        a[n] += fabs(p);
      }
    }
  }
  free(offs);
}
