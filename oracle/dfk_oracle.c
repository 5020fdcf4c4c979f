/*
 * dfk_oracle.c -- fp64 CPU oracle for the decode-stage SwiGLU MLP.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA library; it reads the same bf16 input bytes and
 * computes the plain definition of the method, slowly and obviously, in
 * double precision.
 *
 * What is computed (source: "Deep Kernel Fusion for Transformer Decoding",
 * episode description -- the method fuses the gate projection, the up
 * projection, the SiLU activation and the elementwise multiply into one
 * decode kernel and keeps the down projection as a separate kernel; "Deep
 * Kernel Fusion for Transformers", abstract -- the SwiGLU MLP block is the
 * target; GPULlama3.java PR #78 "fusing dequantize with compute",
 * description of the `rms_ffn_gate_up` task -- RMS normalisation fused in
 * front of the gate/up projection):
 *
 *   r_b    = 1 / sqrt( (1/D) * sum_k x[b,k]^2 + eps )          (RMSNorm, optional)
 *   xn_bk  = x[b,k] * r_b * gamma[k]                            (else xn = x)
 *   a_bj   = sum_k xn_bk * Wg[j,k]                              (gate projection)
 *   u_bj   = sum_k xn_bk * Wu[j,k]                              (up projection)
 *   h_bj   = SiLU(a_bj) * u_bj,  SiLU(a) = a / (1 + exp(-a))    (SwiGLU)
 *   y_bi   = sum_j h_bj * Wd[i,j]                               (down projection)
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - SiLU is applied to the gate branch (GLU-variant convention, "GLU
 *     Variants Improve Transformer", cited on the episode page).
 *   - RMSNorm divides by D (not D-1), adds eps inside the square root and
 *     multiplies by gamma after normalising.
 *   - Weight layouts are resolved by index arithmetic only:
 *       row-major    Wg[j,k] = Wg_mem[j*D + k]          ([F][D])
 *       column-major Wg[j,k] = Wg_mem[k*F + j]          ([D][F], i.e. W^T)
 *       interleaved  Wg[j,k] = W_mem[(2j)*D + k],
 *                    Wu[j,k] = W_mem[(2j+1)*D + k]      ([F][2][D])
 *
 * Low-precision weights (the "fusing dequantize with compute" idea of
 * GPULlama3.java PR #78, applied to the same MLP): W[j][k] = s[j] * Q[j][k]
 * with Q an FP8 E4M3 code (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent 0 is subnormal, S.1111.111 is NaN, no infinities) and s one
 * fp32 scale per output row.  The dequantised weight is formed exactly in
 * double and used in the same sums as above.
 *
 * "Mirror" mode rounds xn, h and y to bf16 (round to nearest, ties to even)
 * at the points where the GPU kernels store bf16; it is a diagnostic only.
 * The contract check uses the pure mode (mirror = 0).
 *
 * Every output element is an independent serial sum in ascending k, so the
 * result does not depend on the number of OpenMP threads.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_LAYOUT_ROW 0
#define ORC_LAYOUT_COL 1
#define ORC_LAYOUT_INTERLEAVED 2

/* bf16 bits -> double: the bf16 value is the upper half of an IEEE binary32. */
double dfk_oracle_bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* double -> bf16 bits, round to nearest, ties to even, in one rounding step
 * (no intermediate binary32 rounding).  Overflow goes to +-inf, NaN stays NaN.
 * bf16 has 8 significand bits (7 stored), exponent range of binary32. */
uint16_t dfk_oracle_double_to_bf16(double v) {
  if (isnan(v)) return (uint16_t)0x7fc0;
  int neg = signbit(v) ? 1 : 0;
  double a = fabs(v);
  uint16_t sign = (uint16_t)(neg ? 0x8000 : 0);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7f80);
  int e;
  (void)frexp(a, &e);          /* a = m * 2^e, m in [0.5, 1) */
  int exp_unb = e - 1;         /* a = 1.f * 2^exp_unb */
  /* bf16 normal exponents: -126 .. 127; subnormals have quantum 2^-133 */
  int q_exp = (exp_unb < -126) ? -133 : exp_unb - 7;   /* quantum = 2^q_exp */
  double scaled = ldexp(a, -q_exp);                     /* exact */
  double fl = floor(scaled);
  double rem = scaled - fl;
  double n = fl;
  if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) n = fl + 1.0;
  double r = ldexp(n, q_exp);
  if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7f80);
  float f = (float)r;          /* exact: r is representable in bf16 */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(sign | ((u >> 16) & 0x7fff));
}

static double q_bf16(double v) {
  return dfk_oracle_bf16_to_double(dfk_oracle_double_to_bf16(v));
}

/* SiLU(a) = a * sigmoid(a) = a / (1 + exp(-a)).  For a < about -709,
 * exp(-a) overflows to +inf and the quotient is -0, the correct limit. */
double dfk_oracle_silu(double a) { return a / (1.0 + exp(-a)); }

int dfk_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Set the OpenMP thread count for later calls (n <= 0: leave unchanged). */
void dfk_oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* RMSNorm of each of the B rows of x[B][D]; gamma may be NULL (then 1).
 * xn[B][D] in double.  Returns 0, or -1 on bad arguments. */
int dfk_oracle_rmsnorm(const uint16_t *x, const uint16_t *gamma, double eps,
                       int B, int D, int mirror, double *xn) {
  if (!x || !xn || B < 0 || D <= 0) return -1;
  for (int b = 0; b < B; ++b) {
    double ss = 0.0;
    for (int k = 0; k < D; ++k) {
      double v = dfk_oracle_bf16_to_double(x[(size_t)b * D + k]);
      ss += v * v;
    }
    double r = 1.0 / sqrt(ss / (double)D + eps);
    for (int k = 0; k < D; ++k) {
      double v = dfk_oracle_bf16_to_double(x[(size_t)b * D + k]);
      double g = gamma ? dfk_oracle_bf16_to_double(gamma[k]) : 1.0;
      double o = v * r * g;
      xn[(size_t)b * D + k] = mirror ? q_bf16(o) : o;
    }
  }
  return 0;
}

static double w_gate(const uint16_t *wg, int layout, int j, int k, int D, int F) {
  switch (layout) {
    case ORC_LAYOUT_ROW: return dfk_oracle_bf16_to_double(wg[(size_t)j * D + k]);
    case ORC_LAYOUT_COL: return dfk_oracle_bf16_to_double(wg[(size_t)k * F + j]);
    default:             return dfk_oracle_bf16_to_double(wg[(size_t)(2 * j) * D + k]);
  }
}

static double w_up(const uint16_t *wg, const uint16_t *wu, int layout, int j, int k,
                   int D, int F) {
  switch (layout) {
    case ORC_LAYOUT_ROW: return dfk_oracle_bf16_to_double(wu[(size_t)j * D + k]);
    case ORC_LAYOUT_COL: return dfk_oracle_bf16_to_double(wu[(size_t)k * F + j]);
    default:             return dfk_oracle_bf16_to_double(wg[(size_t)(2 * j + 1) * D + k]);
  }
}

/* Gate/up + SwiGLU for the output columns listed in rows[0..nrows) (all F
 * columns, in order, when rows == NULL; then nrows must equal F).
 *   x      [B][D] bf16 bits
 *   gamma  [D] bf16 bits, or NULL: no RMSNorm (xn = x)
 *   wg,wu  weights in `layout`; for the interleaved layout wg holds both and
 *          wu is ignored
 *   h      [B][nrows] out, SiLU(a)*u; a_out/u_out (optional) [B][nrows]
 * Returns 0, or -1 on bad arguments. */
int dfk_oracle_gate_up(const uint16_t *x, const uint16_t *gamma, double eps,
                       const uint16_t *wg, const uint16_t *wu, int layout,
                       int B, int D, int F, const int *rows, int nrows, int mirror,
                       double *h, double *a_out, double *u_out) {
  if (!x || !wg || !h || B < 0 || D <= 0 || F <= 0) return -1;
  if (layout != ORC_LAYOUT_ROW && layout != ORC_LAYOUT_COL &&
      layout != ORC_LAYOUT_INTERLEAVED) return -1;
  if (layout != ORC_LAYOUT_INTERLEAVED && !wu) return -1;
  if (!rows && nrows != F) return -1;
  if (rows)
    for (int i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= F) return -1;

  /* step 1-2: the normalised activations, once per row b */
  double *xn = (double *)malloc(((size_t)B * D + 1) * sizeof(double));
  if (!xn) return -1;
  if (gamma) {
    dfk_oracle_rmsnorm(x, gamma, eps, B, D, mirror, xn);
  } else {
    for (size_t i = 0; i < (size_t)B * D; ++i) xn[i] = dfk_oracle_bf16_to_double(x[i]);
  }

  /* step 3-4: both projections and the SwiGLU product, one output at a time */
#pragma omp parallel for schedule(static)
  for (int i = 0; i < nrows; ++i) {
    int j = rows ? rows[i] : i;
    for (int b = 0; b < B; ++b) {
      const double *xr = xn + (size_t)b * D;
      double a = 0.0, u = 0.0;
      for (int k = 0; k < D; ++k) {
        a += xr[k] * w_gate(wg, layout, j, k, D, F);
        u += xr[k] * w_up(wg, wu, layout, j, k, D, F);
      }
      double hv = dfk_oracle_silu(a) * u;
      h[(size_t)b * nrows + i] = mirror ? q_bf16(hv) : hv;
      if (a_out) a_out[(size_t)b * nrows + i] = a;
      if (u_out) u_out[(size_t)b * nrows + i] = u;
    }
  }
  free(xn);
  return 0;
}

/* Down projection y[b][i] = sum_j h[b][j] * Wd[i][j] for the rows listed in
 * rows[0..nrows) of W_down (all D rows when rows == NULL; nrows == D).
 *   h   [B][F] double
 *   wd  [D][F] bf16 bits, row-major
 *   y   [B][nrows] out
 * Returns 0, or -1 on bad arguments. */
int dfk_oracle_down(const double *h, const uint16_t *wd, int B, int D, int F,
                    const int *rows, int nrows, int mirror, double *y) {
  if (!h || !wd || !y || B < 0 || D <= 0 || F <= 0) return -1;
  if (!rows && nrows != D) return -1;
  if (rows)
    for (int i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= D) return -1;
#pragma omp parallel for schedule(static)
  for (int i = 0; i < nrows; ++i) {
    int r = rows ? rows[i] : i;
    for (int b = 0; b < B; ++b) {
      double s = 0.0;
      for (int j = 0; j < F; ++j)
        s += h[(size_t)b * F + j] * dfk_oracle_bf16_to_double(wd[(size_t)r * F + j]);
      y[(size_t)b * nrows + i] = mirror ? q_bf16(s) : s;
    }
  }
  return 0;
}

/* Per-row rescale used between decode steps of the layer stack:
 * out[b][k] = y[b][k] / sqrt(mean_k y[b][k]^2 + eps). */
int dfk_oracle_rms_rescale(const double *y, double eps, int B, int D, double *out) {
  if (!y || !out || B < 0 || D <= 0) return -1;
  for (int b = 0; b < B; ++b) {
    double ss = 0.0;
    for (int k = 0; k < D; ++k) ss += y[(size_t)b * D + k] * y[(size_t)b * D + k];
    double r = 1.0 / sqrt(ss / (double)D + eps);
    for (int k = 0; k < D; ++k) out[(size_t)b * D + k] = y[(size_t)b * D + k] * r;
  }
  return 0;
}

/* FP8 E4M3 code -> double (exact). */
double dfk_oracle_e4m3_to_double(uint8_t code) {
  const int sign = (code >> 7) & 1;
  const int e = (code >> 3) & 15;
  const int m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);               /* m/8 * 2^(1-7) */
  else v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

static double w_fp8(const uint8_t *q, const float *sc, int j, int k, int D) {
  return (double)sc[j] * dfk_oracle_e4m3_to_double(q[(size_t)j * D + k]);
}

/* Gate/up + SwiGLU with FP8 weights: Wg[j][k] = sg[j] * qg[j][k] (row-major
 * [F][D] codes), likewise Wu; x, gamma as in dfk_oracle_gate_up. */
int dfk_oracle_gate_up_fp8(const uint16_t *x, const uint16_t *gamma, double eps,
                           const uint8_t *qg, const float *sg, const uint8_t *qu,
                           const float *su, int B, int D, int F, const int *rows, int nrows,
                           double *h, double *a_out, double *u_out) {
  if (!x || !qg || !sg || !qu || !su || !h || B < 0 || D <= 0 || F <= 0) return -1;
  if (!rows && nrows != F) return -1;
  if (rows)
    for (int i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= F) return -1;
  double *xn = (double *)malloc(((size_t)B * D + 1) * sizeof(double));
  if (!xn) return -1;
  if (gamma) {
    dfk_oracle_rmsnorm(x, gamma, eps, B, D, 0, xn);
  } else {
    for (size_t i = 0; i < (size_t)B * D; ++i) xn[i] = dfk_oracle_bf16_to_double(x[i]);
  }
#pragma omp parallel for schedule(static)
  for (int i = 0; i < nrows; ++i) {
    int j = rows ? rows[i] : i;
    for (int b = 0; b < B; ++b) {
      const double *xr = xn + (size_t)b * D;
      double a = 0.0, u = 0.0;
      for (int k = 0; k < D; ++k) {
        a += xr[k] * w_fp8(qg, sg, j, k, D);
        u += xr[k] * w_fp8(qu, su, j, k, D);
      }
      h[(size_t)b * nrows + i] = dfk_oracle_silu(a) * u;
      if (a_out) a_out[(size_t)b * nrows + i] = a;
      if (u_out) u_out[(size_t)b * nrows + i] = u;
    }
  }
  free(xn);
  return 0;
}

/* Down projection with FP8 weights: y[b][i] = sum_j h[b][j] * sd[i] * qd[i][j]. */
int dfk_oracle_down_fp8(const double *h, const uint8_t *qd, const float *sd, int B, int D,
                        int F, const int *rows, int nrows, double *y) {
  if (!h || !qd || !sd || !y || B < 0 || D <= 0 || F <= 0) return -1;
  if (!rows && nrows != D) return -1;
  if (rows)
    for (int i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= D) return -1;
#pragma omp parallel for schedule(static)
  for (int i = 0; i < nrows; ++i) {
    int r = rows ? rows[i] : i;
    for (int b = 0; b < B; ++b) {
      double acc = 0.0;
      for (int j = 0; j < F; ++j) acc += h[(size_t)b * F + j] * w_fp8(qd, sd, r, j, F);
      y[(size_t)b * nrows + i] = acc;
    }
  }
  return 0;
}
