/*
 * Oracle for static per-tensor FP8 E4M3 W8A8 Linear blocks.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * CPU definition that the CUDA path is checked against.  It is compiled into
 * its own shared library and may be loaded only by the tests, by the smoke
 * check and by the CPU-baseline leg of the benchmark.  It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never loads
 * it.
 *
 * Sources (the three pages the method is described on):
 *  [MC]  Hugging Face model card "Cosmos3-Nano-Policy-DROID, FP8 + RTN +
 *        moving-average activation observer (ModelOpt W8A8, per-tensor
 *        static)": Scheme table, Verification table, experiment-setup table
 *        (evaluation paths).
 *  [PR]  TensorRT-LLM pull request "Load static FP8 Cosmos3 Nano/Super
 *        checkpoints without re-quantizing them": Description, What changed,
 *        Test Coverage.
 *  [BLOG] "Running Cosmos 3 Robot Policies on a Single RTX 4090".
 *
 * Readings where the pages are silent (each one also listed in the design
 * notes):
 *  - E4M3 is the OCP 8-bit float with 4 exponent bits (bias 7), 3 mantissa
 *    bits, no infinities, codes 0x7F/0xFF are NaN, largest finite 448.
 *  - Quantize divides by the scale in IEEE fp32, saturates to +-448 and rounds
 *    to the nearest code, ties to the code with an even mantissa.
 *  - The observer averages the per-batch absolute maxima with constant 0.01,
 *    starting from the first batch's maximum.
 *  - SiLU(g) = g / (1 + exp(-g)).
 *
 * Every floating-point step is in fp64 unless a step says fp32.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* E4M3 codebook (format named in [MC] Scheme table: "FP8 E4M3").            */
/* ------------------------------------------------------------------------ */

static double g_codebook[256];
static int g_codebook_ready = 0;

/* Enumerate every code: sign s, exponent field e (4 bits, bias 7), mantissa
 * field m (3 bits).  e == 0 is subnormal: m * 2^-9.  Otherwise
 * (1 + m/8) * 2^(e-7).  0x7F and 0xFF are NaN. */
static void build_codebook(void) {
  for (int c = 0; c < 256; ++c) {
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) {
      mag = NAN;
    } else if (e == 0) {
      mag = (double)m * 0.001953125; /* m * 2^-9 */
    } else {
      double p = 1.0;
      for (int i = 0; i < e - 7; ++i) p *= 2.0;
      for (int i = 0; i < 7 - e; ++i) p *= 0.5;
      mag = (1.0 + (double)m / 8.0) * p;
    }
    g_codebook[c] = s ? -mag : mag;
  }
  g_codebook_ready = 1;
}

static const double *codebook(void) {
  if (!g_codebook_ready) build_codebook();
  return g_codebook;
}

/* Copy the 256-entry table out (NaN for the two NaN codes). */
void oracle_e4m3_codebook(double *out256) {
  const double *cb = codebook();
  memcpy(out256, cb, 256 * sizeof(double));
}

double oracle_e4m3_decode(uint8_t code) { return codebook()[code]; }

/* Nearest code to a real value t (already divided by the scale).  Positive
 * finite codes 0x00..0x7E are strictly increasing in their low 7 bits, so a
 * binary search over them finds the bracket.  Saturating: |t| >= 448 gives the
 * largest finite code.  Ties go to the code whose mantissa LSB is 0 (the even
 * code).  The sign bit follows the sign of t, including -0. */
static uint8_t nearest_code(double t) {
  const double *cb = codebook();
  if (isnan(t)) return 0x7F;
  uint8_t sign = signbit(t) ? 0x80 : 0x00;
  double a = fabs(t);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  /* largest lo in [0, 0x7E] with cb[lo] <= a */
  int lo = 0, hi = 0x7E;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (cb[mid] <= a) lo = mid; else hi = mid - 1;
  }
  int pick = lo;
  if (lo < 0x7E) {
    double dlo = a - cb[lo];
    double dhi = cb[lo + 1] - a;
    if (dhi < dlo) pick = lo + 1;
    else if (dhi == dlo) pick = (lo & 1) ? lo + 1 : lo;
  }
  return (uint8_t)(sign | pick);
}

/* bf16 bits -> value (exact). */
static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static float bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round a double to bf16 (8 significant bits, fp32 exponent range), nearest,
 * ties to even, in one step (no intermediate fp32 rounding). */
uint16_t oracle_round_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  /* largest finite bf16 is (2 - 2^-7) * 2^127; halfway to 2^128 rounds up */
  double maxf = (2.0 - 1.0 / 128.0) * ldexp(1.0, 127);
  double half_up = (2.0 - 1.0 / 256.0) * ldexp(1.0, 127);
  if (a >= half_up) return (uint16_t)(sign | 0x7F80);
  int e;
  frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1): 2^(e-1) <= a < 2^e */
  int exp2 = e - 1;      /* floor(log2 a) */
  if (exp2 < -126) exp2 = -126; /* subnormal range keeps the min-normal quantum */
  double quantum = ldexp(1.0, exp2 - 7);
  double r = a / quantum; /* exact: power-of-two division */
  double fl = floor(r);
  double frac = r - fl;
  double ri;
  if (frac > 0.5) ri = fl + 1.0;
  else if (frac < 0.5) ri = fl;
  else ri = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  double v = ri * quantum;
  if (v > maxf) return (uint16_t)(sign | 0x7F80);
  float f = (float)v; /* exact: v has <= 8 significant bits in fp32 range */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

void oracle_round_bf16_array(const double *x, int64_t n, uint16_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_bf16(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Quantize ([MC] Scheme table: activations FP8 E4M3 with one static scale;  */
/* [PR] What changed: the shared activation is quantized once).             */
/* ------------------------------------------------------------------------ */

/* q(v, s): t = fp32(v) / fp32(s) in IEEE fp32, then saturate and round to the
 * nearest code. */
uint8_t oracle_quant_f32(float v, float s) {
  volatile float t = v / s; /* fp32 division, correctly rounded */
  return nearest_code((double)t);
}

/* q64(v, s): t = v / s in fp64, then saturate and round to the nearest code. */
uint8_t oracle_quant_f64(double v, double s) { return nearest_code(v / s); }

/* Quantize a bf16 tensor of n elements with a static scale. */
void oracle_quantize_bf16(const uint16_t *x, int64_t n, float s, uint8_t *q) {
  for (int64_t i = 0; i < n; ++i) q[i] = oracle_quant_f32(bf16_to_float(x[i]), s);
}

/* ------------------------------------------------------------------------ */
/* Calibration ([MC] Scheme table: round-to-nearest weights with one scale   */
/* per tensor; activation scales from the MOVING_AVERAGE_MINMAX observer     */
/* with averaging constant 0.01; the card's header says the observer        */
/* averages the maxima of the calibration calls instead of taking the max).  */
/* ------------------------------------------------------------------------ */

/* max |x| over a bf16 tensor (exact). */
double oracle_absmax_bf16(const uint16_t *x, int64_t n) {
  double m = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    double a = fabs(bf16_to_double(x[i]));
    if (a > m) m = a;
  }
  return m;
}

/* Moving average of per-batch maxima: A_1 = a_1, A_b = A_{b-1} + c (a_b - A_{b-1}). */
double oracle_moving_average(const double *amax, int nbatch, double c) {
  if (nbatch <= 0) return 0.0;
  double A = amax[0];
  for (int b = 1; b < nbatch; ++b) A = A + c * (amax[b] - A);
  return A;
}

/* Static scale from a calibrated amax: s = fp32(A / 448) (A in fp64). */
float oracle_scale_from_amax_f64(double A) { return (float)(A / 448.0); }

/* RTN weight quantization: s_w = fp32(max|W|) / 448 in fp32, codes q(W, s_w). */
float oracle_rtn_weight(const uint16_t *w, int64_t n, uint8_t *wq) {
  float amax = (float)oracle_absmax_bf16(w, n); /* exact: a bf16 magnitude */
  volatile float s = amax / 448.0f;
  float sw = s;
  oracle_quantize_bf16(w, n, sw, wq);
  return sw;
}

/* ------------------------------------------------------------------------ */
/* W8A8 Linear ([PR] What changed: each Linear applies its own scale in the  */
/* GEMM epilogue; [MC] experiment-setup table: dequantized FP8 weights times */
/* a quantize-dequantized input).                                            */
/*   y[m,n] = bf16( (s_in * s_w) * sum_k deq(xq[m,k]) * deq(wq[n,k]) )       */
/* Products of two E4M3 values are multiples of 2^-18 below 2^18; a sum of   */
/* up to 2^13 of them stays below 2^31 and is therefore exact in fp64.       */
/* ------------------------------------------------------------------------ */
void oracle_linear(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N,
                   int64_t K, float s_in, float s_w, uint16_t *y) {
  const double *cb = codebook();
  double scale = (double)s_in * (double)s_w; /* exact: 24 x 24 bits */
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t m = 0; m < M; ++m) {
    const uint8_t *xr = xq + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t *wr = wq + n * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += cb[xr[k]] * cb[wr[k]];
      y[m * N + n] = oracle_round_bf16(scale * acc);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Two-input SwiGLU with FP8 output ([PR] What changed: SiLU(G) * U from two */
/* separate tensors, quantized directly for the FP8 down_proj).             */
/*   h = q64(SiLU(g) * u, s_down), SiLU(g) = g / (1 + exp(-g)), fp64.        */
/* ------------------------------------------------------------------------ */
static uint8_t silu_mul_code(uint16_t gb, uint16_t ub, double s) {
  double g = bf16_to_double(gb);
  double u = bf16_to_double(ub);
  double silu = g / (1.0 + exp(-g));
  return oracle_quant_f64(silu * u, s);
}

void oracle_silu_mul_2in(const uint16_t *g, const uint16_t *u, int64_t n,
                         float s_down, uint8_t *h) {
  double s = (double)s_down;
  for (int64_t i = 0; i < n; ++i) h[i] = silu_mul_code(g[i], u[i], s);
}

/* The shipped fused form: one [rows, 2I] tensor, gate in the first I columns
 * and up in the last I columns ([PR] What changed: silu_and_mul needs gate and
 * up adjacent in one tensor). */
void oracle_silu_and_mul_fused(const uint16_t *gu, int64_t rows, int64_t I,
                               float s_down, uint8_t *h) {
  double s = (double)s_down;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t i = 0; i < I; ++i)
      h[r * I + i] = silu_mul_code(gu[r * 2 * I + i], gu[r * 2 * I + I + i], s);
}

/* ------------------------------------------------------------------------ */
/* SwiGLU variants ([PR] commit notes on the two-input SwiGLU: alpha is a gain */
/* inside the sigmoid, beta an offset on up; swiglu_limit is named there and  */
/* read here as the clamp of the "swigluoai" shape: gate <= limit,            */
/* -limit <= up <= limit).                                                   */
/*   h = q64( g' * sigmoid(alpha g') * (u' + beta), s_down )                 */
/* with g' = min(g, limit), u' = clamp(u, -limit, limit) when has_limit,     */
/* and the offset added only when beta != 0 (so that alpha = 1, beta = 0 and */
/* no limit is the plain two-input SwiGLU, bit for bit).                     */
/* ------------------------------------------------------------------------ */
static uint8_t swiglu_code(uint16_t gb, uint16_t ub, double s, double alpha, double beta,
                           int has_limit, double limit) {
  double g = bf16_to_double(gb);
  double u = bf16_to_double(ub);
  if (has_limit) {
    if (g > limit) g = limit;
    if (u > limit) u = limit;
    if (u < -limit) u = -limit;
  }
  double act = g / (1.0 + exp(-(alpha * g)));
  double up = (beta != 0.0) ? u + beta : u;
  return oracle_quant_f64(act * up, s);
}

void oracle_swiglu_2in(const uint16_t *g, const uint16_t *u, int64_t n, float s_down,
                       float alpha, float beta, int has_limit, float limit, uint8_t *h) {
  for (int64_t i = 0; i < n; ++i)
    h[i] = swiglu_code(g[i], u[i], (double)s_down, (double)alpha, (double)beta, has_limit,
                       (double)limit);
}

void oracle_swiglu_fused(const uint16_t *gu, int64_t rows, int64_t I, float s_down, float alpha,
                         float beta, int has_limit, float limit, uint8_t *h) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t i = 0; i < I; ++i)
      h[r * I + i] = swiglu_code(gu[r * 2 * I + i], gu[r * 2 * I + I + i], (double)s_down,
                                 (double)alpha, (double)beta, has_limit, (double)limit);
}

/* Unquantized SiLU(g) * u in fp64 (the value the down_proj input observer
 * sees), for calibration of s_down. */
void oracle_silu_mul_f64(const double *g, const double *u, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
}

/* ------------------------------------------------------------------------ */
/* Per-channel weight / per-token activation scales ([MC] comparison report, */
/* table 3.2: the exploratory per-row builds).  One scale per row of a       */
/* [rows, K] tensor: s[r] = fp32(max_k |x[r,k]|) / 448 in fp32 (1 for an     */
/* all-zero row, where every code is 0 whatever the scale), codes            */
/* q(x[r,k], s[r]).  For weights the rows are output channels; for           */
/* activations they are tokens, computed at run time.                       */
/* ------------------------------------------------------------------------ */
void oracle_quantize_rows(const uint16_t *x, int64_t rows, int64_t K, float *s, uint8_t *q) {
  for (int64_t r = 0; r < rows; ++r) {
    float amax = (float)oracle_absmax_bf16(x + r * K, K);
    volatile float sr = amax / 448.0f;
    float sv = (amax > 0.0f) ? (float)sr : 1.0f;
    s[r] = sv;
    oracle_quantize_bf16(x + r * K, K, sv, q + r * K);
  }
}

/* Linear with vector scales: y[m,n] = bf16( sx[m] * sw[n] * sum_k ... ),    */
/* sx of length M (per token) or 1, sw of length N (per channel) or 1.       */
void oracle_linear_scaled(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N, int64_t K,
                          const float *sx, int x_per_row, const float *sw, int w_per_col,
                          uint16_t *y) {
  const double *cb = codebook();
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t m = 0; m < M; ++m) {
    const uint8_t *xr = xq + m * K;
    double a = (double)sx[x_per_row ? m : 0];
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t *wr = wq + n * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += cb[xr[k]] * cb[wr[k]];
      double scale = a * (double)sw[w_per_col ? n : 0]; /* exact: 24 x 24 bits */
      y[m * N + n] = oracle_round_bf16(scale * acc);
    }
  }
}

/* Two-input SwiGLU with per-token FP8 output: v = SiLU(g) * u in fp64 per   */
/* row, s[r] = fp32(max |v| / 448) (1 for an all-zero row), codes q64(v, s).  */
void oracle_silu_mul_2in_rows(const uint16_t *g, const uint16_t *u, int64_t rows, int64_t I,
                              float *s, uint8_t *h) {
  for (int64_t r = 0; r < rows; ++r) {
    double amax = 0.0;
    for (int64_t i = 0; i < I; ++i) {
      double gv = bf16_to_double(g[r * I + i]), uv = bf16_to_double(u[r * I + i]);
      double v = fabs(gv / (1.0 + exp(-gv)) * uv);
      if (v > amax) amax = v;
    }
    float sv = (amax > 0.0) ? (float)(amax / 448.0) : 1.0f;
    s[r] = sv;
    for (int64_t i = 0; i < I; ++i) h[r * I + i] = silu_mul_code(g[r * I + i], u[r * I + i], (double)sv);
  }
}

/* ------------------------------------------------------------------------ */
/* The re-quantization the fused loader did ([PR] Description):              */
/*   qW' = FP8-round((s_i * deq(qW_i)) / max(s))                             */
/* ------------------------------------------------------------------------ */
void oracle_requant_group_member(const uint8_t *qw, int64_t n, float s_i,
                                 float s_max, uint8_t *out) {
  const double *cb = codebook();
  for (int64_t i = 0; i < n; ++i)
    out[i] = oracle_quant_f64((double)s_i * cb[qw[i]], (double)s_max);
}

/* Dequantize codes to fp64 values (test helper). */
void oracle_dequant(const uint8_t *q, int64_t n, double *out) {
  const double *cb = codebook();
  for (int64_t i = 0; i < n; ++i) out[i] = cb[q[i]];
}

/* Number of OpenMP threads the parallel loops use (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
void oracle_set_num_threads(int n) { omp_set_num_threads(n); }
#else
int oracle_num_threads(void) { return 1; }
void oracle_set_num_threads(int n) { (void)n; }
#endif
