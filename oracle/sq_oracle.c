/*
 * sq_oracle.c -- plain, slow CPU oracle for the SmoothQuant W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline / reference leg may load this code.  The product path (the CUDA
 * library under w8a8_smoothquant_gemm_b200/) shares no code with it.
 *
 * Every function below is the plain definition of one step of the method, written
 * as loops over host arrays.  Floating-point work is IEEE-754 binary32 with
 * round-to-nearest-even, one rounding per written operation (build with
 * -ffp-contract=off, no fast-math); fmaf() appears only where the definition says
 * "fused".  Sources (page title, section / equation):
 *
 *   [SQ-eq]   "4.2 W8A8 量化与 SmoothQuant", sec. 3 (Y = (X diag(s)^-1)(diag(s) W)) and
 *             sec. 4 (s_j = max|X_j|^a / max|W_j|^(1-a)); "量化：只压权重，与训练后量化（PTQ）",
 *             SmoothQuant section (W_j is row j of W; statistics on calibration data).
 *   [SQ-LN]   "4.2 W8A8 量化与 SmoothQuant", sec. 6 (fold s^-1 into LayerNorm gamma, beta).
 *   [SQ-pipe] "4.2 W8A8 量化与 SmoothQuant", sec. 7.1 (weights per-channel static,
 *             activations per-token dynamic).
 *   [Q8]      "SmoothQuant大模型平滑量化技术", Python demo quantize_int8
 *             (scale = max|.| / 127, round half to even, clip to [-127, 127]).
 *   [INT8GEMM] "4.2 W8A8 量化与 SmoothQuant", intro (GEMM entirely on INT8 tensor cores);
 *             "量化：只压权重…", SmoothQuant section (per-token / per-channel scales
 *             factor out of the sum; per-input-channel activation scales do not).
 *   [FP8]     "量化：只压权重，与训练后量化（PTQ）", the W8A8-FP8 rows of the decode
 *             roofline (FP8 tensor-core peak twice BF16) and "4.2 W8A8 量化与
 *             SmoothQuant", closing questions (FP8 as the 8-bit format that may need no
 *             explicit smoothing).  The pages do not define the FP8 encoding; the reading
 *             taken is E4M3 of the OCP 8-bit floating point specification (OFP8): bias 7,
 *             3 mantissa bits, no infinities, S.1111.111 = NaN, largest finite 448, with the
 *             same symmetric scheme as INT8 -- scale = max|.| / 448 and code = E4M3 of
 *             RN(v / scale), round to nearest even, saturating at +-448.
 *
 * Readings where the pages are silent (each is a convention shared with the GPU
 * path so that results can be compared bit for bit; no page value checks them,
 * so they are "parity unpinned" as conventions):
 *   - s_j = 1 when max|X_j| = 0 or max|W_j| = 0 (the pages mention a stability
 *     term without giving it).
 *   - s_j is evaluated in binary64 and rounded once to binary32: sqrt(ax/aw) at
 *     a = 1/2, ax at a = 1, 1/aw at a = 0, exp(a log ax - (1-a) log aw) otherwise.
 *   - LayerNorm: sigma = sqrt(var + eps), biased variance, two passes, and the
 *     fixed reduction order documented at ln_reduce() below.
 *   - A zero absmax gives scale 0 and all-zero codes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes, same numbering as the library's public header */
enum { SQO_F32 = 0, SQO_BF16 = 1, SQO_I32 = 2 };

int sqo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads for the following parallel loops (timing only: every result is row- or
 * column-parallel and identical for any thread count). */
void sqo_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* bfloat16 is the top half of a binary32; widening is exact. */
static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* binary32 -> bfloat16, round to nearest, ties to even (NaN kept quiet). */
static uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

uint16_t sqo_f32_to_bf16(float f) { return f32_to_bf16(f); }

static float load_elt(const void* base, int dt, int64_t idx) {
  if (dt == SQO_BF16) return bf16_to_f32(((const uint16_t*)base)[idx]);
  return ((const float*)base)[idx];
}

/* ---------------------------------------------------------------------------
 * Calibration absmax  [SQ-eq], [SQ-pipe]
 *   axis 0: out[j] = max_i |x[i, j]|   (per input channel, over tokens)
 *   axis 1: out[i] = max_j |x[i, j]|   (per row: row j of W[K, N] is input channel j)
 * accumulate != 0 folds the previous contents of out[] into the max.
 * ------------------------------------------------------------------------- */
void sqo_calib_absmax(const void* x, int dt, int64_t rows, int64_t cols, int64_t ld,
                      int axis, int accumulate, float* out) {
  if (axis == 0) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < cols; ++j) {
      float m = accumulate ? out[j] : 0.0f;
      for (int64_t i = 0; i < rows; ++i) {
        float a = fabsf(load_elt(x, dt, i * ld + j));
        if (a > m) m = a;
      }
      out[j] = m;
    }
  } else {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
      float m = accumulate ? out[i] : 0.0f;
      for (int64_t j = 0; j < cols; ++j) {
        float a = fabsf(load_elt(x, dt, i * ld + j));
        if (a > m) m = a;
      }
      out[i] = m;
    }
  }
}

/* ---------------------------------------------------------------------------
 * Smoothing factors  [SQ-eq]:  s_j = ax_j^a / aw_j^(1-a)
 * ------------------------------------------------------------------------- */
void sqo_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s) {
  const double a = (double)alpha;
  for (int64_t j = 0; j < K; ++j) {
    const double x = (double)ax[j];
    const double w = (double)aw[j];
    if (!(x > 0.0) || !(w > 0.0)) {
      s[j] = 1.0f;
    } else if (alpha == 0.5f) {
      s[j] = (float)sqrt(x / w);
    } else if (alpha == 1.0f) {
      s[j] = (float)x;
    } else if (alpha == 0.0f) {
      s[j] = (float)(1.0 / w);
    } else {
      const double t1 = a * log(x);
      const double t2 = (1.0 - a) * log(w);
      s[j] = (float)exp(t1 - t2);
    }
  }
}

/* ---------------------------------------------------------------------------
 * Symmetric INT8 code  [Q8]:  clamp(rne(v / scale), -127, 127); scale 0 -> 0
 * ------------------------------------------------------------------------- */
static int8_t quant_code(float v, float scale) {
  if (scale == 0.0f) return 0;
  float q = rintf(v / scale); /* default rounding mode: nearest, ties to even */
  if (q > 127.0f) q = 127.0f;
  if (q < -127.0f) q = -127.0f;
  return (int8_t)q;
}

/* ---------------------------------------------------------------------------
 * Fold + per-output-channel weight quantisation  [SQ-eq], [SQ-LN], [SQ-pipe]
 *   W'[j, k] = s_j * W[j, k]                    (W is [K, N], row j = input channel)
 *   sw[k]    = max_j |W'[j, k]| / 127
 *   Wq[k, j] = clamp(rne(W'[j, k] / sw[k]))     (stored [N, K], K contiguous)
 *   gamma'_j = gamma_j / s_j, beta'_j = beta_j / s_j   (when given)
 * ------------------------------------------------------------------------- */
void sqo_fold_quant_weights(const void* W, int dt, int64_t K, int64_t N, int64_t ldw,
                            const float* s, const float* gamma, const float* beta,
                            int8_t* Wq, float* sw, float* gamma_f, float* beta_f) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < N; ++k) {
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float wp = s[j] * load_elt(W, dt, j * ldw + k);
      float a = fabsf(wp);
      if (a > m) m = a;
    }
    const float scale = m / 127.0f;
    sw[k] = scale;
    for (int64_t j = 0; j < K; ++j) {
      float wp = s[j] * load_elt(W, dt, j * ldw + k);
      Wq[k * K + j] = quant_code(wp, scale);
    }
  }
  if (gamma && gamma_f)
    for (int64_t j = 0; j < K; ++j) gamma_f[j] = gamma[j] / s[j];
  if (beta && beta_f)
    for (int64_t j = 0; j < K; ++j) beta_f[j] = beta[j] / s[j];
}

/* ---------------------------------------------------------------------------
 * Fixed reduction order for the LayerNorm statistics (a convention; the pages
 * give LN only as (x - mu)/sigma).  The row of K values is cut into 8-element
 * chunks; chunk c belongs to lane c mod 256.  Each lane adds its chunks' values in
 * increasing index order into a binary32 partial that starts at +0 (term(v, acc)
 * is acc + v for the mean and fmaf(v, v, acc) for the variance).  The 256 partials
 * then combine pairwise: inside each group of 32 lanes p[i] = p[i] + p[i + o] for
 * o = 16, 8, 4, 2, 1; then the 8 group results g[i] = g[i] + g[i + o] for
 * o = 4, 2, 1.  The total is g[0].
 * ------------------------------------------------------------------------- */
#define LN_LANES 256
#define LN_CHUNK 8

static float ln_reduce(const float* v, int64_t K, int square) {
  float p[LN_LANES];
  for (int l = 0; l < LN_LANES; ++l) p[l] = 0.0f;
  const int64_t nchunks = K / LN_CHUNK;
  for (int64_t c = 0; c < nchunks; ++c) {
    const int lane = (int)(c % LN_LANES);
    for (int e = 0; e < LN_CHUNK; ++e) {
      const float t = v[c * LN_CHUNK + e];
      p[lane] = square ? fmaf(t, t, p[lane]) : (p[lane] + t);
    }
  }
  for (int g = 0; g < LN_LANES / 32; ++g)
    for (int o = 16; o >= 1; o >>= 1)
      for (int i = 0; i < o; ++i) p[g * 32 + i] = p[g * 32 + i] + p[g * 32 + i + o];
  float gs[LN_LANES / 32];
  for (int g = 0; g < LN_LANES / 32; ++g) gs[g] = p[g * 32];
  for (int o = 4; o >= 1; o >>= 1)
    for (int i = 0; i < o; ++i) gs[i] = gs[i] + gs[i + o];
  return gs[0];
}

/* LayerNorm of one row: y_j = fma((x_j - mu) * rstd, g_j, b_j), rstd = 1/sqrt(var+eps).
 * Needs K % 8 == 0 (the chunking above).  tmp has room for K floats. */
static void layernorm_row(const float* x, int64_t K, const float* g, const float* b,
                          float eps, float* y, float* tmp) {
  const float mu = ln_reduce(x, K, 0) / (float)K;
  for (int64_t j = 0; j < K; ++j) tmp[j] = x[j] - mu;
  const float var = ln_reduce(tmp, K, 1) / (float)K;
  const float rstd = 1.0f / sqrtf(var + eps);
  for (int64_t j = 0; j < K; ++j) {
    const float u = tmp[j] * rstd;
    y[j] = fmaf(u, g[j], b ? b[j] : 0.0f);
  }
}

/* LayerNorm rows in fp32 (test helper: exposes the statistic order above). */
void sqo_layernorm(const void* x, int dt, int64_t M, int64_t K, int64_t ld,
                   const float* gamma, const float* beta, float eps, float* y) {
#pragma omp parallel
  {
    float* xr = (float*)malloc(sizeof(float) * (size_t)K);
    float* tmp = (float*)malloc(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
      for (int64_t j = 0; j < K; ++j) xr[j] = load_elt(x, dt, m * ld + j);
      layernorm_row(xr, K, gamma, beta, eps, y + m * K, tmp);
    }
    free(xr); free(tmp);
  }
}

/* ---------------------------------------------------------------------------
 * Calibration absmax of a LayerNorm output (the linear's input when a LayerNorm
 * precedes it)  [SQ-pipe], [SQ-LN]:  out[j] = max_i |LN(x_i)_j| with the original
 * gamma, beta (beta may be NULL).
 * ------------------------------------------------------------------------- */
void sqo_calib_ln_absmax(const void* x, int dt, int64_t rows, int64_t K, int64_t ld,
                         const float* gamma, const float* beta, float eps,
                         int accumulate, float* out) {
  float* acc = (float*)malloc(sizeof(float) * (size_t)K);
  for (int64_t j = 0; j < K; ++j) acc[j] = accumulate ? out[j] : 0.0f;
#pragma omp parallel
  {
    float* xr = (float*)malloc(sizeof(float) * (size_t)K);
    float* yr = (float*)malloc(sizeof(float) * (size_t)K);
    float* tmp = (float*)malloc(sizeof(float) * (size_t)K);
    float* loc = (float*)calloc((size_t)K, sizeof(float));
#pragma omp for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
      for (int64_t j = 0; j < K; ++j) xr[j] = load_elt(x, dt, i * ld + j);
      layernorm_row(xr, K, gamma, beta, eps, yr, tmp);
      for (int64_t j = 0; j < K; ++j) {
        const float a = fabsf(yr[j]);
        if (a > loc[j]) loc[j] = a;
      }
    }
#pragma omp critical
    for (int64_t j = 0; j < K; ++j)
      if (loc[j] > acc[j]) acc[j] = loc[j];
    free(xr); free(yr); free(tmp); free(loc);
  }
  for (int64_t j = 0; j < K; ++j) out[j] = acc[j];
  free(acc);
}

/* ---------------------------------------------------------------------------
 * Fused LayerNorm -> X diag(s)^-1 -> per-token INT8  [SQ-LN], [SQ-pipe], [Q8]
 *   LN mode (gamma_f != NULL): y = LN(x) with the folded gamma' = gamma/s, beta' = beta/s
 *   plain mode (s != NULL):    y_j = x_j / s_j
 *   sx_m = max_j |y_mj| / 127;  xq_mj = clamp(rne(y_mj / sx_m))
 * ------------------------------------------------------------------------- */
void sqo_ln_smooth_quant(const void* x, int dt, int64_t M, int64_t K, int64_t ldx,
                         const float* gamma_f, const float* beta_f, const float* s,
                         float eps, int8_t* xq, float* sx) {
#pragma omp parallel
  {
    float* xr = (float*)malloc(sizeof(float) * (size_t)K);
    float* yr = (float*)malloc(sizeof(float) * (size_t)K);
    float* tmp = (float*)malloc(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
      for (int64_t j = 0; j < K; ++j) xr[j] = load_elt(x, dt, m * ldx + j);
      if (gamma_f) {
        layernorm_row(xr, K, gamma_f, beta_f, eps, yr, tmp);
      } else {
        for (int64_t j = 0; j < K; ++j) yr[j] = xr[j] / s[j];
      }
      float amax = 0.0f;
      for (int64_t j = 0; j < K; ++j) {
        const float a = fabsf(yr[j]);
        if (a > amax) amax = a;
      }
      const float scale = amax / 127.0f;
      sx[m] = scale;
      for (int64_t j = 0; j < K; ++j) xq[m * K + j] = quant_code(yr[j], scale);
    }
    free(xr); free(yr); free(tmp);
  }
}

/* ---------------------------------------------------------------------------
 * Fused LayerNorm / smoothing -> per-TENSOR INT8 (the coarser activation granularity:
 * one scale for the whole activation tensor)  [SQ-pipe] (O1 and the static end of the
 * granularity ladder), [Q8]
 *   y as in sqo_ln_smooth_quant;
 *   static_scale == 0: scale = max_{m,j} |y_mj| / 127 (dynamic), written to *scale;
 *   static_scale != 0: scale = *scale as given (calibrated); values beyond it clamp.
 *   xq_mj = clamp(rne(y_mj / scale), -127, 127);  sx[m] = scale for every row.
 * ------------------------------------------------------------------------- */
void sqo_ln_smooth_quant_per_tensor(const void* x, int dt, int64_t M, int64_t K, int64_t ldx,
                                    const float* gamma_f, const float* beta_f, const float* s,
                                    float eps, int static_scale, float* scale, int8_t* xq,
                                    float* sx) {
  float* y = (float*)malloc(sizeof(float) * (size_t)(M * K > 0 ? M * K : 1));
  float* xr = (float*)malloc(sizeof(float) * (size_t)K);
  float* tmp = (float*)malloc(sizeof(float) * (size_t)K);
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t j = 0; j < K; ++j) xr[j] = load_elt(x, dt, m * ldx + j);
    if (gamma_f) {
      layernorm_row(xr, K, gamma_f, beta_f, eps, y + m * K, tmp);
    } else {
      for (int64_t j = 0; j < K; ++j) y[m * K + j] = xr[j] / s[j];
    }
  }
  float sc;
  if (static_scale) {
    sc = *scale;
  } else {
    float amax = 0.0f;
    for (int64_t i = 0; i < M * K; ++i) {
      const float a = fabsf(y[i]);
      if (a > amax) amax = a;
    }
    sc = amax / 127.0f;
    *scale = sc;
  }
  for (int64_t i = 0; i < M * K; ++i) xq[i] = quant_code(y[i], sc);
  for (int64_t m = 0; m < M; ++m) sx[m] = sc;
  free(y); free(xr); free(tmp);
}

/* ---------------------------------------------------------------------------
 * Per-tensor symmetric INT8 (the coarse activation granularity the pages compare
 * against):  scale = max |y| / 127 over the whole tensor  [Q8], [SQ-pipe]
 * ------------------------------------------------------------------------- */
void sqo_quant_per_tensor(const float* y, int64_t n, int8_t* q, float* scale_out) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    const float a = fabsf(y[i]);
    if (a > amax) amax = a;
  }
  const float scale = amax / 127.0f;
  for (int64_t i = 0; i < n; ++i) q[i] = quant_code(y[i], scale);
  *scale_out = scale;
}

/* ---------------------------------------------------------------------------
 * The next linear's smoothing folded into this linear  [SQ-fold-prev]
 *   "量化：只压权重，与训练后量化（PTQ）", SmoothQuant section: diag(s)^-1 folds offline into
 *   the preceding LayerNorm or linear layer.  For a preceding linear the fold lands on its
 *   per-output-channel scale:  sw'[n] = sw[n] / s_next[n]  (binary32), so its output
 *   ((float)acc * sx) * sw' is the next linear's smoothed input y / s_next.
 * ------------------------------------------------------------------------- */
void sqo_fold_next_smoothing(const float* sw, const float* s_next, int64_t N, float* out) {
  for (int64_t n = 0; n < N; ++n) out[n] = sw[n] / s_next[n];
}

/* ---------------------------------------------------------------------------
 * FP8 E4M3 codes  [FP8]
 *   decode: e = bits 6..3, m = bits 2..0; e = 0: (m / 8) 2^-6; else (1 + m / 8) 2^(e-7);
 *           e = 15 and m = 7: NaN
 *   encode: round to nearest even on the E4M3 grid; magnitudes that round above 448
 *           saturate to 448; NaN -> 0x7F; -0 keeps its sign
 * ------------------------------------------------------------------------- */
float sqo_e4m3_decode(uint8_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  float v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexpf((float)m, -9);
  else v = ldexpf((float)(8 + m), e - 10);
  return (c & 0x80) ? -v : v;
}

uint8_t sqo_e4m3_encode(float v) {
  if (isnan(v)) return 0x7F;
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const float a = fabsf(v);
  if (a >= 448.0f) return sign | 0x7E;
  if (a < 0x1p-6f) {                       /* subnormal grid, spacing 2^-9 */
    const float q = rintf(ldexpf(a, 9));   /* 0 .. 8; 8 is the smallest normal, code 8 */
    return sign | (uint8_t)q;
  }
  int e;
  frexpf(a, &e);                           /* a = f 2^e, f in [0.5, 1) */
  e -= 1;                                  /* a in [2^e, 2^(e+1)), e in -6 .. 8 */
  float q = rintf(ldexpf(a, 3 - e));       /* 8 .. 16 steps of 2^(e-3) */
  if (q == 16.0f) {
    q = 8.0f;
    e += 1;
  }
  if (e > 8 || (e == 8 && q > 14.0f)) return sign | 0x7E; /* above 448: saturate */
  return sign | (uint8_t)(((e + 7) << 3) | ((int)q - 8));
}

/* E4M3 code of v with a shared scale: RN(v / scale) on the E4M3 grid; scale 0 -> +0. */
static uint8_t fp8_code(float v, float scale) {
  if (scale == 0.0f) return 0;
  return sqo_e4m3_encode(v / scale);
}

/* Fold + per-output-channel FP8 weights: as sqo_fold_quant_weights with
 * sw[k] = max_j |W'[j, k]| / 448 and E4M3 codes.  [SQ-eq], [SQ-LN], [SQ-pipe], [FP8] */
void sqo_fold_quant_weights_fp8(const void* W, int dt, int64_t K, int64_t N, int64_t ldw,
                                const float* s, const float* gamma, const float* beta,
                                uint8_t* Wq, float* sw, float* gamma_f, float* beta_f) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < N; ++k) {
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float a = fabsf(s[j] * load_elt(W, dt, j * ldw + k));
      if (a > m) m = a;
    }
    const float scale = m / 448.0f;
    sw[k] = scale;
    for (int64_t j = 0; j < K; ++j) Wq[k * K + j] = fp8_code(s[j] * load_elt(W, dt, j * ldw + k), scale);
  }
  if (gamma && gamma_f)
    for (int64_t j = 0; j < K; ++j) gamma_f[j] = gamma[j] / s[j];
  if (beta && beta_f)
    for (int64_t j = 0; j < K; ++j) beta_f[j] = beta[j] / s[j];
}

/* Fused LayerNorm -> X diag(s)^-1 -> per-token FP8: as sqo_ln_smooth_quant with
 * sx_m = max_j |y_mj| / 448 and E4M3 codes.  [SQ-LN], [SQ-pipe], [FP8] */
void sqo_ln_smooth_quant_fp8(const void* x, int dt, int64_t M, int64_t K, int64_t ldx,
                             const float* gamma_f, const float* beta_f, const float* s,
                             float eps, uint8_t* xq, float* sx) {
#pragma omp parallel
  {
    float* xr = (float*)malloc(sizeof(float) * (size_t)K);
    float* yr = (float*)malloc(sizeof(float) * (size_t)K);
    float* tmp = (float*)malloc(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
      for (int64_t j = 0; j < K; ++j) xr[j] = load_elt(x, dt, m * ldx + j);
      if (gamma_f) {
        layernorm_row(xr, K, gamma_f, beta_f, eps, yr, tmp);
      } else {
        for (int64_t j = 0; j < K; ++j) yr[j] = xr[j] / s[j];
      }
      float amax = 0.0f;
      for (int64_t j = 0; j < K; ++j) {
        const float a = fabsf(yr[j]);
        if (a > amax) amax = a;
      }
      const float scale = amax / 448.0f;
      sx[m] = scale;
      for (int64_t j = 0; j < K; ++j) xq[m * K + j] = fp8_code(yr[j], scale);
    }
    free(xr); free(yr); free(tmp);
  }
}

/* FP8 x FP8 GEMM with the dequant epilogue  [FP8], [INT8GEMM]
 *   acc[m, n] = sum_j dec(xq[m, j]) dec(wq[n, j]), exact: every product of two E4M3 values
 *   has at most 8 significant bits and lies in [2^-18, 448^2], so a binary64 running sum
 *   of up to 2^16 of them never rounds.
 *   acc_out (optional): the exact accumulators;  y: ((float)acc * sx[m]) * sw[n] in
 *   binary32 (F32) or its bfloat16 (BF16), (float)acc being the rounded exact sum. */
void sqo_fp8_gemm(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw,
                  int64_t M, int64_t N, int64_t K, double* acc_out, void* y, int ydt, int64_t ldy) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j)
        acc += (double)sqo_e4m3_decode(xq[m * K + j]) * (double)sqo_e4m3_decode(wq[n * K + j]);
      if (acc_out) acc_out[m * N + n] = acc;
      if (y) {
        const float v = ((float)acc * sx[m]) * sw[n];
        if (ydt == SQO_BF16)
          ((uint16_t*)y)[m * ldy + n] = f32_to_bf16(v);
        else
          ((float*)y)[m * ldy + n] = v;
      }
    }
  }
}

/* ---------------------------------------------------------------------------
 * INT8 x INT8 -> int32 GEMM with the dequant epilogue  [INT8GEMM], [SQ-pipe]
 *   acc[m, n] = sum_j xq[m, j] * wq[n, j]      (exact; int64 running sum, checked)
 *   ydt = I32:  y[m, n] = acc
 *   ydt = BF16: y[m, n] = bf16_rne(((float)acc * sx[m]) * sw[n])
 *   ydt = F32:  y[m, n] = ((float)acc * sx[m]) * sw[n]
 * Returns the number of accumulators outside the int32 range (0 expected).
 * ------------------------------------------------------------------------- */
int64_t sqo_w8a8_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                      int64_t M, int64_t N, int64_t K, void* y, int ydt, int64_t ldy) {
  int64_t overflow = 0;
#pragma omp parallel for schedule(static) reduction(+ : overflow)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      int64_t acc = 0;
      for (int64_t j = 0; j < K; ++j) acc += (int64_t)xq[m * K + j] * (int64_t)wq[n * K + j];
      if (acc > INT32_MAX || acc < INT32_MIN) ++overflow;
      const int32_t a32 = (int32_t)acc;
      if (ydt == SQO_I32) {
        ((int32_t*)y)[m * ldy + n] = a32;
      } else {
        const float v = ((float)a32 * sx[m]) * sw[n];
        if (ydt == SQO_BF16)
          ((uint16_t*)y)[m * ldy + n] = f32_to_bf16(v);
        else
          ((float*)y)[m * ldy + n] = v;
      }
    }
  }
  return overflow;
}
