/*
 * wq_oracle.c -- plain, slow, single-threaded CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY: called by the tests, the smoke check and the
 * benchmark's CPU-baseline leg; never by the product path.  Shares no code
 * with the CUDA library.
 *
 * Every step follows the order in which the quantization write-ups state it;
 * each function names the page section it restates.  Floating-point decisions
 * that pick an integer code are taken in binary32, the same precision as the
 * kernels; matrix products are summed in binary64.  The page tags [P1]..[P4]
 * are listed with their titles in wq_oracle.h.
 */
#include "wq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Rounding and format conversion (IEEE-754 definitions)                      */
/* ------------------------------------------------------------------------- */

/* Round a double that holds a non-negative value to the nearest integer,
 * ties to the even integer.  Exact: floor() and the subtraction are exact for
 * the magnitudes used here (< 2^52). */
static double round_half_even_nonneg(double q) {
  double n = floor(q);
  double d = q - n;
  if (d > 0.5) return n + 1.0;
  if (d < 0.5) return n;
  return (fmod(n, 2.0) == 0.0) ? n : n + 1.0;
}

float oracle_round_half_even(float v) {
  /* numpy.round / torch.round round half to even ([P3] sec. 2.1 code,
   * [P4] sec. 2.1 code); reproduce that on a binary32 value. */
  if (!isfinite(v)) return v;
  double a = fabs((double)v);
  if (a >= 8388608.0) return v; /* already an integer (>= 2^23) */
  double r = round_half_even_nonneg(a);
  return (float)(v < 0 ? -r : r);
}

static uint32_t f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

static float f32_from_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* binary32 -> binary16, round to nearest even. */
uint16_t oracle_f32_to_f16(float f) {
  uint16_t sign = (uint16_t)((f32_bits(f) >> 31) << 15);
  if (isnan(f)) return (uint16_t)(sign | 0x7E00u);
  double a = fabs((double)f);
  /* largest finite binary16 is 65504; the midpoint to the next power of two
   * (65520) has an odd neighbour (0x7BFF), so ties round up to infinity. */
  if (a >= 65520.0) return (uint16_t)(sign | 0x7C00u);
  if (a < ldexp(1.0, -14)) {
    /* subnormal range: value = n * 2^-24, n in [0, 1024] (1024 is the
     * smallest normal, whose encoding 0x0400 is exactly n). */
    double n = round_half_even_nonneg(a * ldexp(1.0, 24));
    return (uint16_t)(sign | (uint16_t)n);
  }
  int e;
  double m = frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
  m *= 2.0;
  e -= 1; /* a = m * 2^e, m in [1, 2) */
  double r = round_half_even_nonneg((m - 1.0) * 1024.0);
  if (r == 1024.0) {
    r = 0.0;
    e += 1;
  }
  if (e > 15) return (uint16_t)(sign | 0x7C00u);
  return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)r);
}

float oracle_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int mant = h & 0x3FF;
  double v;
  if (e == 0x1F) {
    if (mant) return NAN;
    v = INFINITY;
  } else if (e == 0) {
    v = ldexp((double)mant, -24);
  } else {
    v = ldexp(1.0 + mant / 1024.0, e - 15);
  }
  return (float)(sign ? -v : v);
}

/* binary32 -> bfloat16 (1 sign, 8 exponent, 7 fraction bits), nearest even. */
uint16_t oracle_f32_to_bf16(float f) {
  uint16_t sign = (uint16_t)((f32_bits(f) >> 31) << 15);
  if (isnan(f)) return (uint16_t)(sign | 0x7FC0u);
  double a = fabs((double)f);
  if (isinf(f)) return (uint16_t)(sign | 0x7F80u);
  /* largest finite bfloat16 is (2 - 2^-7) * 2^127; the midpoint to 2^128 has
   * an odd neighbour, so it rounds up to infinity */
  if (a >= (2.0 - ldexp(1.0, -8)) * ldexp(1.0, 127))
    return (uint16_t)(sign | 0x7F80u);
  if (a < ldexp(1.0, -126)) {
    double n = round_half_even_nonneg(a * ldexp(1.0, 133));
    return (uint16_t)(sign | (uint16_t)n);
  }
  int e;
  double m = frexp(a, &e);
  m *= 2.0;
  e -= 1;
  double r = round_half_even_nonneg((m - 1.0) * 128.0);
  if (r == 128.0) {
    r = 0.0;
    e += 1;
  }
  if (e > 127) return (uint16_t)(sign | 0x7F80u);
  return (uint16_t)(sign | (uint16_t)((e + 127) << 7) | (uint16_t)r);
}

float oracle_bf16_to_f32(uint16_t b) {
  /* bfloat16 is the top half of a binary32 pattern: widening is exact. */
  return f32_from_bits(((uint32_t)b) << 16);
}

void oracle_f32_to_f16_array(const float *in, uint16_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_f16(in[i]);
}
void oracle_f16_to_f32_array(const uint16_t *in, float *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f32(in[i]);
}
void oracle_f32_to_bf16_array(const float *in, uint16_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(in[i]);
}
void oracle_bf16_to_f32_array(const uint16_t *in, float *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_f32(in[i]);
}

static float load_elem(const void *p, int dtype, int64_t i) {
  switch (dtype) {
    case ORACLE_F32:
      return ((const float *)p)[i];
    case ORACLE_BF16:
      return oracle_bf16_to_f32(((const uint16_t *)p)[i]);
    default:
      return oracle_f16_to_f32(((const uint16_t *)p)[i]);
  }
}

static int clamp_int(int v, int lo, int hi) {
  return v < lo ? lo : (v > hi ? hi : v);
}

/* ------------------------------------------------------------------------- */
/* INT4 group-wise quantize and pack                                          */
/* ------------------------------------------------------------------------- */

/*
 * For each output row n and each group of `group_size` consecutive input
 * columns ([P4] sec. 2.2: W is [out_features, in_features], one scale per 128
 * input dims; [P3] sec. 2.2 per-group):
 *
 * symmetric ([P3] sec. 2.1 symmetric_quantize, [P4] sec. 2.1):
 *   amax = max |x|;  s = amax / (2^(b-1) - 1) = amax / 7;
 *   q = clip(round(x / s), -8, 7);  zero point 0.
 *   Degenerate range (amax < 1e-8): q = 0 and the returned scale is amax.
 * asymmetric ([P3] sec. 2.1 asymmetric_quantize, [P4] sec. 2.1):
 *   s = (max - min) / (2^b - 1) = (max - min) / 15;
 *   z = clip(round(-min / s), 0, 15);  q = clip(round(x / s) + z, 0, 15).
 *   Degenerate range (max - min < 1e-8): q = 0, s = 1.0, z = 0.
 *
 * Readings where the pages leave a step open:
 *   - the scale is stored as fp16 ([P4] sec. 2.2 and 8 keep one fp16 scale
 *     for every 128 INT4 weights) and the rounded, stored scale is the one the codes
 *     are computed with, so dequantization reproduces exactly what the codes
 *     mean; a scale that rounds to fp16 zero is treated as a degenerate range;
 *   - round-then-add (round(x/s) + z), as in [P1] sec. 2.2, [P2] sec. 2 and
 *     [P4] sec. 2.1; rounding is half to even as numpy/torch round;
 *   - the fp32 division is a single IEEE division (x / s, not x * (1/s));
 *   - storage: unsigned nibble u = q - qmin (sym: q + 8, asym: q), two per
 *     byte, element k of row n in byte n*K/2 + k/2, low nibble = even k;
 *     zero points are stored as fp16 integers 0..15 (asym only).
 */
/* Scale (fp16 bits), zero point and degeneracy of one group of n values
 * ([P3] sec. 2.1 / [P4] sec. 2.1, readings in the header): sym s = amax/7,
 * asym s = (max - min)/15 and z = clamp(round(-min/s), 0, 15); the fp32
 * scale is rounded to fp16 and the fp16 value is the one used. */
static void group_params(const float *x, int64_t n, int sym, uint16_t *s16_out,
                         int *z_out, int *degenerate_out, int *nonfinite) {
  float mn = INFINITY, mx = -INFINITY, amax = 0.0f;
  for (int64_t k = 0; k < n; ++k) {
    if (!isfinite(x[k])) *nonfinite = 1;
    if (x[k] < mn) mn = x[k];
    if (x[k] > mx) mx = x[k];
    if (fabsf(x[k]) > amax) amax = fabsf(x[k]);
  }
  uint16_t s16;
  int z = 0;
  int degenerate;
  if (sym) {
    float s32 = amax / 7.0f;
    s16 = oracle_f32_to_f16(s32);
    degenerate = (amax < 1e-8f) || (oracle_f16_to_f32(s16) == 0.0f);
    if (degenerate) s16 = oracle_f32_to_f16(amax);
  } else {
    float range = mx - mn;
    float s32 = range / 15.0f;
    s16 = oracle_f32_to_f16(s32);
    degenerate = (range < 1e-8f) || (oracle_f16_to_f32(s16) == 0.0f);
    if (degenerate) {
      s16 = oracle_f32_to_f16(1.0f);
      z = 0;
    } else {
      float sf = oracle_f16_to_f32(s16);
      float zr = oracle_round_half_even(-mn / sf);
      z = (int)fmaxf(0.0f, fminf(15.0f, zr));
    }
  }
  *s16_out = s16;
  *z_out = z;
  *degenerate_out = degenerate;
}

static void put_nibble(uint8_t *codes, int64_t idx, uint8_t u) {
  uint8_t *byte = &codes[idx / 2];
  if ((idx & 1) == 0)
    *byte = (uint8_t)((*byte & 0xF0u) | u);
  else
    *byte = (uint8_t)((*byte & 0x0Fu) | (uint8_t)(u << 4));
}

int oracle_quantize_int4(const void *W, int w_dtype, int64_t N, int64_t K,
                         int group_size, int sym, uint8_t *codes,
                         uint16_t *scales, uint16_t *zeros) {
  if (N < 0 || K < 0 || group_size <= 0 || (K % group_size) != 0 ||
      (K % 2) != 0)
    return ORACLE_ERR_ARG;
  if (!sym && zeros == NULL) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
  const int64_t G = K / group_size;
  const int qmin = sym ? -8 : 0;
  const int qmax = sym ? 7 : 15;
  float *grp = (float *)malloc((size_t)group_size * sizeof(float));
  if (!grp) return ORACLE_ERR_ARG;
  memset(codes, 0, (size_t)(N * (K / 2)));
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      const int64_t k0 = g * group_size;
      for (int64_t k = 0; k < group_size; ++k) grp[k] = load_elem(W, w_dtype, n * K + k0 + k);
      uint16_t s16;
      int z, degenerate, nonfinite = 0;
      group_params(grp, group_size, sym, &s16, &z, &degenerate, &nonfinite);
      if (nonfinite) status = ORACLE_ERR_NONFINITE;
      if (!sym) zeros[n * G + g] = oracle_f32_to_f16((float)z);
      if (isinf(oracle_f16_to_f32(s16))) status = ORACLE_ERR_NONFINITE;
      scales[n * G + g] = s16;
      const float sf = oracle_f16_to_f32(s16);
      for (int64_t k = 0; k < group_size; ++k) {
        int q;
        if (degenerate) {
          q = 0;
        } else {
          float r = oracle_round_half_even(grp[k] / sf);
          /* clamp in float first so huge quotients do not overflow int */
          r = fmaxf(-64.0f, fminf(64.0f, r));
          q = clamp_int((int)r + z, qmin, qmax);
        }
        put_nibble(codes + n * (K / 2), k0 + k, (uint8_t)(q - qmin));
      }
    }
  }
  free(grp);
  return status;
}

/* ------------------------------------------------------------------------- */
/* INT8 symmetric rows (per-output-channel weights)                           */
/* ------------------------------------------------------------------------- */

/*
 * [P4] sec. 2.2: INT8 weights need only a per-channel scale -- one scale per output
 * row; [P4] sec. 2.1 / [P3] sec. 2.1 symmetric min-max: s = amax / 127,
 * q = clip(round(x / s)).  The clip range is [-127, 127]: [P3] sec. 2.1 maps
 * the symmetric interval onto integers symmetric about zero.  The scale
 * stays fp32 (it feeds the fp32 rescale of the int32 accumulator).
 * Degenerate row (amax < 1e-8): q = 0, scale = amax ([P3] sec. 2.1).
 */
int oracle_quantize_int8_rows(const void *W, int w_dtype, int64_t N, int64_t K,
                              int8_t *q, float *scales) {
  if (N < 0 || K <= 0) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
  for (int64_t n = 0; n < N; ++n) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float x = load_elem(W, w_dtype, n * K + k);
      if (!isfinite(x)) status = ORACLE_ERR_NONFINITE;
      if (fabsf(x) > amax) amax = fabsf(x);
    }
    int degenerate = amax < 1e-8f;
    float s = degenerate ? amax : amax / 127.0f;
    scales[n] = s;
    for (int64_t k = 0; k < K; ++k) {
      int v = 0;
      if (!degenerate) {
        float r = oracle_round_half_even(load_elem(W, w_dtype, n * K + k) / s);
        r = fmaxf(-200.0f, fminf(200.0f, r));
        v = clamp_int((int)r, -127, 127);
      }
      q[n * K + k] = (int8_t)v;
    }
  }
  return status;
}

/* ------------------------------------------------------------------------- */
/* Per-token dynamic INT8 activations                                         */
/* ------------------------------------------------------------------------- */

/*
 * [P4] sec. 6 (quant_kv_per_token, the per-token absmax quantizer; W8A8 uses
 * it for activation rows, [P4] sec. 2.3):
 *   scale = amax(|v|) / 127;  scale = max(scale, 1e-8);
 *   q = clamp(round(v / scale), -128, 127).
 */
int oracle_quant_act_i8(const void *X, int x_dtype, int64_t M, int64_t K,
                        int8_t *q, float *scales) {
  if (M < 0 || K <= 0) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
  for (int64_t m = 0; m < M; ++m) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float x = load_elem(X, x_dtype, m * K + k);
      if (!isfinite(x)) status = ORACLE_ERR_NONFINITE;
      if (fabsf(x) > amax) amax = fabsf(x);
    }
    float s = amax / 127.0f;
    if (s < 1e-8f) s = 1e-8f;
    scales[m] = s;
    for (int64_t k = 0; k < K; ++k) {
      float r = oracle_round_half_even(load_elem(X, x_dtype, m * K + k) / s);
      r = fmaxf(-200.0f, fminf(200.0f, r));
      q[m * K + k] = (int8_t)clamp_int((int)r, -128, 127);
    }
  }
  return status;
}

/* ------------------------------------------------------------------------- */
/* Dequantization                                                             */
/* ------------------------------------------------------------------------- */

/* [P2] sec. 2: f' = S * (q - Z); [P4] sec. 2.1: x_hat = s * (q - z).
 * With the stored unsigned nibble u = q - qmin this is s * (u - z_eff) with
 * z_eff = 8 (symmetric, q = u - 8, Z = 0) or z_eff = z (asymmetric, q = u).
 * The fp16 scale has 11 significant bits and |u - z_eff| <= 15, so the
 * binary32 product is exact. */
int oracle_dequant_int4(const uint8_t *codes, const uint16_t *scales,
                        const uint16_t *zeros, int64_t N, int64_t K,
                        int group_size, int sym, float *out) {
  if (group_size <= 0 || (K % group_size) != 0 || (K % 2) != 0)
    return ORACLE_ERR_ARG;
  if (!sym && zeros == NULL) return ORACLE_ERR_ARG;
  const int64_t G = K / group_size;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = codes[n * (K / 2) + k / 2];
      int u = (k & 1) ? (byte >> 4) : (byte & 0x0F);
      int64_t g = k / group_size;
      float s = oracle_f16_to_f32(scales[n * G + g]);
      int zeff = sym ? 8 : (int)oracle_f16_to_f32(zeros[n * G + g]);
      out[n * K + k] = s * (float)(u - zeff);
    }
  }
  return ORACLE_OK;
}

int oracle_dequant_int8_rows(const int8_t *q, const float *scales, int64_t N,
                             int64_t K, float *out) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      out[n * K + k] = scales[n] * (float)q[n * K + k];
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Matrix products                                                            */
/* ------------------------------------------------------------------------- */

/* W4A16 ([P4] sec. 2.3: INT4 weights, 16-bit activations, the weight is
 * dequantized before the product): Y = X * dequant(W)^T, summed in fp64
 * over k = 0 .. K-1 in order. */
int oracle_gemm_w4a16(const uint16_t *X, int64_t M, int64_t K,
                      const uint8_t *codes, const uint16_t *scales,
                      const uint16_t *zeros, int64_t N, int group_size,
                      int sym, int64_t n0, int64_t n1, double *Y) {
  if (n0 < 0 || n1 > N || n0 > n1 || group_size <= 0 ||
      (K % group_size) != 0 || (K % 2) != 0)
    return ORACLE_ERR_ARG;
  if (!sym && zeros == NULL) return ORACLE_ERR_ARG;
  const int64_t G = K / group_size;
  const int64_t W = n1 - n0;
  for (int64_t n = n0; n < n1; ++n) {
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        uint8_t byte = codes[n * (K / 2) + k / 2];
        int u = (k & 1) ? (byte >> 4) : (byte & 0x0F);
        int64_t g = k / group_size;
        float s = oracle_f16_to_f32(scales[n * G + g]);
        int zeff = sym ? 8 : (int)oracle_f16_to_f32(zeros[n * G + g]);
        double w = (double)(s * (float)(u - zeff));
        acc += (double)oracle_bf16_to_f32(X[m * K + k]) * w;
      }
      Y[m * W + (n - n0)] = acc;
    }
  }
  return ORACLE_OK;
}

/* W8A8 ([P4] sec. 2.3 and 4.2: int8 x int8 on the integer tensor core):
 * exact integer sums, checked to fit the int32 accumulator. */
int oracle_gemm_w8a8_acc(const int8_t *qx, const int8_t *qw, int64_t M,
                         int64_t N, int64_t K, int64_t m0, int64_t m1,
                         int64_t n0, int64_t n1, int32_t *acc) {
  if (m0 < 0 || m1 > M || m0 > m1 || n0 < 0 || n1 > N || n0 > n1)
    return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
  const int64_t W = n1 - n0;
  for (int64_t m = m0; m < m1; ++m) {
    for (int64_t n = n0; n < n1; ++n) {
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k)
        s += (int64_t)qx[m * K + k] * (int64_t)qw[n * K + k];
      if (s > INT32_MAX || s < INT32_MIN) status = ORACLE_ERR_OVERFLOW;
      acc[(m - m0) * W + (n - n0)] = (int32_t)s;
    }
  }
  return status;
}

/* Rescale of the integer accumulator by the two per-row scales, in fp64. */
int oracle_w8a8_rescale(const int32_t *acc, const float *sx, const float *sw,
                        int64_t m0, int64_t m1, int64_t n0, int64_t n1,
                        double *Y) {
  const int64_t W = n1 - n0;
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t n = n0; n < n1; ++n)
      Y[(m - m0) * W + (n - n0)] = (double)acc[(m - m0) * W + (n - n0)] *
                                   (double)sx[m] * (double)sw[n];
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* SmoothQuant smoothing                                                      */
/* ------------------------------------------------------------------------- */

/*
 * [P4] sec. 4.2 moves quantization difficulty from the activations to the
 * weights with an exact rewrite of the product, Y = (X diag(s)^-1)(diag(s) W)
 * in the page's [in, out] weight convention.  The statistics are per input
 * channel j: the largest |X_j| seen on calibration tokens (act_scales) and
 * the largest |W_j| over the output channels (w_scales, clamped to >= 1e-5);
 * the migration factor is s_j = act_j^alpha / w_j^(1 - alpha), clamped to
 * >= 1e-5, with alpha = 0.5 the page's recommended split.
 */
int oracle_channel_absmax(const void *A, int dtype, int64_t R, int64_t K,
                          float *out) {
  if (R < 0 || K <= 0) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
  for (int64_t k = 0; k < K; ++k) out[k] = 0.0f;
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      float x = load_elem(A, dtype, r * K + k);
      if (!isfinite(x)) {
        status = ORACLE_ERR_NONFINITE;
        continue;
      }
      if (fabsf(x) > out[k]) out[k] = fabsf(x);
    }
  }
  return status;
}

int oracle_smooth_scales(const float *act, const float *w, int64_t K,
                         double alpha, float *s) {
  if (K <= 0 || !(alpha >= 0.0 && alpha <= 1.0)) return ORACLE_ERR_ARG;
  for (int64_t k = 0; k < K; ++k) {
    const float wc = w[k] < 1e-5f ? 1e-5f : w[k];      /* w_scales.clamp(min=1e-5) */
    double v = pow((double)act[k], alpha) / pow((double)wc, 1.0 - alpha);
    if (v < 1e-5) v = 1e-5;                            /* s.clamp(min=1e-5) */
    s[k] = (float)v;
  }
  return ORACLE_OK;
}

/* diag(s) W: weight column j (input channel j) multiplied by s_j, one binary32
 * product per element, then the per-channel INT8 quantizer. */
int oracle_quantize_int8_rows_smoothed(const void *W, int w_dtype, int64_t N,
                                       int64_t K, const float *s, int8_t *q,
                                       float *scales) {
  if (N < 0 || K <= 0) return ORACLE_ERR_ARG;
  float *ws = (float *)malloc((size_t)(N > 0 ? N : 1) * (size_t)K * sizeof(float));
  if (!ws) return ORACLE_ERR_ARG;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) ws[n * K + k] = load_elem(W, w_dtype, n * K + k) * s[k];
  const int st = oracle_quantize_int8_rows(ws, ORACLE_F32, N, K, q, scales);
  free(ws);
  return st;
}

/* X diag(s)^-1: activation column j divided by s_j, one binary32 division per
 * element, then the per-token INT8 quantizer. */
int oracle_quant_act_i8_smoothed(const void *X, int x_dtype, int64_t M,
                                 int64_t K, const float *s, int8_t *q,
                                 float *scales) {
  if (M < 0 || K <= 0) return ORACLE_ERR_ARG;
  float *xs = (float *)malloc((size_t)(M > 0 ? M : 1) * (size_t)K * sizeof(float));
  if (!xs) return ORACLE_ERR_ARG;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) xs[m * K + k] = load_elem(X, x_dtype, m * K + k) / s[k];
  const int st = oracle_quant_act_i8(xs, ORACLE_F32, M, K, q, scales);
  free(xs);
  return st;
}

/* ------------------------------------------------------------------------- */
/* KV-cache INT8                                                              */
/* ------------------------------------------------------------------------- */

/*
 * [P4] sec. 6: K and V are quantized differently.  V is flat across channels
 * and takes one scale per token (the page's quant_kv_per_token: scale =
 * amax over the head dim / qmax, clamped to >= 1e-8, q = clamp(round(v /
 * scale), -qmax - 1, qmax)).  K carries channel-wise outliers (it meets Q in a
 * dot product and carries RoPE), so it takes one scale per channel: the same
 * quantizer with the maximum taken over the tokens of a head instead.
 */
int oracle_quant_kv(const void *K, const void *V, int dtype, int64_t BH,
                    int64_t S, int64_t D, int8_t *qk, float *sk, int8_t *qv,
                    float *sv) {
  if (BH < 0 || S < 0 || D <= 0) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
  /* V: rows of D elements, the per-token quantizer as it stands */
  if (BH * S > 0) {
    int st = oracle_quant_act_i8(V, dtype, BH * S, D, qv, sv);
    if (st != ORACLE_OK) status = st;
  }
  /* K: for each head, column d over the S tokens */
  for (int64_t h = 0; h < BH; ++h) {
    for (int64_t d = 0; d < D; ++d) {
      float amax = 0.0f;
      for (int64_t t = 0; t < S; ++t) {
        float x = load_elem(K, dtype, (h * S + t) * D + d);
        if (!isfinite(x)) status = ORACLE_ERR_NONFINITE;
        if (fabsf(x) > amax) amax = fabsf(x);
      }
      float s = amax / 127.0f;
      if (s < 1e-8f) s = 1e-8f;
      sk[h * D + d] = s;
      for (int64_t t = 0; t < S; ++t) {
        float r = oracle_round_half_even(load_elem(K, dtype, (h * S + t) * D + d) / s);
        r = fmaxf(-200.0f, fminf(200.0f, r));
        qk[(h * S + t) * D + d] = (int8_t)clamp_int((int)r, -128, 127);
      }
    }
  }
  return status;
}

/* ------------------------------------------------------------------------- */
/* FP8 E4M3                                                                   */
/* ------------------------------------------------------------------------- */

/* Encoding from the format: value = (-1)^s * 2^(e - 7) * (1 + m/8) for
 * exponent field e in 1..15 (except e = 15, m = 7: NaN), and
 * (-1)^s * 2^-6 * (m/8) for e = 0.  Rounding: nearest, ties to the even
 * mantissa; magnitudes that round above 448 saturate to 448. */
uint8_t oracle_f32_to_e4m3(float f) {
  const uint8_t sign = signbit(f) ? 0x80 : 0x00;
  if (isnan(f)) return (uint8_t)(sign | 0x7F);
  float a = fabsf(f);
  if (a >= 448.0f) return (uint8_t)(sign | 0x7E);
  if (a < 0.015625f) {                       /* below 2^-6: subnormal, step 2^-9 */
    const float m = oracle_round_half_even(a * 512.0f);   /* exact scaling */
    return (uint8_t)(sign | (uint8_t)m);     /* m = 8 is the smallest normal, 0x08 */
  }
  int e = 0;
  float t = a;
  while (t >= 2.0f) { t *= 0.5f; ++e; }      /* exact: powers of two */
  while (t < 1.0f) { t *= 2.0f; --e; }
  float m = oracle_round_half_even((t - 1.0f) * 8.0f);   /* (t - 1) * 8 is exact */
  if (m >= 8.0f) { m = 0.0f; ++e; }
  const int field = e + 7;
  uint8_t code = (uint8_t)((field << 3) | (int)m);
  if (code > 0x7E) code = 0x7E;              /* saturate (448 = 0x7E) */
  return (uint8_t)(sign | code);
}

float oracle_e4m3_to_f32(uint8_t c) {
  const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  float v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexpf((float)m / 8.0f, -6);
  else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return sign ? -v : v;
}

/* The W8A8 recipe of [P4] sec. 2.3 / 4.2 with E4M3 in place of int8: one scale
 * per row (output channel or token) mapping the row's largest magnitude onto
 * the largest finite E4M3 value, 448. */
int oracle_quantize_fp8_rows(const void *W, int w_dtype, int64_t R, int64_t K,
                             uint8_t *q, float *scales) {
  if (R < 0 || K <= 0) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
  for (int64_t r = 0; r < R; ++r) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float x = load_elem(W, w_dtype, r * K + k);
      if (!isfinite(x)) status = ORACLE_ERR_NONFINITE;
      if (fabsf(x) > amax) amax = fabsf(x);
    }
    float s = amax / 448.0f;
    if (s < 1e-8f) s = 1e-8f;
    scales[r] = s;
    for (int64_t k = 0; k < K; ++k) q[r * K + k] = oracle_f32_to_e4m3(load_elem(W, w_dtype, r * K + k) / s);
  }
  return status;
}

int oracle_gemm_fp8(const uint8_t *qx, const float *sx, const uint8_t *qw,
                    const float *sw, int64_t M, int64_t N, int64_t K,
                    int64_t m0, int64_t m1, int64_t n0, int64_t n1, double *Y,
                    double *acc) {
  if (m0 < 0 || m1 > M || n0 < 0 || n1 > N || m0 > m1 || n0 > n1 || K <= 0) return ORACLE_ERR_ARG;
  const int64_t W = n1 - n0;
  for (int64_t m = m0; m < m1; ++m) {
    for (int64_t n = n0; n < n1; ++n) {
      double sum = 0.0;
      for (int64_t k = 0; k < K; ++k)
        sum += (double)oracle_e4m3_to_f32(qx[m * K + k]) * (double)oracle_e4m3_to_f32(qw[n * K + k]);
      if (acc) acc[(m - m0) * W + (n - n0)] = sum;
      Y[(m - m0) * W + (n - n0)] = sum * (double)sx[m] * (double)sw[n];
    }
  }
  return ORACLE_OK;
}

/* [P4] sec. 2.3: W8A16 keeps the activations in 16 bits and expands the
 * 8-bit weight before the product; with a per-output-channel scale the
 * expanded weight is s[n] times the code's value. */
int oracle_gemm_w8a16(const uint16_t *X, int64_t M, int64_t K, const uint8_t *qw,
                      int w_fmt, const float *sw, int64_t N, int64_t n0, int64_t n1,
                      double *Y) {
  if (n0 < 0 || n1 > N || n0 > n1 || K <= 0 || M < 0) return ORACLE_ERR_ARG;
  if (w_fmt != ORACLE_W_I8 && w_fmt != ORACLE_W_E4M3) return ORACLE_ERR_ARG;
  const int64_t W = n1 - n0;
  for (int64_t n = n0; n < n1; ++n) {
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const uint8_t c = qw[n * K + k];
        const double v = (w_fmt == ORACLE_W_I8) ? (double)(int8_t)c
                                                : (double)oracle_e4m3_to_f32(c);
        const double w = (double)sw[n] * v;
        acc += (double)oracle_bf16_to_f32(X[m * K + k]) * w;
      }
      Y[m * W + (n - n0)] = acc;
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* GPTQ                                                                       */
/* ------------------------------------------------------------------------- */

/*
 * [P4] sec. 4.3: GPTQ quantizes a layer's weight column by column (input
 * dimension by input dimension) and pushes each column's rounding error onto
 * the columns not yet quantized, weighted by the inverse Hessian of the
 * layer's reconstruction error ||X W^T - X W_hat^T||^2, H = 2 X^T X.  The
 * page's skeleton uses the upper Cholesky factor U of H^-1 (damped by
 * 0.01 * mean(diag(H)) so that H stays invertible): err = (w_i - q_i) / U_ii,
 * W[:, i+1:] -= err * U[i, i+1:]; group parameters are recomputed at every
 * group start from the current (corrected) weights.
 */

/* in-place Cholesky A = L L^T (lower, row-major); 0 on success */
static int chol_lower(double *A, int64_t n) {
  for (int64_t j = 0; j < n; ++j) {
    double d = A[j * n + j];
    for (int64_t k = 0; k < j; ++k) d -= A[j * n + k] * A[j * n + k];
    if (!(d > 0.0)) return -1;
    const double ljj = sqrt(d);
    A[j * n + j] = ljj;
    for (int64_t i = j + 1; i < n; ++i) {
      double v = A[i * n + j];
      for (int64_t k = 0; k < j; ++k) v -= A[i * n + k] * A[j * n + k];
      A[i * n + j] = v / ljj;
    }
    for (int64_t i = 0; i < j; ++i) A[i * n + j] = 0.0;  /* clear the upper part */
  }
  return 0;
}

int oracle_gptq_hinv_chol(const void *X, int x_dtype, int64_t T, int64_t K,
                          double damp, double *U) {
  if (T <= 0 || K <= 0 || damp < 0.0) return ORACLE_ERR_ARG;
  double *H = (double *)calloc((size_t)(K * K), sizeof(double));
  double *Hi = (double *)calloc((size_t)(K * K), sizeof(double));
  if (!H || !Hi) { free(H); free(Hi); return ORACLE_ERR_ARG; }
  for (int64_t t = 0; t < T; ++t)
    for (int64_t a = 0; a < K; ++a) {
      const double xa = load_elem(X, x_dtype, t * K + a);
      for (int64_t b = 0; b < K; ++b) H[a * K + b] += 2.0 * xa * load_elem(X, x_dtype, t * K + b);
    }
  double mean = 0.0;
  for (int64_t a = 0; a < K; ++a) mean += H[a * K + a];
  mean /= (double)K;
  for (int64_t a = 0; a < K; ++a) H[a * K + a] += damp * mean;
  int st = ORACLE_OK;
  if (chol_lower(H, K) != 0) { st = ORACLE_ERR_ARG; goto done; }
  /* H^-1 = L^-T L^-1: solve L y = e_c, then L^T x = y for every column c */
  {
    double *col = (double *)malloc((size_t)K * sizeof(double));
    if (!col) { st = ORACLE_ERR_ARG; goto done; }
    for (int64_t c = 0; c < K; ++c) {
      for (int64_t i = 0; i < K; ++i) {            /* forward: L y = e_c */
        double v = (i == c) ? 1.0 : 0.0;
        for (int64_t k = 0; k < i; ++k) v -= H[i * K + k] * col[k];
        col[i] = v / H[i * K + i];
      }
      for (int64_t i = K - 1; i >= 0; --i) {       /* backward: L^T x = y */
        double v = col[i];
        for (int64_t k = i + 1; k < K; ++k) v -= H[k * K + i] * col[k];
        col[i] = v / H[i * K + i];
      }
      for (int64_t i = 0; i < K; ++i) Hi[i * K + c] = col[i];
    }
    free(col);
  }
  if (chol_lower(Hi, K) != 0) { st = ORACLE_ERR_ARG; goto done; }
  for (int64_t i = 0; i < K; ++i)                  /* U = L^T (upper) */
    for (int64_t j = 0; j < K; ++j) U[i * K + j] = (j >= i) ? Hi[j * K + i] : 0.0;
done:
  free(H);
  free(Hi);
  return st;
}

int oracle_gptq_quantize(const void *W, int w_dtype, int64_t N, int64_t K,
                         const double *U, int group_size, int sym,
                         uint8_t *codes, uint16_t *scales, uint16_t *zeros) {
  if (N < 0 || K <= 0 || group_size <= 0 || (K % group_size) != 0 || (K % 2) != 0)
    return ORACLE_ERR_ARG;
  if (!sym && zeros == NULL) return ORACLE_ERR_ARG;
  const int64_t G = K / group_size;
  const int qmin = sym ? -8 : 0, qmax = sym ? 7 : 15;
  double *work = (double *)malloc((size_t)K * sizeof(double));
  float *grp = (float *)malloc((size_t)group_size * sizeof(float));
  if (!work || !grp) {
    free(work);
    free(grp);
    return ORACLE_ERR_ARG;
  }
  int status = ORACLE_OK;
  memset(codes, 0, (size_t)(N * (K / 2)));
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) work[k] = load_elem(W, w_dtype, n * K + k);
    float sf = 1.0f;
    int z = 0, degenerate = 1;
    for (int64_t k = 0; k < K; ++k) {
      if (k % group_size == 0) {
        /* parameters of the group starting here, from the corrected weights
         * (rounded to binary32, the precision the INT4 rules work in) */
        const int64_t g = k / group_size;
        for (int64_t j = 0; j < group_size; ++j) grp[j] = (float)work[k + j];
        uint16_t s16;
        int nonfinite = 0;
        group_params(grp, group_size, sym, &s16, &z, &degenerate, &nonfinite);
        if (nonfinite) status = ORACLE_ERR_NONFINITE;
        scales[n * G + g] = s16;
        if (!sym) zeros[n * G + g] = oracle_f32_to_f16((float)z);
        sf = oracle_f16_to_f32(s16);
        if (isinf(sf)) status = ORACLE_ERR_NONFINITE;
      }
      const double w = work[k];
      int q = 0;
      double w_hat = 0.0;
      if (!degenerate) {
        /* the INT4 rule on the binary32 value: one fp32 division, half to even */
        float r = oracle_round_half_even((float)w / sf);
        r = fmaxf(-64.0f, fminf(64.0f, r));
        q = clamp_int((int)r + z, qmin, qmax);
        w_hat = (double)sf * (double)(q - (sym ? 0 : z));
      }
      put_nibble(codes + n * (K / 2), k, (uint8_t)(q - qmin));
      /* this column's error, pushed into the columns not yet quantized */
      const double e = (w - w_hat) / U[k * K + k];
      for (int64_t j = k + 1; j < K; ++j) work[j] -= e * U[k * K + j];
    }
  }
  free(work);
  free(grp);
  return status;
}
