/*
 * wq_oracle.h -- CPU oracle for group-wise affine weight quantization and the
 * W4A16 / W8A8 matrix products.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) includes, links or calls this code; only the tests, the
 * smoke check and the benchmark's CPU-baseline leg do.  It shares no code with
 * the CUDA sources.
 *
 * Plain single-threaded C99, compiled with -O2 -ffp-contract=off and no
 * fast-math, so every float operation below is one IEEE-754 binary32 (or
 * binary64) operation rounded to nearest-even.
 *
 * Sources (page titles from the quantization write-ups this library follows):
 *   [P1] "大模型量化技术入门：为什么我们需要量化？" sec. 2.2 (linear quantization formula)
 *   [P2] "从0到1：大模型量化" sec. 2 (q = round(f/S) + Z, f' = S(q - Z))
 *   [P3] "从 FP32 到 INT4：大模型推理加速中的量化优化实战路径" sec. 2.1 (symmetric /
 *        asymmetric quantizers with their degenerate-range rules), sec. 2.2
 *        (per-group granularity), sec. 4 (metadata share)
 *   [P4] "27届大模型面试准备（十九）：模型量化全攻略" sec. 2.1 (affine quantization,
 *        min-max scale), 2.2 (per-group g=128, 4.25-bit), 3 (per-tensor worked
 *        example), 2.3 (FP8 E4M3 as an 8-bit format), 4.2 (SmoothQuant
 *        smoothing), 4.3 (GPTQ), 6 (per-token absmax quantizer, KV-cache: K
 *        per channel, V per token)
 *
 * Status codes returned by the oracle functions.
 */
#ifndef WQ_ORACLE_H
#define WQ_ORACLE_H
#include <stdint.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_NONFINITE (-5)
#define ORACLE_ERR_OVERFLOW (-7)

/* element type tags for raw input buffers */
#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_F16 2

/* IEEE-754 conversions written from the format definitions (round to nearest,
 * ties to even).  f16 = binary16 (1/5/10), bf16 = 1/8/7. */
uint16_t oracle_f32_to_f16(float f);
float oracle_f16_to_f32(uint16_t h);
uint16_t oracle_f32_to_bf16(float f);
float oracle_bf16_to_f32(uint16_t b);
/* element-wise array forms of the four conversions */
void oracle_f32_to_f16_array(const float *in, uint16_t *out, int64_t n);
void oracle_f16_to_f32_array(const uint16_t *in, float *out, int64_t n);
void oracle_f32_to_bf16_array(const float *in, uint16_t *out, int64_t n);
void oracle_bf16_to_f32_array(const uint16_t *in, float *out, int64_t n);
/* round-half-to-even of a float to an integer-valued float */
float oracle_round_half_even(float v);

/* INT4 group-wise quantize + pack ([P4] sec. 2.1-2.2, [P3] sec. 2.1). */
int oracle_quantize_int4(const void *W, int w_dtype, int64_t N, int64_t K,
                         int group_size, int sym, uint8_t *codes,
                         uint16_t *scales, uint16_t *zeros);

/* INT8 symmetric quantization with one fp32 scale per row of K elements.
 * Used for per-output-channel weights ([P4] sec. 2.2) with qmin = -127. */
int oracle_quantize_int8_rows(const void *W, int w_dtype, int64_t N, int64_t K,
                              int8_t *q, float *scales);

/* Per-token dynamic INT8 activation quantization ([P4] sec. 6). */
int oracle_quant_act_i8(const void *X, int x_dtype, int64_t M, int64_t K,
                        int8_t *q, float *scales);

/* Dequantize INT4 codes to fp32: x_hat = s * (u - z_eff) ([P2] sec. 2). */
int oracle_dequant_int4(const uint8_t *codes, const uint16_t *scales,
                        const uint16_t *zeros, int64_t N, int64_t K,
                        int group_size, int sym, float *out);

/* Dequantize INT8 per-row codes to fp32: x_hat = s * q. */
int oracle_dequant_int8_rows(const int8_t *q, const float *scales, int64_t N,
                             int64_t K, float *out);

/* W4A16 product in fp64: Y[m, n - n0] = sum_k X[m,k] * x_hat[n,k] for
 * n in [n0, n1).  X is bf16 [M, K] row-major; Y is [M, n1 - n0]. */
int oracle_gemm_w4a16(const uint16_t *X, int64_t M, int64_t K,
                      const uint8_t *codes, const uint16_t *scales,
                      const uint16_t *zeros, int64_t N, int group_size,
                      int sym, int64_t n0, int64_t n1, double *Y);

/* W8A8 exact integer accumulators: acc[m - m0, n - n0] = sum_k qx[m,k]*qw[n,k]
 * for m in [m0, m1), n in [n0, n1).  Returns ORACLE_ERR_OVERFLOW if a sum
 * does not fit int32. */
int oracle_gemm_w8a8_acc(const int8_t *qx, const int8_t *qw, int64_t M,
                         int64_t N, int64_t K, int64_t m0, int64_t m1,
                         int64_t n0, int64_t n1, int32_t *acc);

/* SmoothQuant smoothing ([P4] sec. 4.2).
 * Per-column maximum |A[r, k]| over the R rows of A [R, K]: act_scales when A
 * is a calibration activation X [tokens, in], w_scales when A is W [out, in]. */
int oracle_channel_absmax(const void *A, int dtype, int64_t R, int64_t K,
                          float *out);
/* s[k] = max(act[k]^alpha / max(w[k], 1e-5)^(1 - alpha), 1e-5), in binary64,
 * rounded once to binary32; 0 <= alpha <= 1. */
int oracle_smooth_scales(const float *act, const float *w, int64_t K,
                         double alpha, float *s);
/* Per-channel INT8 (as oracle_quantize_int8_rows) of W'[n, k] = W[n, k] * s[k]. */
int oracle_quantize_int8_rows_smoothed(const void *W, int w_dtype, int64_t N,
                                       int64_t K, const float *s, int8_t *q,
                                       float *scales);
/* Per-token INT8 (as oracle_quant_act_i8) of X'[m, k] = X[m, k] / s[k]. */
int oracle_quant_act_i8_smoothed(const void *X, int x_dtype, int64_t M,
                                 int64_t K, const float *s, int8_t *q,
                                 float *scales);

/* KV-cache INT8 ([P4] sec. 6).  K and V are [BH, S, D] (batch x kv-heads,
 * tokens, head dim).  V per token: sv[bh, t] = max(max_d |V| / 127, 1e-8),
 * qv = clamp(round(V / sv), -128, 127).  K per channel: sk[bh, d] =
 * max(max_t |K| / 127, 1e-8) over the S tokens of that head, qk likewise. */
int oracle_quant_kv(const void *K, const void *V, int dtype, int64_t BH,
                    int64_t S, int64_t D, int8_t *qk, float *sk, int8_t *qv,
                    float *sv);

/* FP8 E4M3 ([P4] sec. 2.3 naming table): 1 sign, 4 exponent (bias 7), 3
 * mantissa bits, no infinities, S.1111.111 = NaN, largest finite 448.
 * Round to nearest even, saturating to +-448. */
uint8_t oracle_f32_to_e4m3(float f);
float oracle_e4m3_to_f32(uint8_t c);
/* FP8 W8A8 operands: per-output-channel (weights) or per-token (activations)
 * s = max(amax / 448, 1e-8), q = e4m3(x / s). */
int oracle_quantize_fp8_rows(const void *W, int w_dtype, int64_t R, int64_t K,
                             uint8_t *q, float *scales);
/* Y[m - m0, n - n0] = (sum_k e4m3(qx[m,k]) e4m3(qw[n,k])) * sx[m] * sw[n] in
 * binary64; the sum of products is exact in binary64. */
int oracle_gemm_fp8(const uint8_t *qx, const float *sx, const uint8_t *qw,
                    const float *sw, int64_t M, int64_t N, int64_t K,
                    int64_t m0, int64_t m1, int64_t n0, int64_t n1, double *Y,
                    double *acc);

/* W8A16 ([P4] sec. 2.3 naming table: 8-bit weights, 16-bit activations;
 * the weight is expanded to the activation type inside the product).
 * Weights are per-output-channel: x_hat[n, k] = sw[n] * value(qw[n, k]),
 * value = the int8 code (w_fmt ORACLE_W_I8) or the E4M3 value
 * (ORACLE_W_E4M3).  Y[m, n - n0] = sum_k X[m, k] * x_hat[n, k] in binary64
 * for n in [n0, n1); X bf16 bits [M, K]; Y [M, n1 - n0]. */
enum { ORACLE_W_I8 = 0, ORACLE_W_E4M3 = 1 };
int oracle_gemm_w8a16(const uint16_t *X, int64_t M, int64_t K, const uint8_t *qw,
                      int w_fmt, const float *sw, int64_t N, int64_t n0, int64_t n1,
                      double *Y);

/* GPTQ ([P4] sec. 4.3).  Hessian factor from calibration activations X [T, K]:
 * H = 2 X^T X + damp * mean(diag(H)) * I, U = upper Cholesky factor of H^-1
 * (H^-1 = U^T U), binary64 [K, K] row-major.  ORACLE_ERR_ARG if H is not
 * positive definite. */
int oracle_gptq_hinv_chol(const void *X, int x_dtype, int64_t T, int64_t K,
                          double damp, double *U);
/* GPTQ INT4 group-wise quantization of W [N, K] with factor U: columns in
 * order, group parameters from the error-corrected weights at each group
 * start (the rules of oracle_quantize_int4), each column's scaled error pushed
 * into the later columns.  Output format as oracle_quantize_int4. */
int oracle_gptq_quantize(const void *W, int w_dtype, int64_t N, int64_t K,
                         const double *U, int group_size, int sym,
                         uint8_t *codes, uint16_t *scales, uint16_t *zeros);

/* W8A8 rescale in fp64: Y = acc * sx[m] * sw[n] over the same window. */
int oracle_w8a8_rescale(const int32_t *acc, const float *sx, const float *sw,
                        int64_t m0, int64_t m1, int64_t n0, int64_t n1,
                        double *Y);

#endif
