/*
 * wq.h -- C ABI of libwq: group-wise affine weight quantization and the
 * fused-dequantize W4A16 / W8A8 matrix products on NVIDIA B200 (sm_100a).
 *
 * Page tags used in the citations below (quantization write-ups this library
 * implements):
 *   [P1] "大模型量化技术入门：为什么我们需要量化？"
 *   [P2] "从0到1：大模型量化"
 *   [P3] "从 FP32 到 INT4：大模型推理加速中的量化优化实战路径"
 *   [P4] "27届大模型面试准备（十九）：模型量化全攻略"
 *   [P5] "大模型量化技术定义与主流方案解析"
 *
 * Conventions for every entry point:
 *   - All tensor arguments are DEVICE pointers to row-major buffers that the
 *     caller allocates and owns, on the current CUDA device (the one the
 *     stream belongs to).  The library keeps no pointer after return.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on that stream.
 *   - The return value reports host-side argument validation and launch
 *     errors (wq_status).  Errors the kernels detect (non-finite input, a
 *     scale that overflows fp16, a bounded wait that gave up) are recorded in
 *     a library-owned device status word read by wq_get_device_status().
 *   - Pointers must be 16-byte aligned (WQ_ERR_ALIGN otherwise).
 *   - Sizes are int64_t; negative sizes are WQ_ERR_ARG.  Empty problems
 *     (N == 0 or M == 0) return WQ_OK and launch nothing.
 *   - There is no CPU fallback: the calls need an sm_100a device.
 *
 * INT4 storage (the pages leave it open; this library fixes it):
 *   codes  : uint8 [N, K/2]; element k of row n is the nibble in byte
 *            n*K/2 + k/2, low nibble = even k; the nibble is the unsigned code
 *            u = q - qmin (symmetric: u = q + 8, q in [-8, 7]; asymmetric:
 *            u = q, q in [0, 15]).
 *   scales : fp16 [N, K/group_size], one per group of group_size consecutive
 *            input columns of a row.
 *   zeros  : fp16 [N, K/group_size] integer-valued zero points in [0, 15]
 *            (asymmetric only; NULL for symmetric).
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WQ_API __attribute__((visibility("default")))
#else
#define WQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WQ_OK = 0,
  WQ_ERR_ARG = -1,         /* bad size, NULL pointer, inconsistent options */
  WQ_ERR_UNSUPPORTED = -2, /* valid in principle, not implemented (e.g. g != 128 in a GEMM) */
  WQ_ERR_ALIGN = -3,       /* pointer not 16-byte aligned, or K not a multiple the kernel needs */
  WQ_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed */
  WQ_ERR_NONFINITE = -5,   /* device: NaN/Inf input, or a scale that overflows fp16 */
  WQ_ERR_TIMEOUT = -6,     /* device: a bounded wait inside a kernel gave up */
  WQ_ERR_WORKSPACE = -8,   /* workspace pointer NULL or too small */
  WQ_ERR_NO_DEVICE = -9    /* the current device is not sm_100 */
} wq_status;

typedef enum { WQ_F32 = 0, WQ_BF16 = 1, WQ_F16 = 2 } wq_dtype;

/*
 * wq_quantize_pack -- quantize a weight matrix W [N, K].
 *
 * bits == 4: group-wise affine INT4 ([P4] sec. 2.1 affine quantization,
 *   sec. 2.2 per-group g=128; [P3] sec. 2.1 symmetric/asymmetric quantizers,
 *   sec. 2.2 per-group granularity).  For each row n and group j of
 *   group_size columns:
 *     sym : s = fp16(amax / 7); q = clamp(round(x / s), -8, 7)
 *     asym: s = fp16((max - min) / 15); z = clamp(round(-min / s), 0, 15);
 *           q = clamp(round(x / s) + z, 0, 15)
 *   round = half to even; x / s is one IEEE fp32 division by the stored fp16
 *   scale.  Degenerate groups ([P3] sec. 2.1): sym with amax < 1e-8 (or an
 *   fp16 scale of zero) -> q = 0, stored scale fp16(amax); asym with
 *   max - min < 1e-8 (or an fp16 scale of zero) -> q = 0, s = 1, z = 0.
 *   Outputs: codes uint8 [N, K/2], scales fp16 [N, K/g], zeros fp16 [N, K/g]
 *   (asym) -- zeros must be NULL iff sym.
 *   Requires K % group_size == 0, group_size % 32 == 0.
 * bits == 8: symmetric INT8 with one fp32 scale per output row ([P4] sec. 2.2,
 *   per-channel weights): s = amax / 127, q = clamp(round(x / s), -127, 127);
 *   rows with amax < 1e-8 get q = 0 and s = amax.  Requires sym == 1,
 *   group_size == K, zeros == NULL.  Outputs: codes int8 [N, K], scales fp32 [N].
 *
 * W: w_dtype WQ_F32, WQ_BF16 or WQ_F16, row-major [N, K].
 * Errors: WQ_ERR_ARG (sizes, NULL, sym/zeros mismatch), WQ_ERR_UNSUPPORTED
 * (bits not 4/8), WQ_ERR_ALIGN; device: WQ_ERR_NONFINITE (codes of the
 * offending group are then unspecified).
 */
WQ_API int wq_quantize_pack(const void *W, int w_dtype, int64_t N, int64_t K,
                     int group_size, int bits, int sym, void *codes,
                     void *scales, void *zeros, void *stream);

/*
 * wq_dequant -- x_hat = s * (q - z) ([P2] sec. 2 dequantization; [P4]
 * sec. 2.1).  bits == 4: inputs as produced by wq_quantize_pack (zeros NULL
 * iff sym); the fp32 result is exact.  bits == 8: x_hat = s[n] * q (int8
 * codes, fp32 scales, group_size == K, sym == 1).
 * out: [N, K] of out_dtype WQ_F32 or WQ_BF16 (the fp32 value rounded to
 * nearest even).
 */
WQ_API int wq_dequant(const void *codes, const void *scales, const void *zeros,
               int64_t N, int64_t K, int group_size, int bits, int sym,
               void *out, int out_dtype, void *stream);

/*
 * wq_gemm_w4a16 -- Y = X * dequant(W)^T with INT4 group-wise weights and
 * bf16 activations ([P4] sec. 2.3 W4A16; [P5] sec. 四 fused dequantization:
 * the weight is expanded tile by tile inside the kernel and never written back
 * to memory).  X bf16 [M, K]; codes/scales/zeros as above with
 * group_size == 128 (others: WQ_ERR_UNSUPPORTED, [P4] sec. 7.2: the group must
 * divide the kernel tile); Y bf16 [M, N]; fp32 accumulation.
 * M <= 16 runs a decode kernel (every weight byte streamed once from HBM,
 * the work split evenly over all SMs): on the CUDA cores at M <= 4 while a
 * CTA's fp32 row partials (ceil(N / (4 P)) * 4 rows x ceil(K / 1024) chunks x
 * M rounded up to 1, 2 or 4, P = the SM count) fit in shared memory beside
 * its ring (about 160 KB; N = 28672 and K = 28672 both fit with a wide
 * margin), on the tensor cores otherwise; larger M runs the tensor-core GEMM.
 * Requires K % 128 == 0 and N % 8 == 0.
 *
 * Stream order: the CUDA-core decode kernel is launched as a programmatic
 * dependent of the kernel before it on the stream.  It starts streaming
 * codes and scales (and zeros) while that kernel is still finishing, and
 * reads X, and writes Y, only after it has completed.  Weights are inputs
 * that do not change from call to call: they must not be written by the
 * kernel immediately preceding the call on the same stream while that kernel
 * itself triggers its dependents early (of this library's kernels only this
 * decode kernel does, and it writes no weights; a kernel that does not
 * trigger lets the call start only once all its blocks have exited).
 *
 * ws / ws_bytes: device workspace of wq_w4a16_workspace_bytes(M, N, K) bytes
 * (0 for M > 16, where ws may be NULL).  Fill it with zeros once before its
 * first use (e.g. cudaMemset); every call that completes leaves the part that
 * must start at zero (the arrival counters at its start) zeroed again, so it
 * can be reused call after call (its size does not depend on M).  The
 * CUDA-core kernel does not use it.  Calls that may run at the same
 * time on the GPU need separate workspaces.  After a call reported
 * WQ_ERR_TIMEOUT, zero it again.  WQ_ERR_WORKSPACE if NULL or too small.
 */
WQ_API size_t wq_w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K);
WQ_API int wq_gemm_w4a16(const void *X, int64_t M, int64_t K, const void *codes,
                         const void *scales, const void *zeros, int64_t N,
                         int group_size, int sym, void *Y, void *ws,
                         size_t ws_bytes, void *stream);

/*
 * wq_gemm_w4a16_noalloc -- the decode product of wq_gemm_w4a16 (M = 1..16)
 * for callers that cannot hand the library any device memory: a serving loop
 * whose device memory all belongs to another allocator under a fixed budget,
 * a plain C host with no device allocator of its own, or a latency-critical
 * path where a cudaMalloc (which may synchronize the device) is not
 * acceptable.  The quantization write-ups have no counterpart of this call.
 *
 * Same arguments and results as wq_gemm_w4a16 without ws / ws_bytes.  The
 * library allocates nothing, in this call or ever: the scratch is an array of
 * 4 MiB + 4 KiB inside the library's device image, held by every GPU that
 * loads the library until the process exits.  Limits: M <= 16, N <= 131072,
 * at most 256 SMs (WQ_ERR_UNSUPPORTED beyond them, before any launch).  At
 * M <= 4 the CUDA-core kernel runs and no scratch is used.
 *
 * The first call on a device does the set-up: it looks up the array's device
 * address and sets the decode kernels' launch attributes.  Make that first
 * call before any stream capture.  Every call shares the one array, which
 * keeps the last call's contents; each call clears the counters that must
 * start at zero on its own stream.  Calls that overlap on the GPU (other
 * streams, other host threads) race and give wrong results: serialize them.
 */
WQ_API int wq_gemm_w4a16_noalloc(const void *X, int64_t M, int64_t K,
                                 const void *codes, const void *scales,
                                 const void *zeros, int64_t N, int group_size,
                                 int sym, void *Y, void *stream);

/*
 * wq_quant_act_i8 -- per-token dynamic INT8 quantization of activations
 * ([P4] sec. 6 per-token absmax quantizer, used for the A8 of W8A8, [P4]
 * sec. 2.3): s[m] = max(amax_m / 127, 1e-8); q = clamp(round(x / s), -128, 127).
 * X bf16 [M, K] -> q int8 [M, K], s fp32 [M].  Requires K % 16 == 0.
 */
WQ_API int wq_quant_act_i8(const void *X, int64_t M, int64_t K, void *q, void *s,
                    void *stream);

/* Bytes of workspace wq_gemm_w8a8 needs: int8 X [M, K] then fp32 scales [M],
 * each part 256-byte aligned. */
WQ_API size_t wq_w8a8_workspace_bytes(int64_t M, int64_t K);

/*
 * wq_gemm_w8a8 -- W8A8 product on the int8 tensor cores ([P4] sec. 2.3 and
 * 4.2: int8 weights and activations, int32 accumulation, then a floating
 * rescale).  X bf16 [M, K] is quantized per token into `ws` (see
 * wq_quant_act_i8), then acc[m, n] = sum_k qx[m, k] * qw[n, k] (int32) and
 * Y[m, n] = bf16(float(acc) * sx[m] * w_scales[n]).
 * Wq int8 [N, K] and w_scales fp32 [N] come from wq_quantize_pack(bits = 8).
 * acc_out (nullable) receives the raw int32 accumulators [M, N].
 * Requires K % 128 == 0, N % 16 == 0, ws of wq_w8a8_workspace_bytes(M, K).
 */
WQ_API int wq_gemm_w8a8(const void *X, int64_t M, int64_t K, const void *Wq,
                 const void *w_scales, int64_t N, void *Y, void *ws,
                 size_t ws_bytes, void *acc_out, void *stream);

/*
 * SmoothQuant smoothing ([P4] sec. 4.2): Y = (X diag(s)^-1)(diag(s) W) moves
 * quantization difficulty from activations with outlier channels to the
 * weights, with s_j = max|X_j|^alpha / max|W_j|^(1 - alpha) per input
 * channel j.  The five calls below compute the statistics and s, quantize the
 * smoothed weight and activations, and run the W8A8 product on them.
 */

/*
 * wq_channel_absmax -- out[k] = max_r |A[r, k]| over the R rows of A [R, K]
 * (a_dtype WQ_F32 / WQ_BF16 / WQ_F16): act_scales when A is calibration
 * activations [tokens, K], w_scales when A is a weight [N, K].  out fp32 [K].
 * Requires K % 8 == 0.  Non-finite elements are skipped and reported as
 * WQ_ERR_NONFINITE in the device status.
 */
WQ_API int wq_channel_absmax(const void *A, int a_dtype, int64_t R, int64_t K,
                             void *out, void *stream);

/*
 * wq_smooth_scales -- s[k] = max(act[k]^alpha / max(w[k], 1e-5)^(1 - alpha),
 * 1e-5) for fp32 [K] statistics, evaluated in binary64 and rounded to fp32
 * (the clamps of [P4] sec. 4.2's smooth_ln_linear).  0 <= alpha <= 1; the
 * page recommends 0.5.
 */
WQ_API int wq_smooth_scales(const void *act_absmax, const void *w_absmax,
                            int64_t K, float alpha, void *s, void *stream);

/*
 * wq_quantize_i8_smooth -- per-output-channel INT8 (as wq_quantize_pack with
 * bits = 8) of the smoothed weight W'[n, k] = W[n, k] * s[k] (one fp32 product
 * per element; W' is never stored).  W [N, K] of w_dtype, s fp32 [K] -> q int8
 * [N, K], scales fp32 [N].  Requires K % 16 == 0.
 */
WQ_API int wq_quantize_i8_smooth(const void *W, int w_dtype, int64_t N, int64_t K,
                                 const void *s, void *q, void *scales, void *stream);

/*
 * wq_quant_act_i8_smooth -- per-token INT8 (as wq_quant_act_i8) of the
 * smoothed activations X'[m, k] = X[m, k] / s[k] (one IEEE fp32 division per
 * element).  X bf16 [M, K], s fp32 [K] -> q int8 [M, K], sx fp32 [M].
 * Requires K % 16 == 0.
 */
WQ_API int wq_quant_act_i8_smooth(const void *X, int64_t M, int64_t K, const void *s,
                                  void *q, void *sx, void *stream);

/*
 * wq_gemm_w8a8_smooth -- wq_gemm_w8a8 on the smoothed pair: X is quantized
 * per token after division by s (as wq_quant_act_i8_smooth) into `ws`, then
 * multiplied with Wq / w_scales from wq_quantize_i8_smooth with the same s.
 * Same arguments, requirements and workspace as wq_gemm_w8a8, plus s fp32 [K].
 */
WQ_API int wq_gemm_w8a8_smooth(const void *X, int64_t M, int64_t K, const void *Wq,
                               const void *w_scales, const void *s, int64_t N,
                               void *Y, void *ws, size_t ws_bytes, void *acc_out,
                               void *stream);

/*
 * wq_quant_kv -- KV-cache INT8 ([P4] sec. 6: K and V are treated differently).
 * K, V [BH, S, D] of dtype (WQ_F32 / WQ_BF16 / WQ_F16), BH = batch x kv heads,
 * S tokens, D head dim.
 *   V per token:   sv[bh, t] = max(max_d |V[bh, t, d]| / 127, 1e-8),
 *                  qv = clamp(round(V / sv), -128, 127)   (the page's
 *                  quant_kv_per_token; same quantizer as wq_quant_act_i8)
 *   K per channel: sk[bh, d] = max(max_t |K[bh, t, d]| / 127, 1e-8) over the
 *                  S tokens of that head, qk = clamp(round(K / sk), -128, 127)
 * qk, qv int8 [BH, S, D]; sk fp32 [BH, D]; sv fp32 [BH, S].  Rounding is half
 * to even after one IEEE fp32 division.  Requires D % 8 == 0, D <= 256,
 * BH <= 65535.  16-bit caches with D in {16, 32, 64, 128, 256} and S <= 16384
 * read K once (a thread-block cluster per head and channel block holds the
 * head's K in shared memory while its channel maxima are combined); other
 * shapes and fp32 caches read K twice (maxima, then codes).  A NaN is skipped
 * by a maximum and an infinity counts; their codes follow the definition
 * (a NaN quotient gives 127) and the status reports WQ_ERR_NONFINITE.
 * Keeping the most recent tokens unquantized (the page's residual window) is
 * the caller's choice of S.
 */
WQ_API int wq_quant_kv(const void *K, const void *V, int dtype, int64_t BH, int64_t S,
                       int64_t D, void *qk, void *sk, void *qv, void *sv, void *stream);

/*
 * FP8 E4M3 W8A8 ([P4] sec. 2.3 names FP8 E4M3 as the 8-bit float format of
 * the newest tensor cores; the recipe is the W8A8 one with E4M3 in place of
 * int8).  E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, largest
 * finite value 448, no infinities.
 *
 * wq_quantize_fp8_rows -- one scale per row (a weight's output channel, or an
 * activation's token): s[r] = max(max_k |A[r, k]| / 448, 1e-8) and
 * q = E4M3(A / s) (IEEE division, round to nearest even, saturating to
 * +-448).  A [R, K] of a_dtype -> q uint8 E4M3 codes [R, K], s fp32 [R].
 * Requires K % 16 == 0.
 */
WQ_API int wq_quantize_fp8_rows(const void *A, int a_dtype, int64_t R, int64_t K,
                                void *q, void *scales, void *stream);

/*
 * wq_gemm_w8a16 -- W8A16 ([P4] sec. 2.3 naming table: 8-bit weights with
 * 16-bit activations; the weight is expanded to the activation type inside
 * the product, never written back): Y = bf16(w_scales[n] * acc[m, n]) with
 * acc = sum_k X[m, k] * value(Wq[n, k]) accumulated in fp32.
 * X bf16 [M, K]; Wq [N, K] per-output-channel codes, w_fmt WQ_W8_INT8 (int8
 * codes with fp32 scales, as wq_quantize_pack with bits 8 writes them) or
 * WQ_W8_E4M3 (E4M3 codes with fp32 scales, as wq_quantize_fp8_rows writes
 * them); w_scales fp32 [N]; Y bf16 [M, N].  Every code value is exact in
 * bf16, so the expanded weight is not rounded.  M <= 4 runs on the CUDA
 * cores (every weight byte streamed once), larger M on the tensor cores
 * (tcgen05.mma kind::f16).  With int8 codes and M <= 4 the CUDA-core product
 * takes X in 16-bit fixed point, as the W4A16 decode does: per activation
 * row and 128-element group of K, x' = rint(x 2^e) with the group's largest
 * |x| scaled into [2^12, 2^13), exact integer dot products with the codes,
 * scaled by 2^-e in fp32 (values below 2^-5 of the group maximum move by at
 * most 2^-13 of it; a chunk of X holding a NaN or an infinity is multiplied
 * in fp32).  Requires K % 64 == 0; all pointers 16-byte aligned.
 */
enum { WQ_W8_INT8 = 0, WQ_W8_E4M3 = 1 };
WQ_API int wq_gemm_w8a16(const void *X, int64_t M, int64_t K, const void *Wq, int w_fmt,
                         const void *w_scales, int64_t N, void *Y, void *stream);

/*
 * wq_gemm_fp8 -- Y = bf16(acc * sx[m] * w_scales[n]) with acc[m, n] =
 * sum_k E4M3(qx[m, k]) * E4M3(qw[n, k]) accumulated in fp32 on the tensor cores
 * (tcgen05.mma kind::f8f6f4).  X bf16 [M, K] is quantized per token into ws
 * first (as wq_quantize_fp8_rows); Wq / w_scales come from
 * wq_quantize_fp8_rows on the weight.  acc_out (nullable) receives the fp32
 * accumulators [M, N].  Same requirements and workspace as wq_gemm_w8a8.
 */
WQ_API int wq_gemm_fp8(const void *X, int64_t M, int64_t K, const void *Wq,
                       const void *w_scales, int64_t N, void *Y, void *ws,
                       size_t ws_bytes, void *acc_out, void *stream);

/*
 * wq_gptq_quantize -- GPTQ INT4 group-wise quantization with error feedback
 * ([P4] sec. 4.3).  Columns (input dims) are quantized in order; each column's
 * error (w - w_hat) / U[i, i] is pushed into the columns not yet quantized
 * with weights U[i, j]; at every group start the group's scale (and zero
 * point) come from the corrected weights by the rules of wq_quantize_pack.
 * U: fp64 [K, K] row-major, the upper Cholesky factor of the damped inverse
 * Hessian, H^-1 = U^T U with H = 2 X^T X + damp * mean(diag(H)) * I from
 * calibration activations X (damp 0.01 in [P4]); computing it is the
 * caller's (it is a per-layer calibration step).  W [N, K] of w_dtype;
 * outputs as wq_quantize_pack (bits 4, group_size 128 only).  The
 * corrections run in binary64 and the rounding decision in binary32.
 * ws: wq_gptq_workspace_bytes(N, K) bytes (fp64 errors), any contents.
 * Requires K % 128 == 0.
 */
WQ_API size_t wq_gptq_workspace_bytes(int64_t N, int64_t K);
WQ_API int wq_gptq_quantize(const void *W, int w_dtype, int64_t N, int64_t K,
                            const void *U, int group_size, int sym, void *codes,
                            void *scales, void *zeros, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * wq_get_device_status -- synchronize `stream`, then return the first error
 * any kernel recorded since the last reset (WQ_OK if none); clear it when
 * reset != 0.  Returns WQ_ERR_CUDA if the synchronization itself fails.
 */
WQ_API int wq_get_device_status(void *stream, int reset);

/*
 * wq_selftest_wait_timeout -- exercises the bounded-wait path that every
 * tensor-core kernel of this library uses for its pipeline barriers.  It
 * launches one CTA that waits on a barrier nothing will ever complete; after
 * limit_us microseconds (1 .. 1e6) the wait gives up, records WQ_ERR_TIMEOUT in
 * the device status word and the kernel returns normally (no fault, the
 * context stays usable).  Read the result with wq_get_device_status().
 * The quantization pages have no counterpart: this is a failure-detection hook.
 */
WQ_API int wq_selftest_wait_timeout(int limit_us, void *stream);

/* Human-readable name of a wq_status value (static storage). */
WQ_API const char *wq_status_str(int status);

/* Text of the last CUDA error seen on the host side by this thread. */
WQ_API const char *wq_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* WQ_H */
