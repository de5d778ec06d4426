// kernels.h -- internal launchers behind the C ABI (not part of the public API).
// Each launcher assumes its arguments were validated by wq_api.cu and returns
// a wq_status.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace wq_host {

int launch_quantize_int4(const void* W, int w_dtype, int64_t N, int64_t K, int group_size,
                         int sym, void* codes, void* scales, void* zeros, cudaStream_t s);
// smooth (nullable): SmoothQuant factors s [K]; activations are divided by
// them, weights multiplied, before quantization.
int launch_quantize_rows_i8(const void* W, int w_dtype, int64_t N, int64_t K, bool activation,
                            const float* smooth, void* q, void* scales, cudaStream_t s);
int launch_channel_absmax(const void* A, int a_dtype, int64_t R, int64_t K, float* out,
                          cudaStream_t s);
int launch_smooth_scales(const float* act, const float* w, int64_t K, float alpha, float* out,
                         cudaStream_t s);
int launch_quant_kv(const void* Kc, const void* Vc, int dtype, int64_t BH, int64_t S, int64_t D,
                    void* qk, void* sk, void* qv, void* sv, cudaStream_t s);
// One-launch KV quantizer for 16-bit caches with D in {16, 32, 64, 128, 256}
// and S <= 16384 (kv_fused_plan picks the cluster size, the tokens per CTA and
// the channel block); WQ_ERR_UNSUPPORTED otherwise, and launch_quant_kv takes
// the multi-kernel path instead.
bool kv_fused_plan(int dtype, int64_t BH, int64_t S, int64_t D, int* CS, int* R, int* CW);
int launch_quant_kv_fused(const void* Kc, const void* Vc, int dtype, int64_t BH, int64_t S,
                          int64_t D, void* qk, void* sk, void* qv, void* sv, cudaStream_t s);
int launch_quantize_rows_fp8(const void* W, int w_dtype, int64_t R, int64_t K, void* q,
                             void* scales, cudaStream_t s);
size_t gptq_workspace_bytes(int64_t N, int64_t K);
int launch_gptq(const void* W, int w_dtype, int64_t N, int64_t K, const double* U, int sym,
                void* codes, void* scales, void* zeros, void* ws, cudaStream_t s);
int launch_gemm_fp8(const void* X, int64_t M, int64_t K, const void* Wq, const void* w_scales,
                    int64_t N, void* Y, void* ws, void* acc_out, cudaStream_t s);
// W8A16 (int8 or E4M3 per-channel weights, bf16 activations): CUDA-core
// kernel for M <= kGemvW8a16MaxM, tensor-core GEMM above.
constexpr int64_t kGemvW8a16MaxM = 4;
int launch_gemm_w8a16(const void* X, int64_t M, int64_t K, const void* Wq, int w_fmt,
                      const float* w_scales, int64_t N, void* Y, cudaStream_t s);
int launch_dequant_int4(const void* codes, const void* scales, const void* zeros, int64_t N,
                        int64_t K, int group_size, int sym, void* out, int out_dtype,
                        cudaStream_t s);
int launch_dequant_int8_rows(const void* q, const void* scales, int64_t N, int64_t K, void* out,
                             int out_dtype, cudaStream_t s);

// Decode products (M <= 16): the CUDA-core kernel (no workspace) for M <=
// kGemvCcMaxM when its ring and row partials fit in shared memory
// (gemv_cc_fits), the tensor-core kernel otherwise.  The decode workspace
// holds the tensor-core kernel's tile counters (zeroed by the caller once,
// left zeroed by every completed call) and then its tile partials; it has the
// same size for every M.
constexpr int64_t kGemvCcMaxM = 4;
bool gemv_cc_fits(int64_t M, int64_t N, int64_t K);
int launch_gemv_w4a16_cc(const void* X, int64_t M, int64_t K, const void* codes,
                         const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                         cudaStream_t s);
int launch_gemv_w4a16_tc(const void* X, int64_t M, int64_t K, const void* codes,
                         const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                         void* ws, cudaStream_t s);
size_t gemv_workspace_bytes(int64_t N, int64_t K);
size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K);
bool decode_on_cuda_cores(int64_t M, int64_t N, int64_t K);
int launch_decode_w4a16(const void* X, int64_t M, int64_t K, const void* codes,
                        const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                        void* ws, cudaStream_t s);
// Set the decode kernels' launch attributes on the current device (done
// lazily by the launchers otherwise); WQ_OK or an error status.
int prepare_decode_kernels();
int prepare_cc_kernels();
int prepare_tc_kernels();
int launch_gemm_w4a16(const void* X, int64_t M, int64_t K, const void* codes,
                      const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                      cudaStream_t s);

int launch_gemm_w8a8(const void* X, int64_t M, int64_t K, const void* Wq, const void* w_scales,
                     const float* smooth, int64_t N, void* Y, void* ws, void* acc_out,
                     cudaStream_t s);

}  // namespace wq_host
