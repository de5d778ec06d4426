// wq_api.cu -- the C ABI declared in include/wq.h: argument validation,
// dispatch to the kernels, and the device status word.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

// Library-owned device status word: the first error a kernel detects.  One
// copy per device (a __device__ variable is instantiated on every device the
// library's module is loaded on).
__device__ int g_wq_status = 0;

namespace wq_host {

namespace {
constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
int g_arch_ok[kMaxDevices] = {};  // 0 unknown, 1 ok, -1 not sm_100
std::mutex g_mu;
thread_local char g_last_err[256] = "";

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

int init_device(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_arch_ok[dev] != 0) return g_arch_ok[dev] > 0 ? WQ_OK : WQ_ERR_NO_DEVICE;
  cudaDeviceProp prop;
  cudaError_t e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0) {
    g_arch_ok[dev] = -1;
    snprintf(g_last_err, sizeof(g_last_err), "device %d is sm_%d%d, libwq needs sm_100", dev,
             prop.major, prop.minor);
    return WQ_ERR_NO_DEVICE;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_wq_status);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_wq_status)");
  g_status_ptr[dev] = static_cast<int*>(p);
  g_sms[dev] = prop.multiProcessorCount;
  g_arch_ok[dev] = 1;
  return WQ_OK;
}
}  // namespace

int cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_err, sizeof(g_last_err), "%s: %s", where, cudaGetErrorString(e));
  return WQ_ERR_CUDA;
}

int* status_ptr() {
  const int d = current_device();
  return (d >= 0 && d < kMaxDevices) ? g_status_ptr[d] : nullptr;
}

int sm_count() {
  const int d = current_device();
  return (d >= 0 && d < kMaxDevices && g_sms[d] > 0) ? g_sms[d] : 148;
}

// Validate the current device once per device; every entry point calls it.
int ensure_device() {
  const int d = current_device();
  if (d < 0) {
    cudaError_t e = cudaGetLastError();
    return cuda_fail(e == cudaSuccess ? cudaErrorNoDevice : e, "cudaGetDevice");
  }
  if (d >= kMaxDevices) return WQ_ERR_NO_DEVICE;
  if (g_arch_ok[d] > 0) return WQ_OK;
  return init_device(d);
}

const char* last_error_text() { return g_last_err; }

}  // namespace wq_host

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

}  // namespace

extern "C" {

int wq_quantize_pack(const void* W, int w_dtype, int64_t N, int64_t K, int group_size, int bits,
                     int sym, void* codes, void* scales, void* zeros, void* stream) {
  if (N < 0 || K < 0) return WQ_ERR_ARG;
  if (w_dtype != WQ_F32 && w_dtype != WQ_BF16 && w_dtype != WQ_F16) return WQ_ERR_ARG;
  if (sym != 0 && sym != 1) return WQ_ERR_ARG;
  if (bits == 4) {
    if (group_size <= 0 || (K % group_size) != 0) return WQ_ERR_ARG;
    if ((sym == 1) != (zeros == nullptr)) return WQ_ERR_ARG;
    if ((group_size % 32) != 0 || group_size > 1024 ||
        (group_size & (group_size - 1)) != 0)
      return WQ_ERR_UNSUPPORTED;
  } else if (bits == 8) {
    if (sym != 1 || zeros != nullptr || group_size != K) return WQ_ERR_ARG;
    if ((K % 16) != 0) return WQ_ERR_ALIGN;
  } else {
    return WQ_ERR_UNSUPPORTED;
  }
  if (N == 0 || K == 0) return WQ_OK;
  if (!W || !codes || !scales) return WQ_ERR_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(scales) || (zeros && !aligned16(zeros)))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  if (bits == 4)
    return wq_host::launch_quantize_int4(W, w_dtype, N, K, group_size, sym, codes, scales, zeros,
                                         as_stream(stream));
  return wq_host::launch_quantize_rows_i8(W, w_dtype, N, K, false, nullptr, codes, scales,
                                          as_stream(stream));
}

int wq_dequant(const void* codes, const void* scales, const void* zeros, int64_t N, int64_t K,
               int group_size, int bits, int sym, void* out, int out_dtype, void* stream) {
  if (N < 0 || K < 0) return WQ_ERR_ARG;
  if (out_dtype != WQ_F32 && out_dtype != WQ_BF16) return WQ_ERR_ARG;
  if (sym != 0 && sym != 1) return WQ_ERR_ARG;
  if (bits == 4) {
    if (group_size <= 0 || (K % group_size) != 0) return WQ_ERR_ARG;
    if ((sym == 1) != (zeros == nullptr)) return WQ_ERR_ARG;
    if ((group_size % 32) != 0) return WQ_ERR_UNSUPPORTED;
  } else if (bits == 8) {
    if (sym != 1 || zeros != nullptr || group_size != K) return WQ_ERR_ARG;
    if ((K % 16) != 0) return WQ_ERR_ALIGN;
  } else {
    return WQ_ERR_UNSUPPORTED;
  }
  if (N == 0 || K == 0) return WQ_OK;
  if (!codes || !scales || !out) return WQ_ERR_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(out) || (zeros && !aligned16(zeros)))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  if (bits == 4)
    return wq_host::launch_dequant_int4(codes, scales, zeros, N, K, group_size, sym, out,
                                        out_dtype, as_stream(stream));
  return wq_host::launch_dequant_int8_rows(codes, scales, N, K, out, out_dtype,
                                           as_stream(stream));
}

size_t wq_w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || M > 16 || N <= 0 || K < 128) return 0;
  if (wq_host::ensure_device() != WQ_OK) return 0;
  return wq_host::decode_workspace_bytes(M, N, K);
}

int wq_gemm_w4a16(const void* X, int64_t M, int64_t K, const void* codes, const void* scales,
                  const void* zeros, int64_t N, int group_size, int sym, void* Y, void* ws,
                  size_t ws_bytes, void* stream) {
  if (M < 0 || K < 0 || N < 0) return WQ_ERR_ARG;
  if (sym != 0 && sym != 1) return WQ_ERR_ARG;
  if ((sym == 1) != (zeros == nullptr)) return WQ_ERR_ARG;
  if (group_size != 128) return WQ_ERR_UNSUPPORTED;
  if ((K % 128) != 0 || (N % 8) != 0) return WQ_ERR_ALIGN;
  if (N > (int64_t(1) << 30) || K > (int64_t(1) << 24)) return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (K == 0) return WQ_ERR_ARG;
  if (!X || !codes || !scales || !Y) return WQ_ERR_ARG;
  if (!aligned16(X) || !aligned16(codes) || !aligned16(scales) || !aligned16(Y) ||
      (zeros && !aligned16(zeros)) || (ws && (reinterpret_cast<uintptr_t>(ws) & 255u)))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  if (M <= 16) {
    if (!ws || ws_bytes < wq_host::decode_workspace_bytes(M, N, K)) return WQ_ERR_WORKSPACE;
    return wq_host::launch_decode_w4a16(X, M, K, codes, scales, zeros, N, sym, Y, ws,
                                        as_stream(stream));
  }
  return wq_host::launch_gemm_w4a16(X, M, K, codes, scales, zeros, N, sym, Y, as_stream(stream));
}

int wq_quant_act_i8(const void* X, int64_t M, int64_t K, void* q, void* s, void* stream) {
  if (M < 0 || K < 0) return WQ_ERR_ARG;
  if ((K % 16) != 0) return WQ_ERR_ALIGN;
  if (M == 0 || K == 0) return WQ_OK;
  if (!X || !q || !s) return WQ_ERR_ARG;
  if (!aligned16(X) || !aligned16(q) || !aligned16(s)) return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_quantize_rows_i8(X, WQ_BF16, M, K, true, nullptr, q, s, as_stream(stream));
}

size_t wq_w8a8_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  const size_t a = (size_t(M) * size_t(K) + 255) & ~size_t(255);
  const size_t b = (size_t(M) * 4 + 255) & ~size_t(255);
  return a + b;
}

int wq_gemm_w8a8(const void* X, int64_t M, int64_t K, const void* Wq, const void* w_scales,
                 int64_t N, void* Y, void* ws, size_t ws_bytes, void* acc_out, void* stream) {
  if (M < 0 || K < 0 || N < 0) return WQ_ERR_ARG;
  if ((K % 16) != 0 || (N % 16) != 0) return WQ_ERR_ALIGN;
  if (M > (int64_t(1) << 31) / 2 || N > (int64_t(1) << 31) / 2 || K > (int64_t(1) << 24))
    return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (K == 0) return WQ_ERR_ARG;
  if (!X || !Wq || !w_scales || !Y) return WQ_ERR_ARG;
  if (!ws || ws_bytes < wq_w8a8_workspace_bytes(M, K)) return WQ_ERR_WORKSPACE;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(w_scales) || !aligned16(Y) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || (acc_out && !aligned16(acc_out)))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_gemm_w8a8(X, M, K, Wq, w_scales, nullptr, N, Y, ws, acc_out,
                                   as_stream(stream));
}

// ------------------------------------------------------------- SmoothQuant

int wq_channel_absmax(const void* A, int a_dtype, int64_t R, int64_t K, void* out,
                      void* stream) {
  if (R < 0 || K < 0) return WQ_ERR_ARG;
  if (a_dtype != WQ_F32 && a_dtype != WQ_BF16 && a_dtype != WQ_F16) return WQ_ERR_ARG;
  if ((K % 8) != 0) return WQ_ERR_ALIGN;
  if (K == 0) return WQ_OK;
  if (!out || (R > 0 && !A)) return WQ_ERR_ARG;
  if ((A && !aligned16(A)) || !aligned16(out)) return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_channel_absmax(A, a_dtype, R, K, static_cast<float*>(out),
                                        as_stream(stream));
}

int wq_smooth_scales(const void* act_absmax, const void* w_absmax, int64_t K, float alpha,
                     void* s, void* stream) {
  if (K < 0) return WQ_ERR_ARG;
  if (!(alpha >= 0.f && alpha <= 1.f)) return WQ_ERR_ARG;
  if (K == 0) return WQ_OK;
  if (!act_absmax || !w_absmax || !s) return WQ_ERR_ARG;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_smooth_scales(static_cast<const float*>(act_absmax),
                                       static_cast<const float*>(w_absmax), K, alpha,
                                       static_cast<float*>(s), as_stream(stream));
}

int wq_quantize_i8_smooth(const void* W, int w_dtype, int64_t N, int64_t K, const void* smooth,
                          void* q, void* scales, void* stream) {
  if (N < 0 || K < 0) return WQ_ERR_ARG;
  if (w_dtype != WQ_F32 && w_dtype != WQ_BF16 && w_dtype != WQ_F16) return WQ_ERR_ARG;
  if ((K % 16) != 0) return WQ_ERR_ALIGN;
  if (N == 0 || K == 0) return WQ_OK;
  if (!W || !smooth || !q || !scales) return WQ_ERR_ARG;
  if (!aligned16(W) || !aligned16(smooth) || !aligned16(q) || !aligned16(scales))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_quantize_rows_i8(W, w_dtype, N, K, false,
                                          static_cast<const float*>(smooth), q, scales,
                                          as_stream(stream));
}

int wq_quant_act_i8_smooth(const void* X, int64_t M, int64_t K, const void* smooth, void* q,
                           void* s, void* stream) {
  if (M < 0 || K < 0) return WQ_ERR_ARG;
  if ((K % 16) != 0) return WQ_ERR_ALIGN;
  if (M == 0 || K == 0) return WQ_OK;
  if (!X || !smooth || !q || !s) return WQ_ERR_ARG;
  if (!aligned16(X) || !aligned16(smooth) || !aligned16(q) || !aligned16(s)) return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_quantize_rows_i8(X, WQ_BF16, M, K, true,
                                          static_cast<const float*>(smooth), q, s,
                                          as_stream(stream));
}

int wq_gemm_w8a8_smooth(const void* X, int64_t M, int64_t K, const void* Wq,
                        const void* w_scales, const void* smooth, int64_t N, void* Y, void* ws,
                        size_t ws_bytes, void* acc_out, void* stream) {
  if (!smooth) return WQ_ERR_ARG;
  if (!aligned16(smooth)) return WQ_ERR_ALIGN;
  if (M < 0 || K < 0 || N < 0) return WQ_ERR_ARG;
  if ((K % 16) != 0 || (N % 16) != 0) return WQ_ERR_ALIGN;
  if (M > (int64_t(1) << 31) / 2 || N > (int64_t(1) << 31) / 2 || K > (int64_t(1) << 24))
    return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (K == 0) return WQ_ERR_ARG;
  if (!X || !Wq || !w_scales || !Y) return WQ_ERR_ARG;
  if (!ws || ws_bytes < wq_w8a8_workspace_bytes(M, K)) return WQ_ERR_WORKSPACE;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(w_scales) || !aligned16(Y) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || (acc_out && !aligned16(acc_out)))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_gemm_w8a8(X, M, K, Wq, w_scales, static_cast<const float*>(smooth), N,
                                   Y, ws, acc_out, as_stream(stream));
}

// ---------------------------------------------------------------- KV cache

int wq_quant_kv(const void* K, const void* V, int dtype, int64_t BH, int64_t S, int64_t D,
                void* qk, void* sk, void* qv, void* sv, void* stream) {
  if (BH < 0 || S < 0 || D < 0) return WQ_ERR_ARG;
  if (dtype != WQ_F32 && dtype != WQ_BF16 && dtype != WQ_F16) return WQ_ERR_ARG;
  if ((D % 8) != 0) return WQ_ERR_ALIGN;
  if (D > 256 || BH > 65535) return WQ_ERR_UNSUPPORTED;
  if (BH == 0 || D == 0) return WQ_OK;
  if (!K || !V || !qk || !sk || !qv || !sv) return WQ_ERR_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(qk) || !aligned16(sk) || !aligned16(qv) ||
      !aligned16(sv))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_quant_kv(K, V, dtype, BH, S, D, qk, sk, qv, sv, as_stream(stream));
}

// --------------------------------------------------------------------- FP8

int wq_quantize_fp8_rows(const void* A, int a_dtype, int64_t R, int64_t K, void* q, void* scales,
                         void* stream) {
  if (R < 0 || K < 0) return WQ_ERR_ARG;
  if (a_dtype != WQ_F32 && a_dtype != WQ_BF16 && a_dtype != WQ_F16) return WQ_ERR_ARG;
  if ((K % 16) != 0) return WQ_ERR_ALIGN;
  if (R == 0 || K == 0) return WQ_OK;
  if (!A || !q || !scales) return WQ_ERR_ARG;
  if (!aligned16(A) || !aligned16(q) || !aligned16(scales)) return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_quantize_rows_fp8(A, a_dtype, R, K, q, scales, as_stream(stream));
}

int wq_gemm_fp8(const void* X, int64_t M, int64_t K, const void* Wq, const void* w_scales,
                int64_t N, void* Y, void* ws, size_t ws_bytes, void* acc_out, void* stream) {
  if (M < 0 || K < 0 || N < 0) return WQ_ERR_ARG;
  if ((K % 16) != 0 || (N % 16) != 0) return WQ_ERR_ALIGN;
  if (M > (int64_t(1) << 31) / 2 || N > (int64_t(1) << 31) / 2 || K > (int64_t(1) << 24))
    return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (K == 0) return WQ_ERR_ARG;
  if (!X || !Wq || !w_scales || !Y) return WQ_ERR_ARG;
  if (!ws || ws_bytes < wq_w8a8_workspace_bytes(M, K)) return WQ_ERR_WORKSPACE;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(w_scales) || !aligned16(Y) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || (acc_out && !aligned16(acc_out)))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_gemm_fp8(X, M, K, Wq, w_scales, N, Y, ws, acc_out, as_stream(stream));
}

int wq_gemm_w8a16(const void* X, int64_t M, int64_t K, const void* Wq, int w_fmt,
                  const void* w_scales, int64_t N, void* Y, void* stream) {
  if (M < 0 || K < 0 || N < 0) return WQ_ERR_ARG;
  if (w_fmt != WQ_W8_INT8 && w_fmt != WQ_W8_E4M3) return WQ_ERR_ARG;
  if ((K % 64) != 0) return WQ_ERR_ALIGN;
  if (M > (int64_t(1) << 31) / 2 || N > (int64_t(1) << 31) / 2 || K > (int64_t(1) << 24))
    return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (K == 0) return WQ_ERR_ARG;
  if (!X || !Wq || !w_scales || !Y) return WQ_ERR_ARG;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(w_scales) || !aligned16(Y))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_gemm_w8a16(X, M, K, Wq, w_fmt, static_cast<const float*>(w_scales), N,
                                    Y, as_stream(stream));
}

// -------------------------------------------------------------------- GPTQ

size_t wq_gptq_workspace_bytes(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0) return 0;
  return wq_host::gptq_workspace_bytes(N, K);
}

int wq_gptq_quantize(const void* W, int w_dtype, int64_t N, int64_t K, const void* U,
                     int group_size, int sym, void* codes, void* scales, void* zeros, void* ws,
                     size_t ws_bytes, void* stream) {
  if (N < 0 || K < 0) return WQ_ERR_ARG;
  if (w_dtype != WQ_F32 && w_dtype != WQ_BF16 && w_dtype != WQ_F16) return WQ_ERR_ARG;
  if (sym != 0 && sym != 1) return WQ_ERR_ARG;
  if ((sym == 1) != (zeros == nullptr)) return WQ_ERR_ARG;
  if (group_size != 128) return WQ_ERR_UNSUPPORTED;
  if ((K % 128) != 0) return WQ_ERR_ALIGN;
  if (N > (int64_t(1) << 30) || K > (int64_t(1) << 20)) return WQ_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return WQ_OK;
  if (!W || !U || !codes || !scales) return WQ_ERR_ARG;
  if (!ws || ws_bytes < wq_host::gptq_workspace_bytes(N, K)) return WQ_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(U) || !aligned16(codes) || !aligned16(scales) ||
      (zeros && !aligned16(zeros)) || !aligned16(ws))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  return wq_host::launch_gptq(W, w_dtype, N, K, static_cast<const double*>(U), sym, codes,
                              scales, zeros, ws, as_stream(stream));
}

int wq_get_device_status(void* stream, int reset) {
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  cudaStream_t s = as_stream(stream);
  int value = 0;
  WQ_CUDA_CHECK(cudaMemcpyFromSymbolAsync(&value, g_wq_status, sizeof(int), 0,
                                          cudaMemcpyDeviceToHost, s));
  if (reset) {
    const int zero = 0;
    WQ_CUDA_CHECK(cudaMemcpyToSymbolAsync(g_wq_status, &zero, sizeof(int), 0,
                                          cudaMemcpyHostToDevice, s));
  }
  WQ_CUDA_CHECK(cudaStreamSynchronize(s));
  return value;
}

const char* wq_status_str(int status) {
  switch (status) {
    case WQ_OK: return "WQ_OK";
    case WQ_ERR_ARG: return "WQ_ERR_ARG";
    case WQ_ERR_UNSUPPORTED: return "WQ_ERR_UNSUPPORTED";
    case WQ_ERR_ALIGN: return "WQ_ERR_ALIGN";
    case WQ_ERR_CUDA: return "WQ_ERR_CUDA";
    case WQ_ERR_NONFINITE: return "WQ_ERR_NONFINITE";
    case WQ_ERR_TIMEOUT: return "WQ_ERR_TIMEOUT";
    case WQ_ERR_WORKSPACE: return "WQ_ERR_WORKSPACE";
    case WQ_ERR_NO_DEVICE: return "WQ_ERR_NO_DEVICE";
  }
  return "WQ_ERR_UNKNOWN";
}

const char* wq_last_cuda_error(void) { return wq_host::last_error_text(); }

}  // extern "C"
