// gemv_w4a16.cu -- dispatch of the W4A16 decode product (M <= 16) and its
// entry point without allocation.
//
// Two kernels compute the decode product ("大模型面试准备（十九）…" sec. 1.2 and
// 2.3: decode is bound by HBM bandwidth and stays W4A16):
//   * gemv_w4a16_cc.cu -- CUDA cores, M = 1 .. 4: the multiply-adds of a few
//     activation rows fit the issue budget of a stream (at M = 3, 4 with less
//     margin, still ahead of the tensor-core kernel on every measured shape);
//   * gemv_w4a16_tc.cu -- tensor cores (tcgen05), M = 5 .. 16: M multiply-adds
//     per weight element no longer fit, so they go to the MMA units.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace wq_host {

// One workspace size for every M <= 16 (the CUDA-core kernel needs none), so
// a caller's workspace serves both decode kernels.
size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)M;
  return gemv_workspace_bytes(N, K);
}

bool decode_on_cuda_cores(int64_t M, int64_t N, int64_t K) {
  return M <= kGemvCcMaxM && gemv_cc_fits(M, N, K);
}

int prepare_decode_kernels() {
  const int st = prepare_cc_kernels();
  return st != WQ_OK ? st : prepare_tc_kernels();
}

int launch_decode_w4a16(const void* X, int64_t M, int64_t K, const void* codes,
                        const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                        void* ws, cudaStream_t s) {
  if (decode_on_cuda_cores(M, N, K))
    return launch_gemv_w4a16_cc(X, M, K, codes, scales, zeros, N, sym, Y, s);
  return launch_gemv_w4a16_tc(X, M, K, codes, scales, zeros, N, sym, Y, ws, s);
}

}  // namespace wq_host

// ---------------------------------------------------------------------------
// Decode product without any allocation
// ---------------------------------------------------------------------------
// wq_gemm_w4a16 asks its caller for a workspace (the tensor-core kernel's
// per-tile arrival counters and per-CTA partial sums of the tiles it splits
// between CTAs).  Some callers cannot provide one: a serving loop whose device
// memory is all owned by another allocator under a fixed budget, a plain C
// host with no device allocator of its own, or a latency-critical path where
// a cudaMalloc (which may synchronize the device) is not acceptable.
// wq_gemm_w4a16_noalloc runs the same kernels on scratch that lives in this
// library's own device image: a file-scope array that every GPU which loads
// the library holds until the process exits.
namespace {
constexpr int64_t kNoAllocMaxN = 131072;                              // 1024 row tiles of 128
constexpr int64_t kNoAllocMaxCtas = 256;                              // one CTA per SM
constexpr size_t kNoAllocCntBytes = size_t(kNoAllocMaxN / 128) * 4;   // 4 KiB
constexpr size_t kNoAllocPartBytes = size_t(kNoAllocMaxCtas) * 2 * 128 * 16 * 4;  // 4 MiB
constexpr size_t kNoAllocBytes = kNoAllocCntBytes + kNoAllocPartBytes;
}  // namespace

// The scratch itself.  Its name, used in host code, is only a host-side
// stand-in for the symbol: the device address comes from
// cudaGetSymbolAddress, taken once per device with that device current.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocBytes];

namespace {
void* g_noalloc_ptr[64] = {};
std::mutex g_noalloc_mu;
}  // namespace

extern "C" int wq_gemm_w4a16_noalloc(const void* X, int64_t M, int64_t K, const void* codes,
                                     const void* scales, const void* zeros, int64_t N,
                                     int group_size, int sym, void* Y, void* stream) {
  if (M < 0 || K < 0 || N < 0) return WQ_ERR_ARG;
  if (sym != 0 && sym != 1) return WQ_ERR_ARG;
  if ((sym == 1) != (zeros == nullptr)) return WQ_ERR_ARG;
  if (group_size != 128) return WQ_ERR_UNSUPPORTED;
  if ((K % 128) != 0 || (N % 8) != 0) return WQ_ERR_ALIGN;
  if (M > 16 || N > kNoAllocMaxN || K > (int64_t(1) << 24)) return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (K == 0) return WQ_ERR_ARG;
  if (!X || !codes || !scales || !Y) return WQ_ERR_ARG;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(X) || !a16(codes) || !a16(scales) || !a16(Y) || (zeros && !a16(zeros)))
    return WQ_ERR_ALIGN;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  int dev = 0;
  WQ_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev >= 64) return WQ_ERR_UNSUPPORTED;
  // the scratch must hold every tile's counter and every CTA's partials
  if (int64_t(wq_host::sm_count()) > kNoAllocMaxCtas ||
      wq_host::decode_workspace_bytes(M, N, K) > kNoAllocBytes)
    return WQ_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  {
    // set-up on the first call for this device (this device is current):
    // the array's device address and the decode kernels' launch attributes
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      st = wq_host::prepare_decode_kernels();
      if (st != WQ_OK) return st;
      void* p = nullptr;
      WQ_CUDA_CHECK(cudaGetSymbolAddress(&p, g_decode_scratch));
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (wq_host::decode_on_cuda_cores(M, N, K))  // no scratch at all
    return wq_host::launch_gemv_w4a16_cc(X, M, K, codes, scales, zeros, N, sym, Y, s);
  // the arrival counters must start at zero: clear them on the call's stream
  const size_t cnt = (size_t((N + 127) / 128) * 4 + 255) & ~size_t(255);
  WQ_CUDA_CHECK(cudaMemsetAsync(scratch, 0, cnt, s));
  return wq_host::launch_gemv_w4a16_tc(X, M, K, codes, scales, zeros, N, sym, Y, scratch, s);
}
