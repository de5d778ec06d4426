// tc_host.cu -- host helpers of the tensor-core kernels: TMA tensor-map
// encoding (driver entry point fetched through the runtime, so the library
// needs no -lcuda) and the bounded-wait budget; plus the self-test kernel that
// exercises the bounded-wait path.
#include <stdlib.h>

#include <mutex>

#include "tc.cuh"

namespace wq_host {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  else if (g_encode_err == cudaSuccess)
    g_encode_err = cudaErrorSymbolNotFound;
}
}  // namespace

int make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                 uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                 int swizzle_bytes) {
  std::call_once(g_encode_once, load_encode);
  if (g_encode == nullptr) return cuda_fail(g_encode_err, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * uint64_t(elem_bytes)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                        : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
  return WQ_OK;
}

uint64_t wait_limit_ns() {
  static uint64_t v = [] {
    const char* e = getenv("WQ_WAIT_LIMIT_MS");
    long ms = e ? atol(e) : 0;
    return uint64_t(ms > 0 ? ms : 2000) * 1000000ull;
  }();
  return v;
}

}  // namespace wq_host

namespace wq {

// One CTA of 64 threads: warp 0 waits on a barrier that nothing will ever
// complete; warp 1 waits on the CTA's abort flag through the same helper.
// Both give up at the deadline; the kernel records WQ_ERR_TIMEOUT and returns.
__global__ void selftest_wait_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  const tc::Watchdog wd{tc::globaltimer_ns() + limit_ns, &abort_flag, status};
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = tc::wait_bounded(&bar, 0, wd);  // phase 0 never completes
  __syncwarp();
  __syncthreads();
  if (threadIdx.x == 0 && ok) record_error(status, WQ_ERR_ARG);  // must not happen
}

}  // namespace wq

extern "C" int wq_selftest_wait_timeout(int limit_us, void* stream) {
  if (limit_us <= 0 || limit_us > 1000000) return WQ_ERR_ARG;
  int st = wq_host::ensure_device();
  if (st != WQ_OK) return st;
  wq::selftest_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      uint64_t(limit_us) * 1000ull, wq_host::status_ptr());
  WQ_LAUNCH_CHECK("selftest_wait_kernel");
  return WQ_OK;
}
