// gemv_simt.cu -- W4A16 decode product on the CUDA cores (M <= 16).
//
// Y[m, n] = sum_g s[n, g] * sum_{k in g} X[m, k] * (u[n, k] - z_eff[n, g])
// ("大模型面试准备（十九）…" sec. 2.3 W4A16; the weight is expanded in registers,
// "大模型量化技术定义与主流方案解析" sec. 四).
//
// Each warp owns ROWS consecutive weight rows and walks K in 1024-element
// chunks: lane l reads 16 bytes of codes per row (32 elements, one quarter of a
// 128-group), converts them to exact small integers u - z in fp32, takes the
// fp32 dot product with X and scales it by the group's fp16 scale.  The lanes'
// partial sums are reduced with shuffles at the end.  Each weight byte is
// read once from HBM with a streaming 16-byte load; X (a few KB per row) stays
// in L1/L2.
#include "common.cuh"
#include "kernels.h"

namespace wq {

template <int MT, int ROWS>
__global__ void __launch_bounds__(256) gemv_w4a16_simt_kernel(
    const __nv_bfloat16* __restrict__ X, int M, int64_t K, const uint8_t* __restrict__ codes,
    const __half* __restrict__ scales, const __half* __restrict__ zeros, int64_t N, int sym,
    __nv_bfloat16* __restrict__ Y) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t n0 = warp * ROWS;
  if (n0 >= N) return;
  const int64_t G = K / 128;
  float acc[ROWS][MT];
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;

  for (int64_t k0 = int64_t(lane) * 32; k0 < K; k0 += 1024) {
    uint4 w[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      if (n0 + r < N)
        w[r] = __ldcs(reinterpret_cast<const uint4*>(codes + (n0 + r) * (K / 2) + k0 / 2));
    const int64_t g = k0 >> 7;
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      if (n0 + r >= N) break;
      const float s = __half2float(scales[(n0 + r) * G + g]);
      const float zf = sym ? 8.f : __half2float(zeros[(n0 + r) * G + g]);
      const uint32_t words[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
      float d[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) d[i] = float((words[i >> 3] >> (4 * (i & 7))) & 0xFu) - zf;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m >= M) break;
        const uint4* xp = reinterpret_cast<const uint4*>(X + int64_t(m) * K + k0);
        float inner = 0.f;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          union {
            uint4 u;
            __nv_bfloat162 h[4];
          } xv;
          xv.u = __ldg(xp + v);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(xv.h[j]);
            inner = fmaf(f.x, d[8 * v + 2 * j], inner);
            inner = fmaf(f.y, d[8 * v + 2 * j + 1], inner);
          }
        }
        acc[r][m] = fmaf(s, inner, acc[r][m]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float v = warp_sum(acc[r][m]);
      if (lane == 0 && m < M && n0 + r < N) Y[int64_t(m) * N + n0 + r] = __float2bfloat16_rn(v);
    }
}

}  // namespace wq

namespace wq_host {

template <int MT, int ROWS>
static void gemv_launch(const void* X, int64_t M, int64_t K, const void* codes,
                        const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                        cudaStream_t s) {
  const int64_t warps = (N + ROWS - 1) / ROWS;
  const int64_t blocks = (warps + 7) / 8;
  wq::gemv_w4a16_simt_kernel<MT, ROWS><<<unsigned(blocks), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(X), int(M), K, static_cast<const uint8_t*>(codes),
      static_cast<const __half*>(scales), static_cast<const __half*>(zeros), N, sym,
      static_cast<__nv_bfloat16*>(Y));
}

int launch_gemv_w4a16(const void* X, int64_t M, int64_t K, const void* codes,
                      const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                      cudaStream_t s) {
  if (M == 1)
    gemv_launch<1, 4>(X, M, K, codes, scales, zeros, N, sym, Y, s);
  else if (M <= 4)
    gemv_launch<4, 1>(X, M, K, codes, scales, zeros, N, sym, Y, s);
  else if (M <= 8)
    gemv_launch<8, 1>(X, M, K, codes, scales, zeros, N, sym, Y, s);
  else
    gemv_launch<16, 1>(X, M, K, codes, scales, zeros, N, sym, Y, s);
  WQ_LAUNCH_CHECK("gemv_w4a16_simt_kernel");
  return WQ_OK;
}

}  // namespace wq_host
