// gemm_w8a8.cu -- W8A8 product on the int8 tensor cores of sm_100a
// ("大模型面试准备（十九）…" sec. 2.3 W8A8 and sec. 4.2: int8 weights and
// activations on the INT8 tensor core, int32 accumulation, floating rescale).
//
//   acc[m, n] = sum_k qx[m, k] * qw[n, k]            (int32, exact)
//   Y[m, n]   = bf16(float(acc) * sx[m] * sw[n])      (per-token x per-channel)
//
// Persistent kernel, one 192-thread CTA per SM, 128 x 256 output tiles:
//   warp 0      TMA producer: qx tile [128 x 128 B] and qw tile [256 x 128 B]
//               per k-block into a 4-stage ring (128-byte swizzle)
//   warp 1      TMEM owner + MMA issuer: 4 x tcgen05.mma.kind::i8 (M=128,
//               N=256, K=32) per stage into one of two TMEM accumulators
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, rescale, store;
//               overlaps the next tile's mainloop (double-buffered TMEM)
#include "kernels.h"
#include "tc.cuh"

namespace wq {
namespace w8a8 {

constexpr int BM = 128, BN = 256, BK = 128;  // BK in bytes = int8 elements
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;  // 16 KB
constexpr int B_BYTES = BN * BK;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;  // two 128 x 256 int32 accumulators
constexpr int THREADS = 192;
constexpr uint32_t IDESC = tc::idesc_s8_s32(BM, BN);
constexpr uint32_t IDESC_FP8 = tc::idesc_e4m3_f32(BM, BN);

struct Smem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + size_t(STAGES) * STAGE_BYTES + sizeof(Smem);

// FP8 = false: int8 operands, tcgen05.mma kind::i8, int32 accumulators;
// FP8 = true: E4M3 operands, kind::f8f6f4, fp32 accumulators (same tiles,
// same 32-element K steps, same epilogue up to the accumulator type).
template <bool FP8>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const float* __restrict__ sx, const float* __restrict__ sw,
                     __nv_bfloat16* __restrict__ Y, uint32_t* __restrict__ acc_out, int M, int N,
                     int K, int* status, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* tiles = base;  // stage s: A at s*STAGE_BYTES, B right after
  Smem& sm = *reinterpret_cast<Smem*>(base + size_t(STAGES) * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mtiles = (M + BM - 1) / BM;
  const int ntiles = (N + BN - 1) / BN;
  const int total = mtiles * ntiles;
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&sm.full[s], 1);
      tc::mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&sm.tfull[b], 1);
      tc::mbar_init(&sm.tempty[b], 128);
    }
    tc::mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tc::tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem_base;
  const tc::Watchdog wd{tc::globaltimer_ns() + limit_ns, &sm.abort_flag, status};

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const int mt = tile % mtiles, nt = tile / mtiles;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!(ok = tc::wait_bounded(&sm.empty[s], ph ^ 1u, wd))) break;
          uint8_t* a = tiles + size_t(s) * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          tc::mbar_arrive_expect_tx(&sm.full[s], STAGE_BYTES);
          tc::tma_load_2d(a, &tmA, &sm.full[s], kb * BK, mt * BM);
          tc::tma_load_2d(b, &tmB, &sm.full[s], kb * BK, nt * BN);
        }
      }
      // drain: the last load issued into each stage has landed before exit
      const uint64_t dl = tc::globaltimer_ns() + tc::kDrainNs;
      const uint32_t n = it < uint32_t(STAGES) ? it : uint32_t(STAGES);
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        tc::wait_until(&sm.full[i % STAGES], (i / STAGES) & 1u, dl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1u;
        if (!(ok = tc::wait_bounded(&sm.tempty[buf], ((tcount >> 1) & 1u) ^ 1u, wd))) break;
        tc::fence_after_sync();
        const uint32_t d = tmem + buf * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          if (!(ok = tc::wait_bounded(&sm.full[s], (it / STAGES) & 1u, wd))) break;
          tc::fence_after_sync();
          const uint32_t a = tc::smem_u32(tiles + size_t(s) * STAGE_BYTES);
          const uint32_t b = a + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            if (FP8)
              tc::mma_f8_ss(d, tc::sdesc_k_sw128(a + k * 32), tc::sdesc_k_sw128(b + k * 32),
                            IDESC_FP8, (kb | k) != 0);
            else
              tc::mma_i8_ss(d, tc::sdesc_k_sw128(a + k * 32), tc::sdesc_k_sw128(b + k * 32),
                            IDESC, (kb | k) != 0);
          }
          tc::mma_commit(&sm.empty[s]);
        }
        if (ok) tc::mma_commit(&sm.tfull[buf]);
      }
      // drain: every MMA this thread issued has completed
      tc::mma_commit(&sm.drain);
      tc::wait_until(&sm.drain, 0, tc::globaltimer_ns() + tc::kDrainNs);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
      const int mt = tile % mtiles, nt = tile / mtiles;
      const uint32_t buf = tcount & 1u;
      if (!tc::wait_bounded(&sm.tfull[buf], (tcount >> 1) & 1u, wd)) break;
      tc::fence_after_sync();
      const int row = mt * BM + q * 32 + lane;
      const float srow = row < M ? sx[row] : 0.f;
      const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + buf * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tc::tmem_ld_x32(taddr + c * 32, r);
        tc::tmem_wait_ld();
        const int n0 = nt * BN + c * 32;
        if (row < M) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {  // 8 columns = one 16-byte store
            const int n = n0 + g * 8;
            if (n >= N) break;
            union {
              uint4 v;
              __nv_bfloat162 h[4];
            } o;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t a0 = r[g * 8 + 2 * j], a1 = r[g * 8 + 2 * j + 1];
              const float f0 = FP8 ? __uint_as_float(a0) : float(int32_t(a0));
              const float f1 = FP8 ? __uint_as_float(a1) : float(int32_t(a1));
              const float v0 = f0 * srow * __ldg(sw + n + 2 * j);
              const float v1 = f1 * srow * __ldg(sw + n + 2 * j + 1);
              o.h[j] = __floats2bfloat162_rn(v0, v1);
            }
            *reinterpret_cast<uint4*>(Y + size_t(row) * N + n) = o.v;
            if (acc_out != nullptr) {
              uint32_t* dst = acc_out + size_t(row) * N + n;
              reinterpret_cast<uint4*>(dst)[0] =
                  make_uint4(r[g * 8 + 0], r[g * 8 + 1], r[g * 8 + 2], r[g * 8 + 3]);
              reinterpret_cast<uint4*>(dst)[1] =
                  make_uint4(r[g * 8 + 4], r[g * 8 + 5], r[g * 8 + 6], r[g * 8 + 7]);
            }
          }
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.tempty[buf]);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace w8a8
}  // namespace wq

namespace wq_host {

static int launch_gemm_8bit(bool fp8, const void* qx, const float* sx, int64_t M, int64_t K,
                            const void* Wq, const void* w_scales, int64_t N, void* Y,
                            void* acc_out, cudaStream_t s) {
  using namespace wq::w8a8;
  CUtensorMap ta, tb;
  int st = make_tmap_2d(&ta, qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(M), uint64_t(K), BM, BK,
                        128);
  if (st != WQ_OK) return st;
  st = make_tmap_2d(&tb, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(N), uint64_t(K), BN, BK,
                    128);
  if (st != WQ_OK) return st;

  static bool attr_done[2][64] = {};
  int dev = 0;
  WQ_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 64 && !attr_done[fp8][dev]) {
    if (fp8)
      WQ_CUDA_CHECK(cudaFuncSetAttribute(gemm_w8a8_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(SMEM_BYTES)));
    else
      WQ_CUDA_CHECK(cudaFuncSetAttribute(gemm_w8a8_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(SMEM_BYTES)));
    attr_done[fp8][dev] = true;
  }
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = int(tiles < sm_count() ? tiles : sm_count());
  auto* y = static_cast<__nv_bfloat16*>(Y);
  auto* acc = static_cast<uint32_t*>(acc_out);
  auto* sw = static_cast<const float*>(w_scales);
  if (fp8)
    gemm_w8a8_kernel<true><<<grid, THREADS, SMEM_BYTES, s>>>(ta, tb, sx, sw, y, acc, int(M),
                                                             int(N), int(K), status_ptr(),
                                                             wait_limit_ns());
  else
    gemm_w8a8_kernel<false><<<grid, THREADS, SMEM_BYTES, s>>>(ta, tb, sx, sw, y, acc, int(M),
                                                              int(N), int(K), status_ptr(),
                                                              wait_limit_ns());
  WQ_LAUNCH_CHECK("gemm_w8a8_kernel");
  return WQ_OK;
}

int launch_gemm_w8a8(const void* X, int64_t M, int64_t K, const void* Wq, const void* w_scales,
                     const float* smooth, int64_t N, void* Y, void* ws, void* acc_out,
                     cudaStream_t s) {
  int8_t* qx = static_cast<int8_t*>(ws);
  float* sx = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                       ((size_t(M) * size_t(K) + 255) & ~size_t(255)));
  int st = launch_quantize_rows_i8(X, WQ_BF16, M, K, true, smooth, qx, sx, s);
  if (st != WQ_OK) return st;
  return launch_gemm_8bit(false, qx, sx, M, K, Wq, w_scales, N, Y, acc_out, s);
}

int launch_gemm_fp8(const void* X, int64_t M, int64_t K, const void* Wq, const void* w_scales,
                    int64_t N, void* Y, void* ws, void* acc_out, cudaStream_t s) {
  uint8_t* qx = static_cast<uint8_t*>(ws);
  float* sx = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                       ((size_t(M) * size_t(K) + 255) & ~size_t(255)));
  int st = launch_quantize_rows_fp8(X, WQ_BF16, M, K, qx, sx, s);
  if (st != WQ_OK) return st;
  return launch_gemm_8bit(true, qx, sx, M, K, Wq, w_scales, N, Y, acc_out, s);
}

}  // namespace wq_host
