// gemm_w4a16.cu -- W4A16 prefill product on the sm_100a tensor cores (M > 16).
//
//   Y[m, n] = sum_k X[m, k] * bf16(s[n, g(k)] * (u[n, k] - z[n, g(k)]))
//
// ("大模型面试准备（十九）…" sec. 2.3 W4A16: the INT4 weight is dequantized to
// the 16-bit type before the matrix product, which keeps prefill compute-bound;
// "大模型量化技术定义与主流方案解析" sec. 四: dequantization fused into the
// product, the expanded weight never written to memory.)
//
// The expanded weight element is s * (u - z) computed exactly in fp32 (11-bit
// scale times a 5-bit integer) and rounded once to bf16 -- bit for bit what
// wq_dequant(..., WQ_BF16) returns -- so the product is X * dequant_bf16(W)^T
// with fp32 accumulation.
//
// Persistent kernel, one CTA per SM, output tiles of 128 weight rows x 256
// activation rows (D[128 x 256] fp32 in TMEM, the MMA's M = weight rows, N =
// activation rows), K walked in 64-wide stages:
//   warp 0      TMA producer: codes [128 rows x 32 B] and X [256 rows x 64]
//               bf16 (128-byte swizzle) per stage into a 5-deep ring
//   warp 1      TMEM owner + MMA issuer: 4 x tcgen05.mma.kind::f16 (M=128,
//               N=256, K=16) per stage, A read from tensor memory
//   warps 4..7  epilogue warpgroup: fp32 accumulator -> bf16 Y, 32 columns
//               per tcgen05.ld; overlaps the next tile's dequantization
//   warps 8..15 two dequant warpgroups (alternate stages): thread = weight
//               row, 64 nibbles -> 32 bf16 pairs -> tcgen05.st into the
//               stage's A buffer (ring of eight).
#include <stdlib.h>

#include "kernels.h"
#include "tc.cuh"

namespace wq {
namespace gemm4 {

constexpr int BW = 128;                // weight rows per tile (MMA M)
constexpr int BX = 256;                // activation rows per tile (MMA N)
constexpr int BK = 64;                 // K per stage
constexpr int CODE_BYTES = BW * BK / 2;  // 4 KB
constexpr int X_BYTES = BX * BK * 2;     // 32 KB (128-byte rows, swizzled)
constexpr int STAGE_BYTES = CODE_BYTES + X_BYTES;
constexpr int STAGES = 5;
constexpr int NDQ = 2;
constexpr int NA = 8;                  // A buffers of 32 TMEM columns
constexpr int A_COL0 = 256;            // D at columns [0, 256)
constexpr int EPI_WARP0 = 4;
constexpr int DQ_WARP0 = 8;
constexpr int THREADS = (DQ_WARP0 + 4 * NDQ) * 32;
constexpr int TMEM_COLS = 512;
constexpr uint32_t IDESC = tc::idesc_bf16_f32(BW, BX);

struct Smem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t a_full[NA];
  uint64_t a_empty[NA];
  uint64_t d_full;
  uint64_t d_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t SMEM_BYTES = 1024 + size_t(STAGES) * STAGE_BYTES + sizeof(Smem);

struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance(int size, int by = 1) {
    slot += by;
    while (slot >= size) {
      slot -= size;
      phase ^= 1u;
    }
  }
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// (a & 0x000F000F) | 0x43004300: two nibbles -> bf16x2 (128 + u0, 128 + u1)
__device__ __forceinline__ uint32_t nib_to_bf16x2(uint32_t a) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(0x000F000Fu), "r"(0x43004300u));
  return d;
}
// two fp32 -> bf16x2, round to nearest even (lo in the low half)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tmW,
                      const __grid_constant__ CUtensorMap tmX, const __half* __restrict__ scales,
                      const __half* __restrict__ zeros, __nv_bfloat16* __restrict__ Y, int M,
                      int N, int K, int sym, int* status, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(base + size_t(STAGES) * STAGE_BYTES);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = K / 128;
  const int KB = K / BK;
  const int WT = (N + BW - 1) / BW;
  const int XT = (M + BX - 1) / BX;
  const int tiles = WT * XT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&sm.full[s], 1);
      tc::mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < NA; ++a) {
      tc::mbar_init(&sm.a_full[a], 128);
      tc::mbar_init(&sm.a_empty[a], 1);
    }
    tc::mbar_init(&sm.d_full, 1);
    tc::mbar_init(&sm.d_empty, 128);
    tc::mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch_desc(&tmW);
    tc::tma_prefetch_desc(&tmX);
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

  // tiles ordered with the activation tile fastest: CTAs running at the same
  // time share weight tiles and cover all of X, both L2-resident
  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      Ring st;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int wt = tile / XT, xt = tile - (tile / XT) * XT;
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = tc::wait_bounded(&sm.empty[st.slot], st.phase ^ 1u, wd))) break;
          uint8_t* dst = base + size_t(st.slot) * STAGE_BYTES;
          tc::mbar_arrive_expect_tx(&sm.full[st.slot], STAGE_BYTES);
          tc::tma_load_2d(dst, &tmW, &sm.full[st.slot], kb * (BK / 2), wt * BW);
          tc::tma_load_2d(dst + CODE_BYTES, &tmX, &sm.full[st.slot], kb * BK, xt * BX);
          st.advance(STAGES);
          ++issued;
        }
      }
      const uint64_t dl = tc::globaltimer_ns() + tc::kDrainNs;
      for (int k = 0; k < (issued < STAGES ? issued : STAGES); ++k) {
        const int i = issued - 1 - k;
        tc::wait_until(&sm.full[i % STAGES], uint32_t((i / STAGES) & 1), dl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dhi = tc::sdesc_k_sw128(0);
      const uint32_t x0 = tc::smem_u32(base) + CODE_BYTES;
      Ring st, ab;
      uint32_t dph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        if (!(ok = tc::wait_bounded(&sm.d_empty, dph ^ 1u, wd))) break;
        tc::fence_after_sync();
        for (int kb = 0; kb < KB; ++kb) {
          if (!(ok = tc::wait_bounded(&sm.full[st.slot], st.phase, wd) &&
                     tc::wait_bounded(&sm.a_full[ab.slot], ab.phase, wd)))
            break;
          tc::fence_after_sync();
          const uint64_t xd = dhi | uint64_t((x0 + uint32_t(st.slot) * STAGE_BYTES) >> 4);
          const uint32_t a = tmem + A_COL0 + 32 * ab.slot;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc::mma_f16_ts(tmem, a + 8 * kk, xd + uint64_t((kk * 32) >> 4), IDESC,
                           (kb | kk) != 0);
          tc::mma_commit(&sm.a_empty[ab.slot]);
          tc::mma_commit(&sm.empty[st.slot]);
          st.advance(STAGES);
          ab.advance(NA);
        }
        if (ok) tc::mma_commit(&sm.d_full);
        dph ^= 1u;
      }
      tc::mma_commit(&sm.drain);
      tc::wait_until(&sm.drain, 0, tc::globaltimer_ns() + tc::kDrainNs);
    }
  } else if (warp >= DQ_WARP0) {
    // ----------------------------------------------------------- dequant w
    const int w = (warp - DQ_WARP0) >> 2;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    Ring st, ab;
    st.advance(STAGES, w);
    ab.advance(NA, w);
    bool ok = true;
    int gi = 0;  // global index of the tile's first stage; ours: index % NDQ == w
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
      const int wt = tile / XT;
      const int n = wt * BW + row;
      const bool row_in = n < N;
      const __half* srow = scales + size_t(row_in ? n : 0) * G;
      const __half* zrow = sym ? nullptr : zeros + size_t(row_in ? n : 0) * G;
      // this warpgroup's first stage of the tile and its group's scale / zero;
      // each iteration fetches the next stage's pair before working, so the
      // loads have a whole stage of work to land
      int kb = (w - gi % NDQ + NDQ) % NDQ;
      float s_nx = 0.f, z_nx = 8.f;
      if (kb < KB && row_in) {
        s_nx = __half2float(srow[kb >> 1]);
        if (!sym) z_nx = __half2float(zrow[kb >> 1]);
      }
      for (; kb < KB; kb += NDQ) {
        const float s = s_nx, zf = sym ? 8.f : z_nx;
        if (kb + NDQ < KB && row_in) {
          const int gn = (kb + NDQ) >> 1;  // two stages per 128-wide group
          s_nx = __half2float(srow[gn]);
          if (!sym) z_nx = __half2float(zrow[gn]);
        }
        if (!(ok = tc::wait_bounded(&sm.full[st.slot], st.phase, wd) &&
                   tc::wait_bounded(&sm.a_empty[ab.slot], ab.phase ^ 1u, wd)))
          break;
        tc::fence_after_sync();
        // x_hat = (128 + u) * s - (128 + z) * s: both products exact in fp32,
        // so the fma returns s * (u - z) exactly; one rounding to bf16 after
        const float c = -(128.f + zf) * s;
        const uint8_t* rowp = base + size_t(st.slot) * STAGE_BYTES + row * (BK / 2);
        const uint4 v0 = *reinterpret_cast<const uint4*>(rowp);
        const uint4 v1 = *reinterpret_cast<const uint4*>(rowp + 16);
        const uint32_t words[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t out[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t wd0 = words[k];
          const uint32_t w4 = wd0 >> 4;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t t = nib_to_bf16x2(prmt(wd0, w4, uint32_t(e) | (uint32_t(4 + e) << 8)));
            const float lo = fmaf(__uint_as_float(t << 16), s, c);
            const float hi = fmaf(__uint_as_float(t & 0xFFFF0000u), s, c);
            out[4 * k + e] = pack_bf16x2(lo, hi);
          }
        }
        tc::tmem_st_x32(tmem + lane_off + A_COL0 + 32 * ab.slot, out);
        tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::mbar_arrive(&sm.a_full[ab.slot]);
        st.advance(STAGES, NDQ);
        ab.advance(NA, NDQ);
      }
      gi += KB;
    }
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    uint32_t dph = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
      const int wt = tile / XT, xt = tile - (tile / XT) * XT;
      if (!tc::wait_bounded(&sm.d_full, dph, wd)) break;
      tc::fence_after_sync();
      const int n = wt * BW + row;
#pragma unroll 1
      for (int c = 0; c < BX / 32; ++c) {
        uint32_t r[32];
        tc::tmem_ld_x32(tmem + lane_off + 32 * c, r);
        tc::tmem_wait_ld();
        if (n < N) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = xt * BX + 32 * c + j;
            if (m < M) Y[size_t(m) * N + n] = __float2bfloat16_rn(__uint_as_float(r[j]));
          }
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.d_empty);
      dph ^= 1u;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace gemm4
}  // namespace wq

namespace wq_host {

int launch_gemm_w4a16(const void* X, int64_t M, int64_t K, const void* codes,
                      const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                      cudaStream_t s) {
  using namespace wq::gemm4;
  CUtensorMap tw, tx;
  int st = make_tmap_2d(&tw, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(N),
                        uint64_t(K / 2), BW, BK / 2, 0);
  if (st != WQ_OK) return st;
  st = make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(M), uint64_t(K), BX,
                    BK, 128);
  if (st != WQ_OK) return st;
  static bool attr_done[64] = {};
  int dev = 0;
  WQ_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 64 && !attr_done[dev]) {
    WQ_CUDA_CHECK(cudaFuncSetAttribute(gemm_w4a16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(SMEM_BYTES)));
    attr_done[dev] = true;
  }
  const int64_t tiles = ((N + BW - 1) / BW) * ((M + BX - 1) / BX);
  const int grid = int(tiles < sm_count() ? tiles : sm_count());
  gemm_w4a16_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(
      tw, tx, static_cast<const __half*>(scales), static_cast<const __half*>(zeros),
      static_cast<__nv_bfloat16*>(Y), int(M), int(N), int(K), sym, status_ptr(), wait_limit_ns());
  WQ_LAUNCH_CHECK("gemm_w4a16_kernel");
  return WQ_OK;
}

}  // namespace wq_host
