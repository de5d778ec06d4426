// gemm_w8a16.cu -- W8A16 product: 8-bit per-output-channel weights (int8 or
// FP8 E4M3 codes, one fp32 scale per weight row) with bf16 activations.
//
//   Y[m, n] = s[n] * sum_k X[m, k] * value(q[n, k])
//
// ("27届大模型面试准备（十九）…" sec. 2.3 naming table: W8A16 keeps the
// activations in 16 bits and quantizes only the weights to 8 bits, so the
// weight is expanded to the activation type inside the product; sec. 2.2:
// 8-bit weights take one scale per output channel.)
//
// Every code value is exact in bf16 (int8: at most 8 significant bits; E4M3:
// 4 significant bits, exponents 2^-9 .. 2^8), so the expanded weight needs no
// rounding: the products are X * value(q) accumulated in fp32, and the row
// scale multiplies the fp32 sum once, in the epilogue.
//
// Two kernels:
//  * gemv_w8a16_kernel (M <= 4): CUDA cores.  A warp takes one weight row at
//    a time, each lane 16 consecutive codes per 16-byte load, eight loads of
//    the row in flight per lane; codes expand to fp32 in registers, X comes
//    through L1 (it is shared by every row), and a warp shuffle ends the row.
//  * gemm_w8a16_kernel (M > 4): tensor cores, the warp-specialised layout of
//    the W4A16 GEMM: TMA producer (codes [128 rows x 64 B] and X [256 x 64]
//    bf16 per stage), one MMA issuer (tcgen05.mma.kind::f16, A = expanded
//    weight in TMEM, B = X in shared memory), two expansion warpgroups
//    (thread = weight row: 64 codes -> 32 bf16 pairs -> tcgen05.st) and an
//    epilogue warpgroup (fp32 accumulator x row scale -> bf16 Y).
#include <stdlib.h>

#include <algorithm>

#include "kernels.h"
#include "tc.cuh"

namespace wq {
namespace w8a16 {

// ------------------------------------------------------------ code values
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Four int8 codes of a word -> fp32, exactly: byte b + 128 (the word xor
// 0x80808080) becomes the low mantissa byte of 2^23, and subtracting
// 2^23 + 128 leaves b.
__device__ __forceinline__ void i8x4_to_f32(uint32_t w, float (&f)[4]) {
  const uint32_t wo = w ^ 0x80808080u;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    f[e] = __uint_as_float(prmt(wo, 0x4B000000u, 0x7540u | uint32_t(e))) - 8388736.0f;
}

// Four E4M3 codes of a word -> fp32, exactly (through the hardware
// E4M3 -> f16 pair conversion; every E4M3 value is a normal fp16 or zero).
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float (&f)[4]) {
  uint32_t h01, h23;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
      : "=r"(h01), "=r"(h23)
      : "r"(w));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h01));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h23));
  f[0] = a.x;
  f[1] = a.y;
  f[2] = b.x;
  f[3] = b.y;
}

template <int FMT>
__device__ __forceinline__ void codes_to_f32(uint32_t w, float (&f)[4]) {
  if constexpr (FMT == WQ_W8_E4M3)
    e4m3x4_to_f32(w, f);
  else
    i8x4_to_f32(w, f);
}

// two fp32 values with at most 8 significant bits -> bf16x2 (their high
// halves, which is exact), lo in the low half
__device__ __forceinline__ uint32_t hi_halves(float lo, float hi) {
  return prmt(__float_as_uint(lo), __float_as_uint(hi), 0x7632u);
}

// ------------------------------------------------------------- decode GEMV
template <int FMT, int MT>
__global__ void __launch_bounds__(256) gemv_w8a16_kernel(const __nv_bfloat16* __restrict__ X,
                                                         int M, int K,
                                                         const uint8_t* __restrict__ Wq,
                                                         const float* __restrict__ sw, int N,
                                                         __nv_bfloat16* __restrict__ Y) {
  constexpr int U = 8;  // 16-byte loads per lane in flight
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int nseg = K / 16;  // 16-code segments per row
  for (int64_t n = warp; n < N; n += nwarps) {
    const uint4* wrow = reinterpret_cast<const uint4*>(Wq + n * K);
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    for (int s0 = 0; s0 < nseg; s0 += 32 * U) {
      uint4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int seg = s0 + u * 32 + lane;
        w[u] = seg < nseg ? __ldcs(wrow + seg) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int seg = s0 + u * 32 + lane;
        if (seg < nseg) {
          const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
          float v[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float f[4];
            codes_to_f32<FMT>(ws[i], f);
#pragma unroll
            for (int e = 0; e < 4; ++e) v[4 * i + e] = f[e];
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m < M) {
              const uint4* xp = reinterpret_cast<const uint4*>(X + size_t(m) * K) + 2 * seg;
              const uint4 xa = __ldg(xp), xb = __ldg(xp + 1);
              const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                acc[m] = fmaf(__uint_as_float(xw[i] << 16), v[2 * i], acc[m]);
                acc[m] = fmaf(__uint_as_float(xw[i] & 0xFFFF0000u), v[2 * i + 1], acc[m]);
              }
            }
          }
        }
      }
    }
    const float s = sw[n];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float t = acc[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0 && m < M) Y[size_t(m) * N + n] = __float2bfloat16_rn(s * t);
    }
  }
}

// ------------------------------------------------ int8 decode on DP2A
// int8 codes times X in 16-bit fixed point: for each activation row and
// 128-element group of K, x' = rint(x 2^e) with e chosen so that the group's
// largest |x| maps into [2^12, 2^13).  bf16 values down to 2^-5 of that
// maximum are exact integers then; smaller ones move by at most 2^-13 of it.
// A lane's 16 codes times x' is an exact integer below 2^24 (eight DP2A),
// scaled by 2^-e into an fp32 accumulator.  A warp owns RB weight rows and
// walks K in 512-wide chunks (16 codes per lane and row, one 16-byte load),
// converting X once per chunk for all RB rows; the next chunk's codes are
// loaded before the current one is multiplied.  A chunk whose X holds a NaN
// or an infinity is multiplied in fp32 instead (the exact-code expansion).
__device__ __forceinline__ int dp2a_lo_ss(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi_ss(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// One activation row's chunk of X for this lane (16 elements at k0), in
// fixed point: xq[j] holds x'(2j) | x'(2j + 1) << 16, inv = 2^-e.  Returns
// false (warp-uniformly) when the chunk holds a non-finite value.
__device__ __forceinline__ bool x_fixed_chunk(const uint4 xa, const uint4 xb, uint32_t (&xq)[8],
                                              float& inv, float (&xf)[16]) {
  const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
  uint32_t m2 = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(xw[0], xw[1]), bf16x2_absmax(xw[2], xw[3])),
                              bf16x2_absmax(bf16x2_absmax(xw[4], xw[5]), bf16x2_absmax(xw[6], xw[7])));
  float amax = fmaxf(fabsf(__uint_as_float(m2 << 16)), fabsf(__uint_as_float(m2 & 0xFFFF0000u)));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    xf[2 * j] = __uint_as_float(xw[j] << 16);
    xf[2 * j + 1] = __uint_as_float(xw[j] & 0xFFFF0000u);
  }
  bool finite = true;
#pragma unroll
  for (int e = 0; e < 16; ++e) finite &= fabsf(xf[e]) <= 3.402823466e38f;
  if (!__all_sync(0xffffffffu, finite)) return false;
  // e = 12 - floor(log2 amax) (amax >= 2^-133 for a nonzero bf16); 2^e is
  // applied as two exact power-of-two factors, 2^-e built from its bits
  const int E = amax > 0.f ? int((__float_as_uint(amax) >> 23) & 0xFFu) - 127 : 0;
  const int ee = amax > 0.f ? (E < -126 ? 130 + __clz(int(__float_as_uint(amax) & 0x7FFFFFu)) : 12 - E) : 0;
  const int e1 = ee / 2, e2 = ee - e1;
  const float s1 = __uint_as_float(uint32_t(127 + e1) << 23);
  const float s2 = __uint_as_float(uint32_t(127 + e2) << 23);
  inv = ee <= 126 ? __uint_as_float(uint32_t(127 - ee) << 23) : __uint_as_float(1u << (149 - ee));
  const float magic = 12582912.f;  // 1.5 * 2^23
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float ta = fmaf(xf[2 * j] * s1, s2, magic);
    const float tb = fmaf(xf[2 * j + 1] * s1, s2, magic);
    xq[j] = prmt(__float_as_uint(ta), __float_as_uint(tb), 0x5410u);
  }
  return true;
}

template <int MT, int RB>
__global__ void __launch_bounds__(256, 2) gemv_w8a16_dp_kernel(const __nv_bfloat16* __restrict__ X,
                                                               int M, int K,
                                                               const uint8_t* __restrict__ Wq,
                                                               const float* __restrict__ sw, int N,
                                                               __nv_bfloat16* __restrict__ Y) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int nchunk = (K + 511) / 512;
  const int64_t nblocks = (int64_t(N) + RB - 1) / RB;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (gw >= nblocks) asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int64_t rb = gw; rb < nblocks; rb += nw) {  // warp-uniform
    const int64_t r0 = rb * RB;
    float acc[RB][MT];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;
    auto load = [&](uint4 (&dst)[RB], int c) {
      const int k0 = c * 512 + lane * 16;
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const int64_t n = r0 + r;
        dst[r] = (k0 < K && n < N)
                     ? __ldcs(reinterpret_cast<const uint4*>(Wq + n * int64_t(K) + k0))
                     : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto multiply = [&](const uint4 (&cw)[RB], int c) {
      const int k0 = c * 512 + lane * 16;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m >= M) break;  // uniform
        uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = xa;
        if (k0 < K) {
          const uint4* xp = reinterpret_cast<const uint4*>(X + size_t(m) * K + k0);
          xa = __ldg(xp);
          xb = __ldg(xp + 1);
        }
        uint32_t xq[8];
        float inv, xf[16];
        if (x_fixed_chunk(xa, xb, xq, inv, xf)) {
#pragma unroll
          for (int r = 0; r < RB; ++r) {
            const uint32_t w4[4] = {cw[r].x, cw[r].y, cw[r].z, cw[r].w};
            int isum = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              isum = dp2a_lo_ss(xq[2 * j], w4[j], isum);
              isum = dp2a_hi_ss(xq[2 * j + 1], w4[j], isum);
            }
            acc[r][m] = fmaf(float(isum), inv, acc[r][m]);
          }
        } else {  // non-finite X in this chunk: fp32 products of the exact codes
#pragma unroll
          for (int r = 0; r < RB; ++r) {
            const uint32_t w4[4] = {cw[r].x, cw[r].y, cw[r].z, cw[r].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float f[4];
              i8x4_to_f32(w4[j], f);
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[r][m] = fmaf(xf[4 * j + e], f[e], acc[r][m]);
            }
          }
        }
      }
    };
    uint4 ca[RB], cb[RB];
    load(ca, 0);
    if (rb == gw) asm volatile("griddepcontrol.wait;" ::: "memory");  // X, Y after this
    for (int c = 0; c < nchunk; c += 2) {  // ca holds chunk c, cb chunk c + 1
      if (c + 1 < nchunk) load(cb, c + 1);
      multiply(ca, c);
      if (c + 1 >= nchunk) break;
      if (c + 2 < nchunk) load(ca, c + 2);
      multiply(cb, c + 1);
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int64_t n = r0 + r;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float t = acc[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (lane == 0 && m < M && n < N) Y[size_t(m) * N + n] = __float2bfloat16_rn(sw[n] * t);
      }
    }
  }
}

// ------------------------------------------------------ tensor-core GEMM
constexpr int BW = 128;                 // weight rows per tile (MMA M)
constexpr int BX = 256;                 // activation rows per tile (MMA N)
constexpr int BK = 64;                  // K per stage
constexpr int CODE_BYTES = BW * BK;     // 8 KB
constexpr int X_BYTES = BX * BK * 2;    // 32 KB (128-byte rows, swizzled)
constexpr int STAGE_BYTES = CODE_BYTES + X_BYTES;
constexpr int STAGES = 5;
constexpr int NDQ = 2;
constexpr int NA = 8;                   // A buffers of 32 TMEM columns
constexpr int A_COL0 = 256;             // D at columns [0, 256)
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

template <int FMT>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_w8a16_kernel(const __grid_constant__ CUtensorMap tmW,
                      const __grid_constant__ CUtensorMap tmX, const float* __restrict__ sw,
                      __nv_bfloat16* __restrict__ Y, int M, int N, int K, int* status,
                      uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(base + size_t(STAGES) * STAGE_BYTES);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
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

  // tiles ordered with the activation tile fastest (weight tiles shared by
  // the CTAs running at the same time stay in L2)
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
          tc::tma_load_2d(dst, &tmW, &sm.full[st.slot], kb * BK, wt * BW);
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
    // ------------------------------------------------ weight expansion w
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
      for (int kb = (w - gi % NDQ + NDQ) % NDQ; kb < KB; kb += NDQ) {
        if (!(ok = tc::wait_bounded(&sm.full[st.slot], st.phase, wd) &&
                   tc::wait_bounded(&sm.a_empty[ab.slot], ab.phase ^ 1u, wd)))
          break;
        tc::fence_after_sync();
        const uint4* rowp =
            reinterpret_cast<const uint4*>(base + size_t(st.slot) * STAGE_BYTES + row * BK);
        uint32_t out[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v = rowp[c];
          const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float f[4];
            codes_to_f32<FMT>(ws[i], f);
            out[8 * c + 2 * i] = hi_halves(f[0], f[1]);
            out[8 * c + 2 * i + 1] = hi_halves(f[2], f[3]);
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
      const int n = wt * BW + row;
      const float s = n < N ? sw[n] : 0.f;
      if (!tc::wait_bounded(&sm.d_full, dph, wd)) break;
      tc::fence_after_sync();
#pragma unroll 1
      for (int c = 0; c < BX / 32; ++c) {
        uint32_t r[32];
        tc::tmem_ld_x32(tmem + lane_off + 32 * c, r);
        tc::tmem_wait_ld();
        if (n < N) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = xt * BX + 32 * c + j;
            if (m < M) Y[size_t(m) * N + n] = __float2bfloat16_rn(s * __uint_as_float(r[j]));
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

}  // namespace w8a16
}  // namespace wq

namespace wq_host {

template <int FMT>
static int launch_w8a16_tc(const void* X, int64_t M, int64_t K, const void* Wq,
                           const float* sw, int64_t N, void* Y, cudaStream_t s) {
  using namespace wq::w8a16;
  CUtensorMap tw, tx;
  int st = make_tmap_2d(&tw, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(N), uint64_t(K), BW,
                        BK, 0);
  if (st != WQ_OK) return st;
  st = make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(M), uint64_t(K), BX,
                    BK, 128);
  if (st != WQ_OK) return st;
  static bool attr_done[64] = {};
  int dev = 0;
  WQ_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 64 && !attr_done[dev]) {
    WQ_CUDA_CHECK(cudaFuncSetAttribute(gemm_w8a16_kernel<FMT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(SMEM_BYTES)));
    attr_done[dev] = true;
  }
  const int64_t tiles = ((N + BW - 1) / BW) * ((M + BX - 1) / BX);
  const int grid = int(tiles < sm_count() ? tiles : sm_count());
  gemm_w8a16_kernel<FMT><<<grid, THREADS, SMEM_BYTES, s>>>(
      tw, tx, sw, static_cast<__nv_bfloat16*>(Y), int(M), int(N), int(K), status_ptr(),
      wait_limit_ns());
  WQ_LAUNCH_CHECK("gemm_w8a16_kernel");
  return WQ_OK;
}

template <int FMT>
static int launch_w8a16_cc(const void* X, int64_t M, int64_t K, const void* Wq, const float* sw,
                           int64_t N, void* Y, cudaStream_t s) {
  using namespace wq::w8a16;
  const int64_t blocks = (N + 7) / 8;  // a warp per row, 8 per block
  const int64_t cap = int64_t(sm_count()) * 8;
  const int grid = int(blocks < cap ? blocks : cap);
  const auto* x = static_cast<const __nv_bfloat16*>(X);
  const auto* w = static_cast<const uint8_t*>(Wq);
  auto* y = static_cast<__nv_bfloat16*>(Y);
  if constexpr (FMT == WQ_W8_INT8) {
    // int8 codes: DP2A against X in fixed point, a warp per block of rows
    const int rb = M <= 2 ? 8 : 4;
    const int64_t warps = (N + rb - 1) / rb;
    const int64_t cap2 = int64_t(sm_count()) * 2;
    const int g = int(std::min<int64_t>((warps + 7) / 8, cap2));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(g), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const int mm = int(M), kk = int(K), nn = int(N);
    if (M == 1)
      WQ_CUDA_CHECK(cudaLaunchKernelEx(&cfg, gemv_w8a16_dp_kernel<1, 8>, x, mm, kk, w, sw, nn, y));
    else if (M == 2)
      WQ_CUDA_CHECK(cudaLaunchKernelEx(&cfg, gemv_w8a16_dp_kernel<2, 8>, x, mm, kk, w, sw, nn, y));
    else
      WQ_CUDA_CHECK(cudaLaunchKernelEx(&cfg, gemv_w8a16_dp_kernel<4, 4>, x, mm, kk, w, sw, nn, y));
    return WQ_OK;
  }
  if (M == 1)
    gemv_w8a16_kernel<FMT, 1><<<grid, 256, 0, s>>>(x, int(M), int(K), w, sw, int(N), y);
  else if (M == 2)
    gemv_w8a16_kernel<FMT, 2><<<grid, 256, 0, s>>>(x, int(M), int(K), w, sw, int(N), y);
  else
    gemv_w8a16_kernel<FMT, 4><<<grid, 256, 0, s>>>(x, int(M), int(K), w, sw, int(N), y);
  WQ_LAUNCH_CHECK("gemv_w8a16_kernel");
  return WQ_OK;
}

int launch_gemm_w8a16(const void* X, int64_t M, int64_t K, const void* Wq, int w_fmt,
                      const float* w_scales, int64_t N, void* Y, cudaStream_t s) {
  if (M <= kGemvW8a16MaxM)
    return w_fmt == WQ_W8_E4M3
               ? launch_w8a16_cc<WQ_W8_E4M3>(X, M, K, Wq, w_scales, N, Y, s)
               : launch_w8a16_cc<WQ_W8_INT8>(X, M, K, Wq, w_scales, N, Y, s);
  return w_fmt == WQ_W8_E4M3 ? launch_w8a16_tc<WQ_W8_E4M3>(X, M, K, Wq, w_scales, N, Y, s)
                             : launch_w8a16_tc<WQ_W8_INT8>(X, M, K, Wq, w_scales, N, Y, s);
}

}  // namespace wq_host
