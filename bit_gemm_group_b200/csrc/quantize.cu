// quantize.cu -- the memory-bound kernels of the path:
//   * INT4 group-wise quantize + pack        ("大模型面试准备（十九）…" sec. 2.1-2.2;
//                                             "从 FP32 到 INT4 …" sec. 2.1 quantizers)
//   * INT8 per-row quantize (weights per output channel, activations per token;
//                                             "大模型面试准备（十九）…" sec. 2.2, sec. 6)
//   * dequantize x_hat = s * (q - z)         ("从0到1：大模型量化" sec. 2)
//
// All of them stream their input once with 16-byte (or element-sized when
// smaller) vector loads, keep several groups in flight per warp, and size the
// grid as a multiple of the SM count.  The per-element IEEE division of the
// codes is replaced by a reciprocal multiply whose rounding decisions are
// proved equal (INT4 for 16-bit inputs; INT8 and E4M3 for every input type;
// see the section below).
#include "common.cuh"
#include "kernels.h"
#include "qmath.cuh"
#include <cuda_fp8.h>

namespace wq {

template <int BYTES>
struct Vec;
template <>
struct Vec<16> { using type = uint4; };
template <>
struct Vec<8> { using type = uint2; };
template <>
struct Vec<4> { using type = uint32_t; };
template <>
struct Vec<2> { using type = uint16_t; };
template <>
struct Vec<1> { using type = uint8_t; };

// E contiguous elements of T, loaded with the widest aligned vectors
// (read-only, streaming: the weight is read exactly once).
template <typename T, int E>
struct Elems {
  static constexpr int BYTES = E * int(sizeof(T));
  static constexpr int V = BYTES >= 16 ? 16 : BYTES;
  static constexpr int NV = BYTES / V;
  using VT = typename Vec<V>::type;
  union {
    VT v[NV];
    T e[E];
  } u;
  __device__ __forceinline__ void load(const T* p) {
    const VT* src = reinterpret_cast<const VT*>(p);
#pragma unroll
    for (int i = 0; i < NV; ++i) u.v[i] = __ldcs(src + i);
  }
};

// ---------------------------------------------------------------------------
// INT4 group-wise quantize + pack
// ---------------------------------------------------------------------------
// One warp handles one group of 32*E consecutive elements of a row (lane l owns
// elements [l*E, l*E+E)); U groups per warp iteration are loaded before any is
// processed, so each warp keeps U*32*E*sizeof(T) bytes in flight.  Group i of
// the flattened [N, K/gs] grid starts at element i*gs because gs divides K.
template <typename T, int E, int U>
__global__ void __launch_bounds__(256) quantize_int4_kernel(
    const T* __restrict__ W, int64_t total_groups, int sym, uint8_t* __restrict__ codes,
    __half* __restrict__ scales, __half* __restrict__ zeros, int* status) {
  constexpr int GS = 32 * E;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int qmin = sym ? -8 : 0;
  const int qmax = sym ? 7 : 15;

  for (int64_t base = warp * U; base < total_groups; base += nwarps * U) {
    Elems<T, E> in[U];
#pragma unroll
    for (int j = 0; j < U; ++j)
      if (base + j < total_groups) in[j].load(W + (base + j) * GS + lane * E);
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t gi = base + j;
      if (gi >= total_groups) break;  // warp-uniform
      float x[E];
      float mn = INFINITY, mx = -INFINITY, amax = 0.f;
      bool finite = true;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        x[e] = to_f32<T>(in[j].u.e[e]);
        finite &= isfinite(x[e]);
        mn = fminf(mn, x[e]);
        mx = fmaxf(mx, x[e]);
        amax = fmaxf(amax, fabsf(x[e]));
      }
      unsigned short s_bits;
      float sf;
      int z = 0;
      bool degenerate;
      if (sym) {
        amax = warp_max(amax);
        sf = f16_round_trip(div_rn(amax, 7.f), &s_bits);
        degenerate = (amax < 1e-8f) || (sf == 0.f);
        if (degenerate) sf = f16_round_trip(amax, &s_bits);
      } else {
        mn = warp_min(mn);
        mx = warp_max(mx);
        const float range = mx - mn;
        sf = f16_round_trip(div_rn(range, 15.f), &s_bits);
        degenerate = (range < 1e-8f) || (sf == 0.f);
        if (degenerate) {
          sf = f16_round_trip(1.f, &s_bits);
        } else {
          const float zr = round_even(div_rn(-mn, sf));
          z = int(fmaxf(0.f, fminf(15.f, zr)));
        }
      }
      finite = __all_sync(0xffffffffu, finite);
      if (lane == 0) {
        if (!finite || isinf(sf)) record_error(status, WQ_ERR_NONFINITE);
        scales[gi] = __ushort_as_half(s_bits);
        if (!sym) zeros[gi] = __int2half_rn(z);
      }
      // quantize + pack: E nibbles per lane, low nibble = even element
      uint32_t nib[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        int q = 0;
        if (!degenerate) {
          float r = round_even(div_rn(x[e], sf));
          r = fmaxf(-64.f, fminf(64.f, r));
          q = min(max(int(r) + z, qmin), qmax);
        }
        nib[e] = uint32_t(q - qmin);
      }
      uint8_t* dst = codes + gi * (GS / 2);
      if constexpr (E == 1) {
        const uint32_t other = __shfl_down_sync(0xffffffffu, nib[0], 1);
        if ((lane & 1) == 0) dst[lane >> 1] = uint8_t(nib[0] | (other << 4));
      } else {
        constexpr int NB = E / 2;  // bytes per lane
        union {
          typename Vec<(NB >= 16 ? 16 : NB)>::type v[(NB >= 16 ? NB / 16 : 1)];
          uint8_t b[NB];
        } out;
#pragma unroll
        for (int i = 0; i < NB; ++i) out.b[i] = uint8_t(nib[2 * i] | (nib[2 * i + 1] << 4));
        constexpr int V = NB >= 16 ? 16 : NB;
        using VT = typename Vec<V>::type;
        VT* d = reinterpret_cast<VT*>(dst + lane * NB);
#pragma unroll
        for (int i = 0; i < NB / V; ++i) d[i] = out.v[i];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// INT4 group-wise quantize + pack of 16-bit weights (bf16 / fp16), g <= 512
// ---------------------------------------------------------------------------
// Codes, scales and zeros equal quantize_int4_kernel's bit for bit.  Lane l
// of a group's LPG lanes owns its 16 elements [16 l, 16 l + 16) (two 16-byte
// loads, one 8-byte store of codes); a warp takes 32 / LPG adjacent groups per
// step and U steps are loaded before any is processed.
//
// Codes are the IEEE quotient fl(x / s) itself, rounded to nearest even,
// obtained without a division: with y = rcp_approx(s) (within one ulp),
// q0 = fl(x y) is within 3 ulp of x/s, the residual r = x - q0 s is exact in
// one fma (fewer than 3 * 2^12 units of the last place of q0 s or of x), and
// q0 + r y is within 2^-21 ulp of x/s.  For x a 16-bit float and s an fp16
// value (significands of at most 11 bits) x/s is never an fp32 rounding
// midpoint and lies at least 2^-12 ulp from every one, so fl(q0 + r y) is
// fl(x / s) exactly (Markstein's correction step).  fl(x / s) + 1.5 2^23
// then rounds to even at unit spacing, and its bit pattern is 0x4B400000 plus
// the integer code; codes of |x/s| below 2^-10 are 0 whatever the last bits.
// A quotient that exact half-way tests used to settle is now exact as it
// stands: x/s = j + 1/2 is an fp32 number and the add rounds it to even.
__device__ __forceinline__ float quot16(float x, float s, float y) {
  const float q0 = x * y;
  const float r = fmaf(-q0, s, x);
  return fmaf(r, y, q0);
}

// sum over e = 0..7 of 0x4B400000 * 16^e, modulo 2^32: what eight codes'
// fp32 patterns add to a packed word beyond the codes themselves
__host__ __device__ constexpr uint32_t magic_nibble_sum() {
  uint32_t c = 0u;
  for (int e = 0; e < 8; ++e) c += 0x4B400000u << (4 * e);
  return c;
}

// The 16 codes of a lane as two packed words: nibble e of word h holds
// clamp(code, lo, hi) + zq for element 8 h + e, where the pattern of
// fl(x / s) + 1.5 2^23 (clamped to [1.5 2^23 + lo, 1.5 2^23 + hi] when
// CLAMP) is added in at bit 4 e; the pattern's constant part is taken out
// once per word (the sum stays exact modulo 2^32 and no nibble borrows).
template <typename T, bool CLAMP>
__device__ __forceinline__ uint2 pack_codes16(const uint32_t (&w)[8], float s, float y,
                                              float tlo, float thi, int zq) {
  constexpr float magic = 12582912.f;  // 1.5 * 2^23
  uint32_t acc[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float a, b;
    unpack2<T>(w[i], a, b);
    float ta = quot16(a, s, y) + magic;
    float tb = quot16(b, s, y) + magic;
    if (CLAMP) {
      ta = fminf(fmaxf(ta, tlo), thi);
      tb = fminf(fmaxf(tb, tlo), thi);
    }
    acc[i >> 2] += (__float_as_uint(ta) << (8 * (i & 3))) +
                   (__float_as_uint(tb) << (8 * (i & 3) + 4));
  }
  const uint32_t off = uint32_t(zq) * 0x11111111u - magic_nibble_sum();
  return make_uint2(acc[0] + off, acc[1] + off);
}

template <typename T, bool SYM, int LPG, int U>
__global__ void __launch_bounds__(256) quantize_int4_x16_kernel(
    const T* __restrict__ W, int64_t total_groups, uint8_t* __restrict__ codes,
    __half* __restrict__ scales, __half* __restrict__ zeros, int* status) {
  constexpr int GS = 16 * LPG;   // group size
  constexpr int GPW = 32 / LPG;  // groups per warp and step
  constexpr float magic = 12582912.f;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPG, li = lane % LPG;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  constexpr int qmin = SYM ? -8 : 0;
  bool bad = false;

  for (int64_t base = warp * (U * GPW); base < total_groups; base += nwarps * (U * GPW)) {
    uint4 in[U][2];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t gi = base + j * GPW + sub;
      if (gi < total_groups) {
        const uint4* src = reinterpret_cast<const uint4*>(W + gi * GS) + 2 * li;
        in[j][0] = __ldcs(src);
        in[j][1] = __ldcs(src + 1);
      } else {
        in[j][0] = in[j][1] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      if (base + j * GPW >= total_groups) break;  // warp-uniform
      const int64_t gi = base + j * GPW + sub;
      const bool live = gi < total_groups;
      const uint32_t w[8] = {in[j][0].x, in[j][0].y, in[j][0].z, in[j][0].w,
                             in[j][1].x, in[j][1].y, in[j][1].z, in[j][1].w};
      unsigned short s_bits;
      float sf;
      int z = 0;
      bool degenerate;
      if (SYM) {
        uint32_t m = absmax2<T>(absmax2<T>(absmax2<T>(w[0], w[1]), absmax2<T>(w[2], w[3])),
                                absmax2<T>(absmax2<T>(w[4], w[5]), absmax2<T>(w[6], w[7])));
        float ma, mb;
        unpack2<T>(m, ma, mb);
        float amax = fmaxf(fabsf(ma), fabsf(mb));
        bad |= !(amax <= 3.402823466e38f);  // Inf or NaN in the lane
#pragma unroll
        for (int o = LPG / 2; o > 0; o >>= 1)
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        sf = f16_round_trip(div_rn(amax, 7.f), &s_bits);
        degenerate = (amax < 1e-8f) || (sf == 0.f);
        if (degenerate) sf = f16_round_trip(amax, &s_bits);
      } else {
        uint32_t lo2 = min2<T>(min2<T>(min2<T>(w[0], w[1]), min2<T>(w[2], w[3])),
                               min2<T>(min2<T>(w[4], w[5]), min2<T>(w[6], w[7])));
        uint32_t hi2 = max2<T>(max2<T>(max2<T>(w[0], w[1]), max2<T>(w[2], w[3])),
                               max2<T>(max2<T>(w[4], w[5]), max2<T>(w[6], w[7])));
        float a, b, c, d;
        unpack2<T>(lo2, a, b);
        unpack2<T>(hi2, c, d);
        float mn = fminf(a, b), mx = fmaxf(c, d);
        bad |= !(fabsf(a) <= 3.402823466e38f && fabsf(b) <= 3.402823466e38f &&
                 fabsf(c) <= 3.402823466e38f && fabsf(d) <= 3.402823466e38f);
#pragma unroll
        for (int o = LPG / 2; o > 0; o >>= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const float range = mx - mn;
        sf = f16_round_trip(div_rn(range, 15.f), &s_bits);
        degenerate = (range < 1e-8f) || (sf == 0.f);
        if (degenerate) {
          sf = f16_round_trip(1.f, &s_bits);
        } else {
          const float zr = round_even(div_rn(-mn, sf));
          z = int(fmaxf(0.f, fminf(15.f, zr)));
        }
      }
      if (live && li == 0) {
        scales[gi] = __ushort_as_half(s_bits);
        if (!SYM) zeros[gi] = __int2half_rn(z);
      }
      bad |= isinf(sf);
      // a degenerate group takes code 0 for every element (y = 0)
      const float y = degenerate ? 0.f : rcp_approx(sf);
      const int zq = z - qmin;  // nibble = clamp(q + z, qmin, qmax) - qmin
      const float tlo = magic - float(zq), thi = magic + float(15 - zq);
      uint2 packed;
      if (SYM) {
        // |x/s| <= amax/s < 7.5 for a normal fp16 s = fl16(amax / 7): no clamp;
        // a subnormal s (amax below 4.3e-4) can reach +-8 and takes it
        const bool clamp = !degenerate && sf < 0x1p-14f;
        if (__any_sync(0xffffffffu, clamp))
          packed = pack_codes16<T, true>(w, sf, y, tlo, thi, zq);
        else
          packed = pack_codes16<T, false>(w, sf, y, tlo, thi, zq);
      } else {
        packed = pack_codes16<T, true>(w, sf, y, tlo, thi, zq);
      }
      if (live) *reinterpret_cast<uint2*>(codes + gi * (GS / 2) + li * 8) = packed;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(status, WQ_ERR_NONFINITE);
}

// ---------------------------------------------------------------------------
// INT8 per-row quantization (weights per output channel / activations per token)
// ---------------------------------------------------------------------------
// One 256-thread block per row: pass 1 reduces amax with 16-byte loads, pass 2
// re-reads the row (L1/L2 resident: a row is at most a few tens of KB) and
// writes int8 codes 8 at a time.
// Element e of an 8-vector at column k after the optional SmoothQuant
// migration ("27届大模型面试准备（十九）…" sec. 4.2): activations are divided by
// s[k] (X diag(s)^-1), weights multiplied (W diag(s)); one IEEE operation.
template <bool ACT>
__device__ __forceinline__ void smooth8(float (&x)[8], const float* __restrict__ smooth,
                                        int64_t k) {
  if (smooth == nullptr) return;
  const float4 a = *reinterpret_cast<const float4*>(smooth + k);
  const float4 b = *reinterpret_cast<const float4*>(smooth + k + 4);
  const float sv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = ACT ? div_rn(x[e], sv[e]) : __fmul_rn(x[e], sv[e]);
}

template <typename T, bool ACT>
__global__ void __launch_bounds__(256) quantize_rows_i8_kernel(
    const T* __restrict__ X, int64_t rows, int64_t K, const float* __restrict__ smooth,
    int8_t* __restrict__ q, float* __restrict__ scales, int* status) {
  constexpr int EV = 8;  // elements per vector step
  __shared__ float red[8];
  __shared__ int bad_any;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const T* row = X + r * K;
    float amax = 0.f;
    bool finite = true;
    for (int64_t k = int64_t(threadIdx.x) * EV; k < K; k += int64_t(blockDim.x) * EV) {
      Elems<T, EV> v;
      v.load(row + k);
      float x[EV];
#pragma unroll
      for (int e = 0; e < EV; ++e) x[e] = to_f32<T>(v.u.e[e]);
      smooth8<ACT>(x, smooth, k);
#pragma unroll
      for (int e = 0; e < EV; ++e) {
        finite &= isfinite(x[e]);
        amax = fmaxf(amax, fabsf(x[e]));
      }
    }
    amax = warp_max(amax);
    const int nbad = __syncthreads_or(!finite);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = red[0];
      for (int w = 1; w < int(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
      red[0] = m;
      bad_any = nbad;
    }
    __syncthreads();
    amax = red[0];
    float s;
    bool degenerate = false;
    if (ACT) {
      s = fmaxf(div_rn(amax, 127.f), 1e-8f);
    } else {
      degenerate = amax < 1e-8f;
      s = degenerate ? amax : div_rn(amax, 127.f);
    }
    if (threadIdx.x == 0) {
      scales[r] = s;
      if (bad_any) record_error(status, WQ_ERR_NONFINITE);
    }
    const int lo = ACT ? -128 : -127;
    const float inv = rcp_approx(s);
    for (int64_t k = int64_t(threadIdx.x) * EV; k < K; k += int64_t(blockDim.x) * EV) {
      Elems<T, EV> v;
      v.load(row + k);
      float x[EV];
#pragma unroll
      for (int e = 0; e < EV; ++e) x[e] = to_f32<T>(v.u.e[e]);
      smooth8<ACT>(x, smooth, k);
      union {
        uint2 v2;
        int8_t b[EV];
      } o;
#pragma unroll
      for (int e = 0; e < EV; ++e) {
        int qi = 0;
        if (!degenerate) {
          float rr = rint_quot_i8(x[e], s, inv);
          rr = fmaxf(-200.f, fminf(200.f, rr));
          qi = min(max(int(rr), lo), 127);
        }
        o.b[e] = int8_t(qi);
      }
      *reinterpret_cast<uint2*>(q + r * K + k) = o.v2;
    }
    __syncthreads();  // red[] is reused by the next row
  }
}

// ---------------------------------------------------------------------------
// FP8 E4M3 rows ("27届大模型面试准备（十九）…" sec. 2.3: FP8 as the 8-bit float
// format; the W8A8 recipe with E4M3 in place of int8)
// ---------------------------------------------------------------------------
// One scale per row, s = max(amax / 448, 1e-8), q = e4m3(x / s) rounded to
// nearest even and saturated to +-448 (the hardware conversion).
template <typename T>
__global__ void __launch_bounds__(256) quantize_rows_fp8_kernel(
    const T* __restrict__ X, int64_t rows, int64_t K, uint8_t* __restrict__ q,
    float* __restrict__ scales, int* status) {
  constexpr int EV = 8;
  __shared__ float red[8];
  __shared__ int bad_any;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const T* row = X + r * K;
    float amax = 0.f;
    bool finite = true;
    for (int64_t k = int64_t(threadIdx.x) * EV; k < K; k += int64_t(blockDim.x) * EV) {
      Elems<T, EV> v;
      v.load(row + k);
#pragma unroll
      for (int e = 0; e < EV; ++e) {
        const float x = to_f32<T>(v.u.e[e]);
        finite &= isfinite(x);
        amax = fmaxf(amax, fabsf(x));
      }
    }
    amax = warp_max(amax);
    const int nbad = __syncthreads_or(!finite);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = red[0];
      for (int w = 1; w < int(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
      red[0] = m;
      bad_any = nbad;
    }
    __syncthreads();
    const float s = fmaxf(div_rn(red[0], 448.f), 1e-8f);
    const float inv = rcp_approx(s);
    if (threadIdx.x == 0) {
      scales[r] = s;
      if (bad_any) record_error(status, WQ_ERR_NONFINITE);
    }
    for (int64_t k = int64_t(threadIdx.x) * EV; k < K; k += int64_t(blockDim.x) * EV) {
      Elems<T, EV> v;
      v.load(row + k);
      union {
        uint2 v2;
        uint8_t b[EV];
      } o;
#pragma unroll
      for (int e = 0; e < EV; ++e)
        o.b[e] = uint8_t(__nv_cvt_float_to_fp8(quot_e4m3(to_f32<T>(v.u.e[e]), s, inv),
                                               __NV_SATFINITE, __NV_E4M3));
      *reinterpret_cast<uint2*>(q + r * K + k) = o.v2;
    }
    __syncthreads();  // red[] is reused by the next row
  }
}


// ---------------------------------------------------------------------------
// Per-row quantizers with the row held in registers (16-bit inputs, K in
// {1024, 2048, 4096, 8192}): the activation side of W8A8 / FP8
// ---------------------------------------------------------------------------
// A row is K / 32 threads x 32 elements: thread t owns the 8-element blocks
// t + (K / 256) i, i = 0..3 (each load and store instruction of a warp covers
// contiguous bytes).  The row is read once; its maximum |x| is an integer max
// over the 16-bit magnitude bit patterns (which order like the values; a NaN
// or infinity pattern is at least the infinity pattern, so the same max
// reports non-finite input), a warp shuffle tree and one barrier.  The codes
// come from the same reciprocal-multiply rules as the two-pass kernels, so
// they are identical.  KIND 0: int8 per token (s = max(amax / 127, 1e-8),
// q in [-128, 127], optional SmoothQuant division by s[k]); KIND 1: E4M3
// (s = max(amax / 448, 1e-8)).
template <typename T>
__device__ __forceinline__ uint32_t abs_bits_mask() {
  return 0x7FFF7FFFu;
}
template <typename T>
__device__ __forceinline__ uint32_t inf_bits();
template <>
__device__ __forceinline__ uint32_t inf_bits<__nv_bfloat16>() { return 0x7F80u; }
template <>
__device__ __forceinline__ uint32_t inf_bits<__half>() { return 0x7C00u; }

template <typename T>
__device__ __forceinline__ float half_bits_to_f32(uint32_t h);
template <>
__device__ __forceinline__ float half_bits_to_f32<__nv_bfloat16>(uint32_t h) {
  return __uint_as_float(h << 16);
}
template <>
__device__ __forceinline__ float half_bits_to_f32<__half>(uint32_t h) {
  return __half2float(__ushort_as_half((unsigned short)h));
}

__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

template <typename T, int KIND>
__global__ void __launch_bounds__(256, 3) quantize_rows_reg_kernel(
    const T* __restrict__ X, int64_t rows, int K, const float* __restrict__ smooth,
    uint8_t* __restrict__ q, float* __restrict__ scales, int* status) {
  __shared__ float red[8];
  __shared__ int bad_w[8];
  const int tpr = K >> 5;  // threads per row (a multiple of 32)
  const int rpb = 256 / tpr;
  const int wpr = tpr >> 5;
  const int sub = threadIdx.x / tpr, t = threadIdx.x - sub * tpr;
  const int warp = threadIdx.x >> 5;
  for (int64_t r0 = int64_t(blockIdx.x) * rpb; r0 < rows; r0 += int64_t(gridDim.x) * rpb) {
    const int64_t r = r0 + sub;
    const bool live = r < rows;
    const T* row = X + (live ? r : 0) * int64_t(K);
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i] = make_uint4(0, 0, 0, 0);
      if (live) v[i] = __ldcs(reinterpret_cast<const uint4*>(row) + t + tpr * i);
    }
    float x[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[8 * i + 2 * j] = half_bits_to_f32<T>(w[j] & 0xFFFFu);
        x[8 * i + 2 * j + 1] = half_bits_to_f32<T>(w[j] >> 16);
      }
    }
    float amax = 0.f;
    bool finite = true;
    if (KIND == 0 && smooth != nullptr) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t k = 8 * int64_t(t + tpr * i);
        const float4 a = *reinterpret_cast<const float4*>(smooth + k);
        const float4 b = *reinterpret_cast<const float4*>(smooth + k + 4);
        const float sv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          x[8 * i + e] = div_rn(x[8 * i + e], sv[e]);
          finite &= isfinite(x[8 * i + e]);
          amax = fmaxf(amax, fabsf(x[8 * i + e]));
        }
      }
    } else {
      uint32_t m = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        m = vmax_u16x2(m, v[i].x & abs_bits_mask<T>());
        m = vmax_u16x2(m, v[i].y & abs_bits_mask<T>());
        m = vmax_u16x2(m, v[i].z & abs_bits_mask<T>());
        m = vmax_u16x2(m, v[i].w & abs_bits_mask<T>());
      }
      const uint32_t mb = max(m & 0xFFFFu, m >> 16);
      finite = mb < inf_bits<T>();
      if (finite) {
        amax = half_bits_to_f32<T>(mb);
      } else {
        // non-finite input (reported): the maximum as the two-pass kernels
        // take it, NaN ignored and infinity counted
#pragma unroll
        for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(x[e]));
      }
    }
    amax = warp_max(amax);
    const bool wbad = __any_sync(0xffffffffu, !finite);
    if ((threadIdx.x & 31) == 0) {
      red[warp] = amax;
      bad_w[warp] = wbad;
    }
    __syncthreads();
    int bad = 0;
#pragma unroll 1
    for (int j = 0; j < wpr; ++j) {
      amax = fmaxf(amax, red[sub * wpr + j]);
      bad |= bad_w[sub * wpr + j];
    }
    const float s = fmaxf(div_rn(amax, KIND == 0 ? 127.f : 448.f), 1e-8f);
    const float inv = rcp_approx(s);
    if (live && t == 0) {
      scales[r] = s;
      if (bad) record_error(status, WQ_ERR_NONFINITE);
    }
    if (live) {  // warp-uniform: a row spans whole warps
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        union {
          uint2 v2;
          uint8_t b[8];
        } o;
        uint32_t near = 0u;
        if (KIND == 0 && !bad) {
          // finite row: |x / s| <= 127.5, codes through the fp32 patterns
          const float* xi = x + 8 * i;
          o.v2 = make_uint2(
              codes_i8_x4(xi[0], xi[1], xi[2], xi[3], inv, inv, inv, inv, near, 0),
              codes_i8_x4(xi[4], xi[5], xi[6], xi[7], inv, inv, inv, inv, near, 1));
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (KIND == 0) {
              o.b[e] = uint8_t(int8_t(code_i8_full(x[8 * i + e], s, inv)));
            } else {
              o.b[e] = uint8_t(__nv_cvt_float_to_fp8(quot_e4m3(x[8 * i + e], s, inv),
                                                     __NV_SATFINITE, __NV_E4M3));
            }
          }
        }
        uint8_t* dst = q + r * int64_t(K) + 8 * int64_t(t + tpr * i);
        *reinterpret_cast<uint2*>(dst) = o.v2;
        while (near != 0u) {  // groups with a near-half-way element, rewritten exactly
          const int g = __ffs(near) - 1;
          near &= near - 1u;
          float xg[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) xg[j] = g ? x[8 * i + 4 + j] : x[8 * i + j];
          *reinterpret_cast<char4*>(dst + 4 * g) =
              make_char4(code_i8_exact(xg[0], s, inv), code_i8_exact(xg[1], s, inv),
                         code_i8_exact(xg[2], s, inv), code_i8_exact(xg[3], s, inv));
        }
      }
    }
    __syncthreads();  // red[] is reused by the next rows
  }
}

// ---------------------------------------------------------------------------
// SmoothQuant statistics ("27届大模型面试准备（十九）…" sec. 4.2)
// ---------------------------------------------------------------------------
// out[k] = max_r |A[r, k]| over the rows of A [R, K]: act_scales for a
// calibration activation, w_scales for a weight [out, in].  Each thread keeps
// eight adjacent columns (one 16- or 32-byte load per row) over a strip of
// rows and merges with atomicMax on the bit patterns (non-negative floats
// order like their bits), so the result does not depend on the order.
// Non-finite elements are skipped and reported, as in the oracle.
template <typename T>
__global__ void __launch_bounds__(256) channel_absmax_kernel(const T* __restrict__ A, int64_t R,
                                                             int64_t K,
                                                             unsigned* __restrict__ out,
                                                             int* status) {
  const int64_t col = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (col >= K) return;
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  bool bad = false;
  for (int64_t r = blockIdx.y; r < R; r += gridDim.y) {
    Elems<T, 8> v;
    v.load(A + r * K + col);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = to_f32<T>(v.u.e[e]);
      if (isfinite(x)) {
        m[e] = fmaxf(m[e], fabsf(x));
      } else {
        bad = true;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) atomicMax(out + col + e, __float_as_uint(m[e]));
  if (bad) record_error(status, WQ_ERR_NONFINITE);
}

// s[k] = max(act[k]^alpha / max(w[k], 1e-5)^(1 - alpha), 1e-5), evaluated in
// binary64 and rounded once to binary32 (the page's smooth_ln_linear clamps).
__global__ void __launch_bounds__(256) smooth_scales_kernel(const float* __restrict__ act,
                                                            const float* __restrict__ w,
                                                            int64_t K, double alpha,
                                                            float* __restrict__ s) {
  const int64_t k = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const float wc = fmaxf(w[k], 1e-5f);
  double v = pow(double(act[k]), alpha) / pow(double(wc), 1.0 - alpha);
  if (v < 1e-5) v = 1e-5;
  s[k] = __double2float_rn(v);
}

// ---------------------------------------------------------------------------
// KV-cache INT8 ("27届大模型面试准备（十九）…" sec. 6)
// ---------------------------------------------------------------------------
// K [BH, S, D] per channel: amax over the S tokens of each (head, channel).
// Block (D/8 column groups) x (256 / (D/8) token rows); CTA (strip, bh) walks
// its strip of tokens, reduces its rows in shared memory and merges with
// atomicMax on the fp32 bit patterns (order-free, like channel_absmax).
template <typename T>
__global__ void __launch_bounds__(256) kv_k_absmax_kernel(const T* __restrict__ Kc, int64_t S,
                                                          int D, unsigned* __restrict__ amax,
                                                          int* status) {
  __shared__ float red[256 * 8];
  const int cg = threadIdx.x % (D / 8), ty = threadIdx.x / (D / 8);
  const int rows = blockDim.x / (D / 8);
  const int64_t bh = blockIdx.y;
  const T* base = Kc + bh * S * D + cg * 8;
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  bool bad = false;
  for (int64_t t = int64_t(blockIdx.x) * rows + ty; t < S; t += int64_t(gridDim.x) * rows) {
    Elems<T, 8> v;
    v.load(base + t * D);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = to_f32<T>(v.u.e[e]);
      bad |= !isfinite(x);
      m[e] = fmaxf(m[e], fabsf(x));  // a NaN is skipped, an infinity counts
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x * 8 + e] = m[e];
  __syncthreads();
  if (ty == 0) {
    for (int r = 1; r < rows; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], red[(r * (D / 8) + cg) * 8 + e]);
#pragma unroll
    for (int e = 0; e < 8; ++e) atomicMax(amax + bh * D + cg * 8 + e, __float_as_uint(m[e]));
  }
  if (bad) record_error(status, WQ_ERR_NONFINITE);
}

// V [rows = BH S, D] per token, for head dims D = 8 LPR with LPR a power of two
// <= 32: a row is LPR lanes of eight elements, a warp holds 32 / LPR rows, and
// the row maximum is a shuffle reduction inside the row's lane segment (no
// shared memory, no block barrier).  Same arithmetic as the per-token
// quantizer: s = max(amax / 127, 1e-8), q = clamp(round(v / s), -128, 127).
template <typename T, int LPR>
__global__ void __launch_bounds__(256) kv_v_quant_kernel(const T* __restrict__ V, int64_t rows,
                                                         int8_t* __restrict__ qv,
                                                         float* __restrict__ sv, int* status) {
  constexpr int D = 8 * LPR;
  constexpr int RPW = 32 / LPR;  // rows per warp
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, seg = lane % LPR;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  bool bad = false;
  for (int64_t r0 = warp * RPW; r0 < rows; r0 += nwarps * RPW) {
    const int64_t r = r0 + sub;
    const bool act = r < rows;
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (act) {
      Elems<T, 8> v;
      v.load(V + r * D + seg * 8);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = to_f32<T>(v.u.e[e]);
    }
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      bad |= !isfinite(x[e]);
      amax = fmaxf(amax, fabsf(x[e]));
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = fmaxf(div_rn(amax, 127.f), 1e-8f);
    if (act) {
      const float inv = rcp_approx(sc);
      union {
        uint2 v2;
        int8_t b8[8];
      } o;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float rr = rint_quot_i8(x[e], sc, inv);
        rr = fmaxf(-200.f, fminf(200.f, rr));
        o.b8[e] = int8_t(min(max(int(rr), -128), 127));
      }
      *reinterpret_cast<uint2*>(qv + r * D + seg * 8) = o.v2;
      if (seg == 0) sv[r] = sc;
    }
  }
  if (bad) record_error(status, WQ_ERR_NONFINITE);
}

// sk = max(amax / 127, 1e-8) in place (amax arrives as fp32 bit patterns).
__global__ void __launch_bounds__(256) kv_k_scale_kernel(float* __restrict__ sk, int64_t n) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) sk[i] = fmaxf(div_rn(sk[i], 127.f), 1e-8f);
}

// qk = clamp(round(K / sk[bh, d]), -128, 127), eight channels per thread.
template <typename T>
__global__ void __launch_bounds__(256) kv_k_quant_kernel(const T* __restrict__ Kc, int64_t S,
                                                         int D, const float* __restrict__ sk,
                                                         int8_t* __restrict__ qk,
                                                         int64_t n8) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e0 = i * 8;                  // first element
    const int64_t bh = e0 / (S * D);
    const int d0 = int(e0 % D);
    Elems<T, 8> v;
    v.load(Kc + e0);
    const float4 a = *reinterpret_cast<const float4*>(sk + bh * D + d0);
    const float4 b = *reinterpret_cast<const float4*>(sk + bh * D + d0 + 4);
    const float sc[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    union {
      uint2 v2;
      int8_t b8[8];
    } o;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float r = rint_quot_i8(to_f32<T>(v.u.e[e]), sc[e], rcp_approx(sc[e]));
      r = fmaxf(-200.f, fminf(200.f, r));
      o.b8[e] = int8_t(min(max(int(r), -128), 127));
    }
    *reinterpret_cast<uint2*>(qk + e0) = o.v2;
  }
}

// ---------------------------------------------------------------------------
// Dequantization
// ---------------------------------------------------------------------------
// One thread expands 16 bytes of codes (32 elements) of one row.
template <typename OutT>
__global__ void __launch_bounds__(256) dequant_int4_kernel(
    const uint8_t* __restrict__ codes, const __half* __restrict__ scales,
    const __half* __restrict__ zeros, int64_t N, int64_t K, int gs, int sym,
    OutT* __restrict__ out) {
  const int64_t chunks_per_row = K / 32;
  const int64_t total = N * chunks_per_row;
  const int64_t G = K / gs;
  for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < total;
       c += int64_t(gridDim.x) * blockDim.x) {
    const int64_t n = c / chunks_per_row;
    const int64_t k0 = (c % chunks_per_row) * 32;
    const uint4 w = __ldcs(reinterpret_cast<const uint4*>(codes + n * (K / 2) + k0 / 2));
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    float vals[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int64_t k = k0 + i;
      const int64_t g = k / gs;  // gs >= 32 and 32 | gs: at most one change per chunk
      const float s = __half2float(scales[n * G + g]);
      const int zeff = sym ? 8 : int(__half2float(zeros[n * G + g]));
      const int u = int((words[i >> 3] >> (4 * (i & 7))) & 0xFu);
      vals[i] = s * float(u - zeff);  // exact: 11-bit scale times |u - z| <= 15
    }
    OutT* dst = out + n * K + k0;
    if constexpr (sizeof(OutT) == 4) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        __stcs(reinterpret_cast<float4*>(dst) + i,
               make_float4(vals[4 * i], vals[4 * i + 1], vals[4 * i + 2], vals[4 * i + 3]));
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        union {
          uint4 v;
          __nv_bfloat162 h[4];
        } o;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          o.h[j] = __floats2bfloat162_rn(vals[8 * i + 2 * j], vals[8 * i + 2 * j + 1]);
        __stcs(reinterpret_cast<uint4*>(dst) + i, o.v);
      }
    }
  }
}

template <typename OutT>
__global__ void __launch_bounds__(256) dequant_int8_rows_kernel(
    const int8_t* __restrict__ q, const float* __restrict__ scales, int64_t N, int64_t K,
    OutT* __restrict__ out) {
  const int64_t chunks_per_row = K / 16;
  const int64_t total = N * chunks_per_row;
  for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < total;
       c += int64_t(gridDim.x) * blockDim.x) {
    const int64_t n = c / chunks_per_row;
    const int64_t k0 = (c % chunks_per_row) * 16;
    union {
      uint4 v;
      int8_t b[16];
    } w;
    w.v = __ldcs(reinterpret_cast<const uint4*>(q + n * K + k0));
    const float s = scales[n];
    OutT* dst = out + n * K + k0;
    if constexpr (sizeof(OutT) == 4) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        __stcs(reinterpret_cast<float4*>(dst) + i,
               make_float4(s * w.b[4 * i], s * w.b[4 * i + 1], s * w.b[4 * i + 2],
                           s * w.b[4 * i + 3]));
    } else {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        union {
          uint4 v;
          __nv_bfloat162 h[4];
        } o;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          o.h[j] = __floats2bfloat162_rn(s * w.b[8 * i + 2 * j], s * w.b[8 * i + 2 * j + 1]);
        __stcs(reinterpret_cast<uint4*>(dst) + i, o.v);
      }
    }
  }
}

}  // namespace wq

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
namespace wq_host {

static int grid_for(int64_t work_items, int items_per_block) {
  const int64_t blocks = (work_items + items_per_block - 1) / items_per_block;
  const int64_t cap = int64_t(sm_count()) * 8;  // 8 resident 256-thread blocks per SM
  return int(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

template <typename T, int E>
static void quantize_int4_typed(const void* W, int64_t N, int64_t K, int sym, void* codes,
                                void* scales, void* zeros, cudaStream_t s) {
  constexpr int U = E >= 8 ? 2 : 4;
  const int64_t total = N * (K / (32 * E));
  const int64_t warps = (total + U - 1) / U;
  wq::quantize_int4_kernel<T, E, U><<<grid_for(warps, 8), 256, 0, s>>>(
      static_cast<const T*>(W), total, sym, static_cast<uint8_t*>(codes),
      static_cast<__half*>(scales), static_cast<__half*>(zeros), status_ptr());
}

// 16-bit weights, g = 16 LPG: the reciprocal-multiply kernel.
template <typename T, int LPG>
static void quantize_int4_x16(const void* W, int64_t N, int64_t K, int sym, void* codes,
                              void* scales, void* zeros, cudaStream_t s) {
  constexpr int U = 4;
  const int64_t total = N * (K / (16 * LPG));
  const int64_t steps = (total + U * (32 / LPG) - 1) / (U * (32 / LPG));  // warp steps
  const int grid = grid_for(steps, 8);
  if (sym)
    wq::quantize_int4_x16_kernel<T, true, LPG, U><<<grid, 256, 0, s>>>(
        static_cast<const T*>(W), total, static_cast<uint8_t*>(codes),
        static_cast<__half*>(scales), static_cast<__half*>(zeros), status_ptr());
  else
    wq::quantize_int4_x16_kernel<T, false, LPG, U><<<grid, 256, 0, s>>>(
        static_cast<const T*>(W), total, static_cast<uint8_t*>(codes),
        static_cast<__half*>(scales), static_cast<__half*>(zeros), status_ptr());
}

template <typename T>
static int quantize_int4_dispatch(const void* W, int64_t N, int64_t K, int gs, int sym,
                                  void* codes, void* scales, void* zeros, cudaStream_t s) {
  if constexpr (sizeof(T) == 2) {
    if (gs <= 512) {
      switch (gs) {
        case 32: quantize_int4_x16<T, 2>(W, N, K, sym, codes, scales, zeros, s); break;
        case 64: quantize_int4_x16<T, 4>(W, N, K, sym, codes, scales, zeros, s); break;
        case 128: quantize_int4_x16<T, 8>(W, N, K, sym, codes, scales, zeros, s); break;
        case 256: quantize_int4_x16<T, 16>(W, N, K, sym, codes, scales, zeros, s); break;
        case 512: quantize_int4_x16<T, 32>(W, N, K, sym, codes, scales, zeros, s); break;
        default: return WQ_ERR_UNSUPPORTED;
      }
      WQ_LAUNCH_CHECK("quantize_int4_x16_kernel");
      return WQ_OK;
    }
  }
  switch (gs) {
    case 32: quantize_int4_typed<T, 1>(W, N, K, sym, codes, scales, zeros, s); break;
    case 64: quantize_int4_typed<T, 2>(W, N, K, sym, codes, scales, zeros, s); break;
    case 128: quantize_int4_typed<T, 4>(W, N, K, sym, codes, scales, zeros, s); break;
    case 256: quantize_int4_typed<T, 8>(W, N, K, sym, codes, scales, zeros, s); break;
    case 512: quantize_int4_typed<T, 16>(W, N, K, sym, codes, scales, zeros, s); break;
    case 1024: quantize_int4_typed<T, 32>(W, N, K, sym, codes, scales, zeros, s); break;
    default: return WQ_ERR_UNSUPPORTED;
  }
  WQ_LAUNCH_CHECK("quantize_int4_kernel");
  return WQ_OK;
}

int launch_quantize_int4(const void* W, int w_dtype, int64_t N, int64_t K, int gs, int sym,
                         void* codes, void* scales, void* zeros, cudaStream_t s) {
  switch (w_dtype) {
    case WQ_F32: return quantize_int4_dispatch<float>(W, N, K, gs, sym, codes, scales, zeros, s);
    case WQ_BF16:
      return quantize_int4_dispatch<__nv_bfloat16>(W, N, K, gs, sym, codes, scales, zeros, s);
    case WQ_F16: return quantize_int4_dispatch<__half>(W, N, K, gs, sym, codes, scales, zeros, s);
  }
  return WQ_ERR_ARG;
}

// The register-resident kernel serves 16-bit rows of K = 1024, 2048, 4096 or
// 8192 elements: a row is K / 32 threads of 32 elements, and the 256-thread
// block holds a whole number of rows.
static bool rows_in_registers(int w_dtype, int64_t K) {
  return (w_dtype == WQ_BF16 || w_dtype == WQ_F16) &&
         (K == 1024 || K == 2048 || K == 4096 || K == 8192);
}

template <typename T, int KIND>
static void launch_rows_reg(const void* W, int64_t N, int64_t K, const float* smooth, void* q,
                            void* scales, cudaStream_t s) {
  const int64_t rpb = 8192 / K;
  const int64_t blocks = (N + rpb - 1) / rpb;
  const int64_t cap = int64_t(sm_count()) * 8;
  const int grid = int(blocks < cap ? blocks : cap);
  wq::quantize_rows_reg_kernel<T, KIND><<<grid, 256, 0, s>>>(
      static_cast<const T*>(W), N, int(K), smooth, static_cast<uint8_t*>(q),
      static_cast<float*>(scales), status_ptr());
}

int launch_quantize_rows_i8(const void* W, int w_dtype, int64_t N, int64_t K, bool activation,
                            const float* smooth, void* q, void* scales, cudaStream_t s) {
  if (activation && rows_in_registers(w_dtype, K)) {
    if (w_dtype == WQ_BF16)
      launch_rows_reg<__nv_bfloat16, 0>(W, N, K, smooth, q, scales, s);
    else
      launch_rows_reg<__half, 0>(W, N, K, smooth, q, scales, s);
    WQ_LAUNCH_CHECK("quantize_rows_reg_kernel");
    return WQ_OK;
  }
  const int grid = int(N < int64_t(sm_count()) * 16 ? N : int64_t(sm_count()) * 16);
  int* st = status_ptr();
  auto* qo = static_cast<int8_t*>(q);
  auto* so = static_cast<float*>(scales);
#define WQ_ROWS(T)                                                                           \
  do {                                                                                       \
    if (activation)                                                                          \
      wq::quantize_rows_i8_kernel<T, true><<<grid, 256, 0, s>>>(static_cast<const T*>(W), N, \
                                                                K, smooth, qo, so, st);      \
    else                                                                                     \
      wq::quantize_rows_i8_kernel<T, false><<<grid, 256, 0, s>>>(static_cast<const T*>(W),   \
                                                                 N, K, smooth, qo, so, st);  \
  } while (0)
  switch (w_dtype) {
    case WQ_F32: WQ_ROWS(float); break;
    case WQ_BF16: WQ_ROWS(__nv_bfloat16); break;
    case WQ_F16: WQ_ROWS(__half); break;
    default: return WQ_ERR_ARG;
  }
#undef WQ_ROWS
  WQ_LAUNCH_CHECK("quantize_rows_i8_kernel");
  return WQ_OK;
}

int launch_quantize_rows_fp8(const void* W, int w_dtype, int64_t R, int64_t K, void* q,
                             void* scales, cudaStream_t s) {
  if (rows_in_registers(w_dtype, K)) {
    if (w_dtype == WQ_BF16)
      launch_rows_reg<__nv_bfloat16, 1>(W, R, K, nullptr, q, scales, s);
    else
      launch_rows_reg<__half, 1>(W, R, K, nullptr, q, scales, s);
    WQ_LAUNCH_CHECK("quantize_rows_reg_kernel");
    return WQ_OK;
  }
  const int grid = int(R < int64_t(sm_count()) * 16 ? R : int64_t(sm_count()) * 16);
  int* st = status_ptr();
  auto* qo = static_cast<uint8_t*>(q);
  auto* so = static_cast<float*>(scales);
  switch (w_dtype) {
    case WQ_F32:
      wq::quantize_rows_fp8_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(W), R, K,
                                                               qo, so, st);
      break;
    case WQ_BF16:
      wq::quantize_rows_fp8_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(W), R, K, qo, so, st);
      break;
    case WQ_F16:
      wq::quantize_rows_fp8_kernel<__half><<<grid, 256, 0, s>>>(static_cast<const __half*>(W), R,
                                                                K, qo, so, st);
      break;
    default: return WQ_ERR_ARG;
  }
  WQ_LAUNCH_CHECK("quantize_rows_fp8_kernel");
  return WQ_OK;
}

int launch_channel_absmax(const void* A, int a_dtype, int64_t R, int64_t K, float* out,
                          cudaStream_t s) {
  WQ_CUDA_CHECK(cudaMemsetAsync(out, 0, size_t(K) * 4, s));
  if (R == 0) return WQ_OK;
  const int64_t groups = K / 8;  // 8 columns per thread
  const int gx = int((groups + 255) / 256);
  const int64_t want = int64_t(sm_count()) * 8;
  const int gy = int(R < want / gx + 1 ? R : want / gx + 1);
  const dim3 grid(unsigned(gx), unsigned(gy > 65535 ? 65535 : gy));
  auto* o = reinterpret_cast<unsigned*>(out);
  int* st = status_ptr();
  switch (a_dtype) {
    case WQ_F32:
      wq::channel_absmax_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(A), R, K, o, st);
      break;
    case WQ_BF16:
      wq::channel_absmax_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(A), R, K, o, st);
      break;
    case WQ_F16:
      wq::channel_absmax_kernel<__half><<<grid, 256, 0, s>>>(static_cast<const __half*>(A), R, K, o, st);
      break;
    default: return WQ_ERR_ARG;
  }
  WQ_LAUNCH_CHECK("channel_absmax_kernel");
  return WQ_OK;
}

int launch_quant_kv(const void* Kc, const void* Vc, int dtype, int64_t BH, int64_t S, int64_t D,
                    void* qk, void* sk, void* qv, void* sv, cudaStream_t s) {
  const int fused = launch_quant_kv_fused(Kc, Vc, dtype, BH, S, D, qk, sk, qv, sv, s);
  if (fused != WQ_ERR_UNSUPPORTED) return fused;
  float* skf = static_cast<float*>(sk);
  WQ_CUDA_CHECK(cudaMemsetAsync(skf, 0, size_t(BH) * size_t(D) * 4, s));
  if (BH == 0 || S == 0) return WQ_OK;
  const int groups = int(D / 8);
  const int rows = 256 / groups;
  const int64_t want = int64_t(sm_count()) * 8 / BH + 1;
  const int64_t strips_need = (S + rows - 1) / rows;
  const int strips = int(strips_need < want ? strips_need : want);
  const dim3 ga(unsigned(strips > 65535 ? 65535 : strips), unsigned(BH));
  const int block = groups * rows;
  const int64_t n8 = BH * S * D / 8;
  int* st = status_ptr();
  auto* am = reinterpret_cast<unsigned*>(skf);
  auto* q8 = static_cast<int8_t*>(qk);
#define WQ_KV(T)                                                                               \
  do {                                                                                         \
    wq::kv_k_absmax_kernel<T><<<ga, block, 0, s>>>(static_cast<const T*>(Kc), S, int(D), am,  \
                                                   st);                                        \
    wq::kv_k_scale_kernel<<<grid_for(BH * D, 256), 256, 0, s>>>(skf, BH * D);                  \
    wq::kv_k_quant_kernel<T><<<grid_for(n8, 256), 256, 0, s>>>(static_cast<const T*>(Kc), S,   \
                                                               int(D), skf, q8, n8);           \
  } while (0)
  switch (dtype) {
    case WQ_F32: WQ_KV(float); break;
    case WQ_BF16: WQ_KV(__nv_bfloat16); break;
    case WQ_F16: WQ_KV(__half); break;
    default: return WQ_ERR_ARG;
  }
#undef WQ_KV
  WQ_LAUNCH_CHECK("kv_k_quant_kernel");
  // V: one scale per token row of D elements
  const int64_t vrows = BH * S;
  const int lpr = int(D / 8);
  if ((lpr & (lpr - 1)) != 0)  // head dims that are not 8 x a power of two
    return launch_quantize_rows_i8(Vc, dtype, vrows, D, true, nullptr, qv, sv, s);
  const int64_t warps_needed = (vrows * lpr + 31) / 32;
  const int vgrid = grid_for(warps_needed * 32, 256);
  auto* qvo = static_cast<int8_t*>(qv);
  auto* svo = static_cast<float*>(sv);
#define WQ_KVV(T, L)                                                                             \
  case L:                                                                                        \
    wq::kv_v_quant_kernel<T, L><<<vgrid, 256, 0, s>>>(static_cast<const T*>(Vc), vrows, qvo, svo, \
                                                      st);                                       \
    break;
#define WQ_KVV_ALL(T)                                                                  \
  switch (lpr) {                                                                       \
    WQ_KVV(T, 1) WQ_KVV(T, 2) WQ_KVV(T, 4) WQ_KVV(T, 8) WQ_KVV(T, 16) WQ_KVV(T, 32) \
    default: return WQ_ERR_ARG;                                                        \
  }
  switch (dtype) {
    case WQ_F32: WQ_KVV_ALL(float); break;
    case WQ_BF16: WQ_KVV_ALL(__nv_bfloat16); break;
    default: WQ_KVV_ALL(__half); break;
  }
#undef WQ_KVV_ALL
#undef WQ_KVV
  WQ_LAUNCH_CHECK("kv_v_quant_kernel");
  return WQ_OK;
}

int launch_smooth_scales(const float* act, const float* w, int64_t K, float alpha, float* out,
                         cudaStream_t s) {
  wq::smooth_scales_kernel<<<grid_for(K, 256), 256, 0, s>>>(act, w, K, double(alpha), out);
  WQ_LAUNCH_CHECK("smooth_scales_kernel");
  return WQ_OK;
}

int launch_dequant_int4(const void* codes, const void* scales, const void* zeros, int64_t N,
                        int64_t K, int gs, int sym, void* out, int out_dtype, cudaStream_t s) {
  const int grid = grid_for(N * (K / 32), 256);
  auto* c = static_cast<const uint8_t*>(codes);
  auto* sc = static_cast<const __half*>(scales);
  auto* z = static_cast<const __half*>(zeros);
  if (out_dtype == WQ_F32)
    wq::dequant_int4_kernel<float><<<grid, 256, 0, s>>>(c, sc, z, N, K, gs, sym,
                                                        static_cast<float*>(out));
  else
    wq::dequant_int4_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        c, sc, z, N, K, gs, sym, static_cast<__nv_bfloat16*>(out));
  WQ_LAUNCH_CHECK("dequant_int4_kernel");
  return WQ_OK;
}

int launch_dequant_int8_rows(const void* q, const void* scales, int64_t N, int64_t K, void* out,
                             int out_dtype, cudaStream_t s) {
  const int grid = grid_for(N * (K / 16), 256);
  auto* qi = static_cast<const int8_t*>(q);
  auto* sc = static_cast<const float*>(scales);
  if (out_dtype == WQ_F32)
    wq::dequant_int8_rows_kernel<float><<<grid, 256, 0, s>>>(qi, sc, N, K,
                                                             static_cast<float*>(out));
  else
    wq::dequant_int8_rows_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        qi, sc, N, K, static_cast<__nv_bfloat16*>(out));
  WQ_LAUNCH_CHECK("dequant_int8_rows_kernel");
  return WQ_OK;
}

}  // namespace wq_host
