// gptq.cu -- GPTQ INT4 group-wise quantization with error feedback
// ("27届大模型面试准备（十九）…" sec. 4.3).
//
// Columns (input dims) are quantized in order; each column's rounding error,
// divided by U[i, i], is pushed into the columns not yet quantized with
// weights U[i, j], where U is the upper Cholesky factor of the damped inverse
// Hessian (H^-1 = U^T U, H = 2 X^T X + damp mean(diag H) I from calibration
// activations; the caller supplies U).  At every group start the group's
// scale (and zero point) come from the corrected weights by the same rules as
// the round-to-nearest quantizer.  Output: the packed codes / fp16 scales /
// fp16 zeros of wq_quantize_pack, usable by the W4A16 products as they are.
//
// Rows are independent.  A CTA owns RB = 32 rows and walks the K columns in
// 128-wide groups, in binary64 (the quantization decision itself is the
// binary32 rule of the round-to-nearest quantizer):
//   1. block update: the group's corrected weights
//        wv[r, j] = W[r, j] - sum_{i < group start} err[r, i] U[i, j]
//      as a shared-memory-tiled product of the errors of the earlier groups
//      (kept in the caller's workspace) with the matching blocks of U;
//   2. group parameters from wv, by the round-to-nearest rules;
//   3. the 128 columns in order: eight lanes per row sum the in-group
//      correction, the row's first lane quantizes and stores err[r, j].
#include "common.cuh"
#include "kernels.h"

namespace wq {
namespace gptq {

constexpr int RB = 32;      // rows per CTA
constexpr int GS = 128;     // group size = column block
constexpr int THREADS = 256;
constexpr int LPR = THREADS / RB;  // 8 lanes per row
constexpr int CPT = GS / LPR;      // 16 columns per thread in the block update

// Shared memory: U block [128][129] (rows padded by one double so that the
// eight lanes of a row, reading entries 128 rows apart, hit distinct banks),
// E block [32][129], corrected weights [32][129].
constexpr int LD = GS + 1;
constexpr size_t SMEM_BYTES = size_t(GS) * LD * 8 + size_t(RB) * LD * 8 * 2;

// The round-to-nearest group rules on binary32 values (sym: s = amax / 7;
// asym: s = (max - min) / 15, z = clamp(round(-min / s), 0, 15); the scale
// rounded to fp16 and that value used; degenerate groups code 0).
__device__ __forceinline__ void group_rules(float amax, float mn, float mx, int sym,
                                            __half* s16, int* z, bool* degenerate) {
  if (sym) {
    __half h = __float2half_rn(div_rn(amax, 7.f));
    *degenerate = amax < 1e-8f || __half2float(h) == 0.f;
    if (*degenerate) h = __float2half_rn(amax);
    *s16 = h;
    *z = 0;
  } else {
    const float range = mx - mn;
    __half h = __float2half_rn(div_rn(range, 15.f));
    *degenerate = range < 1e-8f || __half2float(h) == 0.f;
    if (*degenerate) {
      *s16 = __float2half_rn(1.f);
      *z = 0;
    } else {
      *s16 = h;
      const float zr = round_even(div_rn(-mn, __half2float(h)));
      *z = int(fmaxf(0.f, fminf(15.f, zr)));
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(THREADS, 1)
    gptq_kernel(const T* __restrict__ W, int N, int K, const double* __restrict__ U, int sym,
                uint8_t* __restrict__ codes, __half* __restrict__ scales,
                __half* __restrict__ zeros, double* __restrict__ err, int* status) {
  extern __shared__ double smem[];
  double* Us = smem;                  // [GS][LD]
  double* Es = Us + GS * LD;          // [RB][LD]
  double* Ws = Es + RB * LD;          // [RB][LD]
  const int t = threadIdx.x;
  const int r = t / LPR, l8 = t % LPR;  // row within the CTA, lane within the row
  const int n = blockIdx.x * RB + r;
  const bool row_in = n < N;
  const int G = K / GS;
  const int qmin = sym ? -8 : 0, qmax = sym ? 7 : 15;
  bool bad = false;

  for (int g = 0; g < G; ++g) {
    const int j0 = g * GS;
    // ---- 1. block update from the earlier groups' errors
    double c[CPT];
#pragma unroll
    for (int q = 0; q < CPT; ++q) c[q] = 0.0;
    for (int p = 0; p < g; ++p) {
      __syncthreads();
      for (int i = t; i < GS * GS / 2; i += THREADS) {   // U[p block, g block], 16-byte loads
        const int a = i / (GS / 2), b = (i % (GS / 2)) * 2;
        const double2 v = *reinterpret_cast<const double2*>(U + size_t(p * GS + a) * K + j0 + b);
        Us[a * LD + b] = v.x;
        Us[a * LD + b + 1] = v.y;
      }
      for (int i = t; i < RB * GS / 2; i += THREADS) {   // err[rows, p block]
        const int a = i / (GS / 2), b = (i % (GS / 2)) * 2;
        const int na = blockIdx.x * RB + a;
        double2 v = make_double2(0.0, 0.0);
        if (na < N) v = *reinterpret_cast<const double2*>(err + size_t(na) * K + p * GS + b);
        Es[a * LD + b] = v.x;
        Es[a * LD + b + 1] = v.y;
      }
      __syncthreads();
      for (int i = 0; i < GS; ++i) {
        const double e = Es[r * LD + i];
#pragma unroll
        for (int q = 0; q < CPT; ++q) c[q] = fma(e, Us[i * LD + l8 + LPR * q], c[q]);
      }
    }
    // ---- corrected group values and the group's parameters
    float amax = 0.f, mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      const int j = l8 + LPR * q;
      const double w0 = row_in ? double(to_f32<T>(W[size_t(n) * K + j0 + j])) : 0.0;
      const double wv = w0 - c[q];
      Ws[r * LD + j] = wv;
      const float f = float(wv);
      bad |= !isfinite(f);
      amax = fmaxf(amax, fabsf(f));
      mn = fminf(mn, f);
      mx = fmaxf(mx, f);
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) {
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    __half s16;
    int z;
    bool degenerate;
    group_rules(amax, mn, mx, sym, &s16, &z, &degenerate);
    const float sf = __half2float(s16);
    if (l8 == 0 && row_in) {
      const int Gn = K / GS;
      scales[size_t(n) * Gn + g] = s16;
      if (!sym) zeros[size_t(n) * Gn + g] = __float2half_rn(float(z));
      if (isinf(sf)) bad = true;
    }
    // ---- 2. the group's own columns, in order
    __syncthreads();  // every warp is done with Us / Es of the block update
    for (int i = t; i < GS * GS / 2; i += THREADS) {     // U diagonal block
      const int a = i / (GS / 2), b = (i % (GS / 2)) * 2;
      const double2 v = *reinterpret_cast<const double2*>(U + size_t(j0 + a) * K + j0 + b);
      Us[a * LD + b] = v.x;
      Us[a * LD + b + 1] = v.y;
    }
    __syncthreads();
    uint32_t packed = 0;  // the row's first lane assembles 8 nibbles per word
    for (int j = 0; j < GS; ++j) {
      double part = 0.0;
      for (int i = l8; i < j; i += LPR) part = fma(Es[r * LD + i], Us[i * LD + j], part);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (l8 == 0) {
        const double w = Ws[r * LD + j] - part;
        int q = 0;
        double w_hat = 0.0;
        if (!degenerate) {
          float rr = round_even(div_rn(float(w), sf));
          rr = fmaxf(-64.f, fminf(64.f, rr));
          q = min(max(int(rr) + z, qmin), qmax);
          w_hat = double(sf) * double(q - (sym ? 0 : z));
        }
        Es[r * LD + j] = (w - w_hat) / Us[j * LD + j];
        packed |= uint32_t(q - qmin) << (4 * (j & 7));
        if ((j & 7) == 7) {
          if (row_in)
            *reinterpret_cast<uint32_t*>(codes + size_t(n) * (K / 2) + (j0 + j - 7) / 2) = packed;
          packed = 0;
        }
      }
      __syncwarp();
    }
    // this group's errors, for the block updates of the later groups
    if (row_in)
      for (int j = l8; j < GS; j += LPR) err[size_t(n) * K + j0 + j] = Es[r * LD + j];
    __syncthreads();
  }
  if (bad) record_error(status, WQ_ERR_NONFINITE);
}

}  // namespace gptq
}  // namespace wq

namespace wq_host {

size_t gptq_workspace_bytes(int64_t N, int64_t K) { return size_t(N) * size_t(K) * 8; }

int launch_gptq(const void* W, int w_dtype, int64_t N, int64_t K, const double* U, int sym,
                void* codes, void* scales, void* zeros, void* ws, cudaStream_t s) {
  using namespace wq::gptq;
  static bool attr_done[3][64] = {};
  int dev = 0;
  WQ_CUDA_CHECK(cudaGetDevice(&dev));
  const dim3 grid(unsigned((N + RB - 1) / RB));
  auto* c = static_cast<uint8_t*>(codes);
  auto* sc = static_cast<__half*>(scales);
  auto* zp = static_cast<__half*>(zeros);
  auto* e = static_cast<double*>(ws);
  int* st = status_ptr();
#define WQ_GPTQ(T, I)                                                                      \
  do {                                                                                     \
    if (dev < 64 && !attr_done[I][dev]) {                                                  \
      WQ_CUDA_CHECK(cudaFuncSetAttribute(gptq_kernel<T>,                                   \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,      \
                                         int(SMEM_BYTES)));                                \
      attr_done[I][dev] = true;                                                            \
    }                                                                                      \
    gptq_kernel<T><<<grid, THREADS, SMEM_BYTES, s>>>(static_cast<const T*>(W), int(N),    \
                                                     int(K), U, sym, c, sc, zp, e, st);    \
  } while (0)
  switch (w_dtype) {
    case WQ_F32: WQ_GPTQ(float, 0); break;
    case WQ_BF16: WQ_GPTQ(__nv_bfloat16, 1); break;
    case WQ_F16: WQ_GPTQ(__half, 2); break;
    default: return WQ_ERR_ARG;
  }
#undef WQ_GPTQ
  WQ_LAUNCH_CHECK("gptq_kernel");
  return WQ_OK;
}

}  // namespace wq_host
