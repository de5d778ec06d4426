// qmath.cuh -- element arithmetic shared by the quantizing kernels: the
// reciprocal-multiply route to IEEE-division codes, 16-bit pair unpacking and
// packed-pair maxima.
#pragma once

#include "common.cuh"

namespace wq {

// ---------------------------------------------------------------------------
// Reciprocal-multiply quantization with the IEEE-division result
// ---------------------------------------------------------------------------
// The quantizers' codes are defined by round-half-even of the binary32
// quotient fl(x / s).  One reciprocal per scale and one multiply per element
// reach the same codes: r = x * rcp(s), with rcp within one ulp of 1/s, is
// within |x/s| * 1.5 * 2^-23 of x/s, and rint(fl(x/s)) depends only on which
// side of each half-integer x/s lies.  So rint(r) is the IEEE result unless
// x/s is very close to (or exactly on) a half-integer; each kernel below
// recognises those elements and decides them exactly.

// 1/v within one ulp (a single instruction).
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// The two 16-bit floats of a 32-bit word as fp32 (element 0 = low half).
template <typename T>
__device__ __forceinline__ void unpack2(uint32_t w, float& a, float& b);
template <>
__device__ __forceinline__ void unpack2<__nv_bfloat16>(uint32_t w, float& a, float& b) {
  a = __uint_as_float(w << 16);
  b = __uint_as_float(w & 0xFFFF0000u);
}
template <>
__device__ __forceinline__ void unpack2<__half>(uint32_t w, float& a, float& b) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
  a = f.x;
  b = f.y;
}

// rint(fl(x / s)) for an INT8 code, from inv = rcp_approx(s).  Exact for
// |x/s| <= 128.5; larger quotients saturate the code either way.
__device__ __forceinline__ float rint_quot_i8(float x, float s, float inv) {
  // k = rint of the exact product x * inv (one fma with 1.5 2^23); d, the
  // residual x * inv - k rounded once, is within 2^-24 of the true one.  The
  // reciprocal is within one ulp, so x * inv is within 1.01 2^-16 of x / s,
  // and fl(x / s) within 2^-17 more: when |d| is below 0.5 - 2^-14, fl(x / s)
  // lies on k's side of the half-integers and rounds to k as well; otherwise
  // the division decides.
  const float magic = 12582912.f;  // 1.5 * 2^23
  const float k = fmaf(x, inv, magic) - magic;
  const float d = fmaf(x, inv, -k);
  if (fabsf(d) >= 0.5f - 0x1p-14f) return rintf(div_rn(x, s));
  return k;
}

// A binary32 quotient that rounds to the same E4M3 code as fl(x / s), from
// inv = rcp_approx(s).  r = x * inv is within 3 units of the binary32 last
// place of x/s, and fl(x/s) within half a unit; an E4M3 half-way point in the
// normal range has the low 20 mantissa bits 0x80000 (bit 19 alone), so when
// r's low 20 bits are more than 4 units from that pattern, r and fl(x/s) lie
// on the same side of every half-way point and round to the same code
// (powers of two, where the binade changes, are codes themselves).  Nonzero
// |r| < 2^-6 (the E4M3 subnormal range, uniform spacing 2^-9) and the rare
// near-half-way r take the division itself.
__device__ __forceinline__ float quot_e4m3(float x, float s, float inv) {
  const float r = x * inv;
  const int m20 = int(__float_as_uint(r) & 0xFFFFFu) - 0x80000;
  if ((r != 0.f && fabsf(r) < 0x1p-6f) || (m20 >= -4 && m20 <= 4)) return div_rn(x, s);
  return r;
}

// The largest |x| (sym) or the smallest and largest x (asym) of a lane's 16
// 16-bit elements, on the packed pairs.  NaN propagates (.NaN), so a lane
// with a NaN or an infinity yields a non-finite statistic.
template <typename T>
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b);
template <>
__device__ __forceinline__ uint32_t absmax2<__nv_bfloat16>(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <>
__device__ __forceinline__ uint32_t absmax2<__half>(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <typename T>
__device__ __forceinline__ uint32_t min2(uint32_t a, uint32_t b);
template <typename T>
__device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b);
template <>
__device__ __forceinline__ uint32_t min2<__nv_bfloat16>(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <>
__device__ __forceinline__ uint32_t max2<__nv_bfloat16>(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <>
__device__ __forceinline__ uint32_t min2<__half>(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.NaN.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <>
__device__ __forceinline__ uint32_t max2<__half>(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Largest magnitude of each 16-bit lane pair with NaN ignored (a NaN operand
// yields the other one) and infinities kept: the maximum the quantizers'
// scales are defined by.
template <typename T>
__device__ __forceinline__ uint32_t absmax2_skipnan(uint32_t a, uint32_t b);
template <>
__device__ __forceinline__ uint32_t absmax2_skipnan<__nv_bfloat16>(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <>
__device__ __forceinline__ uint32_t absmax2_skipnan<__half>(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// INT8 codes through the fp32 pattern of t = fl(x y + 1.5 2^23), y =
// rcp_approx(s): for |x y| < 2^22 its low byte is the two's complement of
// rint(x y), and d = fl(x y - (t - 1.5 2^23)) is that rounding's residual
// (within 2^-24 of the exact one).  rint(x y) is rint(fl(x / s)) unless x y
// lies within 2^-14 of a half-integer (x y is within 1.01 2^-16 of x / s for
// |x / s| <= 128.5, and fl(x / s) within 2^-17 of x / s).
//
// Those near-half-way elements are decided exactly without a division.  With
// k = rint(x y), sg = sign(d) and h = k + sg / 2 (the half-integer x y is
// close to), e = x - h s is exact in one fma: h has at most 9 significant
// bits, so h s and x lie on the grid of the coarser of their last places,
// and |e| < 2^-12 |x| needs fewer than 24 bits of it.  fl(x / s) = h exactly
// when |x / s - h| <= ulp(h) / 2, i.e. |e| <= s 2^(E - 24) with 2^E <= |h| <
// 2^(E+1) (the tie rounds to h, whose last significand bit is 0); rint(h) is
// then the even one of k and k + sg.  Otherwise fl(x / s) lies on the side of
// h that x / s lies on: beyond it (e of sg's sign) the code is k + sg, else
// k.  (h = 1/2 is a binade edge; both sides give code 0 there.)
__device__ __forceinline__ uint32_t code_i8_fix(float x, float s, float t, float d) {
  const float magic = 12582912.f;  // 1.5 * 2^23
  const float k = t - magic;
  const float sg = d >= 0.f ? 1.f : -1.f;
  const float h = fmaf(0.5f, sg, k);
  const float e = fmaf(-h, s, x);
  const float tol = s * __uint_as_float((__float_as_uint(h) & 0x7F800000u) - (24u << 23));
  float kk = k;
  if (fabsf(e) <= tol) {
    if (int(k) & 1) kk = k + sg;
  } else if ((e > 0.f) == (sg > 0.f)) {
    kk = k + sg;
  }
  return __float_as_uint(kk + magic);
}

// Low bytes of four words, in order, as one word.
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// INT8 codes of four elements (finite x over finite s, |x / s| <= 127.5) as
// one word, from the fp32 patterns of rint(x y) + 1.5 2^23 (y = rcp_approx(s));
// bit g of `near` is raised when one of the four lies near half-way and the
// group needs code_i8_exact.  Near-half-way elements are a few per thousand
// on real data (x = +-amax/2 puts x / s within 2^-18 of 63.5), so the caller
// stores the fast codes and then rewrites the flagged groups.
__device__ __forceinline__ uint32_t codes_i8_x4(float x0, float x1, float x2, float x3, float y0,
                                                float y1, float y2, float y3, uint32_t& near,
                                                int g) {
  const float magic = 12582912.f;
  const float t0 = fmaf(x0, y0, magic), t1 = fmaf(x1, y1, magic);
  const float t2 = fmaf(x2, y2, magic), t3 = fmaf(x3, y3, magic);
  const float d0 = fmaf(x0, y0, magic - t0), d1 = fmaf(x1, y1, magic - t1);
  const float d2 = fmaf(x2, y2, magic - t2), d3 = fmaf(x3, y3, magic - t3);
  const float m = fmaxf(fmaxf(fabsf(d0), fabsf(d1)), fmaxf(fabsf(d2), fabsf(d3)));
  if (m >= 0.5f - 0x1p-14f) near |= 1u << g;
  return low_bytes4(__float_as_uint(t0), __float_as_uint(t1), __float_as_uint(t2),
                    __float_as_uint(t3));
}

// The INT8 code rint(fl(x / s)) of one element (finite x and s, |x / s| <=
// 127.5), from y = rcp_approx(s): the fast code unless the element is near
// half-way, then code_i8_fix.
__device__ __forceinline__ int8_t code_i8_exact(float x, float s, float y) {
  const float magic = 12582912.f;
  const float t = fmaf(x, y, magic);
  const float d = fmaf(x, y, magic - t);
  const uint32_t bits = fabsf(d) >= 0.5f - 0x1p-14f ? code_i8_fix(x, s, t, d) : __float_as_uint(t);
  return int8_t(bits & 0xFFu);
}

// a[i] for a run-time i without dynamic register indexing (rare paths only).
template <typename V, int N>
__device__ __forceinline__ V pick(const V (&a)[N], int i) {
  V v = a[0];
#pragma unroll
  for (int j = 1; j < N; ++j) v = (i == j) ? a[j] : v;
  return v;
}

// The INT8 code of the per-row / per-channel quantizers with every case of
// the definition: clamp(round(x / s), -200, 200), then to [-128, 127]; a NaN
// quotient (NaN x, or an infinite x over an infinite s) gives 127.
__device__ __forceinline__ int code_i8_full(float x, float s, float y) {
  float r = rint_quot_i8(x, s, y);
  r = fmaxf(-200.f, fminf(200.f, r));
  return min(max(int(r), -128), 127);
}

}  // namespace wq
