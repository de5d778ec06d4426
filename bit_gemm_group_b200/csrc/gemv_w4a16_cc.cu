// gemv_w4a16_cc.cu -- W4A16 decode product for one to four activation rows on
// the CUDA cores.
//
//   Y[m, n] = sum_g s[n, g] * sum_{k in g} X[m, k] * (u[n, k] - z[n, g])
//
// ("大模型面试准备（十九）…" sec. 1.2: a decode token reads every weight once,
// about 4 FLOP per weight byte at INT4, so the product is bound by HBM
// bandwidth; sec. 2.3 W4A16; "大模型量化技术定义与主流方案解析" sec. 四: the
// weight is expanded inside the product and never written back.)
//
// At M <= 4 the arithmetic per weight byte is small enough for the CUDA cores,
// and a streaming kernel keeps every SM's loads in flight from its first cycle
// to its last, with none of the tensor-core path's hand-offs between warps.
//
// Exact integer inner products.  Each CTA first rewrites X per (row m, group
// g) as integers x' = rint(x * 2^e), e chosen so that the group's largest |x|
// lands in [2^12, 2^13) (bf16 values down to 2^-5 of the group maximum are
// integers there already; smaller ones lose bits, at most 2^-13 of the
// maximum each).  x' = 128 h + l with h in [-64, 64] and l in [0, 127]
// gives two int8 limbs.  A 32-bit code word holds elements e0..e7 (low nibble
// of byte b = e_2b): w & 0x0F0F0F0F holds the even elements as bytes and
// (w >> 4) & 0x0F0F0F0F the odd ones, so four DP4A instructions take the word
// against the limbs of X.  Per lane (32 elements of one group) the sum
//   sum (u - z) x' = 128 sum u h + sum u l - z sum x'
// is exact in int32 (below 2^22), and only s * 2^-e * (that) is rounded, in
// fp32, when it is accumulated.
//
// Work split.  An item is (block of R = 4 weight rows, 1024-wide K chunk);
// lane l of a warp takes elements [32 l, 32 l + 32) of the chunk, i.e. 16
// coalesced bytes of codes per row.  CTA c of the P-CTA grid (one per SM)
// owns row blocks [c NB / P, (c + 1) NB / P), so SMs differ by at most one row
// block; its I_c items, numbered row-block-major, are split into 16 equal
// contiguous ranges, one per warp.  A row block that one warp covers entirely
// is written straight to Y; the partial sums of the (at most 16) row blocks
// that straddle two warps' ranges go to shared memory and are added in warp
// order after the CTA's barrier (deterministic, no global atomics).
//
// Data movement.  Codes land through a per-warp ring of D items in shared
// memory (cp.async, 16 bytes per lane and row); each lane reads back exactly
// the bytes it copied, so the only synchronisation is the lane's own
// cp.async group count, and D - 1 items per warp are in flight while one is
// computed.  The CTA prepares X for all K while the first items stream in and
// keeps it in shared memory in lane order, so every read of it is a
// conflict-free 16-byte load.
#include "common.cuh"
#include "kernels.h"

namespace wq {
namespace gemv_cc {

constexpr int THREADS = 512;
constexpr int WARPS = THREADS / 32;
constexpr int CHUNK = 1024;               // K elements per item: 32 per lane
constexpr int R = 4;                      // weight rows per item
constexpr int ITEM_BYTES = R * CHUNK / 2; // codes of one item (2 KB)
constexpr int MAXD = 6;
constexpr int SMEM_LIMIT = 227 * 1024;
constexpr int MT_MAX = 4;

// sum of the four byte products a_i * b_i plus c; a unsigned, b signed bytes
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t pack_bytes(int b0, int b1, int b2, int b3) {
  return (uint32_t(b0) & 0xFFu) | ((uint32_t(b1) & 0xFFu) << 8) | ((uint32_t(b2) & 0xFFu) << 16) |
         (uint32_t(b3) << 24);
}
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(d), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ X prep
// The CTA's threads rewrite X [M, K] bf16 into shared memory, one 8-element
// block (row m, elements 8 kb .. 8 kb + 7) per thread and round; the 16 blocks
// of a group sit in one half-warp and the 4 blocks of a lane's 32 elements in
// one quad.  Block (q, l) of chunk c -- elements c * CHUNK + 32 l + 8 q .. --
// becomes 16 bytes {even h, even l, odd h, odd l} (limb bytes of elements
// 0, 2, 4, 6 and 1, 3, 5, 7) at xs[(m C + c) 128 + 32 q + l]; sx[(m C + c) 32
// + l] = the lane's sum of x'; inv[m G + g] = 2^-e.
__device__ __forceinline__ void prepare_x(const __nv_bfloat16* __restrict__ X, int M, int K,
                                          int C, uint4* __restrict__ xs, int* __restrict__ sx,
                                          float* __restrict__ invs) {
  const int kb8 = K / 8;
  const int total = M * kb8;
  for (int base = 0; base < total; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const bool act = i < total;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (act) v = __ldg(reinterpret_cast<const uint4*>(X) + i);
    float x[8];
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      x[2 * r] = __uint_as_float(wv[r] << 16);
      x[2 * r + 1] = __uint_as_float(wv[r] & 0xFFFF0000u);
    }
    float amax = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) amax = fmaxf(amax, fabsf(x[r]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    // amax in [2^(E-127), 2^(E-126)) for its biased exponent E; 2^e puts it
    // in [2^12, 2^13).  A zero (or subnormal) group takes the largest step.
    const int E = int(__float_as_uint(amax) >> 23);
    const int e = max(min(139 - E, 126), -126);
    const float sc = __uint_as_float(uint32_t(127 + e) << 23);
    int xi[8], hi[8], lo[8], sum = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      xi[r] = __float2int_rn(x[r] * sc);  // |xi| <= 2^13
      hi[r] = xi[r] >> 7;                 // floor: xi = 128 hi + lo, lo in [0, 127]
      lo[r] = xi[r] & 127;
      sum += xi[r];
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    if (act) {
      const int m = i / kb8, kb = i - m * kb8;
      const int c = kb >> 7, l = (kb >> 2) & 31, q = kb & 3;
      uint4 o;
      o.x = pack_bytes(hi[0], hi[2], hi[4], hi[6]);
      o.y = pack_bytes(lo[0], lo[2], lo[4], lo[6]);
      o.z = pack_bytes(hi[1], hi[3], hi[5], hi[7]);
      o.w = pack_bytes(lo[1], lo[3], lo[5], lo[7]);
      xs[(m * C + c) * 128 + q * 32 + l] = o;
      if (q == 0) sx[(m * C + c) * 32 + l] = sum;
      if ((threadIdx.x & 15) == 0) invs[i >> 4] = __uint_as_float(uint32_t(127 - e) << 23);
    }
  }
}

// ------------------------------------------------------------------ product
struct Shape {
  int M, N, K, G, C, NB;  // NB = row blocks, C = chunks per row
  int sym;
};

// Position of an item: row block b, chunk c.
struct Pos {
  int b, c;
  __device__ __forceinline__ void next(int C) {
    if (++c == C) {
      c = 0;
      ++b;
    }
  }
};

// Copies the codes of the item at p (when `live`) into ring slot `slot` and
// closes one cp.async group (an empty one otherwise).  Items whose R rows all
// exist take the path without per-row checks.
__device__ __forceinline__ void issue_item(uint4* __restrict__ ring_w, int slot,
                                           const uint8_t* __restrict__ codes, Pos p, bool live,
                                           const Shape& sh, int lane) {
  const int k = p.c * CHUNK + lane * 32;
  if (live && k < sh.K) {
    const size_t rowb = size_t(sh.K >> 1);
    const uint8_t* src = codes + size_t(p.b * R) * rowb + (k >> 1);
    uint4* dst = ring_w + slot * (R * 32) + lane;
    if (p.b * R + R <= sh.N) {
#pragma unroll
      for (int r = 0; r < R; ++r) cp_async16(dst + r * 32, src + r * rowb);
    } else {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (p.b * R + r < sh.N) cp_async16(dst + r * 32, src + r * rowb);
    }
  }
  cp_async_commit();
}

// Scales (as fp32) and zero points (as integers) of one item for its R rows.
struct ItemSZ {
  float s[R];
  int z[R];
};

// Loads v for the item at p when `live` (a lane past K, or a row past N,
// keeps what it had: its values are never used).  Zero points are loaded only
// for asymmetric weights; symmetric ones keep z = 8.
__device__ __forceinline__ void load_sz(ItemSZ& v, const __half* __restrict__ scales,
                                        const __half* __restrict__ zeros, Pos p, bool live,
                                        const Shape& sh, int lane) {
  const int k = p.c * CHUNK + lane * 32;
  if (!live || k >= sh.K) return;
  const size_t gi = size_t(p.b * R) * size_t(sh.G) + (k >> 7);
  const __half* sp = scales + gi;
  const __half* zp = zeros + gi;
  if (p.b * R + R <= sh.N) {
#pragma unroll
    for (int r = 0; r < R; ++r) v.s[r] = __half2float(__ldg(sp + r * sh.G));
    if (!sh.sym) {
#pragma unroll
      for (int r = 0; r < R; ++r) v.z[r] = __half2int_rn(__ldg(zp + r * sh.G));
    }
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (p.b * R + r < sh.N) {
        v.s[r] = __half2float(__ldg(sp + r * sh.G));
        if (!sh.sym) v.z[r] = __half2int_rn(__ldg(zp + r * sh.G));
      }
  }
}

template <int MT>
__device__ __forceinline__ void compute_item(const uint4* __restrict__ words, const ItemSZ& v,
                                             float (&acc)[R][MT], const uint4* __restrict__ xs,
                                             const int* __restrict__ sx,
                                             const float* __restrict__ invs, int c,
                                             const Shape& sh, int lane) {
  const int k = c * CHUNK + lane * 32;
  if (k >= sh.K) return;
  const int g = k >> 7;
  uint4 wr[R];
#pragma unroll
  for (int r = 0; r < R; ++r) wr[r] = words[r * 32];
  int ah[R][MT], al[R][MT];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) ah[r][m] = al[r][m] = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t ev[R], od[R];  // even / odd elements of word q as bytes, per row
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint32_t w = q == 0 ? wr[r].x : q == 1 ? wr[r].y : q == 2 ? wr[r].z : wr[r].w;
      ev[r] = w & 0x0F0F0F0Fu;
      od[r] = (w >> 4) & 0x0F0F0F0Fu;
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < sh.M) {
        const uint4 xq = xs[(m * sh.C + c) * 128 + q * 32 + lane];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          ah[r][m] = dp4a_us(ev[r], xq.x, ah[r][m]);
          al[r][m] = dp4a_us(ev[r], xq.y, al[r][m]);
          ah[r][m] = dp4a_us(od[r], xq.z, ah[r][m]);
          al[r][m] = dp4a_us(od[r], xq.w, al[r][m]);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m < sh.M) {
      const int sxl = sx[(m * sh.C + c) * 32 + lane];
      const float fi = invs[m * sh.G + g];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int t = ah[r][m] * 128 + al[r][m] - v.z[r] * sxl;  // exact
        acc[r][m] = fmaf(float(t), v.s[r] * fi, acc[r][m]);
      }
    }
  }
}

// The warp's sums for row block b: Y directly when the warp covered all of
// it, else a partial in the warp's shared-memory slot (0: the warp's first
// row block, 1: its last).
template <int MT>
__device__ __forceinline__ void emit_block(float (&acc)[R][MT], int b, bool whole, int slot,
                                           float* __restrict__ part_w,
                                           __nv_bfloat16* __restrict__ Y, const Shape& sh,
                                           int lane) {
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v = acc[r][m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[r][m] = 0.f;
      if (lane == 0) {
        if (whole) {
          if (m < sh.M && b * R + r < sh.N) Y[size_t(m) * sh.N + b * R + r] = __float2bfloat16_rn(v);
        } else {
          part_w[(slot * R + r) * MT_MAX + m] = v;
        }
      }
    }
}

// Shared memory: [ring: 16 warps x D x R x 32 lanes x 16 B][X limbs: M C 128 x 16 B]
//                [lane sums: M C 32 ints][2^-e: M G floats][partials: 16 x 2 x R x 2 floats]
template <int MT, int D>
__global__ void __launch_bounds__(THREADS, 1) gemv_cc_kernel(
    const __nv_bfloat16* __restrict__ X, const uint8_t* __restrict__ codes,
    const __half* __restrict__ scales, const __half* __restrict__ zeros,
    __nv_bfloat16* __restrict__ Y, Shape sh) {
  extern __shared__ uint4 smem[];
  uint4* ring = smem;
  uint4* xs = smem + WARPS * D * R * 32;
  int* sx = reinterpret_cast<int*>(xs + sh.M * sh.C * 128);
  float* invs = reinterpret_cast<float*>(sx + sh.M * sh.C * 32);
  float* part = invs + sh.M * sh.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* ring_w = ring + warp * (D * R * 32);

  // this CTA's row blocks and items; warp j takes items [s_j, s_{j+1})
  const int rb0 = int((int64_t(blockIdx.x) * sh.NB) / gridDim.x);
  const int rb1 = int((int64_t(blockIdx.x + 1) * sh.NB) / gridDim.x);
  const int64_t ic = int64_t(rb1 - rb0) * sh.C;
  const int64_t s0 = (ic * warp) / WARPS, s1 = (ic * (warp + 1)) / WARPS;
  const int n_it = int(s1 - s0);
  Pos cur{rb0 + int(s0 / sh.C), int(s0 % sh.C)};
  const int b_first = cur.b;

  // A kernel launched right after this one may be scheduled as soon as SMs
  // free up; it only prefetches weights until this grid has finished.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the warp's first D items go out before anything else
  Pos ahead = cur;
#pragma unroll
  for (int d = 0; d < D; ++d) {
    issue_item(ring_w, d, codes, ahead, d < n_it, sh, lane);
    ahead.next(sh.C);
  }
  // scales and zero points run two items ahead, in two alternating sets
  ItemSZ va, vb;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    va.s[r] = vb.s[r] = 0.f;
    va.z[r] = vb.z[r] = 8;
  }
  Pos szp = cur;
  load_sz(va, scales, zeros, szp, 0 < n_it, sh, lane);
  szp.next(sh.C);
  load_sz(vb, scales, zeros, szp, 1 < n_it, sh, lane);
  szp.next(sh.C);
  // X may be the previous kernel's output, and Y its input: wait for that
  // grid (when launched as its dependent) before touching either
  asm volatile("griddepcontrol.wait;" ::: "memory");
  prepare_x(X, sh.M, sh.K, sh.C, xs, sx, invs);
  __syncthreads();

  float acc[R][MT];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;
  float* part_w = part + warp * (2 * R * MT_MAX);
  int slot = 0;
  int c_start = cur.c;  // first chunk of the current row block this warp holds
  // one item: compute it from the ring and `v`, refill its slot with the item
  // D ahead, load `v` for the item two ahead, emit finished row blocks
  auto step = [&](ItemSZ& v, int it) {
    cp_async_wait<D - 1>();  // this lane's copies of item `it` have landed
    compute_item<MT>(ring_w + slot * R * 32 + lane, v, acc, xs, sx, invs, cur.c, sh, lane);
    // refill the slot just read (its words are in registers) with item it + D
    issue_item(ring_w, slot, codes, ahead, it + D < n_it, sh, lane);
    ahead.next(sh.C);
    slot = (slot + 1 == D) ? 0 : slot + 1;
    load_sz(v, scales, zeros, szp, it + 2 < n_it, sh, lane);
    szp.next(sh.C);
    if (cur.c == sh.C - 1 || it + 1 == n_it) {
      emit_block<MT>(acc, cur.b, c_start == 0 && cur.c == sh.C - 1, cur.b == b_first ? 0 : 1,
                     part_w, Y, sh, lane);
      c_start = 0;
    }
    cur.next(sh.C);
  };
  for (int it = 0; it < n_it; it += 2) {
    step(va, it);
    if (it + 1 == n_it) break;
    step(vb, it + 1);
  }
  cp_async_wait<0>();
  __syncthreads();

  // row blocks that straddle warp ranges: sum the partials in warp order
  const int nbl = rb1 - rb0;
  for (int t = threadIdx.x; t < nbl * R * MT; t += blockDim.x) {
    const int bl = t / (R * MT), rm = t - bl * (R * MT), r = rm / MT, m = rm - r * MT;
    const int64_t f = int64_t(bl) * sh.C, l = f + sh.C - 1;  // the block's first, last item
    int jf = 0, jl = 0;
    for (int j = 1; j < WARPS; ++j) {
      const int64_t sj = (ic * j) / WARPS;
      if (sj <= f) jf = j;
      if (sj <= l) jl = j;
    }
    // jf..jl: warps whose ranges meet the block (empty ranges have no items
    // and are skipped: their start equals the next warp's)
    if (jf == jl) continue;  // one warp held all of it and wrote Y
    float v = 0.f;
    for (int j = jf; j <= jl; ++j) {
      const int64_t sj = (ic * j) / WARPS, ej = (ic * (j + 1)) / WARPS;
      if (sj == ej) continue;
      const int sl = (rb0 + int(sj / sh.C) == rb0 + bl) ? 0 : 1;
      v += part[j * (2 * R * MT_MAX) + (sl * R + r) * MT_MAX + m];
    }
    const int n = (rb0 + bl) * R + r;
    if (m < sh.M && n < sh.N) Y[size_t(m) * sh.N + n] = __float2bfloat16_rn(v);
  }
}

}  // namespace gemv_cc
}  // namespace wq

namespace wq_host {

static int64_t cc_chunks(int64_t K) { return (K + wq::gemv_cc::CHUNK - 1) / wq::gemv_cc::CHUNK; }

// Shared memory of the prepared X (limbs, lane sums, 2^-e factors) and of the
// warps' partial sums.
static size_t cc_x_smem(int64_t M, int64_t K) {
  using namespace wq::gemv_cc;
  const size_t C = size_t(cc_chunks(K));
  return size_t(M) * C * CHUNK * 2 + size_t(M) * C * 32 * 4 + size_t(M) * size_t(K / 128) * 4 +
         size_t(WARPS) * 2 * R * MT_MAX * 4;
}

int gemv_cc_depth(int64_t M, int64_t K) {
  using namespace wq::gemv_cc;
  if (M < 1 || M > kGemvCcMaxM) return 0;
  const int64_t room = int64_t(SMEM_LIMIT) - int64_t(cc_x_smem(M, K));
  const int64_t per_slot = int64_t(WARPS) * ITEM_BYTES;
  const int64_t d = room > 0 ? room / per_slot : 0;
  return d >= 2 ? int(d < MAXD ? d : MAXD) : 0;
}

template <int MT, int D>
static cudaError_t launch_cc(dim3 grid, size_t smem, cudaStream_t s, const __nv_bfloat16* X,
                             const uint8_t* codes, const __half* scales, const __half* zeros,
                             __nv_bfloat16* Y, const wq::gemv_cc::Shape& sh) {
  static bool attr_done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !attr_done[dev]) {
    e = cudaFuncSetAttribute(wq::gemv_cc::gemv_cc_kernel<MT, D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             wq::gemv_cc::SMEM_LIMIT);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  // programmatic dependent launch: the weight prefetch of this kernel
  // overlaps the tail of the kernel before it on the stream
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(wq::gemv_cc::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, wq::gemv_cc::gemv_cc_kernel<MT, D>, X, codes, scales, zeros, Y,
                            sh);
}

int launch_gemv_w4a16_cc(const void* X, int64_t M, int64_t K, const void* codes,
                         const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                         cudaStream_t s) {
  using namespace wq::gemv_cc;
  const int D = gemv_cc_depth(M, K);
  if (D == 0) return WQ_ERR_ARG;
  Shape sh;
  sh.M = int(M);
  sh.N = int(N);
  sh.K = int(K);
  sh.G = int(K / 128);
  sh.C = int(cc_chunks(K));
  sh.NB = int((N + R - 1) / R);
  sh.sym = sym;
  const int P = sm_count();
  const dim3 grid(unsigned(sh.NB < P ? sh.NB : P));
  const size_t smem = size_t(WARPS) * D * ITEM_BYTES + cc_x_smem(M, K);

  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(X);
  const __half* sc = static_cast<const __half*>(scales);
  const __half* zp = static_cast<const __half*>(zeros);
  const uint8_t* cd = static_cast<const uint8_t*>(codes);
  __nv_bfloat16* y = static_cast<__nv_bfloat16*>(Y);
  cudaError_t e = cudaErrorInvalidValue;
  const int mt = M <= 1 ? 1 : M <= 2 ? 2 : 4;  // M = 3 runs the 4-row instance
#define WQ_CC_CASE(MT_, D_) \
  if (mt == MT_ && D == D_) e = launch_cc<MT_, D_>(grid, smem, s, x, cd, sc, zp, y, sh);
  WQ_CC_CASE(1, 2) WQ_CC_CASE(1, 3) WQ_CC_CASE(1, 4) WQ_CC_CASE(1, 5) WQ_CC_CASE(1, 6)
  WQ_CC_CASE(2, 2) WQ_CC_CASE(2, 3) WQ_CC_CASE(2, 4) WQ_CC_CASE(2, 5) WQ_CC_CASE(2, 6)
  WQ_CC_CASE(4, 2) WQ_CC_CASE(4, 3) WQ_CC_CASE(4, 4) WQ_CC_CASE(4, 5) WQ_CC_CASE(4, 6)
#undef WQ_CC_CASE
  if (e != cudaSuccess) return cuda_fail(e, "gemv_cc_kernel");
  return WQ_OK;
}

}  // namespace wq_host
