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
// At M <= 4 there is too little arithmetic per weight byte for the tensor
// cores to help: the kernel is a stream, and what bounds it is how many issue
// slots it spends per byte and how many bytes it keeps in flight (from M = 5
// on, the multiply-adds go to the tensor cores: gemv_w4a16_mma.cu).
//
// Exact integer inner products.  X is rewritten per (activation row m,
// group g of 128 along K) as integers x' = rint(x * 2^e), e chosen so that
// the group's largest |x| lands in [2^12, 2^13): bf16 values down to 2^-5 of
// the group maximum are integers there already, smaller ones lose bits (at
// most 2^-13 of the maximum each).  x' fits in 16 bits, and a pair of them
// is one operand of DP2A.  A 32-bit code word holds elements e0..e7 (the low
// nibble of byte b is e_2b): w & 0x0F0F0F0F holds the even elements as bytes
// and w & 0xF0F0F0F0 sixteen times the odd ones, so four DP2A take the word
// against X (the odd sum is exactly divisible by 16).  A group's
//   sum (u - z) x' = sum u x' - z sum x'
// is exact in int32 (below 2^24, so also exact as a float) and only
// s * 2^-e * (that) is rounded, in fp32.
//
// Work split.  An item is (8 weight rows, one 1024-wide K chunk): 512
// contiguous bytes of codes per row, 16 per lane, lane l covering elements
// [32 l, 32 l + 32) of the chunk (a quarter of group l / 4).  CTA c of the
// one-per-SM grid owns the 4-row blocks [c NB / P, (c + 1) NB / P), so SMs
// differ by at most four rows.  Its items are numbered chunk-major (all of the
// CTA's row tiles for chunk 0, then chunk 1, ...) and split into equal
// contiguous ranges, one per warp, so a warp keeps one chunk's X in registers
// for many items and converts X only when its chunk changes.  Each item ends
// in a transposed reduction: the 4 lanes of a group exchange row sums in two
// shuffle rounds (each lane keeps 2 of the 8 rows, as exact integers), apply
// the group's scale and zero point to those, and three more rounds sum the 8
// groups of the chunk.  The chunk's partial sum of each row lands in shared
// memory; after one barrier the CTA adds a row's chunk partials in chunk
// order (deterministic, no atomics, no workspace).
//
// Data movement.  Each warp has its own ring of D item slots in shared
// memory, filled by TMA (one 2D box of 4 rows x 512 bytes per 4 rows, issued
// by one lane) that completes on the slot's mbarrier.  A warp refills a slot
// as soon as it has read its codes into registers, before computing them, so
// D items per warp are in flight almost all the time.  The launch shape
// (warps per CTA, ring depth) depends on the matrix size (cc_config).
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace wq {
namespace gemv_cc {

constexpr int CHUNK = 1024;               // K elements per item: 32 per lane
constexpr int RB = 8;                     // weight rows per item
constexpr int ROW_BYTES = CHUNK / 2;      // codes of one row of an item
constexpr int ITEM_BYTES = RB * ROW_BYTES;
constexpr int BOX_BYTES = 4 * ROW_BYTES;  // one TMA box: 4 rows of an item
constexpr int SMEM_LIMIT = 227 * 1024;
constexpr uint32_t MAGIC = 0x4B400000u;   // bit pattern of 1.5 * 2^23

// d = c + a.h0 * b.b0 + a.h1 * b.b1 (lo: bytes 0, 1 of b; hi: bytes 2, 3);
// a holds two signed 16-bit values, b four unsigned bytes
__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// elementwise max(|a|, |b|) of two bf16 pairs (the result's sign bits are
// not meaningful)
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(tc::smem_u32(p)));
  return v;
}
struct Shape {
  int M, N, K, G, C;  // G = groups per row, C = chunks per row
  int NB;             // 4-row blocks
  int rows_max;       // rows of the largest CTA range (partials stride)
  int sym;
};

// An item: chunk c, row tile t of the CTA (chunk-major order).
struct Item {
  int c, t;
  __device__ __forceinline__ void next(int T) {
    if (++t == T) {
      t = 0;
      ++c;
    }
  }
};

// Per-lane view of one chunk of X (activation rows m < MT): for each of the
// lane's 4 code words q, x' of its even elements {0, 2}, {4, 6} and odd
// elements {1, 3}, {5, 7} as 16-bit pairs; the group's sum of x' and 2^-e.
template <int MT>
struct XChunk {
  uint32_t w[MT][4][4];
  int sx[MT];
  float inv[MT];
};

template <int MT>
__device__ __forceinline__ void load_x_raw(uint4 (&xr)[MT][4], const __nv_bfloat16* __restrict__ X,
                                           int c, const Shape& sh, int lane) {
  const int k = c * CHUNK + 32 * lane;
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      xr[m][q] = make_uint4(0, 0, 0, 0);
      if (m < sh.M && k < sh.K)
        xr[m][q] = __ldg(reinterpret_cast<const uint4*>(X + size_t(m) * sh.K + k) + q);
    }
}

// Bring the lane's 64 bytes of a chunk of X into L1 ahead of its use.
template <int MT>
__device__ __forceinline__ void prefetch_x(const __nv_bfloat16* __restrict__ X, int c,
                                           const Shape& sh, int lane) {
  const int k = c * CHUNK + 32 * lane;
#pragma unroll
  for (int m = 0; m < MT; ++m)
    if (m < sh.M && k < sh.K)
      asm volatile("prefetch.global.L1 [%0];" ::"l"(X + size_t(m) * sh.K + k));
}

template <int MT>
__device__ __forceinline__ void convert_x(const uint4 (&xr)[MT][4], XChunk<MT>& xc) {
  const float magic = __uint_as_float(MAGIC);
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    uint32_t mx = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      mx = maxabs_bf16x2(mx, xr[m][q].x);
      mx = maxabs_bf16x2(mx, xr[m][q].y);
      mx = maxabs_bf16x2(mx, xr[m][q].z);
      mx = maxabs_bf16x2(mx, xr[m][q].w);
    }
    // |x| bit patterns order like the values; the group is 4 lanes
    uint32_t amax = max(mx & 0x7FFFu, (mx >> 16) & 0x7FFFu);
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    // amax in [2^(E-127), 2^(E-126)) for its biased exponent E; 2^e puts it
    // in [2^12, 2^13).  A zero (or subnormal) group takes the largest step.
    const int E = int(amax >> 7);
    const int e = max(min(139 - E, 126), -126);
    const float sc = __uint_as_float(uint32_t(127 + e) << 23);
    uint32_t sum = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t wv[4] = {xr[m][q].x, xr[m][q].y, xr[m][q].z, xr[m][q].w};
      uint32_t b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // fma rounds x * 2^e (exact) + 1.5 * 2^23 once, to the nearest
        // integer (ties to even): the bit pattern is MAGIC + x'
        b[2 * i] = __float_as_uint(fmaf(__uint_as_float(wv[i] << 16), sc, magic));
        b[2 * i + 1] = __float_as_uint(fmaf(__uint_as_float(wv[i] & 0xFFFF0000u), sc, magic));
        sum += b[2 * i] + b[2 * i + 1];
      }
      xc.w[m][q][0] = prmt(b[0], b[2], 0x5410);  // x'0, x'2
      xc.w[m][q][1] = prmt(b[4], b[6], 0x5410);  // x'4, x'6
      xc.w[m][q][2] = prmt(b[1], b[3], 0x5410);  // x'1, x'3
      xc.w[m][q][3] = prmt(b[5], b[7], 0x5410);  // x'5, x'7
    }
    int s = int(sum - 32u * MAGIC);  // the lane's sum of x' (mod 2^32, exact)
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    xc.sx[m] = s;
    xc.inv[m] = __uint_as_float(uint32_t(127 - e) << 23);
  }
}

// Scales and zero points of the 2 rows a lane finishes in an item: rows
// 2 j, 2 j + 1 (j = lane & 3) of group lane / 4 of the chunk, kept as the
// raw fp16 bits (converted only where they are used, so that the loads stay
// in flight until then: no instruction may consume them at load time).  Rows outside the CTA's range and groups past K get
// s = 0.
struct SZ {
  unsigned short s[2], z[2];
};

__device__ __forceinline__ void load_sz(SZ& v, const __half* __restrict__ scales,
                                        const __half* __restrict__ zeros, Item p, bool live,
                                        int row0, int row1, const Shape& sh, int lane) {
  if (!live) return;
  const int g = p.c * (CHUNK / 128) + (lane >> 2);
  const int r = row0 + p.t * RB + 2 * (lane & 3);
  const unsigned short* sp = reinterpret_cast<const unsigned short*>(scales);
  const unsigned short* zp = reinterpret_cast<const unsigned short*>(zeros);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    v.s[k] = 0;       // +0.0
    v.z[k] = 0x4800;  // 8.0: the symmetric code offset
    if (r + k < row1 && g < sh.G) {
      const size_t i = size_t(r + k) * sh.G + g;
      v.s[k] = __ldg(sp + i);
      if (!sh.sym) v.z[k] = __ldg(zp + i);
    }
  }
}

// Issue the TMA loads of item p into a ring slot: one box of 4 rows x 512
// bytes per 4 rows (the rows of a CTA come in multiples of 4; a chunk past K
// reads zeros).  One lane issues them: a tensor copy takes warp-uniform
// operands, so a single issuing lane needs no per-lane serialisation.
__device__ __forceinline__ void issue_item(uint8_t* slot, uint64_t* bar, const CUtensorMap* tmap,
                                           Item p, int row0, int row1, int lane) {
  if (lane == 0) {
    const int r0 = row0 + p.t * RB;
    const int boxes = min(RB, row1 - r0) / 4;
    tc::mbar_arrive_expect_tx(bar, uint32_t(boxes) * BOX_BYTES);
    tc::tma_load_2d(slot, tmap, bar, p.c * (ROW_BYTES / 4), r0);
    if (boxes > 1) tc::tma_load_2d(slot + BOX_BYTES, tmap, bar, p.c * (ROW_BYTES / 4), r0 + 4);
  }
}

// Bounded wait of the whole warp on a slot's mbarrier; false (and the error
// recorded) when the deadline passed.
__device__ __forceinline__ bool wait_slot(uint64_t* bar, uint32_t parity, uint64_t deadline,
                                          int* status) {
  bool ok = tc::mbar_try_wait(bar, parity);
  uint32_t spins = 0;
  while (!ok) {
    ok = tc::mbar_try_wait(bar, parity);
    if (!ok && (++spins & 31u) == 0 && tc::globaltimer_ns() > deadline) break;
  }
  const bool all = __all_sync(0xffffffffu, ok);
  if (!all && (threadIdx.x & 31) == 0) record_error(status, WQ_ERR_TIMEOUT);
  return all;
}

// Shared memory: [ring: W x D x ITEM_BYTES][mbarriers: W x D]
//                [chunk partials: rows_max x C x MT floats]
template <int MT, int D, int W>
__global__ void __launch_bounds__(W * 32, (W <= 8 && MT <= 2) ? 2 : 1)
    gemv_cc_kernel(const __grid_constant__ CUtensorMap tmap, const __nv_bfloat16* __restrict__ X,
                   const __half* __restrict__ scales, const __half* __restrict__ zeros,
                   __nv_bfloat16* __restrict__ Y, Shape sh, int* status, uint64_t wait_ns) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring_w = smem + size_t(warp) * D * ITEM_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(W) * D * ITEM_BYTES) + warp * D;
  float* part = reinterpret_cast<float*>(smem + size_t(W) * D * ITEM_BYTES +
                                         size_t(W) * D * sizeof(uint64_t));

  // this CTA's rows, row tiles and items; warp w takes items [s_w, s_{w+1})
  const int row0 = 4 * int(int64_t(blockIdx.x) * sh.NB / gridDim.x);
  const int row1 = min(4 * int(int64_t(blockIdx.x + 1) * sh.NB / gridDim.x), sh.N);
  const int T = (row1 - row0 + RB - 1) / RB;
  const int64_t I = int64_t(T) * sh.C;
  const int64_t s0 = I * warp / W, s1 = I * (warp + 1) / W;
  const int n_it = int(s1 - s0);
  Item cur{int(s0 / T), int(s0 % T)};

  if (lane == 0) {
#pragma unroll
    for (int d = 0; d < D; ++d) tc::mbar_init(bars + d, 1);
    tc::fence_mbar_init();
    tc::tma_prefetch_desc(&tmap);
  }
  __syncwarp();
  // The next kernel on the stream may be scheduled as soon as SMs have room;
  // it only prefetches weights until this grid has finished.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint64_t deadline = tc::globaltimer_ns() + wait_ns;

  // the warp's first D items go out before anything else
  Item ahead = cur;
#pragma unroll
  for (int d = 0; d < D; ++d) {
    if (d < n_it) issue_item(ring_w + d * ITEM_BYTES, bars + d, &tmap, ahead, row0, row1, lane);
    ahead.next(T);
  }
  // scales and zero points run two items ahead, in two alternating sets
  SZ va, vb;
  Item szp = cur;
  load_sz(va, scales, zeros, szp, 0 < n_it, row0, row1, sh, lane);
  szp.next(T);
  load_sz(vb, scales, zeros, szp, 1 < n_it, row0, row1, sh, lane);
  szp.next(T);

  // X may be the previous kernel's output, and Y its input: wait for that
  // grid (when launched as its dependent) before touching either
  asm volatile("griddepcontrol.wait;" ::: "memory");

  XChunk<MT> xc;
  int xchunk = -1;
  int slot = 0;
  uint32_t parity = 0;
  bool ok = true;
  int done = 0;  // items whose slot wait has completed

  auto step = [&](SZ& v, int it) {
    if (cur.c != xchunk) {
      uint4 xr[MT][4];
      load_x_raw<MT>(xr, X, cur.c, sh, lane);
      convert_x<MT>(xr, xc);
      xchunk = cur.c;
    }
    Item nx = cur;
    nx.next(T);
    // the next chunk's X is brought into L1 one item before it is needed
    if (it + 1 < n_it && nx.c != cur.c) prefetch_x<MT>(X, nx.c, sh, lane);

    ok = wait_slot(bars + slot, parity, deadline, status);
    if (!ok) return;
    ++done;
    const uint8_t* sb = ring_w + slot * ITEM_BYTES + lane * 16;
    uint4 w4[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) w4[r] = lds128(sb + r * ROW_BYTES);
    // The slot's codes are read (the warp barrier orders every lane's reads
    // before the copies that overwrite them): refill it with the item D
    // ahead before computing, so that D items per warp stay in flight.
    __syncwarp();
    if (it + D < n_it)
      issue_item(ring_w + slot * ITEM_BYTES, bars + slot, &tmap, ahead, row0, row1, lane);
    ahead.next(T);
    if (++slot == D) {
      slot = 0;
      parity ^= 1u;
    }

    int tr[RB][MT];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const uint32_t wv[4] = {w4[r].x, w4[r].y, w4[r].z, w4[r].w};
      int ae[MT], ao[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) ae[m] = ao[m] = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t ev = wv[q] & 0x0F0F0F0Fu;  // u of elements 0, 2, 4, 6
        const uint32_t od = wv[q] & 0xF0F0F0F0u;  // 16 u of elements 1, 3, 5, 7
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          ae[m] = dp2a_lo(xc.w[m][q][0], ev, ae[m]);
          ae[m] = dp2a_hi(xc.w[m][q][1], ev, ae[m]);
          ao[m] = dp2a_lo(xc.w[m][q][2], od, ao[m]);
          ao[m] = dp2a_hi(xc.w[m][q][3], od, ao[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) tr[r][m] = ae[m] + (ao[m] >> 4);  // exact
    }

    // 4 lanes of a group: lane j keeps rows 2 j, 2 j + 1 (exact integers)
    const bool b1 = lane & 2, b0 = lane & 1, b2 = lane & 4;
    int u4[4][MT];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int keep = b1 ? tr[4 + k][m] : tr[k][m];
        const int send = b1 ? tr[k][m] : tr[4 + k][m];
        u4[k][m] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
    float p[2][MT];
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int keep = b0 ? u4[2 + k][m] : u4[k][m];
        const int send = b0 ? u4[k][m] : u4[2 + k][m];
        const int zk = __half2int_rn(__ushort_as_half(v.z[k]));
        const int t = keep + __shfl_xor_sync(0xffffffffu, send, 1) - zk * xc.sx[m];
        p[k][m] = (float(t) * __half2float(__ushort_as_half(v.s[k]))) * xc.inv[m];
      }
    // the 8 groups of the chunk: lane keeps row 2 j + b2, then sums over b3, b4
    float P[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float keep = b2 ? p[1][m] : p[0][m];
      const float send = b2 ? p[0][m] : p[1][m];
      P[m] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      P[m] += __shfl_xor_sync(0xffffffffu, P[m], 8);
      P[m] += __shfl_xor_sync(0xffffffffu, P[m], 16);
    }
    if (lane < 8) {
      const int rl = cur.t * RB + 4 * int(b1) + 2 * int(b0) + int(b2);  // row within the CTA
      if (row0 + rl < row1) {
#pragma unroll
        for (int m = 0; m < MT; ++m) part[(size_t(rl) * sh.C + cur.c) * MT + m] = P[m];
      }
    }
    load_sz(v, scales, zeros, szp, it + 2 < n_it, row0, row1, sh, lane);
    szp.next(T);
    cur = nx;
  };
  for (int it = 0; it < n_it && ok; it += 2) {
    step(va, it);
    if (it + 1 == n_it || !ok) break;
    step(vb, it + 1);
  }
  if (!ok) {
    // a copy did not land in time: wait (bounded) for the copies this warp
    // still has in flight so that none lands after the kernel has exited
    const uint64_t drain = tc::globaltimer_ns() + tc::kDrainNs;
    for (int i = done; i < n_it && i < done + D; ++i) {
      tc::wait_until(bars + slot, parity, drain);
      if (++slot == D) {
        slot = 0;
        parity ^= 1u;
      }
    }
  }
  __syncthreads();

  // a row's chunk partials, added in chunk order
  const int nrows = row1 - row0;
  for (int idx = threadIdx.x; idx < nrows * MT; idx += W * 32) {
    const int r = idx / MT, m = idx - r * MT;
    if (m >= sh.M) continue;
    const float* pr = part + size_t(r) * sh.C * MT + m;
    float acc = 0.f;
    for (int c = 0; c < sh.C; ++c) acc += pr[size_t(c) * MT];
    Y[size_t(m) * sh.N + row0 + r] = __float2bfloat16_rn(acc);
  }
}

}  // namespace gemv_cc
}  // namespace wq

namespace wq_host {

namespace {

using namespace wq::gemv_cc;

int cc_mt(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : 4; }  // M = 3 runs the 4-row instance

Shape cc_shape(int64_t M, int64_t N, int64_t K, int sym, int P) {
  Shape sh;
  sh.M = int(M);
  sh.N = int(N);
  sh.K = int(K);
  sh.G = int(K / 128);
  sh.C = int((K + CHUNK - 1) / CHUNK);
  sh.NB = int((N + 3) / 4);
  sh.rows_max = 4 * int((int64_t(sh.NB) + P - 1) / P);
  sh.sym = sym;
  return sh;
}

int cc_grid(int64_t N) {
  const int64_t nb = (N + 3) / 4;
  const int P = sm_count();
  return int(nb < P ? nb : P);
}

size_t cc_smem(int mt, int D, int W, const Shape& sh) {
  return size_t(W) * D * ITEM_BYTES + size_t(W) * D * sizeof(uint64_t) +
         size_t(sh.rows_max) * size_t(sh.C) * size_t(mt) * sizeof(float);
}

// Launch shape.  Small matrices (N K <= 2^25): 8 warps with 3 ring slots
// each (96 KB, at most 128 registers per thread at M <= 2), so that the next
// decode kernel's CTA fits on the same SM and streams its first items under
// the programmatic dependent launch -- on these shapes the fixed cost of a
// launch dominates.  Larger ones: 12 warps with 2 slots each, which keeps
// more items in compute at once and streams faster, at the price of
// occupying the SM alone.  Measured on B200 at M = 1: 4096 x 4096 3.6 vs
// 4.2 us, 11008 x 4096 7.4 vs 6.7 us, 28672 x 8192 32 vs 23.5 us.
struct CcConfig {
  int W, D;
};

CcConfig cc_config(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > kGemvCcMaxM || N < 1 || K < 128) return {0, 0};
  const Shape sh = cc_shape(M, N, K, 1, cc_grid(N));
  const CcConfig pref = N * K <= (int64_t(1) << 25) ? CcConfig{8, 3} : CcConfig{12, 2};
  const CcConfig tries[3] = {pref, {8, 2}, {0, 0}};
  for (const CcConfig& c : tries)
    if (c.W > 0 && cc_smem(cc_mt(M), c.D, c.W, sh) <= size_t(SMEM_LIMIT)) return c;
  return {0, 0};
}

std::mutex g_cc_attr_mu;

// the kernel's dynamic shared memory limit, once per device
template <int MT, int D, int W>
cudaError_t cc_attr() {
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_cc_attr_mu);
  if (!done[dev]) {
    e = cudaFuncSetAttribute(gemv_cc_kernel<MT, D, W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_LIMIT);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

template <int MT, int D, int W>
cudaError_t launch_cc(int grid, size_t smem, cudaStream_t s, const CUtensorMap& tmap,
                      const __nv_bfloat16* X, const __half* scales, const __half* zeros,
                      __nv_bfloat16* Y, const Shape& sh) {
  cudaError_t e = cc_attr<MT, D, W>();
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: the weight prefetch of this kernel
  // overlaps the tail of the kernel before it on the stream
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_cc_kernel<MT, D, W>, tmap, X, scales, zeros, Y, sh,
                            status_ptr(), wait_limit_ns());
}

}  // namespace

bool gemv_cc_fits(int64_t M, int64_t N, int64_t K) { return cc_config(M, N, K).W > 0; }

int prepare_cc_kernels() {
  const cudaError_t es[9] = {cc_attr<1, 3, 8>(), cc_attr<1, 2, 8>(), cc_attr<1, 2, 12>(),
                             cc_attr<2, 3, 8>(), cc_attr<2, 2, 8>(), cc_attr<2, 2, 12>(),
                             cc_attr<4, 3, 8>(), cc_attr<4, 2, 8>(), cc_attr<4, 2, 12>()};
  for (cudaError_t e : es)
    if (e != cudaSuccess) return cuda_fail(e, "gemv_cc_kernel attributes");
  return WQ_OK;
}

int launch_gemv_w4a16_cc(const void* X, int64_t M, int64_t K, const void* codes,
                         const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                         cudaStream_t s) {
  const CcConfig cf = cc_config(M, N, K);
  if (cf.W == 0) return WQ_ERR_ARG;
  const int grid = cc_grid(N);
  const Shape sh = cc_shape(M, N, K, sym, grid);
  const int mt = cc_mt(M);
  const size_t smem = cc_smem(mt, cf.D, cf.W, sh);

  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(X);
  const __half* sc = static_cast<const __half*>(scales);
  const __half* zp = static_cast<const __half*>(zeros);
  __nv_bfloat16* y = static_cast<__nv_bfloat16*>(Y);
  // the codes as rows of K / 8 32-bit words; a box is 4 rows x 128 words
  CUtensorMap tmap;
  const int st = make_tmap_2d(&tmap, codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, uint64_t(N),
                              uint64_t(K / 8), 4, ROW_BYTES / 4, 0);
  if (st != WQ_OK) return st;
  cudaError_t e = cudaErrorInvalidValue;
#define WQ_CC_CASE(MT_, D_, W_)                   \
  if (mt == MT_ && cf.D == D_ && cf.W == W_) \
    e = launch_cc<MT_, D_, W_>(grid, smem, s, tmap, x, sc, zp, y, sh);
  WQ_CC_CASE(1, 3, 8) WQ_CC_CASE(1, 2, 8) WQ_CC_CASE(1, 2, 12)
  WQ_CC_CASE(2, 3, 8) WQ_CC_CASE(2, 2, 8) WQ_CC_CASE(2, 2, 12)
  WQ_CC_CASE(4, 3, 8) WQ_CC_CASE(4, 2, 8) WQ_CC_CASE(4, 2, 12)
#undef WQ_CC_CASE
  if (e != cudaSuccess) return cuda_fail(e, "gemv_cc_kernel");
  return WQ_OK;
}

}  // namespace wq_host
