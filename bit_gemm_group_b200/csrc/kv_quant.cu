// kv_quant.cu -- KV-cache INT8 ("27届大模型面试准备（十九）…" sec. 6: K per
// channel, V per token) reading K and V once each: a streaming per-token
// kernel for V and a cluster kernel for K.
//
// K's per-channel scale spans all S tokens of a head, so the tokens of one head
// and one block of CW channels are split over a cluster of CS CTAs: each CTA
// brings its [R, CW] slab of K into shared memory with TMA, reduces its channel
// maxima, and the cluster combines the CS partial maxima through distributed
// shared memory.  Every CTA then quantizes its slab from shared memory, so K
// crosses HBM once (the two-pass kernels of quantize.cu read it twice).
//
// Codes equal the IEEE-division definition bit for bit: the reciprocal
// multiply of qmath.cuh, with near-half-way elements rewritten exactly and
// non-finite input redone by the full definition.
#include "kernels.h"
#include "qmath.cuh"
#include "tc.cuh"

#include <mutex>
#include <type_traits>

namespace wq {
namespace kvq {

constexpr int kThreads = 256;               // V rows kernel
constexpr int kKThreads = 256;              // K cluster kernel
constexpr int kBoxRows = 256;                // TMA box height (rows of K)
constexpr int kMaxSlabBytes = 64 * 1024;     // shared memory for one K slab
constexpr int kMaxCluster = 8;               // portable cluster size
constexpr int kNearQueue = 1024;            // deferred near-half-way groups per K CTA
constexpr int kMaxBoxes = kMaxSlabBytes / (kBoxRows * 16 * 2);  // boxes of a slab, CW >= 16

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
// Arrive without release: only says that this CTA's reads of the others'
// shared memory are over (their values are already in registers), so it does
// not wait for this CTA's global stores to drain.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// 32-bit load from the shared memory of CTA `rank` of this cluster, at the
// offset of `local` in its own shared memory.
__device__ __forceinline__ uint32_t ld_cluster_u32(const void* local, uint32_t rank) {
  uint32_t remote, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(remote)
               : "r"(tc::smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

// V rows of D = 16 LPR elements (per token): LPR lanes per row, 16 elements
// (32 bytes) per lane, 32 / LPR rows per warp and step, U steps loaded ahead;
// warps stride over all BH S rows.
template <typename T, int LPR>
__global__ void __launch_bounds__(kThreads) kv_v_rows_kernel(const T* __restrict__ V, int64_t nrows,
                                                            int8_t* __restrict__ qv,
                                                            float* __restrict__ sv, int* status) {
  constexpr int D = 16 * LPR;
  constexpr int RPW = 32 / LPR;
  constexpr int U = 4;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, seg = lane % LPR;
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int64_t row1 = nrows;
  bool bad = false;
  // per warp: groups of four codes with a near-half-way element, (row << 8) |
  // group, rewritten by the whole warp once half the queue is used
  constexpr int kQ = 128;
  __shared__ unsigned long long vq[kThreads / 32][kQ];
  __shared__ int vq_n[kThreads / 32];
  const int wib = threadIdx.x >> 5;
  if (lane == 0) vq_n[wib] = 0;
  __syncwarp();
  auto flush = [&]() {
    __syncwarp();  // the queued groups' 16-byte stores and scales are visible
    const int n = min(vq_n[wib], kQ);
    for (int i = lane; i < n; i += 32) {
      const int64_t r = int64_t(vq[wib][i] >> 8);
      const int c = 4 * int(vq[wib][i] & 0xFFu);
      const uint2 v = *reinterpret_cast<const uint2*>(V + r * D + c);
      const float sc = sv[r], y = rcp_approx(sc);
      float a0, b0, a1, b1;
      unpack2<T>(v.x, a0, b0);
      unpack2<T>(v.y, a1, b1);
      *reinterpret_cast<char4*>(qv + r * D + c) =
          make_char4(code_i8_exact(a0, sc, y), code_i8_exact(b0, sc, y),
                     code_i8_exact(a1, sc, y), code_i8_exact(b1, sc, y));
    }
    __syncwarp();
    if (lane == 0) vq_n[wib] = 0;
    __syncwarp();
  };
  for (int64_t vb = gw * (U * RPW); vb < row1; vb += nw * (U * RPW)) {
    uint4 in[U][2];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t r = vb + u * RPW + sub;
      if (r < row1) {
        const uint4* src = reinterpret_cast<const uint4*>(V + r * D) + 2 * seg;
        in[u][0] = __ldcs(src);
        in[u][1] = __ldcs(src + 1);
      } else {
        in[u][0] = in[u][1] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (vb + u * RPW >= row1) break;  // warp-uniform
      const int64_t r = vb + u * RPW + sub;
      const bool live = r < row1;
      const uint32_t w[8] = {in[u][0].x, in[u][0].y, in[u][0].z, in[u][0].w,
                             in[u][1].x, in[u][1].y, in[u][1].z, in[u][1].w};
      uint32_t m2 = absmax2<T>(absmax2<T>(absmax2<T>(w[0], w[1]), absmax2<T>(w[2], w[3])),
                               absmax2<T>(absmax2<T>(w[4], w[5]), absmax2<T>(w[6], w[7])));
      float ma, mb;
      unpack2<T>(m2, ma, mb);
      // a NaN or an infinity among the lane's elements (the pair maxima
      // propagate NaN); the warp vote below sends its row to the full path
      const bool special = !(fabsf(ma) <= 3.402823466e38f && fabsf(mb) <= 3.402823466e38f);
      float amax = fmaxf(fabsf(ma), fabsf(mb));
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      float sc = fmaxf(div_rn(amax, 127.f), 1e-8f);
      float y = rcp_approx(sc);
      uint32_t ow[4];
      uint32_t near = 0u;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float a0, b0, a1, b1;
        unpack2<T>(w[2 * g], a0, b0);
        unpack2<T>(w[2 * g + 1], a1, b1);
        ow[g] = codes_i8_x4(a0, b0, a1, b1, y, y, y, y, near, g);
      }
      uint4 o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      if (__any_sync(0xffffffffu, special)) {
        // the row maximum by the definition (NaN skipped, infinities kept)
        const uint32_t p2 =
            absmax2_skipnan<T>(absmax2_skipnan<T>(absmax2_skipnan<T>(w[0], w[1]),
                                                  absmax2_skipnan<T>(w[2], w[3])),
                               absmax2_skipnan<T>(absmax2_skipnan<T>(w[4], w[5]),
                                                  absmax2_skipnan<T>(w[6], w[7])));
        float pa, pb;
        unpack2<T>(p2, pa, pb);
        float am = fmaxf(fabsf(pa), fabsf(pb));
#pragma unroll
        for (int o2 = LPR / 2; o2 > 0; o2 >>= 1)
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o2));
        sc = fmaxf(div_rn(am, 127.f), 1e-8f);
        y = rcp_approx(sc);
        uint32_t c[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float a, b;
          unpack2<T>(w[i], a, b);
          const uint32_t ca = uint32_t(code_i8_full(a, sc, y)) & 0xFFu;
          const uint32_t cb = uint32_t(code_i8_full(b, sc, y)) & 0xFFu;
          c[i >> 1] |= (ca | (cb << 8)) << (16 * (i & 1));
        }
        o = make_uint4(c[0], c[1], c[2], c[3]);
        near = 0u;
      }
      bad |= live && special;
      if (live) {
        int8_t* dst = qv + r * D + seg * 16;
        *reinterpret_cast<uint4*>(dst) = o;
        if (seg == 0) sv[r] = sc;
        while (near != 0u) {  // groups with a near-half-way element: queued
          const int g = __ffs(near) - 1;
          near &= near - 1u;
          const int slot = atomicAdd(&vq_n[wib], 1);
          if (slot < kQ) {
            vq[wib][slot] = (static_cast<unsigned long long>(r) << 8) | unsigned(seg * 4 + g);
            continue;
          }
          // queue full: rewritten here
          float a0, b0, a1, b1;
          unpack2<T>(pick(w, 2 * g), a0, b0);
          unpack2<T>(pick(w, 2 * g + 1), a1, b1);
          *reinterpret_cast<char4*>(dst + 4 * g) =
              make_char4(code_i8_exact(a0, sc, y), code_i8_exact(b0, sc, y),
                         code_i8_exact(a1, sc, y), code_i8_exact(b1, sc, y));
        }
      }
    }
    __syncwarp();
    if (vq_n[wib] >= kQ / 2) flush();  // warp-uniform
  }
  flush();
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(status, WQ_ERR_NONFINITE);
}

// K per channel.  Grid (CS, D / CW, BH) in clusters of (CS, 1, 1): the
// cluster is one head and one block of CW channels; CTA `rank` owns tokens
// [rank R, rank R + R).
template <typename T, int CW, int D>
__global__ void __launch_bounds__(kKThreads, 3) kv_k_cluster_kernel(
    const __grid_constant__ CUtensorMap kmap, int64_t S, int R, int8_t* __restrict__ qk,
    float* __restrict__ sk, int* status, uint64_t wait_ns) {
  constexpr int WPR = CW / 2;          // 32-bit words (channel pairs) per slab row
  constexpr int TPR = CW / 8;          // threads per slab row, 16 bytes each
  constexpr int RPS = kKThreads / TPR;  // slab rows per CTA step
  extern __shared__ __align__(128) unsigned char smem_raw[];
  T* slab = reinterpret_cast<T*>(smem_raw);  // [boxes * kBoxRows][CW]
  __shared__ __align__(8) uint64_t bars[kMaxBoxes];  // one per TMA box
  __shared__ uint32_t part[2][WPR];          // this CTA's channel-pair maxima
  __shared__ uint32_t comb[kMaxCluster][WPR];  // the cluster's partial maxima
  __shared__ int s_fail;
  __shared__ uint32_t wred[kKThreads / 32][WPR];
  __shared__ float s_sc[CW], s_y[CW];
  __shared__ int s_special;
  // groups of four codes with a near-half-way element: (slab row << 8) |
  // first channel; rewritten by the whole CTA after the slab is quantized
  __shared__ uint32_t nq[kNearQueue];
  __shared__ int nq_n;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int CS = int(gridDim.x);
  const int cb = int(blockIdx.y);
  const int64_t bh = blockIdx.z;
  const int64_t r0 = int64_t(rank) * R;
  const int rows = int(r0 < S ? (S - r0 < R ? S - r0 : R) : 0);  // K rows of this CTA
  const int boxes = (rows + kBoxRows - 1) / kBoxRows;

  if (tid == 0) {
    for (int b = 0; b < boxes; ++b) tc::mbar_init(&bars[b], 1);
    tc::fence_mbar_init();
    s_special = 0;
    s_fail = 0;
    nq_n = 0;
  }
  __syncthreads();
  if (tid == 0) {
    tc::tma_prefetch_desc(&kmap);
    for (int b = 0; b < boxes; ++b) {
      tc::mbar_arrive_expect_tx(&bars[b], uint32_t(kBoxRows * CW * sizeof(T)));
      tc::tma_load_2d(slab + size_t(b) * kBoxRows * CW, &kmap, &bars[b], cb * CW,
                      int32_t(bh * S + r0 + int64_t(b) * kBoxRows));
    }
  }

  // channel-pair maxima of the slab (NaN-propagating), box by box as each
  // lands (bounded waits; after a timeout the rest of the slab is not read)
  const int cg = tid % TPR, rl = tid / TPR;
  uint32_t m[4] = {0u, 0u, 0u, 0u};
  const uint64_t deadline = tc::globaltimer_ns() + wait_ns;
  for (int b = 0; b < boxes; ++b) {
    if (!__all_sync(0xffffffffu, tc::wait_until(&bars[b], 0, deadline))) {
      if (lane == 0) {
        s_fail = 1;
        record_error(status, WQ_ERR_TIMEOUT);
      }
      break;
    }
    const int rend = rows < (b + 1) * kBoxRows ? rows : (b + 1) * kBoxRows;
    for (int r = b * kBoxRows + rl; r < rend; r += RPS) {
      const uint4 v = *reinterpret_cast<const uint4*>(slab + size_t(r) * CW + cg * 8);
      m[0] = absmax2<T>(m[0], v.x);
      m[1] = absmax2<T>(m[1], v.y);
      m[2] = absmax2<T>(m[2], v.z);
      m[3] = absmax2<T>(m[3], v.w);
    }
  }
#pragma unroll
  for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = absmax2<T>(m[i], __shfl_xor_sync(0xffffffffu, m[i], o));
  if (lane < TPR)
#pragma unroll
    for (int i = 0; i < 4; ++i) wred[warp][cg * 4 + i] = m[i];
  __syncthreads();
  const bool ok = s_fail == 0;
  if (tid < WPR) {
    uint32_t v = wred[0][tid];
#pragma unroll
    for (int w = 1; w < kKThreads / 32; ++w) v = absmax2<T>(v, wred[w][tid]);
    part[0][tid] = v;
  }
  cluster_arrive();
  cluster_wait();  // every CTA's partial maxima are visible

  // one remote load per thread, then the reduction over the ranks
  if (tid < WPR * CS) comb[tid / WPR][tid % WPR] = ld_cluster_u32(&part[0][tid % WPR], tid / WPR);
  __syncthreads();
  uint32_t pair = 0u;
  if (tid < WPR) {
    for (int k = 0; k < CS; ++k) pair = absmax2<T>(pair, comb[k][tid]);
    float a, b;
    unpack2<T>(pair, a, b);
    if (!(fabsf(a) <= 3.402823466e38f && fabsf(b) <= 3.402823466e38f)) s_special = 1;
  }
  __syncthreads();
  // The combined maxima are the same in every CTA of the cluster, so all of
  // them take this branch or none does.
  const bool special = s_special != 0;
  if (special) {
    // a NaN or an infinity in these channels: maxima by the definition
    uint32_t p[4] = {0u, 0u, 0u, 0u};
    if (ok) {
      for (int r = rl; r < rows; r += RPS) {
        const uint4 v = *reinterpret_cast<const uint4*>(slab + size_t(r) * CW + cg * 8);
        p[0] = absmax2_skipnan<T>(p[0], v.x);
        p[1] = absmax2_skipnan<T>(p[1], v.y);
        p[2] = absmax2_skipnan<T>(p[2], v.z);
        p[3] = absmax2_skipnan<T>(p[3], v.w);
      }
    }
#pragma unroll
    for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        p[i] = absmax2_skipnan<T>(p[i], __shfl_xor_sync(0xffffffffu, p[i], o));
    __syncthreads();  // wred is reused
    if (lane < TPR)
#pragma unroll
      for (int i = 0; i < 4; ++i) wred[warp][cg * 4 + i] = p[i];
    __syncthreads();
    if (tid < WPR) {
      uint32_t v = wred[0][tid];
#pragma unroll
      for (int w = 1; w < kKThreads / 32; ++w) v = absmax2_skipnan<T>(v, wred[w][tid]);
      part[1][tid] = v;
    }
    cluster_arrive();
    cluster_wait();
    if (tid < WPR * CS)
      comb[tid / WPR][tid % WPR] = ld_cluster_u32(&part[1][tid % WPR], tid / WPR);
    __syncthreads();
    if (tid < WPR) {
      pair = 0u;
      for (int k = 0; k < CS; ++k) pair = absmax2_skipnan<T>(pair, comb[k][tid]);
    }
    if (tid == 0 && rank == 0) record_error(status, WQ_ERR_NONFINITE);
  }
  if (tid < WPR) {
    float a, b;
    unpack2<T>(pair, a, b);
    const float sa = fmaxf(div_rn(fabsf(a), 127.f), 1e-8f);
    const float sb = fmaxf(div_rn(fabsf(b), 127.f), 1e-8f);
    s_sc[2 * tid] = sa;
    s_sc[2 * tid + 1] = sb;
    s_y[2 * tid] = rcp_approx(sa);
    s_y[2 * tid + 1] = rcp_approx(sb);
    if (rank == 0) {
      sk[bh * D + cb * CW + 2 * tid] = sa;
      sk[bh * D + cb * CW + 2 * tid + 1] = sb;
    }
  }
  cluster_arrive_relaxed();  // this CTA is done reading the others' shared memory
  __syncthreads();

  // quantize the slab: 8 channels per thread, fixed over the rows
  float sc[8], y[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    sc[e] = s_sc[cg * 8 + e];
    y[e] = s_y[cg * 8 + e];
  }
  int8_t* qk_head = qk + bh * S * D + cb * CW + cg * 8;
  // one slab row segment (8 channels) of this thread: codes, store, and the
  // near-half-way groups queued
  auto quant_row = [&](const uint4 v, const int r, const bool live) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint2 o;
    uint32_t near = 0u;
    if (!special) {
      uint32_t ow[2];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        float a0, b0, a1, b1;
        unpack2<T>(w[2 * g], a0, b0);
        unpack2<T>(w[2 * g + 1], a1, b1);
        ow[g] = codes_i8_x4(a0, b0, a1, b1, y[4 * g], y[4 * g + 1], y[4 * g + 2], y[4 * g + 3],
                            near, g);
      }
      o = make_uint2(ow[0], ow[1]);
    } else {
      uint32_t c[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a, b;
        unpack2<T>(w[i], a, b);
        const uint32_t ca = uint32_t(code_i8_full(a, sc[2 * i], y[2 * i])) & 0xFFu;
        const uint32_t cb2 = uint32_t(code_i8_full(b, sc[2 * i + 1], y[2 * i + 1])) & 0xFFu;
        c[i >> 1] |= (ca | (cb2 << 8)) << (16 * (i & 1));
      }
      o = make_uint2(c[0], c[1]);
    }
    int8_t* dst = qk_head + (r0 + r) * D;
    if (live) *reinterpret_cast<uint2*>(dst) = o;
    // groups with a near-half-way element: queued, one shared atomic per warp
    const uint32_t bal0 = __ballot_sync(0xffffffffu, near & 1u);
    const uint32_t bal1 = __ballot_sync(0xffffffffu, near & 2u);
    if ((bal0 | bal1) != 0u) {
      const uint32_t lt = (1u << lane) - 1u;
      int base = 0;
      if (lane == 0) base = atomicAdd(&nq_n, __popc(bal0) + __popc(bal1));
      base = __shfl_sync(0xffffffffu, base, 0);
      const int slot[2] = {base + __popc(bal0 & lt), base + __popc(bal0) + __popc(bal1 & lt)};
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        if (!((near >> g) & 1u)) continue;
        if (slot[g] < kNearQueue) {
          nq[slot[g]] = (uint32_t(r) << 8) | uint32_t(cg * 8 + 4 * g);
          continue;
        }
        // queue full: rewritten here
        float a0, b0, a1, b1;
        unpack2<T>(g ? w[2] : w[0], a0, b0);
        unpack2<T>(g ? w[3] : w[1], a1, b1);
        float sg[4], yg[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sg[j] = g ? sc[4 + j] : sc[j];
          yg[j] = g ? y[4 + j] : y[j];
        }
        *reinterpret_cast<char4*>(dst + 4 * g) =
            make_char4(code_i8_exact(a0, sg[0], yg[0]), code_i8_exact(b0, sg[1], yg[1]),
                       code_i8_exact(a1, sg[2], yg[2]), code_i8_exact(b1, sg[3], yg[3]));
      }
    }
  };
  if (ok) {
    // two rows per thread and step, both loaded before either is processed
    for (int base = 0; base < rows; base += 2 * RPS) {
      const int ra = base + rl, rb = base + RPS + rl;
      const bool la = ra < rows, lb = rb < rows;
      uint4 va = make_uint4(0u, 0u, 0u, 0u), vb = va;
      if (la) va = *reinterpret_cast<const uint4*>(slab + size_t(ra) * CW + cg * 8);
      if (lb) vb = *reinterpret_cast<const uint4*>(slab + size_t(rb) * CW + cg * 8);
      quant_row(va, ra, la);
      quant_row(vb, rb, lb);
    }
  }
  // The queued groups, one per thread: exact codes from the slab (the group's
  // 8-byte store above is ordered before this one by the block barrier).
  __syncthreads();
  const int nn = nq_n < kNearQueue ? nq_n : kNearQueue;
  for (int i = tid; i < nn; i += kKThreads) {
    const int r = int(nq[i] >> 8), c = int(nq[i] & 0xFFu);
    const uint2 v = *reinterpret_cast<const uint2*>(slab + size_t(r) * CW + c);
    float a0, b0, a1, b1;
    unpack2<T>(v.x, a0, b0);
    unpack2<T>(v.y, a1, b1);
    *reinterpret_cast<char4*>(qk + bh * S * D + (r0 + r) * D + cb * CW + c) =
        make_char4(code_i8_exact(a0, s_sc[c], s_y[c]), code_i8_exact(b0, s_sc[c + 1], s_y[c + 1]),
                   code_i8_exact(a1, s_sc[c + 2], s_y[c + 2]),
                   code_i8_exact(b1, s_sc[c + 3], s_y[c + 3]));
  }
  if (!ok)  // own copies still in flight
    for (int b = 0; b < boxes; ++b)
      tc::wait_until(&bars[b], 0, tc::globaltimer_ns() + tc::kDrainNs);
  cluster_wait();  // no CTA leaves while another may still read its partials
}

}  // namespace kvq
}  // namespace wq

namespace wq_host {

namespace {
template <typename T, int CW, int D>
int launch_k_cluster(const void* Kc, int64_t BH, int64_t S, int CS, int R, void* qk, void* sk,
                     cudaStream_t s) {
  auto kern = wq::kvq::kv_k_cluster_kernel<T, CW, D>;
  static std::mutex mu;
  static bool attr_set[64] = {};
  int dev = 0;
  WQ_CUDA_CHECK(cudaGetDevice(&dev));
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 64 && !attr_set[dev]) {
      WQ_CUDA_CHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         wq::kvq::kMaxSlabBytes));
      attr_set[dev] = true;
    }
  }
  CUtensorMap map;
  const CUtensorMapDataType dt = std::is_same<T, __half>::value
                                     ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                     : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  int st = make_tmap_2d(&map, Kc, dt, 2, uint64_t(BH * S), uint64_t(D), wq::kvq::kBoxRows,
                        uint32_t(CW), 0);
  if (st != WQ_OK) return st;
  const int boxes = (R + wq::kvq::kBoxRows - 1) / wq::kvq::kBoxRows;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(CS), unsigned(D / CW), unsigned(BH));
  cfg.blockDim = dim3(wq::kvq::kKThreads, 1, 1);
  cfg.dynamicSmemBytes = size_t(boxes) * wq::kvq::kBoxRows * CW * 2;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = unsigned(CS);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  WQ_CUDA_CHECK(cudaLaunchKernelEx(&cfg, kern, map, S, R, static_cast<int8_t*>(qk),
                                   static_cast<float*>(sk), status_ptr(), wait_limit_ns()));
  return WQ_OK;
}

template <typename T, int D>
int launch_kv(int CW, const void* Kc, const void* Vc, int64_t BH, int64_t S, int CS, int R,
              void* qk, void* sk, void* qv, void* sv, cudaStream_t s) {
  // V rows first: they need nothing from K
  constexpr int LPR = D / 16;
  const int64_t nrows = BH * S;
  const int64_t warp_steps = (nrows + 4 * (32 / LPR) - 1) / (4 * (32 / LPR));
  int64_t blocks = (warp_steps + 7) / 8;
  const int64_t cap = int64_t(sm_count()) * 3;  // resident 256-thread blocks
  if (blocks > cap) blocks = cap;
  wq::kvq::kv_v_rows_kernel<T, LPR><<<unsigned(blocks), wq::kvq::kThreads, 0, s>>>(
      static_cast<const T*>(Vc), nrows, static_cast<int8_t*>(qv), static_cast<float*>(sv),
      status_ptr());
  WQ_LAUNCH_CHECK("kv_v_rows_kernel");
  switch (CW) {
    case 64:
      if constexpr (D >= 64) return launch_k_cluster<T, 64, D>(Kc, BH, S, CS, R, qk, sk, s);
      break;
    case 32:
      if constexpr (D >= 32) return launch_k_cluster<T, 32, D>(Kc, BH, S, CS, R, qk, sk, s);
      break;
    case 16: return launch_k_cluster<T, 16, D>(Kc, BH, S, CS, R, qk, sk, s);
  }
  return WQ_ERR_UNSUPPORTED;
}

template <typename T>
int dispatch_d(int64_t D, int CW, const void* Kc, const void* Vc, int64_t BH, int64_t S, int CS,
               int R, void* qk, void* sk, void* qv, void* sv, cudaStream_t s) {
  switch (D) {
    case 16: return launch_kv<T, 16>(CW, Kc, Vc, BH, S, CS, R, qk, sk, qv, sv, s);
    case 32: return launch_kv<T, 32>(CW, Kc, Vc, BH, S, CS, R, qk, sk, qv, sv, s);
    case 64: return launch_kv<T, 64>(CW, Kc, Vc, BH, S, CS, R, qk, sk, qv, sv, s);
    case 128: return launch_kv<T, 128>(CW, Kc, Vc, BH, S, CS, R, qk, sk, qv, sv, s);
    case 256: return launch_kv<T, 256>(CW, Kc, Vc, BH, S, CS, R, qk, sk, qv, sv, s);
  }
  return WQ_ERR_UNSUPPORTED;
}
}  // namespace

bool kv_fused_plan(int dtype, int64_t BH, int64_t S, int64_t D, int* CS, int* R, int* CW) {
  if (dtype != WQ_BF16 && dtype != WQ_F16) return false;
  if (BH <= 0 || S <= 0 || BH > 65535) return false;
  if (D != 16 && D != 32 && D != 64 && D != 128 && D != 256) return false;
  int64_t cs = (S + wq::kvq::kBoxRows - 1) / wq::kvq::kBoxRows;
  if (cs > wq::kvq::kMaxCluster) cs = wq::kvq::kMaxCluster;
  const int64_t r = (S + cs - 1) / cs;
  const int64_t boxes = (r + wq::kvq::kBoxRows - 1) / wq::kvq::kBoxRows;
  for (int cw = 64; cw >= 16; cw >>= 1) {
    if (D % cw != 0) continue;
    if (boxes * wq::kvq::kBoxRows * cw * 2 <= wq::kvq::kMaxSlabBytes) {
      *CS = int(cs);
      *R = int(r);
      *CW = cw;
      return true;
    }
  }
  return false;
}

int launch_quant_kv_fused(const void* Kc, const void* Vc, int dtype, int64_t BH, int64_t S,
                          int64_t D, void* qk, void* sk, void* qv, void* sv, cudaStream_t s) {
  int CS = 0, R = 0, CW = 0;
  if (!kv_fused_plan(dtype, BH, S, D, &CS, &R, &CW)) return WQ_ERR_UNSUPPORTED;
  if (dtype == WQ_BF16)
    return dispatch_d<__nv_bfloat16>(D, CW, Kc, Vc, BH, S, CS, R, qk, sk, qv, sv, s);
  return dispatch_d<__half>(D, CW, Kc, Vc, BH, S, CS, R, qk, sk, qv, sv, s);
}

}  // namespace wq_host
