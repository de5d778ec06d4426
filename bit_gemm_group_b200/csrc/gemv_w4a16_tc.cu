// gemv_w4a16_tc.cu -- W4A16 decode product on the sm_100a tensor cores (M = 5..16).
//
//   Y[m, n] = sum_g s[n, g] * sum_{k in g} X[m, k] * (u[n, k] - z[n, g])
//
// ("大模型面试准备（十九）…" sec. 1.2: a decode token reads every weight once,
// about 4 FLOP per byte for INT4, so the bound is HBM bandwidth; sec. 2.3
// W4A16; "大模型量化技术定义与主流方案解析" sec. 四: the weight is expanded inside
// the product and never written back to memory.)
//
// Work decomposition (stream-K): the units are (128-row tile t, 128-wide K
// group g), ordered tile-major; the persistent grid has one CTA per SM and CTA
// c takes the contiguous unit range [c*U/P, (c+1)*U/P), so every SM streams the
// same number of weight bytes whatever the shape.  A CTA's range covers whole
// tiles in its middle and at most two partial tiles at its ends; a partial
// result goes to a per-CTA slot of the caller's workspace and the last CTA to
// finish a tile (per-tile arrival counter) sums the slots in CTA order
// (deterministic), writes Y and resets the counter to zero.
//
// Roles (640 threads, one CTA per SM, 512 TMEM columns):
//   warp 0       TMA producer: per group, packed codes [128 rows x 64 B]
//                (64-byte swizzle) and X [16 rows x 128] bf16 (two 128-byte
//                swizzled slices), into a STAGES-deep ring.
//   warps 1..3   MMA issuers (warp 1 also owns TMEM): issuer k takes groups
//                i = k mod 3; per group 8 x tcgen05.mma.kind::f16, M=128
//                (weight rows), N=16 (X rows, zero-padded), K=16, A read from
//                tensor memory.  One thread issues a small MMA only every ~44
//                cycles, so the issue is spread over three warps.
//   warps 4..7   epilogue warpgroup: per group, reads the fp32 [128 x 16]
//                result (tcgen05.ld) and adds s * D to per-row accumulators;
//                at the end of each tile segment writes Y or the partial.
//   warps 8..19  three dequant warpgroups, group i to warpgroup i mod 3.
//                Thread = weight row: 128 nibbles -> exact bf16 (u - z) pairs
//                -> tcgen05.st into the group's A buffer (ring of six).
// The group scale multiplies an exact per-group integer-weighted sum; all
// accumulation is fp32.
#include <stdlib.h>

#include <mutex>

#include "kernels.h"
#include "tc.cuh"

namespace wq {
namespace gemv {

constexpr int BN = 128;              // weight rows per tile (MMA M)
constexpr int MPAD = 16;             // X rows padded (MMA N)
constexpr int QG = 4;                // groups per stage (one stream-K unit)
constexpr int CBOX = BN * 128;       // codes box: 128 rows x 128 B (two groups)
constexpr int CODE_BYTES = 2 * CBOX; // 128 rows x 256 B: four groups
constexpr int XSLICE = MPAD * 128;   // [16 rows x 64 bf16], 128-byte rows
constexpr int X_BYTES = 2 * QG * XSLICE;  // X for 4 x 128 K elements
constexpr int STAGE_BYTES = CODE_BYTES + X_BYTES;  // 48 KB
constexpr int STAGES = 4;
constexpr int NI = 3;                // MMA issuer warps
constexpr int NDQ = 3;               // dequant warpgroups
constexpr int NAB = 6;               // A buffers (64 TMEM columns each)
constexpr int ND = 8;                // D buffers (16 TMEM columns each)
constexpr int EPI_WARP0 = 4;
constexpr int DQ_WARP0 = 8;
constexpr int THREADS = (DQ_WARP0 + 4 * NDQ) * 32;
constexpr int TMEM_COLS = 512;
constexpr int D_COL0 = 64 * NAB;
constexpr uint32_t IDESC = tc::idesc_bf16_f32(BN, MPAD);
constexpr int EPI_BAR = 1;           // named barrier of the epilogue warpgroup

struct Smem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t a_full[NAB];
  uint64_t a_empty[NAB];
  uint64_t d_full[ND];
  uint64_t d_empty[ND];
  uint64_t drain[NI];
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
};
constexpr size_t SMEM_BYTES = 1024 + size_t(STAGES) * STAGE_BYTES + sizeof(Smem);

// Unit range of CTA c among P over U units.
__host__ __device__ __forceinline__ int unit_begin(int c, int P, int U) {
  return int((int64_t(c) * U) / P);
}
// CTA owning unit u.
__device__ __forceinline__ int owner(int u, int P, int U) {
  int c = int((int64_t(u) * P) / U);
  while (c > 0 && unit_begin(c, P, U) > u) --c;
  while (c + 1 < P && unit_begin(c + 1, P, U) <= u) ++c;
  return c;
}

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
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Position in a ring of `size` slots: slot index and the parity of the phase
// the current use waits for, advanced without divisions.
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

__global__ void __launch_bounds__(THREADS, 1)
    gemv_w4a16_tc_kernel(const __grid_constant__ CUtensorMap tmW,
                         const __grid_constant__ CUtensorMap tmX,
                         const __half* __restrict__ scales, const __half* __restrict__ zeros,
                         __nv_bfloat16* __restrict__ Y, float* __restrict__ ws_part,
                         int* __restrict__ ws_cnt, int M, int N, int G, int sym, int* status,
                         uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(base + size_t(STAGES) * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int T = (N + BN - 1) / BN;
  const int Q = (G + QG - 1) / QG;  // 4-group units per tile (the last may hold fewer)
  const int U = T * Q;
  const int P = gridDim.x;
  const int c = blockIdx.x;
  const int u0 = unit_begin(c, P, U), u1 = unit_begin(c + 1, P, U);
  const int nunits = u1 - u0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&sm.full[s], 1);
      tc::mbar_init(&sm.empty[s], QG);  // one MMA commit per group of the stage
    }
    for (int b = 0; b < NAB; ++b) {
      tc::mbar_init(&sm.a_full[b], 128);
      tc::mbar_init(&sm.a_empty[b], 1);
    }
    for (int d = 0; d < ND; ++d) {
      tc::mbar_init(&sm.d_full[d], 1);
      tc::mbar_init(&sm.d_empty[d], 128);
    }
    for (int k = 0; k < NI; ++k) tc::mbar_init(&sm.drain[k], 1);
    sm.abort_flag = 0;
    sm.last_flag = 0;
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

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      Ring st;
      int issued = 0;
      int t = u0 / Q, qq = u0 - (u0 / Q) * Q;
      for (; issued < nunits; ++issued) {
        if (!tc::wait_bounded(&sm.empty[st.slot], st.phase ^ 1u, wd)) break;
        uint8_t* cdst = base + size_t(st.slot) * STAGE_BYTES;
        uint64_t* bar = &sm.full[st.slot];
        tc::mbar_arrive_expect_tx(bar, STAGE_BYTES);
        tc::tma_load_2d(cdst, &tmW, bar, qq * 256, t * BN);
        tc::tma_load_2d(cdst + CBOX, &tmW, bar, qq * 256 + 128, t * BN);
#pragma unroll
        for (int h = 0; h < 2 * QG; ++h)
          tc::tma_load_2d(cdst + CODE_BYTES + h * XSLICE, &tmX, bar, qq * (QG * 128) + h * 64, 0);
        st.advance(STAGES);
        if (++qq == Q) {
          qq = 0;
          ++t;
        }
      }
      // drain: the last load issued into each stage has landed before exit
      const uint64_t dl = tc::globaltimer_ns() + tc::kDrainNs;
      for (int k = 0; k < (issued < STAGES ? issued : STAGES); ++k) {
        const int i = issued - 1 - k;
        tc::wait_until(&sm.full[i % STAGES], uint32_t((i / STAGES) & 1), dl);
      }
    }
  } else if (warp <= NI) {
    // ------------------------------------------------------------ MMA issuer k
    if (lane == 0) {
      const int k = warp - 1;
      const uint64_t dhi = tc::sdesc_k_sw128(0);
      const uint32_t x0 = tc::smem_u32(base) + CODE_BYTES;
      Ring st, ab, db;
      ab.advance(NAB, k);
      db.advance(ND, k);
      bool ok = true;
      int i = 0;  // group index in the CTA's sequence
      int qq = u0 - (u0 / Q) * Q;
      for (int un = 0; un < nunits && ok; ++un) {
        const int ng = min(QG, G - qq * QG);
        for (int p = 0; p < ng; ++p, ++i) {
          if (i % NI != k) continue;
          if (!(ok = tc::wait_bounded(&sm.full[st.slot], st.phase, wd) &&
                     tc::wait_bounded(&sm.a_full[ab.slot], ab.phase, wd) &&
                     tc::wait_bounded(&sm.d_empty[db.slot], db.phase ^ 1u, wd)))
            break;
          tc::fence_after_sync();
          const uint64_t xd =
              dhi | uint64_t((x0 + uint32_t(st.slot) * STAGE_BYTES + uint32_t(p) * 2 * XSLICE) >> 4);
          const uint32_t a = tmem + 64 * ab.slot;
          const uint32_t d = tmem + D_COL0 + 16 * db.slot;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_f16_ts(d, a + 8 * kk,
                           xd + uint64_t(((kk >> 2) * XSLICE + (kk & 3) * 32) >> 4), IDESC,
                           kk > 0);
          tc::mma_commit(&sm.d_full[db.slot]);
          tc::mma_commit(&sm.a_empty[ab.slot]);
          // the stage is released after one commit per group; the issuer of
          // the last group of a short unit adds the missing arrivals
          for (int e = (p == ng - 1) ? ng - 1 : QG - 1; e < QG; ++e)
            tc::mma_commit(&sm.empty[st.slot]);
          ab.advance(NAB, NI);
          db.advance(ND, NI);
        }
        st.advance(STAGES);
        if (++qq == Q) qq = 0;
      }
      tc::mma_commit(&sm.drain[k]);
      tc::wait_until(&sm.drain[k], 0, tc::globaltimer_ns() + tc::kDrainNs);
    }
  } else if (warp >= DQ_WARP0) {
    // ----------------------------------------------------------- dequant w
    const int w = (warp - DQ_WARP0) >> 2;
    const int q = warp & 3;  // TMEM lane quarter
    const int row = q * 32 + lane;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    Ring st, ab;
    ab.advance(NAB, w);
    bool ok = true;
    int i = 0;
    int t = u0 / Q, qq = u0 - (u0 / Q) * Q;
    for (int un = 0; un < nunits && ok; ++un) {
      const int ng = min(QG, G - qq * QG);
      for (int p = 0; p < ng; ++p, ++i) {
        if (i % NDQ != w) continue;
        const int n = t * BN + row, g = qq * QG + p;
        const int zi = sym ? 8 : (n < N ? int(__half2float(zeros[size_t(n) * G + g])) : 0);
        if (!(ok = tc::wait_bounded(&sm.full[st.slot], st.phase, wd) &&
                   tc::wait_bounded(&sm.a_empty[ab.slot], ab.phase ^ 1u, wd)))
          break;
        tc::fence_after_sync();
        const uint32_t zb = 0x4300u | uint32_t(zi);  // bf16(128 + z), exact
        const uint32_t z2 = zb | (zb << 16);
        // group p = half (p & 1) of box (p >> 1); 16-byte chunk c of a row
        // sits at c ^ (row & 7) (128-byte swizzle)
        const uint8_t* rowp = base + size_t(st.slot) * STAGE_BYTES + (p >> 1) * CBOX + row * 128;
        const int c0 = (p & 1) * 4;
        const uint32_t a = tmem + lane_off + 64 * ab.slot;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4 v0 = *reinterpret_cast<const uint4*>(rowp + (((c0 + 2 * half) ^ (row & 7)) << 4));
          const uint4 v1 =
              *reinterpret_cast<const uint4*>(rowp + (((c0 + 2 * half + 1) ^ (row & 7)) << 4));
          const uint32_t words[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          uint32_t out[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t wd0 = words[k];
            const uint32_t w4 = wd0 >> 4;
#pragma unroll
            for (int e = 0; e < 4; ++e)  // byte e: elements 2e (bits 0..3), 2e+1 (bits 16..19)
              out[4 * k + e] = bf16x2_sub(
                  nib_to_bf16x2(prmt(wd0, w4, uint32_t(e) | (uint32_t(4 + e) << 8))), z2);
          }
          tc::tmem_st_x32(a + 32 * half, out);
        }
        tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::mbar_arrive(&sm.a_full[ab.slot]);
        ab.advance(NAB, NDQ);
      }
      st.advance(STAGES);
      if (++qq == Q) {
        qq = 0;
        ++t;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    const int etid = threadIdx.x - EPI_WARP0 * 32;  // 0..127
    float acc[MPAD];
#pragma unroll
    for (int m = 0; m < MPAD; ++m) acc[m] = 0.f;
    Ring db;
    bool ok = true;
    int t = u0 / Q, qq = u0 - (u0 / Q) * Q;
    const int t_first = t;
    // scales of the current unit, loaded one unit ahead
    float s_cur[QG];
    {
      const int n = t * BN + row;
#pragma unroll
      for (int p = 0; p < QG; ++p) {
        const int g = qq * QG + p;
        s_cur[p] = (n < N && g < G) ? __half2float(scales[size_t(n) * G + g]) : 0.f;
      }
    }
    for (int un = 0; un < nunits; ++un) {
      const int ng = min(QG, G - qq * QG);
      const int n = t * BN + row;
      const bool row_in = n < N;
      // issue the next unit's scale loads now; they are consumed one unit later
      float s_nxt[QG];
      {
        const int qn = (qq + 1 == Q) ? 0 : qq + 1;
        const int tn = (qq + 1 == Q) ? t + 1 : t;
        const int nn = tn * BN + row;
        const bool live = un + 1 < nunits && nn < N;
#pragma unroll
        for (int p = 0; p < QG; ++p) {
          const int g = qn * QG + p;
          s_nxt[p] = (live && g < G) ? __half2float(scales[size_t(nn) * G + g]) : 0.f;
        }
      }
      // the unit's results, two groups at a time: wait, load back to back, release
#pragma unroll
      for (int h = 0; h < QG; h += 2) {
        uint32_t r[2][16];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (h + e < ng && ok) {
            Ring dp = db;
            dp.advance(ND, h + e);
            ok = tc::wait_bounded(&sm.d_full[dp.slot], dp.phase, wd);
          }
        }
        if (ok && h < ng) {
          tc::fence_after_sync();
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            Ring dp = db;
            dp.advance(ND, h + e);
            if (h + e < ng) tc::tmem_ld_x16(tmem + lane_off + D_COL0 + 16 * dp.slot, r[e]);
          }
          tc::tmem_wait_ld();
          tc::fence_before_sync();
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            Ring dp = db;
            dp.advance(ND, h + e);
            if (h + e < ng) tc::mbar_arrive(&sm.d_empty[dp.slot]);
          }
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            if (h + e < ng) {
              const float sc = row_in ? s_cur[h + e] : 0.f;
#pragma unroll
              for (int m = 0; m < MPAD; ++m) acc[m] = fmaf(sc, __uint_as_float(r[e][m]), acc[m]);
            }
          }
        }
      }
      db.advance(ND, ng);
#pragma unroll
      for (int p = 0; p < QG; ++p) s_cur[p] = s_nxt[p];
      const int g = qq * QG + ng - 1;  // last group of this unit
      // end of this tile's segment: write Y, or the partial for the tile's last CTA
      if (g == G - 1 || un == nunits - 1) {
        const bool whole = (g == G - 1) && (t * Q >= u0);
        if (whole) {
          if (row_in) {
#pragma unroll
            for (int m = 0; m < MPAD; ++m)
              if (m < M) Y[size_t(m) * N + n] = __float2bfloat16_rn(acc[m]);
          }
        } else {
          const int which = (t == t_first) ? 0 : 1;
          float* dst = ws_part + (size_t(c) * 2 + which) * (MPAD * BN);
#pragma unroll
          for (int m = 0; m < MPAD; ++m)
            if (m < M) dst[m * BN + row] = acc[m];
          named_bar_sync(EPI_BAR, 128);
          if (etid == 0) {
            // one cumulative fence releases the warpgroup's partial (ordered
            // before it by the barrier); the second one acquires the other
            // CTAs' partials if this is the tile's last arrival
            const int first = owner(t * Q, P, U), last = owner(t * Q + Q - 1, P, U);
            fence_acq_rel_gpu();
            const int old = atomicAdd(ws_cnt + t, 1);
            fence_acq_rel_gpu();
            sm.last_flag = (old == last - first) ? 1 : 0;
          }
          named_bar_sync(EPI_BAR, 128);
          if (sm.last_flag) {
            const int first = owner(t * Q, P, U), last = owner(t * Q + Q - 1, P, U);
            float tot[MPAD];
#pragma unroll
            for (int m = 0; m < MPAD; ++m) tot[m] = 0.f;
#pragma unroll 2
            for (int cc = first; cc <= last; ++cc) {
              const int wh = (t == unit_begin(cc, P, U) / Q) ? 0 : 1;
              const float* src = ws_part + (size_t(cc) * 2 + wh) * (MPAD * BN);
#pragma unroll
              for (int m = 0; m < MPAD; ++m)
                if (m < M) tot[m] += __ldcg(src + m * BN + row);
            }
            if (row_in) {
#pragma unroll
              for (int m = 0; m < MPAD; ++m)
                if (m < M) Y[size_t(m) * N + n] = __float2bfloat16_rn(tot[m]);
            }
            if (etid == 0) ws_cnt[t] = 0;  // ready for the next call
          }
          named_bar_sync(EPI_BAR, 128);
        }
#pragma unroll
        for (int m = 0; m < MPAD; ++m) acc[m] = 0.f;
      }
      if (++qq == Q) {
        qq = 0;
        ++t;
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace gemv
}  // namespace wq

namespace wq_host {

// CTAs of the decode kernel: one per SM, never more than the units.
static int64_t gemv_ctas(int64_t N, int64_t K) {
  const int64_t U = ((N + 127) / 128) * ((K / 128 + 3) / 4);
  const int64_t P = sm_count();
  return U < P ? U : P;
}

size_t gemv_workspace_bytes(int64_t N, int64_t K) {
  const int64_t T = (N + 127) / 128;
  const size_t cnt = (size_t(T) * 4 + 255) & ~size_t(255);
  const size_t part = size_t(gemv_ctas(N, K)) * 2 * 128 * 16 * 4;
  return cnt + part;
}

namespace {
std::mutex g_tc_attr_mu;
bool g_tc_attr_done[64] = {};
}  // namespace

// The kernel's dynamic shared memory size, once per device (under a lock:
// several host threads may launch on the same device).
int prepare_tc_kernels() {
  int dev = 0;
  WQ_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev >= 64) return WQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_tc_attr_mu);
  if (!g_tc_attr_done[dev]) {
    WQ_CUDA_CHECK(cudaFuncSetAttribute(wq::gemv::gemv_w4a16_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(wq::gemv::SMEM_BYTES)));
    g_tc_attr_done[dev] = true;
  }
  return WQ_OK;
}

int launch_gemv_w4a16_tc(const void* X, int64_t M, int64_t K, const void* codes,
                         const void* scales, const void* zeros, int64_t N, int sym, void* Y,
                         void* ws, cudaStream_t s) {
  using namespace wq::gemv;
  const int64_t T = (N + 127) / 128;
  int* cnt = static_cast<int*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                         ((size_t(T) * 4 + 255) & ~size_t(255)));
  CUtensorMap tw, tx;
  int st = make_tmap_2d(&tw, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(N),
                        uint64_t(K / 2), BN, 128, 128);
  if (st != WQ_OK) return st;
  st = make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(M), uint64_t(K), MPAD,
                    64, 128);
  if (st != WQ_OK) return st;
  st = prepare_tc_kernels();
  if (st != WQ_OK) return st;
  const int grid = int(gemv_ctas(N, K));
  gemv_w4a16_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(
      tw, tx, static_cast<const __half*>(scales), static_cast<const __half*>(zeros),
      static_cast<__nv_bfloat16*>(Y), part, cnt, int(M), int(N), int(K / 128), sym,
      status_ptr(), wait_limit_ns());
  WQ_LAUNCH_CHECK("gemv_w4a16_tc_kernel");
  return WQ_OK;
}

}  // namespace wq_host
