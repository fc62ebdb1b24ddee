// Fused Lloyd K-means: every round of every task in ONE launch (bfloat16 rows, D = 64,
// at most 128 clusters per task).
//
// Separate K-means over queries and over keys: pith.science review of arXiv
// 2509.10406, "What carries the argument" / "Core claim"; gist.science
// "Technische Samenvatting", "Kernmechanismen" item 1.  Same rounds as kmeans.cu:
// start from the first C rows; a round assigns every row to its nearest centroid
// (ties to the lowest index) and replaces every centroid by the mean of its members
// (an empty cluster keeps its centroid); the labels of the last round are sorted
// stably into the CSR layout (perm, offsets) that every later stage reads.
//
// A task (one segment of one problem) is owned by a group of g = 1, 2, 4 or 8 CTAs
// of one thread-block cluster of 8; groups are packed into clusters on the host.
// Each CTA streams its share of the task's 128-row tiles through shared memory (TMA,
// 4 stages) every round and keeps the centroids in shared memory:
//   S = X_tile . (c_hi + c_lo)^T      tcgen05.mma, M = 128 rows, N = clusters, fp32 TMEM
//   label = argmin_c ||c||^2 - 2 S    two groups of 4 epilogue warps (tiles by parity),
//                                     a thread per row
//   Sum += OneHot^T . X_tile          tcgen05.mma, M = 128 clusters, N = D, K = rows:
//                                     the centroid sums as a contraction with the
//                                     0/1 membership matrix (exact products, no atomics)
// The centroid split c = c_hi + c_lo (bfloat16 parts) keeps the distance error below
// 2^-18 (||x||^2 + ||c||^2), inside the near-tie band of the label parity rule.
// End of a round: each CTA publishes its partial sums and member counts in shared
// memory; the group's CTAs reduce disjoint cluster slices by reading every member's
// partials through distributed shared memory in group order (deterministic), then
// every CTA gathers the new centroids.  Three cluster barriers per round; the third
// is split so that its wait overlaps the next round's tiles.
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (+ TMEM owner), warps 2-9 =
// epilogue.  Every mbarrier wait is bounded (MUSE_ERR_TIMEOUT); every CTA, idle
// padding CTAs included, executes the same sequence of cluster barriers.
#include <algorithm>
#include <numeric>
#include <vector>

#include "internal.h"
#include "tc_ptx.cuh"

namespace muse {
namespace kmf {

constexpr int TM = 128;        // rows per tile
constexpr int D = 64;          // row width handled by this kernel
constexpr int CMAX = 128;      // clusters per task
constexpr int GMAX = 8;        // CTAs per thread-block cluster (at most)
constexpr int TPC = 8;         // row tiles per CTA that a group size aims for
constexpr int kEpi = 8;        // epilogue warps
constexpr int kThreads = 64 + 32 * kEpi;
constexpr int PLD = D + 4;     // padded row stride (floats) of the partial sums
// Two variants by the largest cluster count CM of a launch: CM = 128, and CM = 64, whose
// shared memory (two row stages, one 64-cluster block per one-hot buffer) and TMEM fit
// two CTAs on an SM.
template <int CM> struct KCfg {
  static constexpr int NSX = CM == 64 ? 2 : 4;  // row-tile stages
  static constexpr int NOH = 2;                 // one-hot buffers
  static constexpr int OHB = CM / 64;           // 64-cluster blocks per one-hot buffer
  static constexpr uint32_t kTmemCols = CM == 64 ? 256 : 512;
  static constexpr uint32_t kSumCol = 2 * CM;   // TMEM column of the centroid-sum accumulator
};

struct PlanEntry {
  uint8_t seg, g;
  uint16_t pos;  // first CTA of the group inside the problem's span
};
struct Job {
  const void *X;
  SegTable tab;
  KmeansOut out;
  int span;  // CTAs per problem (multiple of the job's largest group)
  int base;  // first CTA of the job
  int nent;
  PlanEntry ent[kMaxSeg];
};
struct Params {
  int njobs, P, N, iters;
  Job job[2];
};

template <int CM> struct __align__(1024) Smem {
  using Cf = KCfg<CM>;
  // one-hot rows [row][cluster] in 64-cluster blocks; the row tiles follow them, so that
  // with one block (CM = 64) the sums contraction's second M block (clusters 64-127, whose
  // TMEM lanes are never read) reads finite data inside the CTA's shared memory
  __nv_bfloat16 oh[Cf::NOH][Cf::OHB][TM * 64];
  __nv_bfloat16 x[Cf::NSX][TM * 64];  // row tiles, rows of 128 B, 128-byte swizzle
  __nv_bfloat16 hi[CM * 64];          // centroid split, K-major, 128-byte swizzle
  __nv_bfloat16 lo[CM * 64];
  float part[CM * PLD];               // partial sums; the reducer's new centroids in place
  float cn[CM];                       // squared centroid norms (+inf on padding rows)
  int cnt[CM];                        // this CTA's member counts of the round
  int tot[CM];                        // group totals of the clusters this CTA reduces
  int totall[CM];                     // group totals of every cluster
  int base[CM];                       // final sort: next position per cluster
  int wc[4][CM];                      // final sort: members per (warp, cluster) of a tile
  uint64_t xfull[Cf::NSX], xempty[Cf::NSX], sfull[2], sfree[2], ohfull[Cf::NOH], ohempty[Cf::NOH];
  uint64_t sumdone, fin;
  uint32_t tmem_base;
  int abort_flag;
};

using namespace ptx;

// ------------------------------------------------------------------ cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t peer_addr(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_peer_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a)
               : "memory");
  return v;
}
__device__ __forceinline__ int ld_peer_s32(uint32_t a) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Shared-memory descriptor of an MN-major operand with 128-byte swizzle: rows of
// 128 B hold 64 consecutive M (or N) elements of one K index, 8 K-rows per 1024-B
// atom (SBO), `lbo` bytes between successive 64-element blocks along M (or N).
__device__ __forceinline__ uint64_t sdesc_mn(const void *p, uint32_t lbo) {
  const uint32_t a = saddr(p);
  uint64_t d = 0;
  d |= (uint64_t)((a & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// kind::f16 instruction descriptor with both operands MN-major.
__host__ __device__ constexpr uint32_t idesc_mn(int M, int N) {
  return idesc(M, N) | (1u << 15) | (1u << 16);
}


// Writes half h (32 values) of centroid row c into the K-major split operands and
// returns the partial squared norm.
template <int CM>
__device__ __forceinline__ float put_centroid(Smem<CM> &sm, int c, int h, const float (&v)[32]) {
  float sq = 0.f;
#pragma unroll
  for (int j4 = 0; j4 < 4; ++j4) {
    const int j = 4 * h + j4;
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float a = v[8 * j4 + e], b = v[8 * j4 + e + 1];
      const __nv_bfloat162 hh = __floats2bfloat162_rn(a, b);
      const float2 hf = __bfloat1622float2(hh);
      const __nv_bfloat162 ll = __floats2bfloat162_rn(a - hf.x, b - hf.y);
      hw[e >> 1] = *reinterpret_cast<const uint32_t *>(&hh);
      lw[e >> 1] = *reinterpret_cast<const uint32_t *>(&ll);
      sq = fmaf(a, a, sq);
      sq = fmaf(b, b, sq);
    }
    const int off = c * 64 + ((j ^ (c & 7)) << 3);
    *reinterpret_cast<uint4 *>(&sm.hi[off]) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4 *>(&sm.lo[off]) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
  return sq;
}

template <int CM>
__global__ void __launch_bounds__(kThreads, CM == 64 ? 2 : 1)
km_fused(const __grid_constant__ CUtensorMap map0, const __grid_constant__ CUtensorMap map1,
         const __grid_constant__ Params prm, int *status) {
  using Cf = KCfg<CM>;
  constexpr int NSX = Cf::NSX, NOH = Cf::NOH;
  constexpr uint32_t kTmemCols = Cf::kTmemCols, kSumCol = Cf::kSumCol;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem<CM> &sm = *reinterpret_cast<Smem<CM> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &sm.abort_flag;

  // ---------------------------------------------- the group and task of this CTA
  const int jb = (prm.njobs > 1 && (int)blockIdx.x >= prm.job[1].base) ? 1 : 0;
  const Job &J = prm.job[jb];
  const CUtensorMap *map = jb ? &map1 : &map0;
  const int local = (int)blockIdx.x - J.base;
  const int p = local / J.span, lp = local - p * J.span;
  int seg = -1, g = 1, rank = 0;
  if (p < prm.P)
    for (int e = 0; e < J.nent; ++e) {
      const int pos = J.ent[e].pos, ge = J.ent[e].g;
      if (lp >= pos && lp < pos + ge) {
        seg = J.ent[e].seg;
        g = ge;
        rank = lp - pos;
        break;
      }
    }
  const bool active = seg >= 0;  // uniform over the CTA
  Task tk{};
  if (active) tk = make_task(J.tab, p * J.tab.nseg + seg);
  const int C = tk.C;
  const int CP = (C + 31) & ~31;                      // assign N: both halves multiples of 16
  const uint32_t gb = cluster_rank() - (uint32_t)rank;  // cluster rank of the group's first CTA
  const int ntt = (tk.n + TM - 1) / TM;
  const int tpc = (ntt + g - 1) / g;
  const int t0 = rank * tpc;
  const int nt = active ? max(0, min(ntt - t0, tpc)) : 0;  // this CTA's row tiles
  const int64_t grow0 = (int64_t)p * prm.N + tk.row0;
  const int T = prm.iters;

  // ---------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < NSX; ++i) {
      mbar_init(&sm.xfull[i], 1);
      mbar_init(&sm.xempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.sfree[i], kEpi / 2);  // one group per S buffer
    }
    for (int i = 0; i < NOH; ++i) {
      mbar_init(&sm.ohfull[i], kEpi / 2);
      mbar_init(&sm.ohempty[i], 1);
    }
    mbar_init(&sm.sumdone, 1);
    mbar_init(&sm.fin, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (active && warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(&sm.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (active) {
    // starting centroids: the first C rows of the task
    for (int tid = threadIdx.x; tid < 2 * CM; tid += kThreads) {
      const int c = tid >> 1, h = tid & 1;
      float v[32];
      const __nv_bfloat16 *xr = static_cast<const __nv_bfloat16 *>(J.X) + (grow0 + c) * D + h * 32;
#pragma unroll
      for (int k = 0; k < 32; k += 8) {
        uint4 raw = make_uint4(0u, 0u, 0u, 0u);
        if (c < C) raw = *reinterpret_cast<const uint4 *>(xr + k);
        const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b2[e]);
          v[k + 2 * e] = f.x;
          v[k + 2 * e + 1] = f.y;
        }
      }
      float sq = put_centroid(sm, c, h, v);
      sq += __shfl_xor_sync(0xffffffffu, sq, 1);
      if (c < C && c % g == rank) {  // the reducer of c keeps the current centroid in memory
        float4 *gc = reinterpret_cast<float4 *>(J.out.centroids + (tk.cen + c) * D + h * 32);
#pragma unroll
        for (int k = 0; k < 8; ++k) gc[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
      }
      if (h == 0) {
        sm.cn[c] = c < C ? sq : CUDART_INF_F;
        sm.cnt[c] = 0;
      }
    }
    for (int e = threadIdx.x; e < 4 * CM; e += kThreads) (&sm.wc[0][0])[e] = 0;
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  int loaded = 0;  // producer: row tiles issued, counted over all rounds
  for (int r = 0; r < T; ++r) {
    const bool last = r == T - 1;
    const int u0 = r * nt;
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0 && nt > 0 && !*abort_flag) {
        // this round's tiles, then the next round's first stages (the rows do not change)
        const int target = (r + 1) * nt + (last ? 0 : min(NSX, nt));
        for (; loaded < target; ++loaded) {
          const int u = loaded, st = u % NSX, t = u % nt;
          if (u >= NSX && !mbar_wait(&sm.xempty[st], ((u / NSX) - 1) & 1, abort_flag, status)) break;
          mbar_expect_tx(&sm.xfull[st], TM * 128);
          tma_load_2d(sm.x[st], map, 0, (int)(grow0 + (int64_t)(t0 + t) * TM), &sm.xfull[st]);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      // Two in-order streams, whichever is ready goes first: distances of tile u
      // (needs the rows and the S buffer of tile u-2 read by its group) and the
      // centroid sums of tile u (needs its one-hot rows).
      if (lane == 0 && nt > 0 && !*abort_flag) {
        int a = 0, sidx = 0;  // next tile of each stream (within the round)
        int idle = 0;
        uint64_t t_idle = 0;
        bool ok = true;
        while (ok && sidx < nt) {
          bool progressed = false;
          if (a < nt) {
            const int u = u0 + a, st = u % NSX, buf = u & 1;
            if (mbar_test(&sm.xfull[st], (u / NSX) & 1) &&
                (u < 2 || mbar_test(&sm.sfree[buf], ((u - 2) >> 1) & 1))) {
              tc_fence_after();
              const uint32_t id = idesc(TM, CP);
              for (int kk = 0; kk < D / 16; ++kk)
                tc_mma(tmem + buf * CM, sdesc(sm.x[st] + kk * 16), sdesc(sm.hi + kk * 16), id, kk > 0 ? 1u : 0u);
              for (int kk = 0; kk < D / 16; ++kk)
                tc_mma(tmem + buf * CM, sdesc(sm.x[st] + kk * 16), sdesc(sm.lo + kk * 16), id, 1u);
              tc_commit(&sm.sfull[buf]);
              ++a;
              progressed = true;
            }
          }
          if (sidx < a) {
            const int u = u0 + sidx, st = u % NSX, ob = u % NOH;
            if (mbar_test(&sm.ohfull[ob], (u / NOH) & 1)) {
              tc_fence_after();
              const uint32_t id = idesc_mn(TM, D);
              for (int ks = 0; ks < TM / 16; ++ks)
                tc_mma(tmem + kSumCol, sdesc_mn(sm.oh[ob][0] + ks * 16 * 64, TM * 64 * 2),
                       sdesc_mn(sm.x[st] + ks * 16 * 64, TM * 64 * 2), id, (sidx == 0 && ks == 0) ? 0u : 1u);
              tc_commit(&sm.ohempty[ob]);
              tc_commit(&sm.xempty[st]);
              ++sidx;
              progressed = true;
            }
          }
          if (progressed) {
            idle = 0;
            continue;
          }
          if ((++idle & 255) == 0) {  // the same time limit as every other wait
            if (*abort_flag) {
              ok = false;
            } else {
              const uint64_t now = now_ns();
              if (idle == 256) {
                t_idle = now;
              } else if (now - t_idle > kTimeoutNs) {
                *abort_flag = 1;
                report(status, MUSE_ERR_TIMEOUT);
                ok = false;
              }
            }
          }
        }
        tc_commit(&sm.sumdone);  // tracks every MMA issued this round, on the abort path too
      }
      __syncwarp();
    } else {
      // ------------------------------------------------------------ epilogue
      // Two groups of four warps take the tiles of parity 0 and 1; a thread owns one
      // row (TMEM lane) and scans all CP distance columns.
      const int grp = (warp - 2) >> 2, quad = warp & 3;
      const int rr = quad * 32 + lane;
      const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
      for (int t = 0; t < nt; ++t) {
        const int u = u0 + t, buf = u & 1, ob = u % NOH;
        if (buf != grp) continue;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.sfull[buf], (u >> 1) & 1, abort_flag, status))) break;
        tc_fence_after();
        // 16-column chunks in batches of NB (four; two in the 64-cluster variant, which
        // has half the registers), one chain per chunk; chains and batches are merged
        // in column order (strict <: the lowest index wins a tie)
        constexpr int NB = CM == 64 ? 2 : 4;
        float bv = CUDART_INF_F;
        int bc = 0;
        for (int c0 = 0; c0 < CP; c0 += 16 * NB) {
          uint32_t raw[NB][16];
#pragma unroll
          for (int ch = 0; ch < NB; ++ch)
            if (c0 + ch * 16 < CP) tmem_ld16_async(tmem + lane_base + buf * CM + c0 + ch * 16, raw[ch]);
          tmem_ld_wait();
          if (c0 + 16 * NB >= CP) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sfree[buf]);
          }
          float best[NB];
          int bi[NB];
#pragma unroll
          for (int ch = 0; ch < NB; ++ch) {
            best[ch] = CUDART_INF_F;
            bi[ch] = 0;
            if (c0 + ch * 16 < CP) {
#pragma unroll
              for (int e4 = 0; e4 < 4; ++e4) {
                const float4 n4 = *reinterpret_cast<const float4 *>(&sm.cn[c0 + ch * 16 + 4 * e4]);
                const float nn[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float dd = fmaf(-2.f, __uint_as_float(raw[ch][4 * e4 + e]), nn[e]);
                  if (dd < best[ch]) {
                    best[ch] = dd;
                    bi[ch] = c0 + ch * 16 + 4 * e4 + e;
                  }
                }
              }
            }
          }
#pragma unroll
          for (int ch = 0; ch < NB; ++ch)
            if (best[ch] < bv) {
              bv = best[ch];
              bc = bi[ch];
            }
        }
        const int row = (t0 + t) * TM + rr;
        const bool valid = row < tk.n;
        const int L = valid ? min(bc, C - 1) : -1;
        if (valid) {
          atomicAdd(&sm.cnt[L], 1);  // integer: exact in any order
          if (last) J.out.labels[tk.lab + row] = L;
        }
        // this row's one-hot entries (bf16 1.0 = 0x3F80), both 64-cluster blocks
        if (u >= NOH &&
            !__all_sync(0xffffffffu, mbar_wait(&sm.ohempty[ob], ((u / NOH) - 1) & 1, abort_flag, status)))
          break;
        const uint32_t one = (L & 1) ? 0x3F800000u : 0x00003F80u;
        const int w = (L & 7) >> 1;
#pragma unroll
        for (int half = 0; half < Cf::OHB; ++half) {
          unsigned char *dst = reinterpret_cast<unsigned char *>(sm.oh[ob][half]) + rr * 128;
          const int lc = L - half * 64;
          const bool hit = lc >= 0 && lc < 64;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const bool here = hit && (lc >> 3) == j;
            const uint4 val = make_uint4(here && w == 0 ? one : 0u, here && w == 1 ? one : 0u,
                                         here && w == 2 ? one : 0u, here && w == 3 ? one : 0u);
            *reinterpret_cast<uint4 *>(dst + ((j ^ (rr & 7)) << 4)) = val;
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ohfull[ob]);
      }
    }

    // ---------------------------------------------------------------- end of the round
    // (1) this CTA's partial sums (TMEM lane = cluster) into `part`, once every peer has
    //     finished reading the previous round's contents
    if (r > 0) cluster_wait();
    if (active && warp >= 2) {
      const int half = (warp - 2) >> 2, quad = warp & 3;
      const int c = quad * 32 + lane;
      float v[32];
      bool have = false;
      if (nt > 0) have = __all_sync(0xffffffffu, mbar_wait(&sm.sumdone, r & 1, abort_flag, status));
      if (have) {
        tc_fence_after();
        float a[16], b[16];
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + kSumCol + half * 32, a);
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + kSumCol + half * 32 + 16, b);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          v[e] = a[e];
          v[16 + e] = b[e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
      }
      if (c < CM) {  // (lanes past CM hold the second M block's unused sums)
        float4 *dst = reinterpret_cast<float4 *>(&sm.part[c * PLD + half * 32]);
#pragma unroll
        for (int k = 0; k < 8; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
      }
      tc_fence_before();
    }
    __syncwarp();
    cluster_arrive();
    cluster_wait();
    // (2) reduction: this CTA owns the clusters c = rank + g k; members summed in group order
    if (active) {
      const int nslice = (C - rank + g - 1) / g;
      for (int it = threadIdx.x; it < nslice * (D / 4); it += kThreads) {
        const int c = rank + g * (it / (D / 4)), v4 = it % (D / 4);
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        int total = 0;
        for (int m = 0; m < g; ++m) {
          const float4 a = ld_peer_f4(peer_addr(&sm.part[c * PLD + 4 * v4], gb + m));
          s.x += a.x;
          s.y += a.y;
          s.z += a.z;
          s.w += a.w;
          total += ld_peer_s32(peer_addr(&sm.cnt[c], gb + m));
        }
        float4 *gc = reinterpret_cast<float4 *>(J.out.centroids + (tk.cen + c) * D + 4 * v4);
        float4 nv;
        if (total > 0) {
          const float inv = 1.f / (float)total;
          nv = make_float4(s.x * inv, s.y * inv, s.z * inv, s.w * inv);
        } else {
          nv = *gc;  // empty: keeps its centroid
        }
        *reinterpret_cast<float4 *>(&sm.part[c * PLD + 4 * v4]) = nv;
        *gc = nv;
        if (v4 == 0) sm.tot[c] = total;
      }
    }
    __syncwarp();
    cluster_arrive();
    cluster_wait();
    // (3) every CTA gathers the new centroids (split operands, norms) and the totals
    if (active) {
      for (int tid = threadIdx.x; tid < 2 * CM; tid += kThreads) {
        const int c = tid >> 1, h = tid & 1;
        const uint32_t q = gb + (uint32_t)(c % g);
        float v[32];
        if (c < C) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 a = ld_peer_f4(peer_addr(&sm.part[c * PLD + h * 32 + 4 * k], q));
            v[4 * k] = a.x;
            v[4 * k + 1] = a.y;
            v[4 * k + 2] = a.z;
            v[4 * k + 3] = a.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0.f;
        }
        float sq = put_centroid(sm, c, h, v);
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        if (h == 0) {
          sm.cn[c] = c < C ? sq : CUDART_INF_F;
          sm.totall[c] = c < C ? ld_peer_s32(peer_addr(&sm.tot[c], q)) : 0;
          if (!last) sm.cnt[c] = 0;
        }
      }
      if (last) {
        // CSR offsets (exclusive scan of the totals) and, for this CTA's rows, the first
        // position of each cluster: offsets + the members held by earlier CTAs of the group
        __syncthreads();
        if (warp == 2) {
          int tv[4], s = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            tv[k] = 4 * lane + k < CM ? sm.totall[4 * lane + k] : 0;
            s += tv[k];
          }
          int inc = s;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
          }
          int run = inc - s;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int c = 4 * lane + k;
            if (c < C) {
              sm.base[c] = run;
              if (rank == 0) J.out.offsets[tk.off + c] = run;
            }
            run += tv[k];
          }
          if (lane == 31 && rank == 0) J.out.offsets[tk.off + C] = run;
        }
        __syncthreads();
        if (threadIdx.x < C) {
          int b = sm.base[threadIdx.x];
          for (int m = 0; m < rank; ++m) b += ld_peer_s32(peer_addr(&sm.cnt[threadIdx.x], gb + m));
          sm.base[threadIdx.x] = b;
        }
      }
    }
    __syncwarp();
    cluster_arrive();  // its wait comes before the next write of `part` (or before exit)
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  // ------------------------------------------------ stable scatter of the last labels
  const bool aborted = *abort_flag != 0;  // read after the barrier above: uniform
  if (active && !aborted && warp >= 2 && warp < 6) {
    const int quad = warp & 3, rr = quad * 32 + lane;
    for (int t = 0; t < nt; ++t) {
      const int row = (t0 + t) * TM + rr;
      const bool valid = row < tk.n;
      const int L = valid ? J.out.labels[tk.lab + row] : -1;  // written by this thread
      const unsigned peers = __match_any_sync(0xffffffffu, L);
      const int wrank = __popc(peers & ((1u << lane) - 1u));
      if (valid && wrank == 0) sm.wc[quad][L] = __popc(peers);
      named_sync(1, 128);
      if (valid) {
        int pos = sm.base[L] + wrank;
        for (int q2 = 0; q2 < quad; ++q2) pos += sm.wc[q2][L];
        if (pos >= 0 && pos < tk.n)
          J.out.perm[tk.lab + pos] = tk.row0 + row;
        else
          report(status, MUSE_ERR_DEVICE);
      }
      named_sync(1, 128);
      if (rr < C) {
        int s = 0;
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) {
          s += sm.wc[q2][rr];
          sm.wc[q2][rr] = 0;
        }
        sm.base[rr] += s;
      }
      named_sync(1, 128);
    }
  }

  cluster_wait();  // every peer has finished reading this CTA's shared memory
  // ------------------------------------------------ teardown
  if (warp == 0 && lane == 0)
    for (int u = max(0, loaded - NSX); u < loaded; ++u) mbar_drain(&sm.xfull[u % NSX], (u / NSX) & 1, status);
  if (active && warp == 1 && lane == 0) {
    tc_commit(&sm.fin);
    mbar_drain(&sm.fin, 0, status);
  }
  tc_fence_before();
  __syncthreads();
  if (active && warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host side
// Thread-block clusters of Z = 8 or 6 CTAs (a launch attribute); a task's group is a
// divisor of Z, so that groups placed at multiples of their size never straddle a
// cluster.  Clusters of 6 fit 22 to a B200 at this kernel's shared memory, clusters of
// 8 only 15: for 16 tasks of 64 row tiles, groups of 6 (11 tiles per CTA) then beat
// groups of 4 (16 tiles per CTA).
static int group_size(int n, int tpc, int Z) {
  const int tiles = (n + TM - 1) / TM;
  const int want = (tiles + tpc - 1) / tpc;
  for (int g = 1; g < Z; ++g)
    if (Z % g == 0 && g >= want) return g;
  return Z;
}

// Lays the segments of one problem out in CTA slots, largest groups first, each group at
// a multiple of its size.  Returns the least common multiple of the group sizes, the
// alignment of the problem's span and of the job's first CTA.
static int plan_job(Job &J, const SegTable &t, int tpc, int Z) {
  std::vector<int> order(t.nseg);
  for (int s = 0; s < t.nseg; ++s) order[s] = s;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    return group_size(t.nrow[a], tpc, Z) > group_size(t.nrow[b], tpc, Z);
  });
  int pos = 0, L = 1;
  for (int e = 0; e < t.nseg; ++e) {
    const int s = order[e], g = group_size(t.nrow[s], tpc, Z);
    pos = (pos + g - 1) / g * g;
    J.ent[e].seg = (uint8_t)s;
    J.ent[e].g = (uint8_t)g;
    J.ent[e].pos = (uint16_t)pos;
    pos += g;
    L = std::lcm(L, g);
  }
  J.nent = t.nseg;
  J.span = (pos + L - 1) / L * L;
  return L;
}

// Plans every job for cluster size Z and group target tpc; returns the grid (a multiple
// of Z) and the largest number of row tiles a CTA takes.
static int plan_all(Params &prm, int njobs, const void *const *X, const SegTable *const *tabs,
                    const KmeansOut *outs, int tpc, int Z, int &max_tiles) {
  int cursor = 0;
  max_tiles = 0;
  for (int j = 0; j < njobs; ++j) {
    Job &J = prm.job[j];
    J.X = X[j];
    J.tab = *tabs[j];
    J.out = outs[j];
    const int L = plan_job(J, *tabs[j], tpc, Z);
    cursor = (cursor + L - 1) / L * L;
    J.base = cursor;
    cursor += prm.P * J.span;
    for (int e = 0; e < J.nent; ++e) {
      const int tiles = (J.tab.nrow[J.ent[e].seg] + TM - 1) / TM;
      max_tiles = std::max(max_tiles, (tiles + J.ent[e].g - 1) / J.ent[e].g);
    }
  }
  return (cursor + Z - 1) / Z * Z;
}

}  // namespace kmf

// CTAs of the fused kernel (variant CM) that can be resident at once in clusters of Z
// (0: not even one cluster fits).
template <int CM>
static int kmf_capacity(int Z) {
  static int cap[kmf::GMAX + 1] = {-1, -1, -1, -1, -1, -1, -1, -1, -1};
  if (cap[Z] < 0) {
    const size_t smem = sizeof(kmf::Smem<CM>) + 1024;
    int n = 0;
    if (cudaFuncSetAttribute(kmf::km_fused<CM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = Z;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(Z);
      cfg.blockDim = dim3(kmf::kThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, kmf::km_fused<CM>, &cfg) != cudaSuccess) n = 0;
    }
    if (n <= 0) cudaGetLastError();  // the multi-launch path takes over; leave no error behind
    cap[Z] = n * Z;
  }
  return cap[Z];
}

bool kmeans_fused_supported(int dtype, int D, const SegTable &t) {
  if (dtype != MUSE_BF16 || D != kmf::D || t.max_C > kmf::CMAX || t.nseg > 255) return false;
  int span = 0;
  for (int s = 0; s < t.nseg; ++s) span += kmf::group_size(t.nrow[s], kmf::TPC, kmf::GMAX);
  if (span > 65535 / 3) return false;  // positions of any plan (groups of 6 are at most 1.5x, padding < 2x) fit 16 bits
  return (t.max_C <= 64 ? kmf_capacity<64>(kmf::GMAX) : kmf_capacity<128>(kmf::GMAX)) > 0;
}

template <int CM>
static cudaError_t launch_fused(int njobs, const void *const *X, const SegTable *const *tabs,
                                const KmeansOut *outs, int N, int P, int iters, int *status,
                                cudaStream_t st) {
  using namespace kmf;
  Params prm{};
  prm.njobs = njobs;
  prm.P = P;
  prm.N = N;
  prm.iters = iters;
  // Among the plans whose CTAs are all resident at once (clusters of 8 or 6, about
  // 8 .. 64 row tiles per CTA), the one with the fewest row tiles per CTA; if none fits,
  // clusters of 8 with about 8 tiles per CTA, in several waves.
  int bestZ = GMAX, best_tpc = TPC, best_tiles = 1 << 30;
  for (int Z : {GMAX, 6}) {
    const int cap = kmf_capacity<CM>(Z);
    if (cap <= 0) continue;
    for (int tpc = TPC; tpc <= 8 * TPC; tpc *= 2) {
      int tiles = 0;
      const int grid = plan_all(prm, njobs, X, tabs, outs, tpc, Z, tiles);
      if (grid <= cap && tiles < best_tiles) {
        best_tiles = tiles;
        bestZ = Z;
        best_tpc = tpc;
      }
    }
  }
  int tiles = 0;
  const int grid = plan_all(prm, njobs, X, tabs, outs, best_tpc, bestZ, tiles);
  CUtensorMap m0, m1;
  if (!ptx::make_map(&m0, X[0], D, (uint64_t)P * N, D, TM) ||
      !ptx::make_map(&m1, X[njobs > 1 ? 1 : 0], D, (uint64_t)P * N, D, TM))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem<CM>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(km_fused<CM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = bestZ;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, km_fused<CM>, m0, m1, prm, status);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The 64-cluster variant (two CTAs per SM) when every task of the launch has C <= 64.
cudaError_t run_kmeans_fused(int njobs, const void *const *X, const SegTable *const *tabs,
                             const KmeansOut *outs, int N, int P, int iters, int *status,
                             cudaStream_t st) {
  int maxC = 0;
  for (int j = 0; j < njobs; ++j) maxC = std::max(maxC, tabs[j]->max_C);
  if (maxC <= 64 && kmf_capacity<64>(kmf::GMAX) > 0)
    return launch_fused<64>(njobs, X, tabs, outs, N, P, iters, status, st);
  return launch_fused<128>(njobs, X, tabs, outs, N, P, iters, status, st);
}

}  // namespace muse
