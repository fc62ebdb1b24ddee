// Lloyd K-means over the segments of one or two SegTables (queries and keys are
// clustered in the same launches), batched over (problem, segment).
//
// Separate K-means over queries and over keys: pith.science review of arXiv
// 2509.10406, "What carries the argument" / "Core claim"; gist.science
// "Technische Samenvatting", "Kernmechanismen" item 1.
//
// One round = assign (nearest centroid, ties to the lowest index) + update (mean of
// the members, an empty cluster keeps its centroid).  The update is a stable
// counting sort of the rows by label (perm/offsets, the CSR layout every later
// stage reads) followed by per-cluster sums over the sorted members in a fixed
// order (fixed member slots, then a fixed-order reduction of the slots): no
// floating-point atomics, bitwise reproducible.
//
// Per round: km_assign (distances ||c||^2 - 2 x.c, argmin, per-chunk label histogram
// and in-chunk stable rank), km_scan (per-cluster chunk bases, offsets), km_scatter
// (perm), km_centroid (means).
//
// bfloat16 inputs take km_assign_tc: the x.c products on the tensor cores
// (tcgen05.mma, fp32 accumulation in TMEM) against the centroids split into two
// bfloat16 parts, c = c_hi + c_lo + r with |r| <= 2^-18 |c| elementwise, so the
// distance error is at most 2^-17 sum_d |x_d c_d| <= 2^-18 (||x||^2 + ||c||^2):
// below the near-tie band 1e-5 (||x||^2 + ||c||^2) inside which labels may differ
// from an exact evaluation.
#include <algorithm>

#include "internal.h"
#include "tc_ptx.cuh"

namespace muse {

constexpr int kChunk = 128;   // rows per counting-sort chunk (= rows per assign CTA)
constexpr int kWarps = kChunk / 32;
constexpr int kTcChunks = 4;  // chunks per tensor-core assign CTA (centroids staged once)
constexpr int kCTile = 64;    // centroids staged in shared memory at a time

struct KmJob {
  const void *X;
  SegTable tab;
  KmeansOut out;
  int32_t *lrank;
};
struct KmJobs {
  int njobs, tasks0, nch, maxC;  // tasks of job 0; chunk count and cluster stride of the scratch
  int CP;                        // padded cluster stride of the split centroids (multiple of 16)
  __nv_bfloat16 *chi, *clo;      // [task][CP][D] bf16 split of the centroids (tensor-core path)
  float *cn;                     // [task][CP] squared centroid norms (+inf on padding rows)
  KmJob job[2];
};

struct KmCtx {
  const KmJob *job;
  Task tk;
  int tg;  // global task index (row of the count/base scratch)
};
__device__ __forceinline__ KmCtx km_ctx(const KmJobs &J, int tg) {
  KmCtx c;
  c.tg = tg;
  const int jb = (J.njobs > 1 && tg >= J.tasks0) ? 1 : 0;
  c.job = &J.job[jb];
  c.tk = make_task(c.job->tab, tg - (jb ? J.tasks0 : 0));
  return c;
}

// Initial centroids (the first C rows), their bf16 split and squared norms; one warp
// per centroid row, rows C..CP-1 are padding (+inf norm: never the nearest).
template <typename T, int D>
__global__ void __launch_bounds__(256)
km_init(KmJobs J, int N) {
  const KmCtx k = km_ctx(J, blockIdx.y);
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (c >= J.CP) return;
  const bool real = c < k.tk.C;
  const T *x = static_cast<const T *>(k.job->X) + ((int64_t)k.tk.p * N + k.tk.row0 + c) * D;
  float sq = 0.f;
#pragma unroll
  for (int u = 0; u < D / 32; ++u) {
    const int d = lane + 32 * u;
    const float v = real ? ld_elem(x + d) : 0.f;
    if (real) k.job->out.centroids[(k.tk.cen + c) * D + d] = v;
    if (J.chi) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      J.chi[((int64_t)k.tg * J.CP + c) * D + d] = hi;
      J.clo[((int64_t)k.tg * J.CP + c) * D + d] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
    sq = fmaf(v, v, sq);
  }
  sq = warp_sum(sq);
  if (J.chi && lane == 0) J.cn[(int64_t)k.tg * J.CP + c] = real ? sq : CUDART_INF_F;
}

// Per-chunk label histogram (cluster-major counts[tg][c][chunk]) and the stable rank
// of every row inside its chunk.  Called by all kChunk threads of the CTA.
__device__ __forceinline__ void chunk_count(const KmJobs &J, const KmCtx &k, int chunk, int r,
                                            bool valid, int L, int *cnt, int32_t *counts) {
  const Task &tk = k.tk;
  __syncthreads();
  for (int e = threadIdx.x; e < kWarps * tk.C; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const unsigned peers = __match_any_sync(0xffffffffu, L);
  const int wrank = __popc(peers & ((1u << lane) - 1u));
  if (valid && wrank == 0) cnt[w * tk.C + L] = __popc(peers);
  __syncthreads();
  if (valid) {
    int before = 0;
    for (int w2 = 0; w2 < w; ++w2) before += cnt[w2 * tk.C + L];
    k.job->lrank[tk.lab + r] = before + wrank;
  }
  for (int c = threadIdx.x; c < tk.C; c += blockDim.x) {
    int s = 0;
#pragma unroll
    for (int w2 = 0; w2 < kWarps; ++w2) s += cnt[w2 * tk.C + c];
    counts[((int64_t)k.tg * J.maxC + c) * J.nch + chunk] = s;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kChunk)
km_assign(KmJobs J, int N, int32_t *__restrict__ counts) {
  extern __shared__ float smem[];
  float *cs = smem;                                   // [kCTile][D]
  float *cn = smem + kCTile * D;                      // [kCTile] squared norms
  int *cnt = reinterpret_cast<int *>(cn + kCTile);    // [kWarps][C]
  const KmCtx k = km_ctx(J, blockIdx.y);
  const Task &tk = k.tk;
  const int chunk = blockIdx.x;
  if (chunk * kChunk >= tk.n) return;  // uniform over the CTA
  const int r = chunk * kChunk + threadIdx.x;
  const bool valid = r < tk.n;

  float x[D];
  {
    const T *xr = static_cast<const T *>(k.job->X) + ((int64_t)tk.p * N + tk.row0 + (valid ? r : 0)) * D;
#pragma unroll
    for (int d = 0; d < D; ++d) x[d] = valid ? ld_elem(xr + d) : 0.f;
  }
  float best = CUDART_INF_F;
  int bi = 0;
  const float *cg = k.job->out.centroids + tk.cen * D;
  for (int c0 = 0; c0 < tk.C; c0 += kCTile) {
    const int ct = min(kCTile, tk.C - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < ct * D; e += blockDim.x) cs[e] = cg[(int64_t)c0 * D + e];
    __syncthreads();
    if (threadIdx.x < ct) {
      float s = 0.f;
      for (int d = 0; d < D; ++d) s = fmaf(cs[threadIdx.x * D + d], cs[threadIdx.x * D + d], s);
      cn[threadIdx.x] = s;
    }
    __syncthreads();
    // ||x - c||^2 - ||x||^2 = ||c||^2 - 2 x.c, four centroids per pass
    int c = 0;
    for (; c + 4 <= ct; c += 4) {
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      const float4 *p0 = reinterpret_cast<const float4 *>(cs + c * D);
#pragma unroll
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 v0 = p0[d4], v1 = p0[D / 4 + d4], v2 = p0[2 * (D / 4) + d4],
                     v3 = p0[3 * (D / 4) + d4];
        const float x0 = x[4 * d4], x1 = x[4 * d4 + 1], x2 = x[4 * d4 + 2], x3 = x[4 * d4 + 3];
        a0 = fmaf(x0, v0.x, fmaf(x1, v0.y, fmaf(x2, v0.z, fmaf(x3, v0.w, a0))));
        a1 = fmaf(x0, v1.x, fmaf(x1, v1.y, fmaf(x2, v1.z, fmaf(x3, v1.w, a1))));
        a2 = fmaf(x0, v2.x, fmaf(x1, v2.y, fmaf(x2, v2.z, fmaf(x3, v2.w, a2))));
        a3 = fmaf(x0, v3.x, fmaf(x1, v3.y, fmaf(x2, v3.z, fmaf(x3, v3.w, a3))));
      }
      const float d0 = fmaf(-2.f, a0, cn[c]), d1 = fmaf(-2.f, a1, cn[c + 1]);
      const float d2 = fmaf(-2.f, a2, cn[c + 2]), d3 = fmaf(-2.f, a3, cn[c + 3]);
      if (d0 < best) { best = d0; bi = c0 + c; }      // strict: the lowest index wins a tie
      if (d1 < best) { best = d1; bi = c0 + c + 1; }
      if (d2 < best) { best = d2; bi = c0 + c + 2; }
      if (d3 < best) { best = d3; bi = c0 + c + 3; }
    }
    for (; c < ct; ++c) {
      float a = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) a = fmaf(x[d], cs[c * D + d], a);
      const float dd = fmaf(-2.f, a, cn[c]);
      if (dd < best) { best = dd; bi = c0 + c; }
    }
  }
  const int L = valid ? bi : -1;
  if (valid) k.job->out.labels[tk.lab + r] = L;
  chunk_count(J, k, chunk, r, valid, L, cnt, counts);
}


// ---------------------------------------------------------------------------
// Tensor-core assign (bfloat16 inputs).  One CTA (4 warps, 128 rows per chunk) takes
// up to kTcChunks consecutive chunks of one task; the centroid split is staged in
// shared memory once per CTA (in tiles of 256 centroids when C > 256).
//   S[row][c] = x_row . (c_hi + c_lo)   (tcgen05.mma, M = 128, N <= 256, fp32 TMEM)
//   label = argmin_c (||c||^2 - 2 S[row][c])  (strict <: the lowest index wins a tie)
// ---------------------------------------------------------------------------
template <int D>
struct TcAssignSmem {
  __nv_bfloat16 x[D / 64][kChunk * 64];  // row tile, K-major SW128 blocks
  __nv_bfloat16 hi[D / 64][256 * 64];    // centroid split, same layout
  __nv_bfloat16 lo[D / 64][256 * 64];
  float cn[256];
  uint64_t xbar, mbar;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kChunk, 1)
km_assign_tc(const __grid_constant__ CUtensorMap map0, const __grid_constant__ CUtensorMap map1,
             KmJobs J, int N, int32_t *__restrict__ counts, int *status) {
  using namespace ptx;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TcAssignSmem<D> &sm = *reinterpret_cast<TcAssignSmem<D> *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  int *cnt = reinterpret_cast<int *>(reinterpret_cast<unsigned char *>(&sm) + sizeof(TcAssignSmem<D>));
  const KmCtx k = km_ctx(J, blockIdx.y);
  const Task &tk = k.tk;
  const int chunk0 = blockIdx.x * kTcChunks;
  if (chunk0 * kChunk >= tk.n) return;  // uniform
  const int jb = (J.njobs > 1 && (int)blockIdx.y >= J.tasks0) ? 1 : 0;
  const CUtensorMap *map = jb ? &map1 : &map0;
  const int warp = threadIdx.x >> 5;
  volatile int *abort_flag = &sm.abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&sm.xbar, 1);
    mbar_init(&sm.mbar, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(&sm.tmem_base)),
                 "r"(256)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const int ntile = (tk.C + 255) / 256;
  int xph = 0, mph = 0;
  bool ok = true;
  for (int chunk = chunk0; chunk < chunk0 + kTcChunks && chunk * kChunk < tk.n; ++chunk) {
    const int r = chunk * kChunk + threadIdx.x;
    const bool valid = r < tk.n;
    if (threadIdx.x == 0) {
      mbar_expect_tx(&sm.xbar, (uint32_t)(D / 64) * kChunk * 128);
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_2d(sm.x[kb], map, kb * 64, (int)((int64_t)tk.p * N + tk.row0 + chunk * kChunk), &sm.xbar);
    }
    float best = CUDART_INF_F;
    int bi = 0;
    for (int t = 0; t < ntile; ++t) {
      const int c0 = t * 256;
      const int ct = min(256, J.CP - c0);  // padded: multiple of 16
      if (chunk == chunk0 || ntile > 1) {
        // stage the centroid split rows [c0, c0 + ct) (16-byte vectors, swizzled)
        const __nv_bfloat16 *gh = J.chi + ((int64_t)k.tg * J.CP + c0) * D;
        const __nv_bfloat16 *gl = J.clo + ((int64_t)k.tg * J.CP + c0) * D;
        for (int e = threadIdx.x; e < ct * (D / 8); e += blockDim.x) {
          const int c = e / (D / 8), v = e % (D / 8);
          const int kb = v >> 3, ch = v & 7;
          const int off = c * 128 + ((ch ^ (c & 7)) << 4);
          *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(sm.hi[kb]) + off) =
              *reinterpret_cast<const uint4 *>(gh + (int64_t)c * D + v * 8);
          *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(sm.lo[kb]) + off) =
              *reinterpret_cast<const uint4 *>(gl + (int64_t)c * D + v * 8);
        }
        for (int c = threadIdx.x; c < ct; c += blockDim.x) sm.cn[c] = J.cn[(int64_t)k.tg * J.CP + c0 + c];
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        if (t == 0) ok = ok && mbar_wait(&sm.xbar, xph & 1, abort_flag, status);
        if (ok) {
          tc_fence_after();
          const uint32_t id = idesc(kChunk, ct);
          for (int kk = 0; kk < D / 16; ++kk)
            tc_mma(tmem, sdesc(sm.x[kk >> 2] + (kk & 3) * 16), sdesc(sm.hi[kk >> 2] + (kk & 3) * 16),
                   id, kk > 0 ? 1u : 0u);
          for (int kk = 0; kk < D / 16; ++kk)
            tc_mma(tmem, sdesc(sm.x[kk >> 2] + (kk & 3) * 16), sdesc(sm.lo[kk >> 2] + (kk & 3) * 16),
                   id, 1u);
        }
        tc_commit(&sm.mbar);
      }
      __syncwarp();
      mbar_drain(&sm.mbar, mph & 1, status);
      ++mph;
      tc_fence_after();
      for (int cb = 0; cb < ct / 16; ++cb) {
        float x[16];
        tmem_ld16(tmem + lane_base + cb * 16, x);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float dd = fmaf(-2.f, x[e], sm.cn[cb * 16 + e]);
          if (dd < best) {
            best = dd;
            bi = c0 + cb * 16 + e;
          }
        }
      }
      tc_fence_before();
      __syncthreads();  // TMEM and the staged tiles are reused next
    }
    ++xph;
    if (*abort_flag) break;  // uniform: read after the barrier above
    const int L = valid ? bi : -1;
    if (valid) k.job->out.labels[tk.lab + r] = L;
    chunk_count(J, k, chunk, r, valid, L, cnt, counts);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256)
                 : "memory");
  }
}

// One CTA of 32 warps per task: a warp scans one cluster's chunk counts (lanes over
// chunks), then the block scans the cluster totals into offsets.
__global__ void __launch_bounds__(1024)
km_scan(KmJobs J, const int32_t *__restrict__ counts, int32_t *__restrict__ base) {
  __shared__ int tot[kMaxClusters];
  const KmCtx k = km_ctx(J, blockIdx.x);
  const Task &tk = k.tk;
  const int nch = (tk.n + kChunk - 1) / kChunk;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int c = w; c < kMaxClusters; c += 32) {
    if (c >= tk.C) {
      if (lane == 0) tot[c] = 0;
      continue;
    }
    const int64_t row = ((int64_t)k.tg * J.maxC + c) * J.nch;
    int run = 0;
    for (int ch0 = 0; ch0 < nch; ch0 += 32) {
      const int ch = ch0 + lane;
      const int v = ch < nch ? counts[row + ch] : 0;
      int inc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      if (ch < nch) base[row + ch] = run + inc - v;
      run += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) tot[c] = run;
  }
  __syncthreads();
  const int c = threadIdx.x;
  const int mine = tot[c];
  for (int o = 1; o < kMaxClusters; o <<= 1) {
    const int v = (c >= o) ? tot[c - o] : 0;
    __syncthreads();
    tot[c] += v;
    __syncthreads();
  }
  int32_t *offsets = k.job->out.offsets;
  if (c < tk.C) offsets[tk.off + c] = tot[c] - mine;
  if (c == 0) offsets[tk.off + tk.C] = tk.n;
}

__global__ void __launch_bounds__(kChunk)
km_scatter(KmJobs J, const int32_t *__restrict__ base, int *status) {
  const KmCtx k = km_ctx(J, blockIdx.y);
  const Task &tk = k.tk;
  const int chunk = blockIdx.x;
  const int r = chunk * kChunk + threadIdx.x;
  if (r >= tk.n) return;
  const int L = k.job->out.labels[tk.lab + r];
  const int pos = k.job->out.offsets[tk.off + L] +
                  base[((int64_t)k.tg * J.maxC + L) * J.nch + chunk] + k.job->lrank[tk.lab + r];
  if (pos < 0 || pos >= tk.n) {
    report(status, MUSE_ERR_DEVICE);
    return;
  }
  k.job->out.perm[tk.lab + pos] = tk.row0 + r;  // sequence row index
}

// One warp per (cluster, task), 8 clusters per CTA.  Lane t owns one 16-byte vector
// of the row and one member slot; slots take members b+slot, b+slot+SLOTS, ... in
// order and are then summed in slot order (shuffles): the result depends only on
// the data.
template <typename T, int D>
__global__ void __launch_bounds__(256)
km_centroid(KmJobs J, int N) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int VPR = D / VEC;      // lanes per row (8, 16 or 32)
  constexpr int SLOTS = 32 / VPR;   // member slots per warp
  const KmCtx k = km_ctx(J, blockIdx.y);
  const Task &tk = k.tk;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (c >= tk.C) return;
  const int32_t *offsets = k.job->out.offsets;
  const int b = offsets[tk.off + c], e = offsets[tk.off + c + 1];
  if (e <= b) return;  // empty: keep the previous centroid
  const int v = lane % VPR, slot = lane / VPR;
  const T *xp = static_cast<const T *>(k.job->X) + (int64_t)tk.p * N * D;
  const int32_t *perm = k.job->out.perm + tk.lab;
  float acc[VEC];
#pragma unroll
  for (int u = 0; u < VEC; ++u) acc[u] = 0.f;
  // this slot's members b+slot, b+slot+SLOTS, ... in order, eight loads in flight
  for (int m0 = b + slot; m0 < e; m0 += 8 * SLOTS) {
    int rows[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) rows[t] = (m0 + t * SLOTS < e) ? perm[m0 + t * SLOTS] : -1;
    uint4 raw[8];
#pragma unroll
    for (int t = 0; t < 8; ++t)
      raw[t] = rows[t] >= 0 ? *reinterpret_cast<const uint4 *>(xp + (int64_t)rows[t] * D + v * VEC)
                            : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (rows[t] < 0) break;
      const T *el = reinterpret_cast<const T *>(&raw[t]);
#pragma unroll
      for (int u = 0; u < VEC; ++u) acc[u] += ld_elem(el + u);
    }
  }
  // fixed-order reduction over the slots (lane bits above the vector index)
#pragma unroll
  for (int o = VPR; o < 32; o <<= 1)
#pragma unroll
    for (int u = 0; u < VEC; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
  const float inv = 1.f / (float)(e - b);
  float sq = 0.f;
  if (slot == 0) {
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
      const float val = acc[u] * inv;
      const int d = v * VEC + u;
      k.job->out.centroids[(tk.cen + c) * D + d] = val;
      if (J.chi) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(val);
        J.chi[((int64_t)k.tg * J.CP + c) * D + d] = hi;
        J.clo[((int64_t)k.tg * J.CP + c) * D + d] = __float2bfloat16_rn(val - __bfloat162float(hi));
      }
      sq = fmaf(val, val, sq);
    }
  }
  if (J.chi) {
    sq = warp_sum(sq);  // lanes of slot > 0 contribute 0
    if (lane == 0) J.cn[(int64_t)k.tg * J.CP + c] = sq;
  }
}

static int nch_of(const SegTable &t) { return (t.max_rows + kChunk - 1) / kChunk; }

static int cp_of(int maxC) { return (maxC + 15) & ~15; }

size_t kmeans_pair_ws_bytes(const SegTable *tq, const SegTable *tk, int P, int D) {
  const int64_t tasks = (int64_t)P * tq->nseg + (tk ? (int64_t)P * tk->nseg : 0);
  const int nch = std::max(nch_of(*tq), tk ? nch_of(*tk) : 0);
  const int maxC = std::max(tq->max_C, tk ? tk->max_C : 0);
  const size_t cnt = (size_t)(tasks * nch * maxC) * sizeof(int32_t);
  const size_t lr = (size_t)P * (tq->row_stride + (tk ? tk->row_stride : 0)) * sizeof(int32_t);
  const size_t split = (size_t)tasks * cp_of(maxC) * D * sizeof(__nv_bfloat16);
  const size_t norms = (size_t)tasks * cp_of(maxC) * sizeof(float);
  return align_up(cnt) * 2 + align_up(lr) + 2 * align_up(split) + align_up(norms);
}

size_t kmeans_ws_bytes(const SegTable &t, int P, int D) {
  return kmeans_pair_ws_bytes(&t, nullptr, P, D);
}

template <typename T, int D>
static cudaError_t run_kmeans_t(KmJobs &J, int N, int P, int iters, char *ws, int *status,
                                cudaStream_t st) {
  const int tasks = J.tasks0 + (J.njobs > 1 ? P * J.job[1].tab.nseg : 0);
  const int nch = J.nch;
  const size_t cnt_bytes = align_up((size_t)tasks * nch * J.maxC * sizeof(int32_t));
  int32_t *counts = reinterpret_cast<int32_t *>(ws);
  int32_t *base = reinterpret_cast<int32_t *>(ws + cnt_bytes);
  int32_t *lr = reinterpret_cast<int32_t *>(ws + 2 * cnt_bytes);
  const size_t lr_bytes =
      align_up((size_t)P * (J.job[0].tab.row_stride + (J.njobs > 1 ? J.job[1].tab.row_stride : 0)) *
               sizeof(int32_t));
  J.job[0].lrank = lr;
  if (J.njobs > 1) J.job[1].lrank = lr + (size_t)P * J.job[0].tab.row_stride;
  J.CP = cp_of(J.maxC);
  constexpr bool kTc = sizeof(T) == 2;  // bfloat16 inputs: tensor-core assign
  if (kTc) {
    const size_t split = align_up((size_t)tasks * J.CP * D * sizeof(__nv_bfloat16));
    char *sp = ws + 2 * cnt_bytes + lr_bytes;
    J.chi = reinterpret_cast<__nv_bfloat16 *>(sp);
    J.clo = reinterpret_cast<__nv_bfloat16 *>(sp + split);
    J.cn = reinterpret_cast<float *>(sp + 2 * split);
  } else {
    J.chi = J.clo = nullptr;
    J.cn = nullptr;
  }
  cudaError_t err;
  const size_t smem = (size_t)kCTile * (D + 1) * sizeof(float) + kWarps * (size_t)J.maxC * sizeof(int);
  const size_t smem_tc = sizeof(TcAssignSmem<D>) + 1024 + kWarps * (size_t)J.maxC * sizeof(int);
  CUtensorMap m0, m1;
  if (kTc) {
    err = cudaFuncSetAttribute(km_assign_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem_tc);
    if (err != cudaSuccess) return err;
    if (!ptx::make_map(&m0, J.job[0].X, D, (uint64_t)P * N, D, kChunk) ||
        !ptx::make_map(&m1, J.job[J.njobs > 1 ? 1 : 0].X, D, (uint64_t)P * N, D, kChunk))
      return cudaErrorInvalidValue;
  } else {
    err = cudaFuncSetAttribute(km_assign<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    if (err != cudaSuccess) return err;
  }
  km_init<T, D><<<dim3((J.CP + 7) / 8, tasks), 256, 0, st>>>(J, N);
  count_launches(1 + 4 * iters);
  for (int it = 0; it < iters; ++it) {
    if (kTc)
      km_assign_tc<D><<<dim3((nch + kTcChunks - 1) / kTcChunks, tasks), kChunk, smem_tc, st>>>(
          m0, m1, J, N, counts, status);
    else
      km_assign<T, D><<<dim3(nch, tasks), kChunk, smem, st>>>(J, N, counts);
    km_scan<<<tasks, 1024, 0, st>>>(J, counts, base);
    km_scatter<<<dim3(nch, tasks), kChunk, 0, st>>>(J, base, status);
    km_centroid<T, D><<<dim3((J.maxC + 7) / 8, tasks), 256, 0, st>>>(J, N);
  }
  return cudaGetLastError();
}

static cudaError_t dispatch(KmJobs &J, int dtype, int D, int N, int P, int iters, char *ws,
                            int *status, cudaStream_t st) {
  if (dtype == MUSE_F32)
    return D == 64 ? run_kmeans_t<float, 64>(J, N, P, iters, ws, status, st)
                   : run_kmeans_t<float, 128>(J, N, P, iters, ws, status, st);
  return D == 64 ? run_kmeans_t<__nv_bfloat16, 64>(J, N, P, iters, ws, status, st)
                 : run_kmeans_t<__nv_bfloat16, 128>(J, N, P, iters, ws, status, st);
}

cudaError_t run_kmeans(const void *X, int dtype, int D, int N, const SegTable &tab, int P,
                       int iters, const KmeansOut &o, char *ws, int *status, cudaStream_t st) {
  if (kmeans_fused_supported(dtype, D, tab)) {
    const SegTable *t[1] = {&tab};
    return run_kmeans_fused(1, &X, t, &o, N, P, iters, status, st);
  }
  KmJobs J;
  J.njobs = 1;
  J.tasks0 = P * tab.nseg;
  J.nch = nch_of(tab);
  J.maxC = tab.max_C;
  J.job[0].X = X;
  J.job[0].tab = tab;
  J.job[0].out = o;
  J.job[1] = J.job[0];
  return dispatch(J, dtype, D, N, P, iters, ws, status, st);
}

cudaError_t run_kmeans_pair(const void *Xq, const SegTable &tq, const KmeansOut &oq,
                            const void *Xk, const SegTable &tk, const KmeansOut &ok, int dtype,
                            int D, int N, int P, int iters, char *ws, int *status,
                            cudaStream_t st) {
  if (kmeans_fused_supported(dtype, D, tq) && kmeans_fused_supported(dtype, D, tk)) {
    const void *X[2] = {Xq, Xk};
    const SegTable *t[2] = {&tq, &tk};
    const KmeansOut o[2] = {oq, ok};
    return run_kmeans_fused(2, X, t, o, N, P, iters, status, st);
  }
  KmJobs J;
  J.njobs = 2;
  J.tasks0 = P * tq.nseg;
  J.nch = std::max(nch_of(tq), nch_of(tk));
  J.maxC = std::max(tq.max_C, tk.max_C);
  J.job[0].X = Xq;
  J.job[0].tab = tq;
  J.job[0].out = oq;
  J.job[1].X = Xk;
  J.job[1].tab = tk;
  J.job[1].out = ok;
  return dispatch(J, dtype, D, N, P, iters, ws, status, st);
}

}  // namespace muse
