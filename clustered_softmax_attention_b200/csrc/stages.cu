// Stage kernels (CUDA cores) of the MuSe forward pass, batched over
// (problem, instance): sorted copies, tilt logits / log-normalisers / weights,
// tilted moments, the refinement coefficients, and the refinement itself.
//
// Stage 1 (tilted monopole summaries and dipole): pith.science review of arXiv
// 2509.10406, "What carries the argument" and "Assumptions & free parameters"
// (M_j(q) = E exp(q.k)); referee minor comment on Algorithm 3 (tilted Cov_ij(v,k)).
// Stage 2 (refinement that drops only qt.kt): same page, "What carries the
// argument"; gist.science "Technische Samenvatting", "Kernmechanismen" 1-2.
//
// The refinement uses the identity
//   mu_v,ij + s C_ij qt = sum_{k in S_j} w_ik (1 - s qt.mu_k,ij + s qt.k) v_k
// (the weights w_ik sum to one and sum_k w_ik (k - mu_k,ij) = 0), so with
//   c0_nj = p_nj (1 - s u_nj),  c1_nj = s p_nj,  u_nj = qt_n.mu_k,ij,
//   O_n = sum_k w_{i(n),k} (c0_{n,j(k)} + c1_{n,j(k)} qt_n.k) v_k :
// two contractions over the cluster-sorted keys with an element-wise step between
// them, and C_ij is never formed.
#include <type_traits>
#include "internal.h"

namespace muse {

__device__ __forceinline__ Task q_task(const MuseTables &mt, int p, int s) {
  return make_task(mt.q, p * mt.q.nseg + s);
}
__device__ __forceinline__ Task k_task(const MuseTables &mt, int p, int s) {
  return make_task(mt.k, p * mt.k.nseg + s);
}

// ---------------------------------------------------------------------------
// Sorted copies: position m of a task's perm holds row perm[m] (minus its
// cluster's centroid when `centroids` is given: the query residuals).
// One CTA per 64 sorted positions of a task (compact grid); a position's cluster is
// the last one whose offset is <= it (a binary search over the task's offsets).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
sort_side(const T *__restrict__ X, int N, int W, SegTable tab, const int32_t *__restrict__ perm,
          const int32_t *__restrict__ offsets, const float *__restrict__ centroids,
          T *__restrict__ rows, int32_t *__restrict__ cluster, const __grid_constant__ BlockMap bm) {
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte vector
  int bfirst;
  const int sg = map_block(bm, tab.nseg, blockIdx.x, bfirst);
  const Task tk = make_task(tab, blockIdx.y * tab.nseg + sg);
  const int m0 = ((int)blockIdx.x - bfirst) * 64, m1 = min(m0 + 64, tk.n);
  if (m0 >= tk.n) return;
  const int32_t *off = offsets + tk.off;
  const int vpr = W / VEC, slots = 256 / vpr;
  const int v = threadIdx.x % vpr, slot = threadIdx.x / vpr;
  for (int m = m0 + slot; m < m1; m += slots) {
    int lo = 0, hi = tk.C - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(off + mid) <= m) lo = mid;
      else hi = mid - 1;
    }
    const int c = lo;
    float cv[VEC];
#pragma unroll
    for (int u = 0; u < VEC; ++u) cv[u] = centroids ? centroids[(tk.cen + c) * W + v * VEC + u] : 0.f;
    const int row = perm[tk.lab + m];
    uint4 raw = *reinterpret_cast<const uint4 *>(X + ((int64_t)tk.p * N + row) * W + v * VEC);
    if (centroids) {
      T *el = reinterpret_cast<T *>(&raw);
#pragma unroll
      for (int u = 0; u < VEC; ++u) st_elem(el + u, ld_elem(el + u) - cv[u]);
    }
    *reinterpret_cast<uint4 *>(rows + (tk.lab + m) * W + v * VEC) = raw;
    if (v == 0) cluster[tk.lab + m] = c;
  }
}

// ---------------------------------------------------------------------------
// Transposed sorted copy: vt[p][c][lab0 + m] = X[p][perm[m]][c] (keys innermost,
// row length vt_ld(row_stride)), so that the values are a K-major operand of the
// P.V contraction.  64 sorted positions per CTA, staged through shared memory.
// ---------------------------------------------------------------------------
template <typename T, int W>
__global__ void __launch_bounds__(256)
sort_side_t(const T *__restrict__ X, int N, SegTable tab, const int32_t *__restrict__ perm,
            T *__restrict__ vt, BlockMap bm) {
  int bfirst;
  const int sg = map_block(bm, tab.nseg, blockIdx.x, bfirst);
  const Task tk = make_task(tab, blockIdx.y * tab.nseg + sg);
  const int m0 = ((int)blockIdx.x - bfirst) * 64;
  if (m0 >= tk.n) return;
  __shared__ T buf[64][W + 2];
  const int mt = min(64, tk.n - m0);
  constexpr int VEC = 16 / sizeof(T), VPR = W / VEC;  // 16-byte vectors per row
  for (int e = threadIdx.x; e < mt * VPR; e += blockDim.x) {
    const int mm = e / VPR, cv = e % VPR;
    const int row = perm[tk.lab + m0 + mm];
    const uint4 raw = *reinterpret_cast<const uint4 *>(X + ((int64_t)tk.p * N + row) * W + cv * VEC);
    const T *el = reinterpret_cast<const T *>(&raw);
#pragma unroll
    for (int u = 0; u < VEC; ++u) buf[mm][cv * VEC + u] = el[u];
  }
  __syncthreads();
  const int ld = vt_ld(tab.row_stride);
  const int64_t col0 = (int64_t)(tk.lab - (int64_t)tk.p * tab.row_stride) + m0;
  for (int e = threadIdx.x; e < mt * W; e += blockDim.x) {
    const int c = e / mt, mm = e % mt;
    vt[((int64_t)tk.p * W + c) * ld + col0 + mm] = buf[mm][c];
  }
  // The 16 columns after the segment are read (and multiplied by zero weights) by a
  // key tile that overhangs the segment's end: make them zeros, not stale memory.
  if (m0 + 64 >= tk.n) {
    const int64_t end = (int64_t)(tk.lab - (int64_t)tk.p * tab.row_stride) + tk.n;
    for (int e = threadIdx.x; e < 16 * W; e += blockDim.x) {
      const int c = e >> 4;
      const int64_t col = end + (e & 15);
      if (col < ld) vt[((int64_t)tk.p * W + c) * ld + col] = T(0.f);
    }
  }
}

// ---------------------------------------------------------------------------
// Tilt logits W[i][pos] = s qbar_i . k_pos over the sorted keys (64 x 64 tiles).
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256)
tilt_logits(MuseTables mt, float scale, const float *__restrict__ qcen, const T *__restrict__ ks,
            float *__restrict__ W, BlockMap bm) {
  // blockIdx.x: a 64-key block of one instance (compact grid), blockIdx.z: the problem
  int bfirst;
  const int p = blockIdx.z, s = map_block(bm, mt.in.ninst, blockIdx.x, bfirst);
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int Cq = q.C, nk = k.n;
  const int i0 = blockIdx.y * 64, k0 = ((int)blockIdx.x - bfirst) * 64;
  if (i0 >= Cq || k0 >= nk) return;
  __shared__ float As[32][65];
  __shared__ float Bs[32][65];
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float *qc = qcen + (q.cen + i0) * D;
  const T *kr = ks + (k.lab + k0) * D;
  for (int d0 = 0; d0 < D; d0 += 32) {
    for (int e = threadIdx.x; e < 64 * 32; e += 256) {
      const int r = e >> 5, dd = e & 31;
      As[dd][r] = (i0 + r < Cq) ? qc[(int64_t)r * D + d0 + dd] : 0.f;
      Bs[dd][r] = (k0 + r < nk) ? ld_elem(kr + (int64_t)r * D + d0 + dd) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int dd = 0; dd < 32; ++dd) {
      float av[4], bv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) av[a] = As[dd][ty * 4 + a];
#pragma unroll
      for (int b = 0; b < 4; ++b) bv[b] = Bs[dd][tx * 4 + b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }
    __syncthreads();
  }
  float *wo = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty * 4 + a;
    if (i >= Cq) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int kk = k0 + tx * 4 + b;
      if (kk < nk) wo[(int64_t)i * w_ld(nk) + kk] = scale * acc[a][b];
    }
  }
}

// ---------------------------------------------------------------------------
// logZ_ij = logsumexp of W[i][S_j] (one warp per (i, j)), then W <- exp(W - logZ).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
tilt_lse(MuseTables mt, const int32_t *__restrict__ k_offsets, float *__restrict__ W,
         float *__restrict__ logZ) {
  const int p = blockIdx.y / mt.in.ninst, s = blockIdx.y % mt.in.ninst;
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int Cq = q.C, Ck = k.C, nk = k.n;
  const int wid = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (wid >= Cq * Ck) return;
  const int i = wid / Ck, j = wid % Ck;
  const int b = k_offsets[k.off + j], e = k_offsets[k.off + j + 1];
  float *w = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s] + (int64_t)i * w_ld(nk);
  float m = -CUDART_INF_F;
  for (int pos = b + lane; pos < e; pos += 32) m = fmaxf(m, w[pos]);
  m = warp_max(m);
  float l = 0.f;
  for (int pos = b + lane; pos < e; pos += 32) l += expf(w[pos] - m);
  l = warp_sum(l);
  const float lz = (e > b) ? m + logf(l) : -CUDART_INF_F;
  for (int pos = b + lane; pos < e; pos += 32) w[pos] = expf(w[pos] - lz);
  if (lane == 0) logZ[(int64_t)p * mt.in.z_stride + mt.in.z0[s] + (int64_t)i * Ck + j] = lz;
}

// ---------------------------------------------------------------------------
// The same for short key clusters (a few keys each): one warp per row i, one lane
// per key cluster j, each lane scanning its cluster's keys in order.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
tilt_lse_short(MuseTables mt, const int32_t *__restrict__ k_offsets, float *__restrict__ W,
               float *__restrict__ logZ) {
  const int p = blockIdx.y / mt.in.ninst, s = blockIdx.y % mt.in.ninst;
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (i >= q.C) return;
  const int Ck = k.C;
  float *w = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s] + (int64_t)i * w_ld(k.n);
  float *lzr = logZ + (int64_t)p * mt.in.z_stride + mt.in.z0[s] + (int64_t)i * Ck;
  for (int j = lane; j < Ck; j += 32) {
    const int b = k_offsets[k.off + j], e = k_offsets[k.off + j + 1];
    float m = -CUDART_INF_F;
    for (int pos = b; pos < e; ++pos) m = fmaxf(m, w[pos]);
    float l = 0.f;
    for (int pos = b; pos < e; ++pos) l += expf(w[pos] - m);
    const float lz = (e > b) ? m + logf(l) : -CUDART_INF_F;
    for (int pos = b; pos < e; ++pos) w[pos] = expf(w[pos] - lz);
    lzr[j] = lz;
  }
}

// ---------------------------------------------------------------------------
// W <- exp(W - logZ[i][j(pos)]) for externally supplied log-normalisers.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
tilt_weights(MuseTables mt, const int32_t *__restrict__ k_cluster, const float *__restrict__ logZ,
             float *__restrict__ W) {
  const int p = blockIdx.z / mt.in.ninst, s = blockIdx.z % mt.in.ninst;
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int i = blockIdx.y;
  if (i >= q.C) return;
  const int pos = blockIdx.x * 256 + threadIdx.x;
  if (pos >= k.n) return;
  const int j = k_cluster[k.lab + pos];
  const float lz = logZ[(int64_t)p * mt.in.z_stride + mt.in.z0[s] + (int64_t)i * k.C + j];
  float *w = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s] + (int64_t)i * w_ld(k.n) + pos;
  *w = expf(*w - lz);
}

// ---------------------------------------------------------------------------
// Tilted means mu[i][j][:] = sum_{pos in S_j} w_i,pos x_pos (x = keys or values).
// CTA per (j, group of 32 query centroids); a warp handles 4 centroids, lanes
// cover the coordinates.
// ---------------------------------------------------------------------------
template <typename T, int WD>
__global__ void __launch_bounds__(256)
tilt_moments(MuseTables mt, const int32_t *__restrict__ k_offsets, const float *__restrict__ W,
             const T *__restrict__ xs, float *__restrict__ mu) {
  constexpr int PW = WD / 16;  // coordinates per thread (interleaved by 16)
  __shared__ float Ws[64][33];
  __shared__ float Xs[32][WD + 4];
  const int p = blockIdx.z / mt.in.ninst, s = blockIdx.z % mt.in.ninst;
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int Cq = q.C, Ck = k.C, nk = k.n;
  const int j = blockIdx.x, i0 = blockIdx.y * 64;
  if (j >= Ck || i0 >= Cq) return;
  const int b = k_offsets[k.off + j], e = k_offsets[k.off + j + 1];
  const int ti = threadIdx.x >> 4, td = threadIdx.x & 15;
  float acc[4][PW];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int u = 0; u < PW; ++u) acc[a][u] = 0.f;
  const float *wb = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s];
  const int wl = w_ld(nk);
  for (int pc = b; pc < e; pc += 32) {
    const int pt = min(32, e - pc);
    __syncthreads();
    for (int x = threadIdx.x; x < 64 * 32; x += 256) {
      const int ii = x >> 5, pp = x & 31;
      Ws[ii][pp] = (i0 + ii < Cq && pp < pt) ? wb[(int64_t)(i0 + ii) * wl + pc + pp] : 0.f;
    }
    for (int x = threadIdx.x; x < 32 * WD; x += 256) {
      const int pp = x / WD, d = x % WD;
      Xs[pp][d] = pp < pt ? ld_elem(xs + (k.lab + pc + pp) * WD + d) : 0.f;
    }
    __syncthreads();
    for (int pp = 0; pp < pt; ++pp) {
      float xv[PW];
#pragma unroll
      for (int u = 0; u < PW; ++u) xv[u] = Xs[pp][td + 16 * u];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float w = Ws[ti * 4 + a][pp];
#pragma unroll
        for (int u = 0; u < PW; ++u) acc[a][u] = fmaf(w, xv[u], acc[a][u]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ti * 4 + a;
    if (i >= Cq) continue;
    float *o = mu + ((int64_t)p * mt.in.z_stride + mt.in.z0[s] + (int64_t)i * Ck + j) * WD;
#pragma unroll
    for (int u = 0; u < PW; ++u) o[td + 16 * u] = acc[a][u];
  }
}

// ---------------------------------------------------------------------------
// logits, log-normalisers, tilt weights and tilted key means in one kernel.  CTA per
// (G consecutive key clusters, 64 query centroids, instance), G chosen per instance so
// that a CTA covers about one chunk of keys (G = 1 for large clusters, up to 16 for
// clusters of a few keys); the centroids are staged once for all G clusters.  A cluster
// of at most KC keys takes one step: its logits stay in registers, give logZ by a
// 16-lane reduction and then the weights and the tilted key mean.  A larger cluster takes
// a first pass over chunks of KC keys (running maximum and sum) and a second pass that
// recomputes the logits.  The next step's keys are loaded into registers while the
// current step computes.  Thread (ti, td): centroids 4 ti .. 4 ti + 3, keys td + 16 c of
// a chunk, coordinates 4 td + 64 h of the means (the 16 threads of a centroid are
// consecutive lanes).
// ---------------------------------------------------------------------------
template <typename T, int D> struct TiltCfg {
  static constexpr int KC = 16384 / (D * (int)sizeof(T));  // keys per chunk (16 KB)
  static constexpr int UR = D * (int)sizeof(T) / 16;       // 16-byte units per key row
  static constexpr int EPU = 16 / (int)sizeof(T);          // elements per unit
  static constexpr int QS = D + 4, WS = 68;                // shared-memory row strides
  static constexpr int GMAX = 16;
  // centroids, keys (fp32), weights, and the raw key chunk the next step copies into
  static constexpr size_t smem = ((size_t)64 * QS + (size_t)KC * QS + (size_t)KC * WS) * 4 + 16384;
};

// 16-byte asynchronous global -> shared copy (src_bytes = 0 writes zeros), its commit
// and the wait for all of this thread's copies.
__device__ __forceinline__ void tilt_cp16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void tilt_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void tilt_cp_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// clusters per CTA for an instance of n keys in C clusters
__host__ __device__ __forceinline__ int tilt_group(int n, int C, int kc) {
  if (C <= 0 || n <= 0) return TiltCfg<float, 64>::GMAX;
  const int64_t g = (int64_t)kc * C / n;
  return (int)(g < 1 ? 1 : g > TiltCfg<float, 64>::GMAX ? TiltCfg<float, 64>::GMAX : g);
}

__device__ __forceinline__ void tilt_unpack(const uint4 u, float *o) {  // 8 bf16
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const float2 f = __bfloat1622float2(h[x]);
    o[2 * x] = f.x;
    o[2 * x + 1] = f.y;
  }
}

struct TiltStep {
  // clusters j .. je-1, keys [b, e), chunk start pc; pass 0: one cluster in one chunk;
  // 1, 2: first, second pass over a larger cluster; 3: a window of several whole
  // clusters that fit in one chunk together
  int j, je, b, e, pc, pass;
};

// PRE: the logits s qbar_i . k are already in W (logits_tc.cu, tensor cores); the kernel
// reads them instead of computing them, and overwrites them with the weights.
template <typename T, int D, bool PRE>
__global__ void __launch_bounds__(256, 2)
tilt_fused(MuseTables mt, float scale, const float *__restrict__ qcen, const T *__restrict__ ks,
           const int32_t *__restrict__ k_offsets, float *__restrict__ W, float *__restrict__ logZ,
           float *__restrict__ mu, const __grid_constant__ BlockMap bm) {
  // blockIdx.x: a group of G key clusters of one instance (compact grid), blockIdx.z: the problem
  using Cf = TiltCfg<T, D>;
  constexpr int KC = Cf::KC, QS = Cf::QS, WS = Cf::WS, PQ = D / 64;
  extern __shared__ float4 tilt_smem[];
  float *Qs = reinterpret_cast<float *>(tilt_smem);  // [64][QS] the group's centroids
  float *Ks = Qs + 64 * QS;                           // [KC][QS] a chunk of keys
  float *Ws = Ks + KC * QS;                           // [KC][WS] the chunk's weights
  uint4 *Kr = reinterpret_cast<uint4 *>(Ws + KC * WS); // [1024] raw 16-byte units of a chunk
  __shared__ int offs[Cf::GMAX + 1];
  __shared__ float LZs[Cf::GMAX * 64];  // window steps: logZ per (cluster, centroid)
  __shared__ unsigned char segk[KC];    // window steps: cluster of each key of the chunk
  int bfirst;
  const int p = blockIdx.z, s = map_block(bm, mt.in.ninst, blockIdx.x, bfirst);
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int Cq = q.C, Ck = k.C, nk = k.n;
  const int G = tilt_group(nk, Ck, KC);
  const int j0 = ((int)blockIdx.x - bfirst) * G, j1 = min(Ck, j0 + G), i0 = blockIdx.y * 64;
  if (j0 >= Ck || i0 >= Cq) return;  // uniform
  const int tid = threadIdx.x, ti = tid >> 4, td = tid & 15;
  if (tid <= j1 - j0) offs[tid] = k_offsets[k.off + j0 + tid];
  if (!PRE) {
    constexpr int QU = D / 4, NR = 64 * QU / 256;
    float4 v[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int u = tid + 256 * r, ii = u / QU;
      v[r] = i0 + ii < Cq ? __ldg(reinterpret_cast<const float4 *>(qcen + (q.cen + i0 + ii) * D) + u % QU)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int u = tid + 256 * r;
      *reinterpret_cast<float4 *>(Qs + (u / QU) * QS + 4 * (u % QU)) = v[r];
    }
  }
  __syncthreads();
  float *wb = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s];
  const int wl = w_ld(nk);
  const int64_t zrow = (int64_t)p * mt.in.z_stride + mt.in.z0[s];
  // outputs of cluster j: logZ and the tilted mean of each of the thread's centroids
  auto put = [&](int j, const float (&lz)[4], const float (&acc)[4][PQ][4]) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = i0 + ti * 4 + a;
      if (i >= Cq) continue;
      const int64_t z = zrow + (int64_t)i * Ck + j;
      if (td == 0) logZ[z] = lz[a];
#pragma unroll
      for (int h = 0; h < PQ; ++h)
        *reinterpret_cast<float4 *>(mu + z * D + 64 * h + 4 * td) =
            make_float4(acc[a][h][0], acc[a][h][1], acc[a][h][2], acc[a][h][3]);
    }
  };
  float lz[4], m[4], l[4], acc[4][PQ][4];
  auto clear_acc = [&]() {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int h = 0; h < PQ; ++h)
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[a][h][x] = 0.f;
  };
  // first non-empty cluster from j on (empty clusters get logZ = -inf and a zero mean)
  auto open = [&](int j) {
    while (j < j1 && offs[j - j0 + 1] == offs[j - j0]) {
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int i = i0 + ti * 4 + a;
        if (i >= Cq) continue;
        const int64_t z = zrow + (int64_t)i * Ck + j;
        if (td == 0) logZ[z] = -CUDART_INF_F;
#pragma unroll
        for (int h = 0; h < PQ; ++h)
          *reinterpret_cast<float4 *>(mu + z * D + 64 * h + 4 * td) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      ++j;
    }
    TiltStep t;
    t.j = j;
    t.je = j + 1;
    t.b = j < j1 ? offs[j - j0] : 0;
    t.e = j < j1 ? offs[j - j0 + 1] : 0;
    t.pc = t.b;
    t.pass = t.e - t.b > KC ? 1 : 0;
    if (j < j1 && t.pass == 0) {  // the following clusters that fit in the same chunk
      int je = j + 1;
      while (je < j1 && offs[je + 1 - j0] - t.b <= KC) ++je;
      if (je - j >= 2) {
        t.je = je;
        t.e = offs[je - j0];
        t.pass = 3;
      }
    }
    return t;
  };
  auto advance = [&](TiltStep t) {
    if (t.pass == 3) return open(t.je);
    if (t.pc + KC < t.e) {
      t.pc += KC;
      return t;
    }
    if (t.pass == 1) {
      t.pass = 2;
      t.pc = t.b;
      return t;
    }
    return open(t.je);
  };
  // each thread copies, and later converts, the same four 16-byte units of a chunk
  auto fetch = [&](const TiltStep &t) {
    const int pt = min(KC, t.e - t.pc);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int u = tid + 256 * r, row = u / Cf::UR;
      const bool in = row < pt;
      tilt_cp16(Kr + u, in ? (const void *)(reinterpret_cast<const uint4 *>(ks + (k.lab + t.pc + row) * D) + u % Cf::UR)
                           : (const void *)ks, in ? 16u : 0u);
    }
    tilt_cp_commit();
  };
  TiltStep cur = open(j0);
  if (cur.j < j1) fetch(cur);
  while (cur.j < j1) {
    const int pt = min(KC, cur.e - cur.pc);
    __syncthreads();  // the previous step is done with Ks and Ws
    tilt_cp_wait();
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int u = tid + 256 * r;
      float *dst = Ks + (u / Cf::UR) * QS + (u % Cf::UR) * Cf::EPU;
      const uint4 raw = Kr[u];
      if constexpr (sizeof(T) == 2) {
        float f[8];
        tilt_unpack(raw, f);
        *reinterpret_cast<float4 *>(dst) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4 *>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
      } else {
        *reinterpret_cast<uint4 *>(dst) = raw;
      }
    }
    if (cur.pass == 3 && tid < pt) {  // cluster of each key of the window
      int cl = 0;
      while (offs[cur.j + cl + 1 - j0] - cur.b <= tid) ++cl;
      segk[tid] = (unsigned char)cl;
    }
    const TiltStep nxt = advance(cur);
    if (nxt.j < j1) fetch(nxt);
    __syncthreads();
    const bool first = cur.pc == cur.b, last = cur.pc + KC >= cur.e;
    auto body = [&](auto ncv) {
      constexpr int NC = decltype(ncv)::value;
      float L[4][NC];
      if constexpr (PRE) {
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const int i = i0 + ti * 4 + a;
#pragma unroll
          for (int c = 0; c < NC; ++c)
            L[a][c] = (i < Cq && td + 16 * c < pt) ? wb[(int64_t)i * wl + cur.pc + td + 16 * c] : -CUDART_INF_F;
        }
      } else {
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < NC; ++c) L[a][c] = 0.f;
#pragma unroll 2
      for (int d = 0; d < D; d += 4) {
        float4 qv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) qv[a] = *reinterpret_cast<const float4 *>(Qs + (ti * 4 + a) * QS + d);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const float4 kv = *reinterpret_cast<const float4 *>(Ks + (td + 16 * c) * QS + d);
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            L[a][c] = fmaf(qv[a].x, kv.x, L[a][c]);
            L[a][c] = fmaf(qv[a].y, kv.y, L[a][c]);
            L[a][c] = fmaf(qv[a].z, kv.z, L[a][c]);
            L[a][c] = fmaf(qv[a].w, kv.w, L[a][c]);
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < NC; ++c) L[a][c] = td + 16 * c < pt ? scale * L[a][c] : -CUDART_INF_F;
      }
      if (cur.pass == 3) {
        // a window of whole clusters: the logits go through shared memory, logZ per
        // (cluster, centroid) by a scan of the cluster's keys, then the weights and one
        // tilted mean per cluster from the same key tile
        const int ncl = cur.je - cur.j;
#pragma unroll
        for (int c = 0; c < NC; ++c)
          *reinterpret_cast<float4 *>(Ws + (td + 16 * c) * WS + 4 * ti) =
              make_float4(L[0][c], L[1][c], L[2][c], L[3][c]);
        __syncthreads();
        for (int x = tid; x < 64 * ncl; x += 256) {
          const int il = x & 63, cl = x >> 6;
          const int kb = offs[cur.j + cl - j0] - cur.b, ke = offs[cur.j + cl + 1 - j0] - cur.b;
          float mx = -CUDART_INF_F;
          for (int kk = kb; kk < ke; ++kk) mx = fmaxf(mx, Ws[kk * WS + il]);
          float sm = 0.f;
          for (int kk = kb; kk < ke; ++kk) sm += expf(Ws[kk * WS + il] - mx);
          LZs[cl * 64 + il] = ke > kb ? mx + logf(sm) : -CUDART_INF_F;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const int kk = td + 16 * c;
          const int cl = kk < pt ? segk[kk] : 0;
          float w[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            w[a] = kk < pt ? expf(L[a][c] - LZs[cl * 64 + ti * 4 + a]) : 0.f;
            if (kk < pt && i0 + ti * 4 + a < Cq) wb[(int64_t)(i0 + ti * 4 + a) * wl + cur.b + kk] = w[a];
          }
          *reinterpret_cast<float4 *>(Ws + kk * WS + 4 * ti) = make_float4(w[0], w[1], w[2], w[3]);
        }
        __syncthreads();
        for (int cl = 0; cl < ncl; ++cl) {
          const int kb = offs[cur.j + cl - j0] - cur.b, ke = offs[cur.j + cl + 1 - j0] - cur.b;
          clear_acc();
          for (int pp = kb; pp < ke; ++pp) {
            const float4 wv = *reinterpret_cast<const float4 *>(Ws + pp * WS + 4 * ti);
            const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int h = 0; h < PQ; ++h) {
              const float4 kv = *reinterpret_cast<const float4 *>(Ks + pp * QS + 64 * h + 4 * td);
#pragma unroll
              for (int a = 0; a < 4; ++a) {
                acc[a][h][0] = fmaf(wa[a], kv.x, acc[a][h][0]);
                acc[a][h][1] = fmaf(wa[a], kv.y, acc[a][h][1]);
                acc[a][h][2] = fmaf(wa[a], kv.z, acc[a][h][2]);
                acc[a][h][3] = fmaf(wa[a], kv.w, acc[a][h][3]);
              }
            }
          }
          float lzw[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) lzw[a] = LZs[cl * 64 + ti * 4 + a];
          put(cur.j + cl, lzw, acc);
        }
        return;
      }
      if (cur.pass != 2) {  // running maximum and sum of exp over the cluster's keys
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          if (first) {
            m[a] = -CUDART_INF_F;
            l[a] = 0.f;
          }
          float cm = L[a][0];
#pragma unroll
          for (int c = 1; c < NC; ++c) cm = fmaxf(cm, L[a][c]);
#pragma unroll
          for (int o = 1; o < 16; o <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
          const float mn = fmaxf(m[a], cm);
          float cs = 0.f;
#pragma unroll
          for (int c = 0; c < NC; ++c) cs += L[a][c] > -CUDART_INF_F ? expf(L[a][c] - mn) : 0.f;
#pragma unroll
          for (int o = 1; o < 16; o <<= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
          l[a] = (m[a] > -CUDART_INF_F ? l[a] * expf(m[a] - mn) : 0.f) + cs;
          m[a] = mn;
          if (last) lz[a] = m[a] + logf(l[a]);
        }
        if (cur.pass == 1) return;
      }
      if (first) clear_acc();
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int kk = td + 16 * c;
        float w[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          w[a] = kk < pt ? expf(L[a][c] - lz[a]) : 0.f;
          if (kk < pt && i0 + ti * 4 + a < Cq) wb[(int64_t)(i0 + ti * 4 + a) * wl + cur.pc + kk] = w[a];
        }
        *reinterpret_cast<float4 *>(Ws + kk * WS + 4 * ti) = make_float4(w[0], w[1], w[2], w[3]);
      }
      __syncthreads();
      for (int pp = 0; pp < pt; ++pp) {
        const float4 wv = *reinterpret_cast<const float4 *>(Ws + pp * WS + 4 * ti);
        const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int h = 0; h < PQ; ++h) {
          const float4 kv = *reinterpret_cast<const float4 *>(Ks + pp * QS + 64 * h + 4 * td);
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            acc[a][h][0] = fmaf(wa[a], kv.x, acc[a][h][0]);
            acc[a][h][1] = fmaf(wa[a], kv.y, acc[a][h][1]);
            acc[a][h][2] = fmaf(wa[a], kv.z, acc[a][h][2]);
            acc[a][h][3] = fmaf(wa[a], kv.w, acc[a][h][3]);
          }
        }
      }
      if (last) put(cur.j, lz, acc);
    };
    const int nc = (pt + 15) >> 4;
    if (nc <= 1) body(std::integral_constant<int, 1>{});
    else if (nc <= 2) body(std::integral_constant<int, 2>{});
    else if (nc <= 4 || KC < 128) body(std::integral_constant<int, (KC / 16 < 4 ? KC / 16 : 4)>{});
    else body(std::integral_constant<int, KC / 16>{});
    cur = nxt;
  }
}

// ---------------------------------------------------------------------------
// Tilted dipole C_ij = sum_k w (v - mu_v)(k - mu_k)^T, centred (inspection only:
// the forward pass never materialises it).  CTA per (j, i, task).
// ---------------------------------------------------------------------------
template <typename T, int D, int DV>
__global__ void __launch_bounds__(256)
tilt_cov(MuseTables mt, const int32_t *__restrict__ k_offsets, const float *__restrict__ W,
         const T *__restrict__ ks, const T *__restrict__ vs, const float *__restrict__ mu_k,
         const float *__restrict__ mu_v, float *__restrict__ cov) {
  const int p = blockIdx.z / mt.in.ninst, s = blockIdx.z % mt.in.ninst;
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int Cq = q.C, Ck = k.C, nk = k.n;
  const int j = blockIdx.x, i = blockIdx.y;
  if (j >= Ck || i >= Cq) return;
  const int b = k_offsets[k.off + j], e = k_offsets[k.off + j + 1];
  const int64_t z = (int64_t)p * mt.in.z_stride + mt.in.z0[s] + (int64_t)i * Ck + j;
  const float *mk = mu_k + z * D;
  const float *mv = mu_v + z * DV;
  const float *w = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s] + (int64_t)i * w_ld(nk);
  float *out = cov + z * DV * D;
  for (int e2 = threadIdx.x; e2 < DV * D; e2 += blockDim.x) {
    const int dv = e2 / D, d = e2 % D;
    float acc = 0.f;
    for (int pos = b; pos < e; ++pos)
      acc = fmaf(w[pos] * (ld_elem(vs + (k.lab + pos) * DV + dv) - mv[dv]),
                 ld_elem(ks + (k.lab + pos) * D + d) - mk[d], acc);
    out[e2] = acc;
  }
}

// ---------------------------------------------------------------------------
// Refinement coefficients for every sorted query position n of cluster i:
//   a_j = logZ_ij + s u_j, u_j = qt.mu_k,ij;  p = softmax_j(a);
//   c0[j][n] = p_j (1 - sd u_j), c1[j][n] = sd p_j,  lse[n] = logsumexp_j a_j,
// with sd = s (monopole and dipole) or sd = 0 (monopole only: c0 = p, c1 = 0).
// CTA per (query cluster, task), one thread per query.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128)
refine_coeffs(MuseTables mt, float scale, const T *__restrict__ qt_rows,
              const int32_t *__restrict__ q_cluster, const float *__restrict__ logZ,
              const float *__restrict__ mu_k, float *__restrict__ c0, float *__restrict__ c1,
              float *__restrict__ lse, int keep_u, BlockMap bm, float sdip) {
  extern __shared__ float su[];  // [Ck][128] residual projections u_j (when keep_u)
  // blockIdx.x: a 128-row block of one instance (compact grid), blockIdx.y: the problem
  int bfirst;
  const int p = blockIdx.y, s = map_block(bm, mt.in.ninst, blockIdx.x, bfirst);
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int Ck = k.C, nq = q.n;
  const int rb0 = ((int)blockIdx.x - bfirst) * 128;
  const int n = rb0 + threadIdx.x;
  if (rb0 >= nq) return;  // uniform
  const bool v = n < nq;
  const int i = v ? q_cluster[q.lab + n] : 0;
  float qt[D];
#pragma unroll
  for (int d = 0; d < D; ++d) qt[d] = v ? ld_elem(qt_rows + (q.lab + n) * D + d) : 0.f;
  const int64_t zrow = (int64_t)p * mt.in.z_stride + mt.in.z0[s] + (int64_t)i * Ck;
  const float *lz = logZ + zrow;
  const float4 *mk = reinterpret_cast<const float4 *>(mu_k + zrow * D);
  float *C0 = c0 + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  float *C1 = c1 + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  const int cl = w_ld(nq);
  auto proj = [&](int j) {
    float u0 = 0.f, u1 = 0.f;
#pragma unroll
    for (int d4 = 0; d4 < D / 4; d4 += 2) {
      const float4 a = __ldg(mk + (int64_t)j * (D / 4) + d4);
      const float4 b = __ldg(mk + (int64_t)j * (D / 4) + d4 + 1);
      u0 = fmaf(qt[4 * d4], a.x, fmaf(qt[4 * d4 + 1], a.y, fmaf(qt[4 * d4 + 2], a.z, fmaf(qt[4 * d4 + 3], a.w, u0))));
      u1 = fmaf(qt[4 * d4 + 4], b.x, fmaf(qt[4 * d4 + 5], b.y, fmaf(qt[4 * d4 + 6], b.z, fmaf(qt[4 * d4 + 7], b.w, u1))));
    }
    return u0 + u1;
  };
  // pass 0: running max and sum of exp(a_j - max); pass 1: the coefficients
  float m = -CUDART_INF_F, l = 0.f;
  if (v) {
    for (int j = 0; j < Ck; ++j) {
      const float u = proj(j);
      if (keep_u) su[j * 128 + threadIdx.x] = u;
      const float a = lz[j] + scale * u;
      if (a > m) {
        l = l * __expf(m - a) + 1.f;
        m = a;
      } else if (a > -CUDART_INF_F) {
        l += __expf(a - m);
      }
    }
    const float inv = 1.f / l;
    for (int j = 0; j < Ck; ++j) {
      const float u = keep_u ? su[j * 128 + threadIdx.x] : proj(j);
      const float a = lz[j] + scale * u;
      const float pj = (a > -CUDART_INF_F) ? __expf(a - m) * inv : 0.f;
      C0[(int64_t)j * cl + n] = pj * (1.f - sdip * u);
      C1[(int64_t)j * cl + n] = sdip * pj;
    }
    lse[q.lab + n] = m + logf(l);
  }
}

// ---------------------------------------------------------------------------
// The same coefficients as a register-tiled contraction per query cluster i:
// U = Qt_i . mu_k,i^T (rows of cluster i against its Ck tilted key means), one
// CTA per 64-row chunk of a query cluster (the largest clusters set no tail).  The
// means and the chunk's rows are copied as stored by cp.async (no transpose); thread
// (tq, tj) takes rows 4 tq .. 4 tq + 3 and key clusters tj + 16 e and reads 4
// coordinates at a time of each; the 16 threads of a row are consecutive lanes
// (softmax by shuffles); each thread stores its 4 consecutive rows of a cluster j as
// one 16-byte vector.
// ---------------------------------------------------------------------------
// 16- and 4-byte asynchronous global -> shared copies (src_bytes = 0 writes zeros).
__device__ __forceinline__ void coef_cp16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void coef_cp4(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}

template <typename T, int D, int JPT>
__global__ void __launch_bounds__(256)
refine_coeffs_tiled(MuseTables mt, float scale, const T *__restrict__ qt_rows,
                    const int32_t *__restrict__ q_offsets, const float *__restrict__ logZ,
                    const float *__restrict__ mu_k, float *__restrict__ c0, float *__restrict__ c1,
                    float *__restrict__ lse, InstMask skip, float sdip, const __grid_constant__ BlockMap bm) {
  constexpr int CJ = 16 * JPT;                         // key clusters (all of them)
  constexpr int MSD = D + 4;                           // row stride of the means (floats)
  constexpr int QRB = D * (int)sizeof(T) + 16;         // row stride of the raw rows (bytes)
  extern __shared__ float4 tiled_smem[];
  float *Ms = reinterpret_cast<float *>(tiled_smem);   // [CJ][MSD] tilted key means of cluster i
  float *lz = Ms + CJ * MSD;                           // [CJ]
  unsigned char *Qr = reinterpret_cast<unsigned char *>(lz + CJ);  // [64][QRB] residual rows
  // blockIdx.x: a chunk slot of one instance (compact grid over this kernel's instances),
  // blockIdx.y: the problem
  int bfirst;
  const int p = blockIdx.y, s = map_block(bm, mt.in.ninst, blockIdx.x, bfirst);
  const int chunk = (int)blockIdx.x - bfirst;
  if ((skip.w[s >> 5] >> (s & 31)) & 1u) return;  // uniform: another kernel's instance
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  // this CTA's 64-row chunk: chunk g of the instance, counting ceil(rows/64) chunks
  // per query cluster in cluster order (rows start on 4-row boundaries)
  __shared__ int s_i, s_r0;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int run = 0, found = -1, fr0 = 0;
    for (int c0 = 0; c0 < q.C && found < 0; c0 += 32) {
      const int c = c0 + lane;
      int nch = 0, bb = 0;
      if (c < q.C) {
        bb = q_offsets[q.off + c];
        const int ee = q_offsets[q.off + c + 1];
        nch = ee > bb ? (ee - (bb & ~3) + 63) / 64 : 0;
      }
      int inc = nch;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const int first = run + inc - nch;  // chunk index of this cluster's first chunk
      const bool mine = chunk >= first && chunk < first + nch;
      const unsigned bal = __ballot_sync(0xffffffffu, mine);
      if (bal) {
        const int src = __ffs(bal) - 1;
        found = __shfl_sync(0xffffffffu, c, src);
        fr0 = __shfl_sync(0xffffffffu, (bb & ~3) + 64 * (chunk - first), src);
      }
      run += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) {
      s_i = found;
      s_r0 = fr0;
    }
  }
  __syncthreads();
  const int i = s_i;
  if (i < 0) return;  // uniform: past the instance's last chunk
  const int Ck = k.C;
  const int b = q_offsets[q.off + i], e = q_offsets[q.off + i + 1];
  const int64_t zrow = (int64_t)p * mt.in.z_stride + mt.in.z0[s] + (int64_t)i * Ck;
  const int r0 = s_r0;
  // Ms[j][d]: the cluster's tilted key means as stored (rows of D floats, padded);
  // Qr: the chunk's residual rows as stored (rows outside [b, e) zero); both by cp.async
  for (int u = threadIdx.x; u < CJ * (D / 4); u += 256) {
    const int j = u / (D / 4), c = u % (D / 4);
    const bool in = j < Ck;
    coef_cp16(Ms + j * MSD + 4 * c, in ? (const void *)(mu_k + (zrow + j) * D + 4 * c) : (const void *)mu_k,
              in ? 16u : 0u);
  }
  {
    constexpr int UR = D * (int)sizeof(T) / 16;
    for (int u = threadIdx.x; u < 64 * UR; u += 256) {
      const int rr = u / UR, c = u % UR;
      const bool in = r0 + rr >= b && r0 + rr < e;
      coef_cp16(Qr + rr * QRB + 16 * c,
                in ? (const void *)(reinterpret_cast<const uint4 *>(qt_rows + (q.lab + r0 + rr) * D) + c)
                   : (const void *)qt_rows,
                in ? 16u : 0u);
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int j = threadIdx.x; j < CJ; j += 256) lz[j] = j < Ck ? logZ[zrow + j] : -CUDART_INF_F;
  const int tq = threadIdx.x >> 4, tj = threadIdx.x & 15;
  float *C0 = c0 + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  float *C1 = c1 + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  const int cl = w_ld(q.n);
  // chunks start on 4-row boundaries of the coefficient arrays (16-byte stores);
  // rows outside [b, e) belong to other clusters and are neither read nor written
  {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    float acc[4][JPT];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int u = 0; u < JPT; ++u) acc[a][u] = 0.f;
#pragma unroll 2
    for (int d = 0; d < D; d += 4) {
      float qv[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const unsigned char *qrow = Qr + (4 * tq + a) * QRB;
        if constexpr (sizeof(T) == 2) {
          const uint2 raw = *reinterpret_cast<const uint2 *>(qrow + 2 * d);
          const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
          const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
          qv[a][0] = x.x;
          qv[a][1] = x.y;
          qv[a][2] = y.x;
          qv[a][3] = y.y;
        } else {
          const float4 x = *reinterpret_cast<const float4 *>(qrow + 4 * d);
          qv[a][0] = x.x;
          qv[a][1] = x.y;
          qv[a][2] = x.z;
          qv[a][3] = x.w;
        }
      }
#pragma unroll
      for (int u = 0; u < JPT; ++u) {
        const float4 m4 = *reinterpret_cast<const float4 *>(Ms + (tj + 16 * u) * MSD + d);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          acc[a][u] = fmaf(qv[a][0], m4.x, acc[a][u]);
          acc[a][u] = fmaf(qv[a][1], m4.y, acc[a][u]);
          acc[a][u] = fmaf(qv[a][2], m4.z, acc[a][u]);
          acc[a][u] = fmaf(qv[a][3], m4.w, acc[a][u]);
        }
      }
    }
    // a_j = logZ_ij + s u_j; p = softmax_j(a) over the 16 lanes of each row
    float pv[4][JPT];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float m = -CUDART_INF_F;
#pragma unroll
      for (int u = 0; u < JPT; ++u) m = fmaxf(m, lz[tj + 16 * u] + scale * acc[a][u]);
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float l = 0.f;
#pragma unroll
      for (int u = 0; u < JPT; ++u) {
        const float av = lz[tj + 16 * u] + scale * acc[a][u];
        l += av > -CUDART_INF_F ? __expf(av - m) : 0.f;
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      const float inv = 1.f / l;
#pragma unroll
      for (int u = 0; u < JPT; ++u) {
        const float av = lz[tj + 16 * u] + scale * acc[a][u];
        const float pj = av > -CUDART_INF_F ? __expf(av - m) * inv : 0.f;
        acc[a][u] = pj * (1.f - sdip * acc[a][u]);  // c0
        pv[a][u] = sdip * pj;                       // c1
      }
      const int n = r0 + 4 * tq + a;
      if (tj == 0 && n >= b && n < e) lse[q.lab + n] = m + logf(l);
    }
    // c0, then c1, through shared memory (the means' space, free after the products):
    // every key cluster's rows of the chunk leave as one contiguous run
    float *Cs = Ms;  // [CJ][65]
    const int lo = max(b, r0) - r0, hi = min(e, r0 + 64) - r0;  // the chunk's rows of cluster i
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      __syncthreads();  // the products (first half) or the previous stores are done
#pragma unroll
      for (int u = 0; u < JPT; ++u)
#pragma unroll
        for (int a = 0; a < 4; ++a) Cs[(tj + 16 * u) * 65 + 4 * tq + a] = half ? pv[a][u] : acc[a][u];
      __syncthreads();
      float *dst = half ? C1 : C0;
      for (int x = threadIdx.x; x < Ck * 64; x += 256) {
        const int j = x >> 6, rr = x & 63;
        if (rr >= lo && rr < hi) dst[(int64_t)j * cl + r0 + rr] = Cs[j * 65 + rr];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// The same coefficients for query clusters of a few rows (the causal squares' small
// instances): CTA per G consecutive query clusters of one instance (compact grid), passes
// of 16 rows of one cluster.  The cluster's Ck tilted key means and log-normalisers and
// the pass's residual rows arrive by cp.async one pass ahead.  Thread (tr, tj): row tr
// of the pass, key clusters tj + 16 u; the softmax runs over the 16 lanes of a row; the
// coefficients go through shared memory so that each key cluster's rows leave as one
// contiguous run.
// ---------------------------------------------------------------------------
template <typename T, int D, int JPT> struct CoefCfg {
  static constexpr int CJ = 16 * JPT;                  // key clusters (all of them)
  static constexpr int MSD = D + 4;                    // row stride of the means (floats)
  static constexpr int QRB = D * (int)sizeof(T) + 16;  // row stride of the raw rows (bytes)
  static constexpr int GMAX = 16;
  static constexpr size_t smem = 2 * (size_t)CJ * MSD * 4 + 2 * (size_t)CJ * 4 + 2 * 16 * (size_t)QRB +
                                 2 * (size_t)CJ * 17 * 4;
};

// query clusters per CTA for an instance of n rows in C clusters (about 64 rows a CTA)
__host__ __device__ __forceinline__ int coef_group(int n, int C) {
  if (C <= 0 || n <= 0) return 16;
  const int64_t g = 64ll * C / n;
  return (int)(g < 1 ? 1 : g > 16 ? 16 : g);
}


template <typename T, int D, int JPT>
__global__ void __launch_bounds__(256)
refine_coeffs_grouped(MuseTables mt, float scale, const T *__restrict__ qt_rows,
                      const int32_t *__restrict__ q_offsets, const float *__restrict__ logZ,
                      const float *__restrict__ mu_k, float *__restrict__ c0, float *__restrict__ c1,
                      float *__restrict__ lse, const __grid_constant__ BlockMap bm, float sdip) {
  using Cf = CoefCfg<T, D, JPT>;
  constexpr int CJ = Cf::CJ, MSD = Cf::MSD, QRB = Cf::QRB;
  extern __shared__ float4 coef_smem[];
  float *Ms = reinterpret_cast<float *>(coef_smem);               // [2][CJ][MSD] means
  float *Lz = Ms + 2 * CJ * MSD;                                  // [2][CJ] logZ row
  unsigned char *Qr = reinterpret_cast<unsigned char *>(Lz + 2 * CJ);  // [2][16][QRB] rows
  float *Cs = reinterpret_cast<float *>(Qr + 2 * 16 * QRB);       // [2][CJ][17] c0, c1
  __shared__ int offs[Cf::GMAX + 1];
  int bfirst;
  const int p = blockIdx.y, s = map_block(bm, mt.in.ninst, blockIdx.x, bfirst);
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int Cq = q.C, Ck = k.C;
  const int G = coef_group(q.n, Cq);
  const int i0 = ((int)blockIdx.x - bfirst) * G, i1 = min(Cq, i0 + G);
  if (i0 >= Cq) return;  // uniform
  const int tid = threadIdx.x, tr = tid >> 4, tj = tid & 15;
  if (tid <= i1 - i0) offs[tid] = q_offsets[q.off + i0 + tid];
  __syncthreads();
  const int64_t zbase = (int64_t)p * mt.in.z_stride + mt.in.z0[s];
  float *C0 = c0 + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  float *C1 = c1 + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  const int cl = w_ld(q.n);
  // a pass: rows r0 .. r0 + 15 (clipped to e) of cluster i
  struct Pass {
    int i, e, r0, mb;  // mb: the means buffer of cluster i
  };
  auto first_of = [&](int i, int mb) {
    while (i < i1 && offs[i - i0 + 1] == offs[i - i0]) ++i;
    Pass t;
    t.i = i;
    t.r0 = i < i1 ? offs[i - i0] : 0;
    t.e = i < i1 ? offs[i - i0 + 1] : 0;
    t.mb = mb;
    return t;
  };
  auto next_of = [&](const Pass &t) {
    if (t.r0 + 16 < t.e) {
      Pass n = t;
      n.r0 += 16;
      return n;
    }
    return first_of(t.i + 1, t.mb ^ 1);
  };
  // copies of pass t's inputs: the rows into row buffer qb and, for a cluster's first
  // pass, its means and log-normalisers into means buffer t.mb
  auto fetch = [&](const Pass &t, int qb, bool means) {
    constexpr int UR = D * (int)sizeof(T) / 16;  // 16-byte units per row
    for (int u = tid; u < 16 * UR; u += 256) {
      const int r = u / UR, c = u % UR;
      const bool in = t.r0 + r < t.e;
      coef_cp16(Qr + (qb * 16 + r) * QRB + 16 * c,
                in ? (const void *)(reinterpret_cast<const uint4 *>(qt_rows + (q.lab + t.r0 + r) * D) + c)
                   : (const void *)qt_rows,
                in ? 16u : 0u);
    }
    if (means) {
      const int64_t zrow = zbase + (int64_t)t.i * Ck;
      for (int u = tid; u < CJ * (D / 4); u += 256) {
        const int j = u / (D / 4), c = u % (D / 4);
        const bool in = j < Ck;
        coef_cp16(Ms + (t.mb * CJ + j) * MSD + 4 * c,
                  in ? (const void *)(mu_k + (zrow + j) * D + 4 * c) : (const void *)mu_k, in ? 16u : 0u);
      }
      for (int j = tid; j < CJ; j += 256)
        coef_cp4(Lz + t.mb * CJ + j, j < Ck ? (const void *)(logZ + zrow + j) : (const void *)logZ,
                 j < Ck ? 4u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  Pass cur = first_of(i0, 0);
  if (cur.i >= i1) return;  // uniform: every cluster of the group is empty
  int qb = 0;
  fetch(cur, qb, true);
  while (cur.i < i1) {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();  // this pass's inputs have landed; the previous pass is done
    const Pass nxt = next_of(cur);
    if (nxt.i < i1) fetch(nxt, qb ^ 1, nxt.i != cur.i);
    const float *M = Ms + cur.mb * CJ * MSD;
    const float *lz = Lz + cur.mb * CJ;
    const unsigned char *qrow = Qr + (qb * 16 + tr) * QRB;
    float acc[JPT];
#pragma unroll
    for (int u = 0; u < JPT; ++u) acc[u] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; d += 4) {
      float qv[4];
      if constexpr (sizeof(T) == 2) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(qrow + 2 * d);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
        qv[0] = a.x;
        qv[1] = a.y;
        qv[2] = b.x;
        qv[3] = b.y;
      } else {
        const float4 a = *reinterpret_cast<const float4 *>(qrow + 4 * d);
        qv[0] = a.x;
        qv[1] = a.y;
        qv[2] = a.z;
        qv[3] = a.w;
      }
#pragma unroll
      for (int u = 0; u < JPT; ++u) {
        const float4 m4 = *reinterpret_cast<const float4 *>(M + (tj + 16 * u) * MSD + d);
        acc[u] = fmaf(qv[0], m4.x, acc[u]);
        acc[u] = fmaf(qv[1], m4.y, acc[u]);
        acc[u] = fmaf(qv[2], m4.z, acc[u]);
        acc[u] = fmaf(qv[3], m4.w, acc[u]);
      }
    }
    // a_j = logZ_ij + s u_j; p = softmax_j(a) over the 16 lanes of the row
    float m = -CUDART_INF_F;
#pragma unroll
    for (int u = 0; u < JPT; ++u)
      m = fmaxf(m, tj + 16 * u < Ck ? lz[tj + 16 * u] + scale * acc[u] : -CUDART_INF_F);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
#pragma unroll
    for (int u = 0; u < JPT; ++u) {
      const float av = tj + 16 * u < Ck ? lz[tj + 16 * u] + scale * acc[u] : -CUDART_INF_F;
      l += av > -CUDART_INF_F ? __expf(av - m) : 0.f;
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    const float inv = 1.f / l;
#pragma unroll
    for (int u = 0; u < JPT; ++u) {
      const int j = tj + 16 * u;
      const float av = j < Ck ? lz[j] + scale * acc[u] : -CUDART_INF_F;
      const float pj = av > -CUDART_INF_F ? __expf(av - m) * inv : 0.f;
      Cs[j * 17 + tr] = pj * (1.f - sdip * acc[u]);
      Cs[(CJ + j) * 17 + tr] = sdip * pj;
    }
    const int nr = min(16, cur.e - cur.r0);
    if (tj == 0 && tr < nr) lse[q.lab + cur.r0 + tr] = m + logf(l);
    __syncthreads();
    for (int x = tid; x < Ck * 16; x += 256) {
      const int j = x >> 4, r = x & 15;
      if (r < nr) {
        C0[(int64_t)j * cl + cur.r0 + r] = Cs[j * 17 + r];
        C1[(int64_t)j * cl + cur.r0 + r] = Cs[(CJ + j) * 17 + r];
      }
    }
    cur = nxt;
    qb ^= 1;
  }
}

// ---------------------------------------------------------------------------
// Refinement on CUDA cores: 64 sorted queries per CTA, 4 threads per query
// (coordinates interleaved by 4), keys staged 32 at a time.
// ---------------------------------------------------------------------------
template <typename T, int D, int DV>
__global__ void __launch_bounds__(256)
refine_simt(MuseTables mt, int N, const T *__restrict__ qt_rows, const int32_t *__restrict__ q_perm,
            const int32_t *__restrict__ q_cluster, const T *__restrict__ ks,
            const int32_t *__restrict__ k_cluster, const T *__restrict__ vs,
            const float *__restrict__ W, const float *__restrict__ c0,
            const float *__restrict__ c1, const float *__restrict__ lse, T *__restrict__ O,
            float *__restrict__ part_o, float *__restrict__ part_lse) {
  const int p = blockIdx.y / mt.in.ninst, s = blockIdx.y % mt.in.ninst;
  const Task q = q_task(mt, p, s), k = k_task(mt, p, s);
  const int nq = q.n, nk = k.n;
  const int n0 = blockIdx.x * 64;
  if (n0 >= nq) return;
  __shared__ float Ks[32][D];
  __shared__ float Vs[32][DV];
  __shared__ int Js[32];
  const int g = threadIdx.x & 3;
  const int n = n0 + (threadIdx.x >> 2);
  const bool v = n < nq;
  constexpr int PD = D / 4, PV = DV / 4;
  float qt[PD];
#pragma unroll
  for (int t = 0; t < PD; ++t) qt[t] = v ? ld_elem(qt_rows + (q.lab + n) * D + g + 4 * t) : 0.f;
  const int i = v ? q_cluster[q.lab + n] : 0;
  const float *wrow = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s] + (int64_t)i * w_ld(nk);
  const float *C0 = c0 + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  const float *C1 = c1 + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  float acc[PV];
#pragma unroll
  for (int t = 0; t < PV; ++t) acc[t] = 0.f;
  int curj = -1;
  float a0 = 0.f, a1 = 0.f;
  for (int k0 = 0; k0 < nk; k0 += 32) {
    const int kt = min(32, nk - k0);
    __syncthreads();
    for (int e = threadIdx.x; e < kt * D; e += blockDim.x)
      Ks[e / D][e % D] = ld_elem(ks + (k.lab + k0) * D + e);
    for (int e = threadIdx.x; e < kt * DV; e += blockDim.x)
      Vs[e / DV][e % DV] = ld_elem(vs + (k.lab + k0) * DV + e);
    if (threadIdx.x < kt) Js[threadIdx.x] = k_cluster[k.lab + k0 + threadIdx.x];
    __syncthreads();
    for (int kk = 0; kk < kt; ++kk) {
      float x = 0.f;
#pragma unroll
      for (int t = 0; t < PD; ++t) x = fmaf(qt[t], Ks[kk][g + 4 * t], x);
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      const int j = Js[kk];
      if (j != curj) {
        curj = j;
        a0 = v ? C0[(int64_t)j * w_ld(nq) + n] : 0.f;
        a1 = v ? C1[(int64_t)j * w_ld(nq) + n] : 0.f;
      }
      const float P = v ? wrow[k0 + kk] * fmaf(a1, x, a0) : 0.f;
#pragma unroll
      for (int t = 0; t < PV; ++t) acc[t] = fmaf(P, Vs[kk][g + 4 * t], acc[t]);
    }
  }
  if (!v) return;
  const int row = q_perm[q.lab + n];
  if (O) {
    T *o = O + ((int64_t)p * N + row) * DV;
#pragma unroll
    for (int t = 0; t < PV; ++t) st_elem(o + g + 4 * t, acc[t]);
  } else {
    const int64_t r = (int64_t)p * mt.in.out_stride + mt.in.out0[s] + row;
#pragma unroll
    for (int t = 0; t < PV; ++t) part_o[r * DV + g + 4 * t] = acc[t];
    if (g == 0) part_lse[r] = lse[q.lab + n];
  }
}

// ---------------------------------------------------------------------------
// Causal: exact attention inside each diagonal block (keys [b*S, n]) merged with
// the level partials of the squares that hold the row (levels whose bit of b is
// set).  64 queries per CTA, 4 threads per query.
// ---------------------------------------------------------------------------
template <typename T, int D, int DV>
__global__ void __launch_bounds__(256)
diag_merge(const T *__restrict__ Qg, const T *__restrict__ Kg, const T *__restrict__ Vg, int N,
           int block, int levels, float scale, const float *__restrict__ part_o,
           const float *__restrict__ part_lse, T *__restrict__ O) {
  const int p = blockIdx.y;
  const int n0 = blockIdx.x * 64;
  const int bidx = n0 / block;
  const int ks0 = bidx * block;
  __shared__ float Ks[32][D];
  __shared__ float Vs[32][DV];
  const int g = threadIdx.x & 3;
  const int n = n0 + (threadIdx.x >> 2);
  constexpr int PD = D / 4, PV = DV / 4;
  const T *Qp = Qg + (int64_t)p * N * D;
  const T *Kp = Kg + (int64_t)p * N * D;
  const T *Vp = Vg + (int64_t)p * N * DV;
  float qv[PD];
#pragma unroll
  for (int t = 0; t < PD; ++t) qv[t] = ld_elem(Qp + (int64_t)n * D + g + 4 * t) * scale;
  float m = -CUDART_INF_F, l = 0.f;
  float acc[PV];
#pragma unroll
  for (int t = 0; t < PV; ++t) acc[t] = 0.f;
  const int kend = min(n0 + 64, N);
  for (int k0 = ks0; k0 < kend; k0 += 32) {
    const int kt = min(32, kend - k0);
    __syncthreads();
    for (int e = threadIdx.x; e < kt * D; e += blockDim.x)
      Ks[e / D][e % D] = ld_elem(Kp + (int64_t)k0 * D + e);
    for (int e = threadIdx.x; e < kt * DV; e += blockDim.x)
      Vs[e / DV][e % DV] = ld_elem(Vp + (int64_t)k0 * DV + e);
    __syncthreads();
    for (int kk = 0; kk < kt; ++kk) {
      float x = 0.f;
#pragma unroll
      for (int t = 0; t < PD; ++t) x = fmaf(qv[t], Ks[kk][g + 4 * t], x);
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      if (k0 + kk <= n) {
        const float mn = fmaxf(m, x);
        const float corr = expf(m - mn);
        const float pe = expf(x - mn);
        l = l * corr + pe;
#pragma unroll
        for (int t = 0; t < PV; ++t) acc[t] = fmaf(pe, Vs[kk][g + 4 * t], acc[t] * corr);
        m = mn;
      }
    }
  }
  // levels < 0: a single partial array, merged into every row
  const int nlev = levels < 0 ? 1 : levels;
  for (int lev = 1; lev <= nlev; ++lev) {
    if (levels > 0 && !((bidx >> (lev - 1)) & 1)) continue;
    const int64_t r = ((int64_t)p * nlev + (lev - 1)) * N + n;
    const float L = part_lse[r];
    if (!(L > -CUDART_INF_F)) continue;
    const float mn = fmaxf(m, L);
    const float ca = expf(m - mn), cb = expf(L - mn);
    l = l * ca + cb;
#pragma unroll
    for (int t = 0; t < PV; ++t) acc[t] = acc[t] * ca + cb * part_o[r * DV + g + 4 * t];
    m = mn;
  }
  const float inv = 1.f / l;
  T *o = O + ((int64_t)p * N + n) * DV;
#pragma unroll
  for (int t = 0; t < PV; ++t) st_elem(o + g + 4 * t, acc[t] * inv);
}

// ===========================================================================
// Host launchers
// ===========================================================================

cudaError_t run_sort_side(const void *X, int dtype, int width, int N, const SegTable &tab, int P,
                          const int32_t *perm, const int32_t *offsets, const float *centroids,
                          SortedSide out, cudaStream_t st) {
  const BlockMap bm = make_block_map(tab, 64);
  if (bm.total == 0) return cudaSuccess;
  dim3 grid(bm.total, P);
  const int threads = 256;
  count_launches(1);
  if (dtype == MUSE_F32)
    sort_side<float><<<grid, threads, 0, st>>>((const float *)X, N, width, tab, perm, offsets,
                                               centroids, (float *)out.rows, out.cluster, bm);
  else
    sort_side<__nv_bfloat16><<<grid, threads, 0, st>>>(
        (const __nv_bfloat16 *)X, N, width, tab, perm, offsets, centroids,
        (__nv_bfloat16 *)out.rows, out.cluster, bm);
  return cudaGetLastError();
}

cudaError_t run_sort_side_t(const void *X, int dtype, int width, int N, const SegTable &tab,
                            int P, const int32_t *perm, void *vt, cudaStream_t st) {
  const BlockMap bm = make_block_map(tab, 64);
  dim3 grid(bm.total, P);
  count_launches(1);
  if (dtype == MUSE_F32) {
    if (width == 64) sort_side_t<float, 64><<<grid, 256, 0, st>>>((const float *)X, N, tab, perm, (float *)vt, bm);
    else sort_side_t<float, 128><<<grid, 256, 0, st>>>((const float *)X, N, tab, perm, (float *)vt, bm);
  } else {
    if (width == 64)
      sort_side_t<__nv_bfloat16, 64><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)X, N, tab, perm, (__nv_bfloat16 *)vt, bm);
    else
      sort_side_t<__nv_bfloat16, 128><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)X, N, tab, perm, (__nv_bfloat16 *)vt, bm);
  }
  return cudaGetLastError();
}

template <typename T, int D, bool PRE>
static cudaError_t launch_tilt_fused(const MuseTables &mt, int P, float scale, const float *qcen,
                                     SortedSide ks, const int32_t *k_offsets, StageBufs b,
                                     cudaStream_t st) {
  using Cf = TiltCfg<T, D>;
  BlockMap bm;  // ceil(C / G) blocks per instance
  bm.pre[0] = 0;
  for (int si = 0; si < mt.in.ninst; ++si) {
    const int C = mt.k.C[si], g = tilt_group(mt.k.nrow[si], C, Cf::KC);
    bm.pre[si + 1] = bm.pre[si] + (C + g - 1) / g;
  }
  for (int si = mt.in.ninst + 1; si <= kMaxSeg; ++si) bm.pre[si] = bm.pre[mt.in.ninst];
  bm.total = bm.pre[mt.in.ninst];
  if (bm.total == 0) return cudaSuccess;
  cudaError_t err = cudaFuncSetAttribute(tilt_fused<T, D, PRE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cf::smem);
  if (err != cudaSuccess) return err;
  tilt_fused<T, D, PRE><<<dim3(bm.total, (mt.q.max_C + 63) / 64, P), 256, Cf::smem, st>>>(
      mt, scale, qcen, (const T *)ks.rows, k_offsets, b.W, b.logZ, b.mu_k, bm);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T, int D, int DV>
static cudaError_t summaries_t(const MuseTables &mt, int P, float scale, const float *qcen,
                               SortedSide ks, const void *vs, const int32_t *k_offsets,
                               StageBufs b, cudaStream_t st) {
  const int tasks = P * mt.in.ninst;
  const int maxCq = mt.q.max_C, maxCk = mt.k.max_C;
  if (b.mu_k && !b.mu_v && !b.cov) {
    // the forward pass: log-normalisers, weights and key means in one launch, from
    // logits of the tensor cores (bfloat16) or its own (float32)
    if (std::is_same<T, __nv_bfloat16>::value && logits_tc_supported(MUSE_BF16, D)) {
      cudaError_t e = run_logits_tc(mt, D, P, scale, qcen, ks.rows, b.W, device_status_word(), st);
      if (e != cudaSuccess) return e;
      return launch_tilt_fused<T, D, true>(mt, P, scale, qcen, ks, k_offsets, b, st);
    }
    return launch_tilt_fused<T, D, false>(mt, P, scale, qcen, ks, k_offsets, b, st);
  }
  const BlockMap kbm = make_block_map(mt.k, 64);
  tilt_logits<T, D><<<dim3(kbm.total, (maxCq + 63) / 64, P), 256, 0, st>>>(
      mt, scale, qcen, (const T *)ks.rows, b.W, kbm);
  int64_t keys = 0, clusters = 0;
  for (int si = 0; si < mt.in.ninst; ++si) {
    keys += mt.k.nrow[si];
    clusters += mt.k.C[si];
  }
  if (keys <= 32 * clusters)  // a few keys per cluster: a lane per cluster
    tilt_lse_short<<<dim3((maxCq + 7) / 8, tasks), 256, 0, st>>>(mt, k_offsets, b.W, b.logZ);
  else
    tilt_lse<<<dim3((maxCq * maxCk + 7) / 8, tasks), 256, 0, st>>>(mt, k_offsets, b.W, b.logZ);
  count_launches(2 + (b.mu_k != nullptr) + (b.mu_v != nullptr) + (b.cov != nullptr));
  if (b.mu_k)
    tilt_moments<T, D><<<dim3(maxCk, (maxCq + 63) / 64, tasks), 256, 0, st>>>(
        mt, k_offsets, b.W, (const T *)ks.rows, b.mu_k);
  if (b.mu_v)
    tilt_moments<T, DV><<<dim3(maxCk, (maxCq + 63) / 64, tasks), 256, 0, st>>>(
        mt, k_offsets, b.W, (const T *)vs, b.mu_v);
  if (b.cov)
    tilt_cov<T, D, DV><<<dim3(maxCk, maxCq, tasks), 256, 0, st>>>(
        mt, k_offsets, b.W, (const T *)ks.rows, (const T *)vs, b.mu_k, b.mu_v, b.cov);
  return cudaGetLastError();
}

#define MUSE_DISPATCH_DDV(dtype, D, Dv, FN, ...)                                        \
  do {                                                                                  \
    if ((dtype) == MUSE_F32) {                                                          \
      if ((D) == 64 && (Dv) == 64) return FN<float, 64, 64>(__VA_ARGS__);               \
      if ((D) == 64 && (Dv) == 128) return FN<float, 64, 128>(__VA_ARGS__);             \
      if ((D) == 128 && (Dv) == 64) return FN<float, 128, 64>(__VA_ARGS__);             \
      return FN<float, 128, 128>(__VA_ARGS__);                                          \
    }                                                                                   \
    if ((D) == 64 && (Dv) == 64) return FN<__nv_bfloat16, 64, 64>(__VA_ARGS__);         \
    if ((D) == 64 && (Dv) == 128) return FN<__nv_bfloat16, 64, 128>(__VA_ARGS__);       \
    if ((D) == 128 && (Dv) == 64) return FN<__nv_bfloat16, 128, 64>(__VA_ARGS__);       \
    return FN<__nv_bfloat16, 128, 128>(__VA_ARGS__);                                    \
  } while (0)

cudaError_t run_summaries(const MuseTables &mt, int dtype, int D, int Dv, int P, float scale,
                          const float *q_centroids, SortedSide ks, const void *vs_rows,
                          const int32_t *k_offsets, StageBufs b, cudaStream_t st) {
  MUSE_DISPATCH_DDV(dtype, D, Dv, summaries_t, mt, P, scale, q_centroids, ks, vs_rows, k_offsets,
                    b, st);
}

template <typename T, int DV>
static cudaError_t values_t(const MuseTables &mt, int P, const int32_t *k_offsets, const float *W,
                            const void *vs_rows, float *mu_v, cudaStream_t st) {
  tilt_moments<T, DV><<<dim3(mt.k.max_C, (mt.q.max_C + 63) / 64, P * mt.in.ninst), 256, 0, st>>>(
      mt, k_offsets, W, (const T *)vs_rows, mu_v);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t run_tilt_values(const MuseTables &mt, int dtype, int Dv, int P, const int32_t *k_offsets,
                            const float *W, const void *vs_rows, float *mu_v, cudaStream_t st) {
  if (dtype == MUSE_F32)
    return Dv == 64 ? values_t<float, 64>(mt, P, k_offsets, W, vs_rows, mu_v, st)
                    : values_t<float, 128>(mt, P, k_offsets, W, vs_rows, mu_v, st);
  return Dv == 64 ? values_t<__nv_bfloat16, 64>(mt, P, k_offsets, W, vs_rows, mu_v, st)
                  : values_t<__nv_bfloat16, 128>(mt, P, k_offsets, W, vs_rows, mu_v, st);
}

template <typename T, int D>
static cudaError_t weights_t(const MuseTables &mt, int P, float scale, const float *qcen,
                             SortedSide ks, const float *logZ, float *W, cudaStream_t st) {
  const int tasks = P * mt.in.ninst;
  const BlockMap kbm = make_block_map(mt.k, 64);
  tilt_logits<T, D><<<dim3(kbm.total, (mt.q.max_C + 63) / 64, P), 256, 0, st>>>(
      mt, scale, qcen, (const T *)ks.rows, W, kbm);
  tilt_weights<<<dim3((mt.k.max_rows + 255) / 256, mt.q.max_C, tasks), 256, 0, st>>>(
      mt, ks.cluster, logZ, W);
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t run_tilt_weights(const MuseTables &mt, int dtype, int D, int P, float scale,
                             const float *q_centroids, SortedSide ks, const float *logZ, float *W,
                             cudaStream_t st) {
  if (dtype == MUSE_F32)
    return D == 64 ? weights_t<float, 64>(mt, P, scale, q_centroids, ks, logZ, W, st)
                   : weights_t<float, 128>(mt, P, scale, q_centroids, ks, logZ, W, st);
  return D == 64 ? weights_t<__nv_bfloat16, 64>(mt, P, scale, q_centroids, ks, logZ, W, st)
                 : weights_t<__nv_bfloat16, 128>(mt, P, scale, q_centroids, ks, logZ, W, st);
}

template <typename T, int D, int JPT>
static cudaError_t coeffs_tiled_t(const MuseTables &mt, int P, float scale, SortedSide qs,
                                  const int32_t *q_offsets, StageBufs b, InstMask skip,
                                  float sdip, cudaStream_t st) {
  constexpr int CJ = 16 * JPT;
  const size_t smem = (size_t)CJ * (D + 4) * 4 + CJ * 4 + 64 * (D * sizeof(T) + 16);
  cudaError_t err = cudaFuncSetAttribute(refine_coeffs_tiled<T, D, JPT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  // chunk slots of an instance (none for the skipped ones): a cluster of n rows starting
  // up to 3 rows past a 4-row boundary takes at most n / 64 + 2 chunks
  BlockMap bm;
  bm.pre[0] = 0;
  for (int si = 0; si < mt.in.ninst; ++si) {
    const bool mine = !((skip.w[si >> 5] >> (si & 31)) & 1u);
    bm.pre[si + 1] = bm.pre[si] + (mine ? mt.q.nrow[si] / 64 + 2 * mt.q.C[si] : 0);
  }
  for (int si = mt.in.ninst + 1; si <= kMaxSeg; ++si) bm.pre[si] = bm.pre[mt.in.ninst];
  bm.total = bm.pre[mt.in.ninst];
  if (bm.total == 0) return cudaSuccess;
  refine_coeffs_tiled<T, D, JPT><<<dim3(bm.total, P), 256, smem, st>>>(
      mt, scale, (const T *)qs.rows, q_offsets, b.logZ, b.mu_k, b.c0, b.c1, b.lse, skip, sdip, bm);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T, int D, int JPT>
static cudaError_t coeffs_grouped_t(const MuseTables &mt, int P, float scale, SortedSide qs,
                                    const int32_t *q_offsets, StageBufs b, InstMask skip,
                                    float sdip, cudaStream_t st) {
  using Cf = CoefCfg<T, D, JPT>;
  BlockMap bm;  // ceil(C / G) blocks per instance this kernel takes
  bm.pre[0] = 0;
  for (int si = 0; si < mt.in.ninst; ++si) {
    const int C = mt.q.C[si], g = coef_group(mt.q.nrow[si], C);
    const bool mine = !((skip.w[si >> 5] >> (si & 31)) & 1u);
    bm.pre[si + 1] = bm.pre[si] + (mine ? (C + g - 1) / g : 0);
  }
  for (int si = mt.in.ninst + 1; si <= kMaxSeg; ++si) bm.pre[si] = bm.pre[mt.in.ninst];
  bm.total = bm.pre[mt.in.ninst];
  if (bm.total == 0) return cudaSuccess;
  cudaError_t err = cudaFuncSetAttribute(refine_coeffs_grouped<T, D, JPT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cf::smem);
  if (err != cudaSuccess) return err;
  refine_coeffs_grouped<T, D, JPT><<<dim3(bm.total, P), 256, Cf::smem, st>>>(
      mt, scale, (const T *)qs.rows, q_offsets, b.logZ, b.mu_k, b.c0, b.c1, b.lse, bm, sdip);
  count_launches(1);
  return cudaGetLastError();
}

// Instances whose query clusters hold fewer than 32 rows on average take the grouped
// kernel (passes of 16 rows), those with at least 64 the tensor-core kernel (bfloat16:
// one CTA per cluster and 128 rows), the others the tiled one (chunks of 64 rows); the
// kinds run side by side when the instances differ (the causal squares).
template <typename T, int D, int JPT>
static cudaError_t coeffs_split_t(const MuseTables &mt, int P, float scale, SortedSide qs,
                                  const int32_t *q_offsets, StageBufs b, float sdip,
                                  cudaStream_t st) {
  const bool tc = std::is_same<T, __nv_bfloat16>::value && coef_tc_supported(MUSE_BF16, D, mt.k.max_C);
  // each mask lists the instances its kernel skips
  InstMask not_small{}, not_mid{}, not_large{};
  bool any[3] = {false, false, false};
  for (int si = 0; si < mt.in.ninst; ++si) {
    const int64_t rows = mt.q.nrow[si], C = mt.q.C[si];
    const int kind = rows < 32 * C ? 0 : (tc && rows >= 64 * C) ? 2 : 1;
    any[kind] = true;
    const uint32_t bit = 1u << (si & 31);
    if (kind != 0) not_small.w[si >> 5] |= bit;
    if (kind != 1) not_mid.w[si >> 5] |= bit;
    if (kind != 2) not_large.w[si >> 5] |= bit;
  }
  cudaError_t err = cudaSuccess;
  if (any[2])
    err = run_coef_tc(mt, D, P, scale, qs.rows, q_offsets, b, not_large, sdip, device_status_word(), st);
  if (err == cudaSuccess && any[1])
    err = coeffs_tiled_t<T, D, JPT>(mt, P, scale, qs, q_offsets, b, not_mid, sdip, st);
  if (err == cudaSuccess && any[0])
    err = coeffs_grouped_t<T, D, JPT>(mt, P, scale, qs, q_offsets, b, not_small, sdip, st);
  return err;
}

template <typename T, int D>
static cudaError_t coeffs_t(const MuseTables &mt, int P, float scale, SortedSide qs,
                            const int32_t *q_offsets, StageBufs b, float sdip, cudaStream_t st) {
  // both forms stage each query cluster's tilted key means once in shared memory
  if (mt.k.max_C <= 64) return coeffs_split_t<T, D, 4>(mt, P, scale, qs, q_offsets, b, sdip, st);
  if (mt.k.max_C <= 128) return coeffs_split_t<T, D, 8>(mt, P, scale, qs, q_offsets, b, sdip, st);
  if (mt.k.max_C <= 256 && D == 64)
    return coeffs_split_t<T, D, 16>(mt, P, scale, qs, q_offsets, b, sdip, st);
  const int keep_u = mt.k.max_C <= 256 ? 1 : 0;
  const size_t smem = keep_u ? (size_t)mt.k.max_C * 128 * sizeof(float) : 0;
  cudaError_t err = cudaFuncSetAttribute(refine_coeffs<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const BlockMap bm = make_block_map(mt.q, 128);
  refine_coeffs<T, D><<<dim3(bm.total, P), 128, smem, st>>>(
      mt, scale, (const T *)qs.rows, qs.cluster, b.logZ, b.mu_k, b.c0, b.c1, b.lse, keep_u, bm, sdip);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t run_coeffs(const MuseTables &mt, int dtype, int D, int P, float scale, SortedSide qs,
                       const int32_t *q_offsets, StageBufs b, float sdip, cudaStream_t st) {
  if (dtype == MUSE_F32)
    return D == 64 ? coeffs_t<float, 64>(mt, P, scale, qs, q_offsets, b, sdip, st)
                   : coeffs_t<float, 128>(mt, P, scale, qs, q_offsets, b, sdip, st);
  return D == 64 ? coeffs_t<__nv_bfloat16, 64>(mt, P, scale, qs, q_offsets, b, sdip, st)
                 : coeffs_t<__nv_bfloat16, 128>(mt, P, scale, qs, q_offsets, b, sdip, st);
}

template <typename T, int D, int DV>
static cudaError_t refine_t(const MuseTables &mt, int N, int P, SortedSide qs,
                            const int32_t *q_perm, SortedSide ks, const void *vs, StageBufs b,
                            void *O, float *part_o, float *part_lse, cudaStream_t st) {
  dim3 grid((mt.q.max_rows + 63) / 64, P * mt.in.ninst);
  refine_simt<T, D, DV><<<grid, 256, 0, st>>>(
      mt, N, (const T *)qs.rows, q_perm, qs.cluster, (const T *)ks.rows, ks.cluster,
      (const T *)vs, b.W, b.c0, b.c1, b.lse, (T *)O, part_o, part_lse);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t run_refine(const MuseTables &mt, int dtype, int D, int Dv, int N, int P,
                       SortedSide qs, const int32_t *q_perm, SortedSide ks, const void *vs_rows,
                       StageBufs b, void *O, float *part_o, float *part_lse, cudaStream_t st) {
  MUSE_DISPATCH_DDV(dtype, D, Dv, refine_t, mt, N, P, qs, q_perm, ks, vs_rows, b, O, part_o,
                    part_lse, st);
}

template <typename T, int D, int DV>
static cudaError_t diag_t(const void *Q, const void *K, const void *V, int N, int P, int block,
                          int levels, float scale, const float *part_o, const float *part_lse,
                          void *O, cudaStream_t st) {
  diag_merge<T, D, DV><<<dim3(N / 64, P), 256, 0, st>>>(
      (const T *)Q, (const T *)K, (const T *)V, N, block, levels, scale, part_o, part_lse, (T *)O);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t run_diag_merge(const void *Q, const void *K, const void *V, int dtype, int D, int Dv,
                           int N, int P, int block, int levels, float scale,
                           const float *part_o, const float *part_lse, void *O, cudaStream_t st) {
  if (diag_tc_supported(dtype, D, Dv, N, block))
    return run_diag_tc(Q, K, V, N, P, block, levels, scale, part_o, part_lse, O, device_status_word(), st);
  MUSE_DISPATCH_DDV(dtype, D, Dv, diag_t, Q, K, V, N, P, block, levels, scale, part_o, part_lse,
                    O, st);
}

}  // namespace muse
