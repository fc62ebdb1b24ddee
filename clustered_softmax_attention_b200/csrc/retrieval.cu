// Causal MuSe with causal accumulation and top-k retrieval.
//
// gist.science "Technische Samenvatting: Multipole Semantic Attention (MuSe)",
// "Kernmechanismen" item 3 (the context is cut into spatial blocks; a block sees the
// summaries of all preceding blocks) and item 4 (top-k1 key clusters by tilted
// summary score, then top-k2 spatial blocks inside them; exact attention on the
// retrieved (cluster, block) pairs and the local block diagonal; the remaining
// interactions through the approximate summaries).
//
// Clusters are global (one K-means over each problem's queries and keys).  Inside
// a key cluster the sorted keys keep their token order, so the keys of cluster j in
// block b' form one contiguous run; pend[j][b'] counts the keys of cluster j in
// blocks < b'.
//
// For query n (block b, cluster i, qt = q - qbar_i):
//   selection: sigma_j = logsumexp_{b'<b} logZb_{i,j,b'}; the k1 largest (ties to the
//     lower j); inside each, the k2 largest logZb_{i,j,b'}, b' < b (ties to lower b');
//   remainder R_j = keys of cluster j in blocks < b minus the selected runs, tilted by
//     qbar_i: logZR_{i,b,j}, and with W_ik = exp(s qbar_i.k - logZ_ij) (the whole
//     cluster's tilt), w^R_ik = W_ik exp(logZ_ij - logZR_{i,b,j});
//     u_j = sum_{k in R_j} w^R_ik qt.k ;  a_j = logZR + s u_j ;  p = softmax_j(a);
//     remainder output = sum_j p_j sum_{k in R_j} w^R_ik (1 - s u_j + s qt.k) v_k
//     (the monopole + dipole refinement of the acausal path, restricted to R_j);
//   exact part: keys of the selected runs and the diagonal keys [bS, n];
//   both parts are merged into one softmax through their logsumexps.
//
// bfloat16 inputs (D, Dv in {64, 128}) take the tensor-core path: u_j via running
// prefixes over the key blocks (ret_T), the remainder output on tcgen05 (the
// refinement kernel's retrieval mode), the selected runs exactly on the CUDA cores
// (ret_runs) and the diagonal with the merge on tcgen05 (diag_tc) where it applies.
// float32 inputs take the CUDA-core passes below (remainder_pass, exact_merge).
#include <math.h>
#include <string.h>

#include <algorithm>

#include "internal.h"
#include "tc.h"

namespace muse {
namespace ret {

struct Geo {
  int N, S, nb, Cq, Ck, K12, k1, k2;
};

__device__ __forceinline__ float lse_add(float a, float b) {
  if (a == -CUDART_INF_F) return b;
  if (b == -CUDART_INF_F) return a;
  const float m = fmaxf(a, b);
  return m + logf(expf(a - m) + expf(b - m));
}

// cnt[p][j][b'] = rows of cluster j in block b' (integer atomics: exact); C clusters.
__global__ void block_counts(Geo g, int C, const int32_t *__restrict__ labels, int32_t *__restrict__ cnt) {
  const int p = blockIdx.y;
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= g.N) return;
  const int j = labels[(int64_t)p * g.N + k];
  atomicAdd(&cnt[((int64_t)p * C + j) * g.nb + k / g.S], 1);
}

// pend[p][j][b'] = rows of cluster j in blocks < b' (b' = 0..nb).
__global__ void block_prefix(Geo g, int P, int C, const int32_t *__restrict__ cnt,
                             int32_t *__restrict__ pend) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= P * C) return;
  const int32_t *c = cnt + (int64_t)t * g.nb;
  int32_t *o = pend + (int64_t)t * (g.nb + 1);
  int run = 0;
  for (int b = 0; b < g.nb; ++b) {
    o[b] = run;
    run += c[b];
  }
  o[g.nb] = run;
}

// logZb[p][i][j][b'] = logZ_ij + log(sum of W_ik over the run of (j, b')); one thread per
// (p, i, j, b'), the run's weights summed in key order (runs are a few keys long).
__global__ void __launch_bounds__(256)
block_lse(Geo g, int P, const float *__restrict__ W, int w_stride, const float *__restrict__ logZ,
          const int32_t *__restrict__ k_offsets, const int32_t *__restrict__ pend,
          float *__restrict__ logZb) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (int64_t)P * g.Cq * g.Ck * g.nb) return;
  const int b = (int)(t % g.nb);
  const int64_t pij = t / g.nb;
  const int j = (int)(pij % g.Ck);
  const int i = (int)((pij / g.Ck) % g.Cq);
  const int p = (int)(pij / ((int64_t)g.Ck * g.Cq));
  const float *w = W + (int64_t)p * w_stride + (int64_t)i * w_ld(g.N);
  const int off = k_offsets[(int64_t)p * (g.Ck + 1) + j];
  const int32_t *pe = pend + ((int64_t)p * g.Ck + j) * (g.nb + 1);
  const int s0 = off + pe[b], s1 = off + pe[b + 1];
  float acc = 0.f;
  for (int pos = s0; pos < s1; ++pos) acc += w[pos];
  logZb[t] = (s1 > s0) ? logZ[pij] + logf(acc) : -CUDART_INF_F;
}

// pref[p][i][b][j] = logsumexp_{b' < b} logZb[p][i][j][b'] (b = 0..nb), accumulated in block
// order; one thread per (p, i, j).
__global__ void __launch_bounds__(256)
block_prefix_lse(Geo g, int P, const float *__restrict__ logZb, float *__restrict__ pref) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (int64_t)P * g.Cq * g.Ck) return;
  const int j = (int)(t % g.Ck);
  const int64_t pi = t / g.Ck;
  const float *lzb = logZb + t * g.nb;
  float *out = pref + pi * (int64_t)(g.nb + 1) * g.Ck + j;
  float acc = -CUDART_INF_F;
  out[0] = acc;
  for (int b = 0; b < g.nb; ++b) {
    acc = lse_add(acc, lzb[b]);
    out[(int64_t)(b + 1) * g.Ck] = acc;
  }
}

// One warp per (p, i, b): the selection and the remainder log-normalisers.
// sel[p][i][b][slot] = (j, b'), slot = t*k2 + u; logZR[p][i][b][j].  MAXJ: key clusters per
// lane (Ck <= 32 MAXJ).
template <int MAXJ>
__global__ void __launch_bounds__(256)
select_blocks(Geo g, int P, const float *__restrict__ logZb, const float *__restrict__ pref,
              int32_t *__restrict__ sel, float *__restrict__ logZR) {
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)P * g.Cq * g.nb) return;
  const int b = (int)(wid % g.nb);
  const int i = (int)((wid / g.nb) % g.Cq);
  const int p = (int)(wid / ((int64_t)g.nb * g.Cq));
  const float *lzb = logZb + ((int64_t)p * g.Cq + i) * g.Ck * g.nb;  // [j][b']
  int32_t *so = sel + (((int64_t)p * g.Cq + i) * g.nb + b) * g.K12 * 2;
  float *zr = logZR + (((int64_t)p * g.Cq + i) * g.nb + b) * g.Ck;
  for (int e = lane; e < g.K12 * 2; e += 32) so[e] = -1;
  // sigma_j for this lane's clusters j = lane + 32 m
  float sig[MAXJ];
  bool taken[MAXJ];
#pragma unroll
  for (int m = 0; m < MAXJ; ++m) {
    sig[m] = -CUDART_INF_F;
    taken[m] = false;
    const int j = lane + 32 * m;
    if (j < g.Ck) sig[m] = pref[(((int64_t)p * g.Cq + i) * (g.nb + 1) + b) * g.Ck + j];
  }
  int chosen[64];
  int nchosen = 0;
  for (int t = 0; t < g.k1 && b > 0; ++t) {
    // warp argmax of sigma over untaken finite clusters, ties to the lower j
    float bv = -CUDART_INF_F;
    int bj = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < MAXJ; ++m) {
      const int j = lane + 32 * m;
      if (j < g.Ck && !taken[m] && sig[m] > -CUDART_INF_F && (sig[m] > bv || (sig[m] == bv && j < bj))) {
        bv = sig[m];
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (ov > bv || (ov == bv && oj < bj)) {
        bv = ov;
        bj = oj;
      }
    }
    if (bj == 0x7fffffff) break;  // fewer candidates than k1
    if ((bj & 31) == lane) taken[bj >> 5] = true;
    chosen[nchosen++] = bj;
    // top-k2 blocks of cluster bj among b' < b (lanes over b')
    const float *row = lzb + (int64_t)bj * g.nb;
    unsigned used = 0u;  // bit m: block lane + 32 m already chosen
    for (int u = 0; u < g.k2; ++u) {
      float vv = -CUDART_INF_F;
      int vb = 0x7fffffff;
      for (int m = 0; m * 32 < b; ++m) {
        const int bb = lane + 32 * m;
        if (bb < b && !((used >> m) & 1u)) {
          const float x = row[bb];
          if (x > -CUDART_INF_F && (x > vv || (x == vv && bb < vb))) {
            vv = x;
            vb = bb;
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, vv, o);
        const int ob = __shfl_xor_sync(0xffffffffu, vb, o);
        if (ov > vv || (ov == vv && ob < vb)) {
          vv = ov;
          vb = ob;
        }
      }
      if (vb == 0x7fffffff) break;
      if ((vb & 31) == lane) used |= 1u << (vb >> 5);
      if (lane == 0) {
        so[(t * g.k2 + u) * 2] = bj;
        so[(t * g.k2 + u) * 2 + 1] = vb;
      }
    }
  }
  __syncwarp();
  // remainder log-normalisers: blocks b' < b, minus the selected runs (an unselected
  // cluster's is its prefix score, summed in the same order)
#pragma unroll
  for (int m = 0; m < MAXJ; ++m) {
    const int j = lane + 32 * m;
    if (j >= g.Ck) continue;
    int tj = -1;
    for (int t = 0; t < nchosen; ++t)
      if (chosen[t] == j) tj = t;
    if (tj < 0) {
      zr[j] = sig[m];
      continue;
    }
    float acc = -CUDART_INF_F;
    for (int bb = 0; bb < b; ++bb) {
      bool ex = false;
      for (int u = 0; u < g.k2; ++u) ex |= (so[(tj * g.k2 + u) * 2 + 1] == bb);
      if (!ex) acc = lse_add(acc, lzb[(int64_t)j * g.nb + bb]);
    }
    zr[j] = acc;
  }
}

static void launch_select(const Geo &g, int P, int64_t ns, const float *logZb, const float *pref,
                          int32_t *sel, float *logZR, cudaStream_t st) {
  const unsigned grid = (unsigned)((ns + 7) / 8);
  if (g.Ck <= 128)
    select_blocks<4><<<grid, 256, 0, st>>>(g, P, logZb, pref, sel, logZR);
  else if (g.Ck <= 256)
    select_blocks<8><<<grid, 256, 0, st>>>(g, P, logZb, pref, sel, logZR);
  else
    select_blocks<kMaxClusters / 32><<<grid, 256, 0, st>>>(g, P, logZb, pref, sel, logZR);
}

// Excluded blocks of cluster j for a query whose selection row is `so` (<= 64 slots).
__device__ __forceinline__ int excluded_blocks(const int32_t *so, int K12, int j, int (&xb)[8]) {
  int n = 0;
  for (int s = 0; s < K12 && n < 8; ++s)
    if (so[2 * s] == j) xb[n++] = so[2 * s + 1];
  return n;
}
__device__ __forceinline__ bool in_list(int v, const int (&xb)[8], int n) {
  bool r = false;
#pragma unroll
  for (int a = 0; a < 8; ++a) r |= (a < n && xb[a] == v);
  return r;
}

// Passes over the remainder keys of every cluster, 64 queries (one block b) per CTA,
// 4 threads per query.  MODE 0: T[j][n] = sum_{k in R_j} W_ik qt.k.
// MODE 1: o_n = sum_j sum_{k in R_j} W_ik (c0'_{jn} + c1'_{jn} qt.k) v_k.
template <typename T, int D, int DV, int MODE>
__global__ void __launch_bounds__(256)
remainder_pass(Geo g, const T *__restrict__ Q, const float *__restrict__ qcen,
               const int32_t *__restrict__ q_labels, const T *__restrict__ ks,
               const T *__restrict__ vs, const int32_t *__restrict__ k_perm,
               const int32_t *__restrict__ k_offsets, const int32_t *__restrict__ pend,
               const float *__restrict__ W, int w_stride, const int32_t *__restrict__ sel,
               float *__restrict__ Tbuf, const float *__restrict__ c0, const float *__restrict__ c1,
               float *__restrict__ part_o) {
  const int p = blockIdx.y;
  const int n0 = blockIdx.x * 64;
  const int b = n0 / g.S;
  if (b == 0) return;  // block 0 has no remainder
  __shared__ float Ks[32][D];
  __shared__ float Vs[MODE ? 32 : 1][DV];
  __shared__ int Bk[32];
  const int gq = threadIdx.x & 3;
  const int n = n0 + (threadIdx.x >> 2);
  constexpr int PD = D / 4, PV = DV / 4;
  const int i = q_labels[(int64_t)p * g.N + n];
  float qt[PD];
#pragma unroll
  for (int t = 0; t < PD; ++t)
    qt[t] = ld_elem(Q + ((int64_t)p * g.N + n) * D + gq + 4 * t) - qcen[((int64_t)p * g.Cq + i) * D + gq + 4 * t];
  const float *wrow = W + (int64_t)p * w_stride + (int64_t)i * w_ld(g.N);
  const int32_t *so = sel + (((int64_t)p * g.Cq + i) * g.nb + b) * g.K12 * 2;
  float acc[MODE ? PV : 1];
#pragma unroll
  for (int t = 0; t < (MODE ? PV : 1); ++t) acc[t] = 0.f;
  const int32_t *koff = k_offsets + (int64_t)p * (g.Ck + 1);
  const T *kp = ks + (int64_t)p * g.N * D;
  const T *vp = vs + (int64_t)p * g.N * DV;
  for (int j = 0; j < g.Ck; ++j) {
    const int s0 = koff[j];
    const int s1 = s0 + pend[((int64_t)p * g.Ck + j) * (g.nb + 1) + b];
    if (s1 <= s0) continue;  // CTA-uniform
    int xb[8];
    const int nx = excluded_blocks(so, g.K12, j, xb);
    float tsum = 0.f, a0 = 0.f, a1 = 0.f;
    if (MODE) {
      a0 = c0[((int64_t)p * g.Ck + j) * g.N + n];
      a1 = c1[((int64_t)p * g.Ck + j) * g.N + n];
    }
    for (int k0 = s0; k0 < s1; k0 += 32) {
      const int kt = min(32, s1 - k0);
      __syncthreads();
      for (int e = threadIdx.x; e < kt * D; e += blockDim.x) Ks[e / D][e % D] = ld_elem(kp + (int64_t)k0 * D + e);
      if (MODE)
        for (int e = threadIdx.x; e < kt * DV; e += blockDim.x)
          Vs[e / DV][e % DV] = ld_elem(vp + (int64_t)k0 * DV + e);
      if (threadIdx.x < kt) Bk[threadIdx.x] = k_perm[(int64_t)p * g.N + k0 + threadIdx.x] / g.S;
      __syncthreads();
      for (int kk = 0; kk < kt; ++kk) {
        float x = 0.f;
#pragma unroll
        for (int t = 0; t < PD; ++t) x = fmaf(qt[t], Ks[kk][gq + 4 * t], x);
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        if (nx && in_list(Bk[kk], xb, nx)) continue;
        const float w = wrow[k0 + kk];
        if (MODE) {
          const float P = w * fmaf(a1, x, a0);
#pragma unroll
          for (int t = 0; t < PV; ++t) acc[t] = fmaf(P, Vs[kk][gq + 4 * t], acc[t]);
        } else {
          tsum = fmaf(w, x, tsum);
        }
      }
    }
    if (!MODE && gq == 0) Tbuf[((int64_t)p * g.Ck + j) * g.N + n] = tsum;
  }
  if (MODE) {
#pragma unroll
    for (int t = 0; t < PV; ++t) part_o[((int64_t)p * g.N + n) * DV + gq + 4 * t] = acc[t];
  }
}

// Remainder coefficients per query (natural order):
//   U_j = exp(logZ_ij - logZR) T_j;  a_j = logZR + s U_j;  p = softmax(a);
//   c0'_j = p_j (1 - s U_j) exp(logZ_ij - logZR),  c1'_j = s p_j exp(logZ_ij - logZR).
__global__ void __launch_bounds__(128)
remainder_coeffs(Geo g, int P, float scale, const int32_t *__restrict__ q_labels,
                 const float *__restrict__ logZ, const float *__restrict__ logZR,
                 const float *__restrict__ Tbuf, float *__restrict__ c0, float *__restrict__ c1,
                 float *__restrict__ lse_r) {
  const int p = blockIdx.y;
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= g.N) return;
  const int b = n / g.S;
  const int i = q_labels[(int64_t)p * g.N + n];
  const float *lz = logZ + ((int64_t)p * g.Cq + i) * g.Ck;
  const float *zr = logZR + (((int64_t)p * g.Cq + i) * g.nb + b) * g.Ck;
  float m = -CUDART_INF_F, l = 0.f;
  for (int pass = 0; pass < 2; ++pass) {
    const float inv = pass ? 1.f / l : 0.f;
    for (int j = 0; j < g.Ck; ++j) {
      const int64_t at = ((int64_t)p * g.Ck + j) * g.N + n;
      const float r = zr[j];
      if (b == 0 || !(r > -CUDART_INF_F)) {
        if (pass) {
          c0[at] = 0.f;
          c1[at] = 0.f;
        }
        continue;
      }
      const float f = expf(lz[j] - r);
      const float U = f * Tbuf[at];
      const float a = r + scale * U;
      if (!pass) {
        if (a > m) {
          l = l * expf(m - a) + 1.f;
          m = a;
        } else {
          l += expf(a - m);
        }
      } else {
        const float pj = expf(a - m) * inv;
        c0[at] = pj * (1.f - scale * U) * f;
        c1[at] = scale * pj * f;
      }
    }
  }
  lse_r[(int64_t)p * g.N + n] = (l > 0.f) ? m + logf(l) : -CUDART_INF_F;
}

// Exact part (diagonal keys [bS, n] and the selected runs) with online softmax, merged
// with the remainder partial (lse_r, o_r).  64 queries per CTA, 4 threads per query.
template <typename T, int D, int DV>
__global__ void __launch_bounds__(256)
exact_merge(Geo g, float scale, const T *__restrict__ Q, const T *__restrict__ K,
            const T *__restrict__ V, const int32_t *__restrict__ q_labels,
            const T *__restrict__ ks, const T *__restrict__ vs,
            const int32_t *__restrict__ k_offsets, const int32_t *__restrict__ pend,
            const int32_t *__restrict__ sel, const float *__restrict__ part_o,
            const float *__restrict__ lse_r, T *__restrict__ O) {
  const int p = blockIdx.y;
  const int n0 = blockIdx.x * 64;
  const int b = n0 / g.S;
  __shared__ float Ks[32][D];
  __shared__ float Vs[32][DV];
  const int gq = threadIdx.x & 3;
  const int n = n0 + (threadIdx.x >> 2);
  constexpr int PD = D / 4, PV = DV / 4;
  float qv[PD];
#pragma unroll
  for (int t = 0; t < PD; ++t) qv[t] = ld_elem(Q + ((int64_t)p * g.N + n) * D + gq + 4 * t) * scale;
  float m = -CUDART_INF_F, l = 0.f;
  float acc[PV];
#pragma unroll
  for (int t = 0; t < PV; ++t) acc[t] = 0.f;
  auto add = [&](float x, const float *vrow, int stride) {
    const float mn = fmaxf(m, x);
    const float corr = expf(m - mn), pe = expf(x - mn);
    l = l * corr + pe;
#pragma unroll
    for (int t = 0; t < PV; ++t) acc[t] = fmaf(pe, vrow[t * stride], acc[t] * corr);
    m = mn;
  };
  // diagonal block, keys [bS, n]
  const int kend = n0 + 64;
  for (int k0 = b * g.S; k0 < kend; k0 += 32) {
    const int kt = min(32, kend - k0);
    __syncthreads();
    for (int e = threadIdx.x; e < kt * D; e += blockDim.x)
      Ks[e / D][e % D] = ld_elem(K + ((int64_t)p * g.N + k0) * D + e);
    for (int e = threadIdx.x; e < kt * DV; e += blockDim.x)
      Vs[e / DV][e % DV] = ld_elem(V + ((int64_t)p * g.N + k0) * DV + e);
    __syncthreads();
    for (int kk = 0; kk < kt; ++kk) {
      float x = 0.f;
#pragma unroll
      for (int t = 0; t < PD; ++t) x = fmaf(qv[t], Ks[kk][gq + 4 * t], x);
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      if (k0 + kk <= n) add(x, &Vs[kk][gq], 4);
    }
  }
  // selected runs (sorted positions), per query
  if (b > 0) {
    const int i = q_labels[(int64_t)p * g.N + n];
    const int32_t *so = sel + (((int64_t)p * g.Cq + i) * g.nb + b) * g.K12 * 2;
    const int32_t *koff = k_offsets + (int64_t)p * (g.Ck + 1);
    for (int s = 0; s < g.K12; ++s) {
      const int j = so[2 * s], bb = so[2 * s + 1];
      if (j < 0) continue;
      const int32_t *pe = pend + ((int64_t)p * g.Ck + j) * (g.nb + 1);
      const int s0 = koff[j] + pe[bb], s1 = koff[j] + pe[bb + 1];
      for (int pos = s0; pos < s1; ++pos) {
        const T *kr = ks + ((int64_t)p * g.N + pos) * D;
        float x = 0.f;
#pragma unroll
        for (int t = 0; t < PD; ++t) x = fmaf(qv[t], ld_elem(kr + gq + 4 * t), x);
        // the 4 lanes of this query follow the same runs
        const unsigned gm = 0xFu << ((threadIdx.x & 31) & ~3);
        x += __shfl_xor_sync(gm, x, 1);
        x += __shfl_xor_sync(gm, x, 2);
        float vr[PV];
        const T *vrp = vs + ((int64_t)p * g.N + pos) * DV;
#pragma unroll
        for (int t = 0; t < PV; ++t) vr[t] = ld_elem(vrp + gq + 4 * t);
        add(x, vr, 1);
      }
    }
    const float L = lse_r[(int64_t)p * g.N + n];
    if (L > -CUDART_INF_F) {
      const float mn = fmaxf(m, L);
      const float ca = expf(m - mn), cb = expf(L - mn);
      l = l * ca + cb;
#pragma unroll
      for (int t = 0; t < PV; ++t)
        acc[t] = acc[t] * ca + cb * part_o[((int64_t)p * g.N + n) * DV + gq + 4 * t];
      m = mn;
    }
  }
  const float inv = 1.f / l;
  T *o = O + ((int64_t)p * g.N + n) * DV;
#pragma unroll
  for (int t = 0; t < PV; ++t) st_elem(o + gq + 4 * t, acc[t] * inv);
}

// ---------------------------------------------------------------------------
// Tensor-core path (bfloat16).  Query rows are in query-cluster order (sorted
// residuals qt = q - qbar_i), keys in key-cluster order; inside a cluster both keep
// token order, so the rows of (cluster i, block b) and the keys of (cluster j,
// block b') are contiguous runs: [qoff_i + qpend_i(b), qoff_i + qpend_i(b+1)) and
// [koff_j + pend_j(b'), koff_j + pend_j(b'+1)).
// ---------------------------------------------------------------------------

// T[p][j][r] = sum over the remainder keys k of cluster j of W_ik qt_r.k for sorted query
// row r (cluster i, block b): the keys of j in blocks b' < b minus the runs selected for
// (i, b).  A running sum m1_j = sum_{b' < b} sum_{k in (j, b')} W_ik k over the key blocks
// gives qt_r.m1_j; a selected cluster's runs are summed once per (i, b) group into e_j
// and qt_r.(m1_j - e_j) is taken (float32).  One CTA per (problem, query cluster i, group
// of JPC key clusters); DP = D / 8 threads per cluster, 8 coordinates each (few registers,
// so many warps hide the latency of the block-by-block walk); no block-wide barrier (a
// thread's work varies with its cluster's keys per block).
template <int D>
__global__ void __launch_bounds__(256)
ret_T(Geo g, const __nv_bfloat16 *__restrict__ qs, const int32_t *__restrict__ q_offsets,
      const int32_t *__restrict__ qpend, const __nv_bfloat16 *__restrict__ ks,
      const int32_t *__restrict__ k_offsets, const int32_t *__restrict__ pend,
      const float *__restrict__ W, int w_stride, const int32_t *__restrict__ sel,
      float *__restrict__ Tout) {
  constexpr int CPT = 8, DP = D / CPT, JPC = 256 / DP;
  const int p = blockIdx.z, i = blockIdx.y;
  const int jl = threadIdx.x / DP, dp = threadIdx.x % DP;
  const int j = blockIdx.x * JPC + jl;
  const bool live = j < g.Ck;
  const int jj = live ? j : g.Ck - 1;
  const int32_t *qo = q_offsets + (int64_t)p * (g.Cq + 1);
  const int32_t *qpe = qpend + ((int64_t)p * g.Cq + i) * (g.nb + 1);
  const int32_t *pe = pend + ((int64_t)p * g.Ck + jj) * (g.nb + 1);
  const int kbase = k_offsets[(int64_t)p * (g.Ck + 1) + jj];
  const float *wrow = W + (int64_t)p * w_stride + (int64_t)i * w_ld(g.N);
  const __nv_bfloat16 *kp = ks + (int64_t)p * g.N * D + dp * CPT;
  const __nv_bfloat16 *qp = qs + (int64_t)p * g.N * D;
  float *tout = Tout + ((int64_t)p * g.Ck + jj) * g.N;
  const int r_first = qo[i];
  float m1[CPT];
#pragma unroll
  for (int d = 0; d < CPT; ++d) m1[d] = 0.f;
  // acc[d] += w * key[dp * CPT + d] for the key at sorted position pos
  auto add_key = [&](int pos, float w, float (&acc)[CPT]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(kp + (int64_t)pos * D);
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162 *>(&w4[h]);
      acc[2 * h] = fmaf(w, __low2float(b2), acc[2 * h]);
      acc[2 * h + 1] = fmaf(w, __high2float(b2), acc[2 * h + 1]);
    }
  };
  for (int b = 0; b < g.nb; ++b) {
    if (b > 0 && live) {
      // the keys of (j, b - 1) join the prefix
      const int e = kbase + pe[b];
      int pos = kbase + pe[b - 1];
      for (; pos + 1 < e; pos += 2) {
        const float w0 = wrow[pos], w1 = wrow[pos + 1];
        add_key(pos, w0, m1);
        add_key(pos + 1, w1, m1);
      }
      if (pos < e) add_key(pos, wrow[pos], m1);
    }
    const int r0 = r_first + qpe[b], r1 = r_first + qpe[b + 1];
    if (r0 >= r1) continue;  // CTA-uniform
    // a cluster the group selected: the sum of its selected runs, once for the group
    int tj = -1;
    const int32_t *so = sel + (((int64_t)p * g.Cq + i) * g.nb + b) * g.K12 * 2;
    if (b > 0 && live)
      for (int t = 0; t < g.k1; ++t)
        if (so[2 * t * g.k2] == j) tj = t;
    float ex[CPT];
#pragma unroll
    for (int d = 0; d < CPT; ++d) ex[d] = 0.f;
    if (tj >= 0) {
      for (int u = 0; u < g.k2; ++u) {
        const int bb = so[2 * (tj * g.k2 + u) + 1];
        if (bb < 0) continue;
        for (int pos = kbase + pe[bb]; pos < kbase + pe[bb + 1]; ++pos) add_key(pos, wrow[pos], ex);
      }
    }
    // every row of the group: qt.(m1 - e), the thread's CPT coordinates read straight from
    // the sorted residuals (the same addresses for the threads of a coordinate slice)
    for (int r = r0; r < r1; ++r) {
      float acc = 0.f;
      if (b > 0) {
        const uint4 u = *reinterpret_cast<const uint4 *>(qp + (int64_t)r * D + dp * CPT);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162 *>(&w4[h]);
          acc = fmaf(__low2float(b2), m1[2 * h] - ex[2 * h], acc);
          acc = fmaf(__high2float(b2), m1[2 * h + 1] - ex[2 * h + 1], acc);
        }
      }
#pragma unroll
      for (int o = DP / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (live && dp == 0) tout[r] = acc;
    }
  }
}

// kb[p][pos] = block of the key at sorted position pos; kg[p][pos / 8] = smallest | largest
// << 16 block of the 8 keys pos & ~7 .. (pos & ~7) + 7 (N is a multiple of 8).
__global__ void __launch_bounds__(256)
key_blocks(Geo g, const int32_t *__restrict__ k_perm, unsigned short *__restrict__ kb,
           int *__restrict__ kg) {
  const int p = blockIdx.y;
  const int pos = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = pos < g.N ? k_perm[(int64_t)p * g.N + pos] / g.S : 0;
  int lo = b, hi = b;
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (pos < g.N) {
    kb[(int64_t)p * g.N + pos] = (unsigned short)b;
    if ((pos & 7) == 0) kg[(int64_t)p * (g.N / 8) + pos / 8] = lo | (hi << 16);
  }
}

// Remainder coefficients per sorted query row r (cluster i, block b):
//   U_j = exp(logZ_ij - logZR) T_jr;  a_j = logZR + s U_j;  p = softmax(a);
//   c0_jr = p_j (1 - s U_j) exp(logZ_ij - logZR),  c1_jr = s p_j exp(logZ_ij - logZR);
// lse_r[p][r] = logsumexp_j a_j (-inf when nothing remains).
__global__ void __launch_bounds__(128)
ret_coeffs(Geo g, float scale, const int32_t *__restrict__ q_perm,
           const int32_t *__restrict__ q_cluster, const float *__restrict__ logZ,
           const float *__restrict__ logZR, const float *__restrict__ Tbuf,
           float *__restrict__ c0, float *__restrict__ c1, float *__restrict__ lse_r) {
  const int p = blockIdx.y;
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= g.N) return;
  const int b = q_perm[(int64_t)p * g.N + r] / g.S;
  const int i = q_cluster[(int64_t)p * g.N + r];
  const float *lz = logZ + ((int64_t)p * g.Cq + i) * g.Ck;
  const float *zr = logZR + (((int64_t)p * g.Cq + i) * g.nb + b) * g.Ck;
  float m = -CUDART_INF_F, l = 0.f;
  for (int pass = 0; pass < 2; ++pass) {
    const float inv = pass ? 1.f / l : 0.f;
    for (int j = 0; j < g.Ck; ++j) {
      const int64_t at = ((int64_t)p * g.Ck + j) * g.N + r;
      const float z = zr[j];
      if (b == 0 || !(z > -CUDART_INF_F)) {
        if (pass) {
          c0[at] = 0.f;
          c1[at] = 0.f;
        }
        continue;
      }
      const float f = expf(lz[j] - z);
      const float U = f * Tbuf[at];
      const float a = z + scale * U;
      if (!pass) {
        if (a > m) {
          l = l * expf(m - a) + 1.f;
          m = a;
        } else {
          l += expf(a - m);
        }
      } else {
        const float pj = expf(a - m) * inv;
        c0[at] = pj * (1.f - scale * U) * f;
        c1[at] = scale * pj * f;
      }
    }
  }
  lse_r[(int64_t)p * g.N + r] = (l > 0.f) ? m + logf(l) : -CUDART_INF_F;
}

// Exact attention over the (cluster, block) runs selected for (query cluster i, query
// block b), merged into the remainder partial of every row of the group (token order):
// part_lse[p][n], part_o[p][n][:] become the joint (log-normaliser, normalised output) of
// the remainder and the runs.  One warp per (problem, i, b) group, no block-wide
// barrier.  The warp lists the runs (lanes over the slots, a shuffle scan of their
// lengths); the runs are the same for every row of the group.  Up to 16 rows at a time
// form the M side of warp-level tensor-core products (mma.sync m16n8k16, bfloat16 in,
// float32 accumulate), over chunks of 32 selected keys staged in the warp's shared memory
// (keys as sorted, contiguous inside a run; values by token, transposed):
//   S = Q_rows . K_chunk^T (scaled),  online softmax per row,  O += P . V_chunk
// with P (bfloat16) taken from S's accumulator fragments as the A operand.
template <int D, int DV> struct RunsCfg {
  static constexpr int WPC = 4;       // warps (groups) per CTA
  static constexpr int QS = D + 8;    // staged row strides (bf16): 4-byte fragment loads of a
  static constexpr int KS = D + 8;    // quad's 8 rows hit distinct banks
  static constexpr int VS = 32 + 8;   // transposed values: [DV][VS]
  static constexpr size_t warp_bytes = ((size_t)16 * QS + 32 * KS + (size_t)DV * VS) * 2;
  static constexpr size_t smem = WPC * warp_bytes;
};

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

template <int D, int DV>
__global__ void __launch_bounds__(RunsCfg<D, DV>::WPC * 32)
ret_runs(Geo g, int P, float scale, const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ ks,
         const __nv_bfloat16 *__restrict__ V, const int32_t *__restrict__ q_perm,
         const int32_t *__restrict__ q_offsets, const int32_t *__restrict__ qpend,
         const int32_t *__restrict__ k_perm, const int32_t *__restrict__ k_offsets,
         const int32_t *__restrict__ pend, const int32_t *__restrict__ sel,
         float *__restrict__ part_o, float *__restrict__ part_lse) {
  using Cf = RunsCfg<D, DV>;
  constexpr int QS = Cf::QS, KS = Cf::KS, VS = Cf::VS, NV = DV / 8;
  extern __shared__ float4 runs_smem[];
  __shared__ int runs[Cf::WPC][64], cum[Cf::WPC][65];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;  // fragment row group and thread in group
  unsigned char *wbase = reinterpret_cast<unsigned char *>(runs_smem) + warp * Cf::warp_bytes;
  __nv_bfloat16 *sQ = reinterpret_cast<__nv_bfloat16 *>(wbase);  // [16][QS]
  __nv_bfloat16 *sK = sQ + 16 * QS;                                // [32][KS]
  __nv_bfloat16 *sV = sK + 32 * KS;                                // [DV][VS] (transposed)
  const int64_t gid = (int64_t)blockIdx.x * Cf::WPC + warp;  // (p, i, b)
  if (gid >= (int64_t)g.nb * g.Cq * P) return;  // whole warps
  const int b = (int)(gid % g.nb), i = (int)((gid / g.nb) % g.Cq), p = (int)(gid / ((int64_t)g.nb * g.Cq));
  if (b == 0) return;
  const int32_t *qo = q_offsets + (int64_t)p * (g.Cq + 1);
  const int32_t *qpe = qpend + ((int64_t)p * g.Cq + i) * (g.nb + 1);
  const int r0 = qo[i] + qpe[b], r1 = qo[i] + qpe[b + 1];
  if (r0 >= r1) return;
  // the selected runs: slots lane and lane + 32
  const int32_t *so = sel + (((int64_t)p * g.Cq + i) * g.nb + b) * g.K12 * 2;
  int start[2], len[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int t = lane + 32 * h;
    start[h] = 0;
    len[h] = 0;
    if (t < g.K12) {
      const int j = so[2 * t], bb = so[2 * t + 1];
      if (j >= 0) {
        const int32_t *pe = pend + ((int64_t)p * g.Ck + j) * (g.nb + 1);
        start[h] = k_offsets[(int64_t)p * (g.Ck + 1) + j] + pe[bb];
        len[h] = pe[bb + 1] - pe[bb];
      }
    }
  }
  // exclusive scan over the 64 slots (lane-major halves: slots 0..31, then 32..63)
  int inc0 = len[0], inc1 = len[1];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y0 = __shfl_up_sync(0xffffffffu, inc0, o), y1 = __shfl_up_sync(0xffffffffu, inc1, o);
    if (lane >= o) {
      inc0 += y0;
      inc1 += y1;
    }
  }
  const int tot0 = __shfl_sync(0xffffffffu, inc0, 31);
  runs[warp][lane] = start[0];
  runs[warp][lane + 32] = start[1];
  cum[warp][lane] = inc0 - len[0];
  cum[warp][lane + 32] = tot0 + inc1 - len[1];
  if (lane == 31) cum[warp][64] = tot0 + inc1;
  __syncwarp();
  const int total = cum[warp][64];
  if (total == 0) return;
  const int32_t *kperm = k_perm + (int64_t)p * g.N;
  for (int rb = r0; rb < r1; rb += 16) {
    const int nr = min(16, r1 - rb);
    // the tile's query rows (rows past the group repeat its first row)
    __syncwarp();
    for (int x = lane; x < 16 * (D / 8); x += 32) {
      const int rr = x / (D / 8), c = x % (D / 8);
      const int n = q_perm[(int64_t)p * g.N + rb + (rr < nr ? rr : 0)];
      const uint4 v = reinterpret_cast<const uint4 *>(Q + ((int64_t)p * g.N + n) * D)[c];
      uint32_t *dst = reinterpret_cast<uint32_t *>(sQ + rr * QS + 8 * c);
      dst[0] = v.x;
      dst[1] = v.y;
      dst[2] = v.z;
      dst[3] = v.w;
    }
    // rows gq and gq + 8 of the tile: running maximum and sum, output fragments
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
    float o[NV][4];
#pragma unroll
    for (int nt = 0; nt < NV; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    int run = 0;  // run of this lane's key (the lane's keys only move forward)
    for (int c0 = 0; c0 < total; c0 += 32) {
      const int gi = c0 + lane;
      __syncwarp();  // the previous chunk is consumed (and the query tile is written)
      // lane k stages key k of the chunk (zero past the selected keys)
      {
        uint4 kv[D / 8], vv[DV / 8];
        if (gi < total) {
          while (cum[warp][run + 1] <= gi) ++run;
          const int pos = runs[warp][run] + gi - cum[warp][run];  // sorted key position
          const int tok = kperm[pos];
          const uint4 *kr = reinterpret_cast<const uint4 *>(ks + ((int64_t)p * g.N + pos) * D);
          const uint4 *vr = reinterpret_cast<const uint4 *>(V + ((int64_t)p * g.N + tok) * DV);
#pragma unroll
          for (int u = 0; u < D / 8; ++u) kv[u] = kr[u];
#pragma unroll
          for (int u = 0; u < DV / 8; ++u) vv[u] = vr[u];
        } else {
#pragma unroll
          for (int u = 0; u < D / 8; ++u) kv[u] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int u = 0; u < DV / 8; ++u) vv[u] = make_uint4(0u, 0u, 0u, 0u);
        }
        uint32_t *kd = reinterpret_cast<uint32_t *>(sK + lane * KS);
#pragma unroll
        for (int u = 0; u < D / 8; ++u) {
          kd[4 * u] = kv[u].x;
          kd[4 * u + 1] = kv[u].y;
          kd[4 * u + 2] = kv[u].z;
          kd[4 * u + 3] = kv[u].w;
        }
#pragma unroll
        for (int u = 0; u < DV / 8; ++u) {
          const __nv_bfloat16 *h = reinterpret_cast<const __nv_bfloat16 *>(&vv[u]);
#pragma unroll
          for (int e = 0; e < 8; ++e) sV[(8 * u + e) * VS + lane] = h[e];
        }
      }
      __syncwarp();
      // S = Q . K^T: 16 rows x 32 keys (four n-tiles of 8)
      float sacc[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        a[0] = *reinterpret_cast<const uint32_t *>(sQ + gq * QS + kk * 16 + 2 * tq);
        a[1] = *reinterpret_cast<const uint32_t *>(sQ + (gq + 8) * QS + kk * 16 + 2 * tq);
        a[2] = *reinterpret_cast<const uint32_t *>(sQ + gq * QS + kk * 16 + 8 + 2 * tq);
        a[3] = *reinterpret_cast<const uint32_t *>(sQ + (gq + 8) * QS + kk * 16 + 8 + 2 * tq);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const __nv_bfloat16 *kr = sK + (nt * 8 + gq) * KS + kk * 16 + 2 * tq;
          mma_bf16_16816(sacc[nt], a, *reinterpret_cast<const uint32_t *>(kr),
                         *reinterpret_cast<const uint32_t *>(kr + 8));
        }
      }
      // online softmax of rows gq (elements 0, 1) and gq + 8 (elements 2, 3); key of
      // element e of n-tile nt: nt * 8 + 2 * tq + (e & 1)
      float mx0 = m0, mx1 = m1;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool in = c0 + nt * 8 + 2 * tq + (e & 1) < total;
          sacc[nt][e] = in ? sacc[nt][e] * scale : -CUDART_INF_F;
          if (e < 2) mx0 = fmaxf(mx0, sacc[nt][e]);
          else mx1 = fmaxf(mx1, sacc[nt][e]);
        }
#pragma unroll
      for (int o2 = 1; o2 < 4; o2 <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
      }
      const float cr0 = expf(m0 - mx0), cr1 = expf(m1 - mx1);  // (m = -inf: 0)
      float s0 = 0.f, s1 = 0.f;
      uint32_t pa[2][4];  // P as the A operand of two k-steps of 16 keys
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const float p0 = expf(sacc[nt][0] - mx0), p1 = expf(sacc[nt][1] - mx0);
        const float p2 = expf(sacc[nt][2] - mx1), p3 = expf(sacc[nt][3] - mx1);
        s0 += p0 + p1;
        s1 += p2 + p3;
        pa[nt >> 1][(nt & 1) * 2] = pack_bf16(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);
      }
#pragma unroll
      for (int o2 = 1; o2 < 4; o2 <<= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, o2);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o2);
      }
      l0 = l0 * cr0 + s0;
      l1 = l1 * cr1 + s1;
      m0 = mx0;
      m1 = mx1;
#pragma unroll
      for (int nt = 0; nt < NV; ++nt) {
        o[nt][0] *= cr0;
        o[nt][1] *= cr0;
        o[nt][2] *= cr1;
        o[nt][3] *= cr1;
      }
      // O += P . V: two k-steps of 16 keys, NV n-tiles of 8 output columns
#pragma unroll
      for (int ks2 = 0; ks2 < 2; ++ks2) {
#pragma unroll
        for (int nt = 0; nt < NV; ++nt) {
          const __nv_bfloat16 *vr = sV + (nt * 8 + gq) * VS + ks2 * 16 + 2 * tq;
          mma_bf16_16816(o[nt], pa[ks2], *reinterpret_cast<const uint32_t *>(vr),
                         *reinterpret_cast<const uint32_t *>(vr + 8));
        }
      }
    }
    // joint softmax with the remainder partial of each row: this thread holds columns
    // nt * 8 + 2 tq (+1) of rows gq and gq + 8
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rr = gq + 8 * h;
      if (rr >= nr) continue;
      const float m = h ? m1 : m0, l = h ? l1 : l0;
      const int n = q_perm[(int64_t)p * g.N + rb + rr];
      const int64_t at = (int64_t)p * g.N + n;
      const float L = part_lse[at];
      float *po = part_o + at * DV;
      const bool has = L > -CUDART_INF_F;
      const float mn = has ? fmaxf(m, L) : m;
      const float ca = expf(m - mn), cb = has ? expf(L - mn) : 0.f;
      const float lt = l * ca + cb;
#pragma unroll
      for (int nt = 0; nt < NV; ++nt) {
        float2 *dst = reinterpret_cast<float2 *>(po + nt * 8 + 2 * tq);
        const float2 prev = has ? *dst : make_float2(0.f, 0.f);
        *dst = make_float2((o[nt][2 * h] * ca + cb * prev.x) / lt, (o[nt][2 * h + 1] * ca + cb * prev.y) / lt);
      }
      if (tq == 0) part_lse[at] = mn + logf(lt);
    }
  }
}

// Workspace layout.
struct Ws {
  KmeansOut q, k;
  char *km_scratch;
  SortedSide ks;
  void *vs;
  int32_t *v_cluster;
  float *W, *logZ;
  int32_t *cnt, *pend, *sel;
  float *logZb, *logZR, *T, *c0, *c1, *lse_r, *part_o, *pref;
  SortedSide qs;              // tensor-core path: sorted residuals
  int32_t *qcnt, *qpend;      // rows of query cluster i in / before each block
  unsigned short *kb;         // block of every sorted key
  int *kg;                    // block range of every 8 sorted keys
  float *part_lse;            // remainder + runs log-normaliser per token
};

struct Bump2 {
  char *base;
  size_t off = 0;
  explicit Bump2(void *b) : base(static_cast<char *>(b)) {}
  template <typename X>
  X *take(size_t count) {
    const size_t o = off;
    off = align_up(off + count * sizeof(X));
    return base ? reinterpret_cast<X *>(base + o) : nullptr;
  }
};

static SegTable whole(int N, int C) {
  SegTable t;
  memset(&t, 0, sizeof(t));
  t.nseg = 1;
  t.row_stride = N;
  t.cen_stride = C;
  t.off_stride = C + 1;
  t.max_rows = N;
  t.max_C = C;
  t.nrow[0] = N;
  t.C[0] = C;
  return t;
}

static MuseTables tables(int N, int Cq, int Ck) {
  MuseTables mt;
  memset(&mt, 0, sizeof(mt));
  mt.q = whole(N, Cq);
  mt.k = whole(N, Ck);
  mt.in.ninst = 1;
  mt.in.w_stride = Cq * w_ld(N);
  mt.in.z_stride = Cq * Ck;
  mt.in.c_stride = Ck * w_ld(N);
  mt.in.out_stride = N;
  return mt;
}

static void plan(Bump2 &bp, const muse_dims &d, const Geo &g, Ws &w) {
  const int P = d.B * d.H;
  const size_t es = d.dtype == MUSE_F32 ? 4 : 2;
  MuseTables mt = tables(d.N, g.Cq, g.Ck);
  auto side = [&](const SegTable &t, KmeansOut &o) {
    o.labels = bp.take<int32_t>((size_t)P * t.row_stride);
    o.centroids = bp.take<float>((size_t)P * t.cen_stride * d.D);
    o.perm = bp.take<int32_t>((size_t)P * t.row_stride);
    o.offsets = bp.take<int32_t>((size_t)P * t.off_stride);
  };
  side(mt.q, w.q);
  side(mt.k, w.k);
  w.km_scratch = bp.take<char>(kmeans_pair_ws_bytes(&mt.q, &mt.k, P, d.D));
  w.ks.rows = bp.take<char>((size_t)P * d.N * d.D * es);
  w.ks.cluster = bp.take<int32_t>((size_t)P * d.N);
  w.vs = bp.take<char>((size_t)P * d.N * d.Dv * es);
  w.v_cluster = bp.take<int32_t>((size_t)P * d.N);
  w.W = bp.take<float>((size_t)P * mt.in.w_stride);
  w.logZ = bp.take<float>((size_t)P * g.Cq * g.Ck);
  w.cnt = bp.take<int32_t>((size_t)P * g.Ck * g.nb);
  w.pend = bp.take<int32_t>((size_t)P * g.Ck * (g.nb + 1));
  w.sel = bp.take<int32_t>((size_t)P * g.Cq * g.nb * g.K12 * 2);
  w.logZb = bp.take<float>((size_t)P * g.Cq * g.Ck * g.nb);
  w.pref = bp.take<float>((size_t)P * g.Cq * (g.nb + 1) * g.Ck);
  w.logZR = bp.take<float>((size_t)P * g.Cq * g.nb * g.Ck);
  w.T = bp.take<float>((size_t)P * g.Ck * d.N);
  w.c0 = bp.take<float>((size_t)P * g.Ck * d.N);
  w.c1 = bp.take<float>((size_t)P * g.Ck * d.N);
  w.lse_r = bp.take<float>((size_t)P * d.N);
  w.part_o = bp.take<float>((size_t)P * d.N * d.Dv);
  w.qs.rows = bp.take<char>((size_t)P * d.N * d.D * es);
  w.qs.cluster = bp.take<int32_t>((size_t)P * d.N);
  w.qcnt = bp.take<int32_t>((size_t)P * g.Cq * g.nb);
  w.qpend = bp.take<int32_t>((size_t)P * g.Cq * (g.nb + 1));
  w.part_lse = bp.take<float>((size_t)P * d.N);
  w.kb = bp.take<unsigned short>((size_t)P * d.N);
  w.kg = bp.take<int>((size_t)P * (d.N / 8));
}

static bool valid_geo(const muse_dims &d, int block, int Cq, int Ck, int k1, int k2, Geo &g) {
  if (block <= 0 || block % 64 || d.N % block) return false;
  if (Cq < 1 || Ck < 1 || Cq > d.N || Ck > d.N || Cq > kMaxClusters || Ck > kMaxClusters) return false;
  const int nb = d.N / block;
  if (nb > 1024) return false;
  if (k1 < 0 || k2 < 0 || k1 > Ck || k2 > nb || k1 * k2 > 64) return false;
  if (k2 == 0) k1 = 0;  // a cluster retrieved with no block excludes nothing
  g.N = d.N;
  g.S = block;
  g.nb = nb;
  g.Cq = Cq;
  g.Ck = Ck;
  g.k1 = k1;
  g.k2 = k2;
  g.K12 = std::max(1, k1 * k2);
  return true;
}

// The tensor-core path (bfloat16): see the header of this file.
template <int D, int DV>
static cudaError_t run_tc(const void *Q, const void *K, const void *V, const muse_dims &d,
                          const Geo &g, int iters, Ws &w, void *O, int *status, cudaStream_t st) {
  const int P = d.B * d.H;
  MuseTables mt = tables(d.N, g.Cq, g.Ck);
  cudaError_t e;
  if ((e = run_kmeans_pair(Q, mt.q, w.q, K, mt.k, w.k, d.dtype, D, d.N, P, iters, w.km_scratch,
                           status, st)) != cudaSuccess)
    return e;
  if ((e = run_sort_side(Q, d.dtype, D, d.N, mt.q, P, w.q.perm, w.q.offsets, w.q.centroids, w.qs,
                         st)) != cudaSuccess)
    return e;
  if ((e = run_sort_side(K, d.dtype, D, d.N, mt.k, P, w.k.perm, w.k.offsets, nullptr, w.ks, st)) !=
      cudaSuccess)
    return e;
  if ((e = run_sort_side_t(V, d.dtype, DV, d.N, mt.k, P, w.k.perm, w.vs, st)) != cudaSuccess) return e;
  StageBufs sb;
  memset(&sb, 0, sizeof(sb));
  sb.W = w.W;
  sb.logZ = w.logZ;
  if ((e = run_summaries(mt, d.dtype, D, DV, P, d.scale, w.q.centroids, w.ks, nullptr, w.k.offsets,
                         sb, st)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(w.cnt, 0, (size_t)P * g.Ck * g.nb * sizeof(int32_t), st)) != cudaSuccess ||
      (e = cudaMemsetAsync(w.qcnt, 0, (size_t)P * g.Cq * g.nb * sizeof(int32_t), st)) != cudaSuccess)
    return e;
  block_counts<<<dim3((d.N + 255) / 256, P), 256, 0, st>>>(g, g.Ck, w.k.labels, w.cnt);
  block_prefix<<<(P * g.Ck + 127) / 128, 128, 0, st>>>(g, P, g.Ck, w.cnt, w.pend);
  block_counts<<<dim3((d.N + 255) / 256, P), 256, 0, st>>>(g, g.Cq, w.q.labels, w.qcnt);
  block_prefix<<<(P * g.Cq + 127) / 128, 128, 0, st>>>(g, P, g.Cq, w.qcnt, w.qpend);
  const int64_t nw = (int64_t)P * g.Cq * g.Ck;
  block_lse<<<(unsigned)((nw * g.nb + 255) / 256), 256, 0, st>>>(g, P, w.W, mt.in.w_stride, w.logZ,
                                                                  w.k.offsets, w.pend, w.logZb);
  block_prefix_lse<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(g, P, w.logZb, w.pref);
  const int64_t ns = (int64_t)P * g.Cq * g.nb;
  launch_select(g, P, ns, w.logZb, w.pref, w.sel, w.logZR, st);
  constexpr int JPC = 256 / (D / 8);  // (ret_T: 8 coordinates per thread)
  ret_T<D><<<dim3((g.Ck + JPC - 1) / JPC, g.Cq, P), 256, 0, st>>>(
      g, (const __nv_bfloat16 *)w.qs.rows, w.q.offsets, w.qpend, (const __nv_bfloat16 *)w.ks.rows,
      w.k.offsets, w.pend, w.W, mt.in.w_stride, w.sel, w.T);
  ret_coeffs<<<dim3((d.N + 127) / 128, P), 128, 0, st>>>(g, d.scale, w.q.perm, w.qs.cluster, w.logZ,
                                                        w.logZR, w.T, w.c0, w.c1, w.lse_r);
  key_blocks<<<dim3((d.N + 255) / 256, P), 256, 0, st>>>(g, w.k.perm, w.kb, w.kg);
  count_launches(10);
  sb.c0 = w.c0;
  sb.c1 = w.c1;
  sb.lse = w.lse_r;
  if ((e = profile_mark(true, st)) != cudaSuccess) return e;
  if ((e = run_refine_tc_ret(mt, D, DV, d.N, P, w.qs, w.q.perm, w.ks, w.k.offsets, w.vs, sb,
                             w.part_o, w.part_lse, w.kb, w.kg, w.pend, w.sel, g.S, g.k1, g.k2,
                             status, st)) != cudaSuccess)
    return e;
  if ((e = profile_mark(false, st)) != cudaSuccess) return e;
  {
    using Rc = RunsCfg<D, DV>;
    if ((e = cudaFuncSetAttribute(ret_runs<D, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)Rc::smem)) != cudaSuccess)
      return e;
    ret_runs<D, DV><<<(unsigned)(((int64_t)g.nb * g.Cq * P + Rc::WPC - 1) / Rc::WPC), Rc::WPC * 32,
                      Rc::smem, st>>>(
        g, P, d.scale, (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)w.ks.rows,
        (const __nv_bfloat16 *)V, w.q.perm, w.q.offsets, w.qpend, w.k.perm, w.k.offsets, w.pend,
        w.sel, w.part_o, w.part_lse);
  }
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return run_diag_merge(Q, K, V, d.dtype, D, DV, d.N, P, g.S, -1, d.scale, w.part_o, w.part_lse, O,
                        st);
}

template <typename T, int D, int DV>
static cudaError_t run_t(const void *Q, const void *K, const void *V, const muse_dims &d,
                         const Geo &g, int iters, Ws &w, void *O, int *status, cudaStream_t st) {
  const int P = d.B * d.H;
  MuseTables mt = tables(d.N, g.Cq, g.Ck);
  cudaError_t e;
  if ((e = run_kmeans_pair(Q, mt.q, w.q, K, mt.k, w.k, d.dtype, D, d.N, P, iters, w.km_scratch,
                           status, st)) != cudaSuccess)
    return e;
  if ((e = run_sort_side(K, d.dtype, D, d.N, mt.k, P, w.k.perm, w.k.offsets, nullptr, w.ks, st)) !=
      cudaSuccess)
    return e;
  SortedSide vsd{w.vs, w.v_cluster};
  if ((e = run_sort_side(V, d.dtype, DV, d.N, mt.k, P, w.k.perm, w.k.offsets, nullptr, vsd, st)) !=
      cudaSuccess)
    return e;
  StageBufs sb;
  memset(&sb, 0, sizeof(sb));
  sb.W = w.W;
  sb.logZ = w.logZ;
  if ((e = run_summaries(mt, d.dtype, D, DV, P, d.scale, w.q.centroids, w.ks, nullptr, w.k.offsets,
                         sb, st)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(w.cnt, 0, (size_t)P * g.Ck * g.nb * sizeof(int32_t), st)) != cudaSuccess)
    return e;
  block_counts<<<dim3((d.N + 255) / 256, P), 256, 0, st>>>(g, g.Ck, w.k.labels, w.cnt);
  block_prefix<<<(P * g.Ck + 127) / 128, 128, 0, st>>>(g, P, g.Ck, w.cnt, w.pend);
  const int64_t nw = (int64_t)P * g.Cq * g.Ck;
  block_lse<<<(unsigned)((nw * g.nb + 255) / 256), 256, 0, st>>>(g, P, w.W, mt.in.w_stride, w.logZ,
                                                                  w.k.offsets, w.pend, w.logZb);
  block_prefix_lse<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(g, P, w.logZb, w.pref);
  const int64_t ns = (int64_t)P * g.Cq * g.nb;
  launch_select(g, P, ns, w.logZb, w.pref, w.sel, w.logZR, st);
  dim3 qg(d.N / 64, P);
  remainder_pass<T, D, DV, 0><<<qg, 256, 0, st>>>(
      g, (const T *)Q, w.q.centroids, w.q.labels, (const T *)w.ks.rows, (const T *)w.vs, w.k.perm,
      w.k.offsets, w.pend, w.W, mt.in.w_stride, w.sel, w.T, nullptr, nullptr, nullptr);
  remainder_coeffs<<<dim3((d.N + 127) / 128, P), 128, 0, st>>>(g, P, d.scale, w.q.labels, w.logZ,
                                                                w.logZR, w.T, w.c0, w.c1, w.lse_r);
  remainder_pass<T, D, DV, 1><<<qg, 256, 0, st>>>(
      g, (const T *)Q, w.q.centroids, w.q.labels, (const T *)w.ks.rows, (const T *)w.vs, w.k.perm,
      w.k.offsets, w.pend, w.W, mt.in.w_stride, w.sel, nullptr, w.c0, w.c1, w.part_o);
  exact_merge<T, D, DV><<<qg, 256, 0, st>>>(g, d.scale, (const T *)Q, (const T *)K, (const T *)V,
                                            w.q.labels, (const T *)w.ks.rows, (const T *)w.vs,
                                            w.k.offsets, w.pend, w.sel, w.part_o, w.lse_r, (T *)O);
  count_launches(9);
  return cudaGetLastError();
}

}  // namespace ret

size_t muse_retrieval_ws(const muse_dims &d, int block, int Cq, int Ck, int k1, int k2) {
  ret::Geo g;
  if (!ret::valid_geo(d, block, Cq, Ck, k1, k2, g)) return 0;
  ret::Bump2 bp(nullptr);
  ret::Ws w;
  ret::plan(bp, d, g, w);
  return bp.off;
}

int *device_status_word();

}  // namespace muse

using namespace muse;

extern "C" muse_status muse_retrieve_exact(const void *Q, const void *K, const void *V, muse_dims d,
                                           int block, int Cq, int Ck, int iters, int k1, int k2,
                                           int32_t *q_labels_out, int32_t *k_labels_out,
                                           int32_t *selected_pairs, void *O, void *ws,
                                           size_t ws_bytes, muse_stream_t st) {
  if (d.dtype != MUSE_F32 && d.dtype != MUSE_BF16) return MUSE_ERR_DTYPE;
  if (d.B <= 0 || d.H <= 0 || d.N <= 0 || (d.D != 64 && d.D != 128) || (d.Dv != 64 && d.Dv != 128))
    return MUSE_ERR_SHAPE;
  if ((int64_t)d.B * d.H > 65535 || (int64_t)d.N * 128 > ((int64_t)1 << 31)) return MUSE_ERR_SHAPE;
  if (!isfinite(d.scale)) return MUSE_ERR_INVALID_ARG;
  for (const void *p : {Q, K, V, (const void *)O})
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u)) return MUSE_ERR_INVALID_ARG;
  for (const void *p : {(const void *)q_labels_out, (const void *)k_labels_out,
                        (const void *)selected_pairs})
    if (p && (reinterpret_cast<uintptr_t>(p) & 15u)) return MUSE_ERR_INVALID_ARG;
  if (block <= 0 || block % 64 || d.N % block) return MUSE_ERR_SHAPE;
  if (iters < 1 || iters > 1000) return MUSE_ERR_INVALID_ARG;
  ret::Geo g;
  if (!ret::valid_geo(d, block, Cq, Ck, k1, k2, g)) return MUSE_ERR_INVALID_ARG;
  const size_t need = muse_retrieval_ws(d, block, Cq, Ck, k1, k2);
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15u)) return MUSE_ERR_WORKSPACE;
  ret::Bump2 bp(ws);
  ret::Ws w;
  ret::plan(bp, d, g, w);
  if (q_labels_out) w.q.labels = q_labels_out;
  if (k_labels_out) w.k.labels = k_labels_out;
  if (selected_pairs) w.sel = selected_pairs;
  cudaError_t e;
  int *status = device_status_word();
  cudaStream_t cs = (cudaStream_t)st;
  if (d.dtype == MUSE_F32) {
    if (d.D == 64 && d.Dv == 64) e = ret::run_t<float, 64, 64>(Q, K, V, d, g, iters, w, O, status, cs);
    else if (d.D == 64) e = ret::run_t<float, 64, 128>(Q, K, V, d, g, iters, w, O, status, cs);
    else if (d.Dv == 64) e = ret::run_t<float, 128, 64>(Q, K, V, d, g, iters, w, O, status, cs);
    else e = ret::run_t<float, 128, 128>(Q, K, V, d, g, iters, w, O, status, cs);
  } else {
    if (d.D == 64 && d.Dv == 64) e = ret::run_tc<64, 64>(Q, K, V, d, g, iters, w, O, status, cs);
    else if (d.D == 64) e = ret::run_tc<64, 128>(Q, K, V, d, g, iters, w, O, status, cs);
    else if (d.Dv == 64) e = ret::run_tc<128, 64>(Q, K, V, d, g, iters, w, O, status, cs);
    else e = ret::run_tc<128, 128>(Q, K, V, d, g, iters, w, O, status, cs);
  }
  return e == cudaSuccess ? MUSE_OK : cuda_fail(e);
}
