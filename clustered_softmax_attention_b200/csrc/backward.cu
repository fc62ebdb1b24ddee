// Backward pass of the acausal MuSe forward: gradients of sum(O * dO) with respect to
// Q, K and V, the clusterings held fixed (K-means assignments are discrete) and each
// query centroid the mean of its members (as K-means leaves it).
//
// pith.science review of arXiv 2509.10406, referee report and "What carries the
// argument": the method is trained through, i.e. the approximation itself is
// differentiated.  The chain rule runs through the definitions in reverse:
//   refinement  O_n = sum_j p_nj y_nj,  y_nj = mu_v,ij + s C_ij qt_n,
//               p_n = softmax_j(a_nj),  a_nj = logZ_ij + s qt_n.mu_k,ij
//     dy_nj = p_nj dO_n;  dp_nj = dO_n.y_nj;  da_nj = p_nj (dp_nj - sum_j' p_nj' dp_nj')
//     dqt_n = s sum_j (da_nj mu_k,ij + p_nj C_ij^T dO_n)
//     dlogZ_ij = sum_n da_nj;  dmu_k,ij = s sum_n da_nj qt_n;  dmu_v,ij = sum_n p_nj dO_n;
//     dC_ij = s sum_n p_nj dO_n qt_n^T                      (n over the rows of cluster i)
//   summaries   w_ik = exp(s qbar_i.k - logZ_ij),  C_ij = sum w v k^T - mu_v mu_k^T
//     dmu_v' = dmu_v - dC mu_k;  dmu_k' = dmu_k - dC^T mu_v
//     dw_ik = v_k.(dC k_k) + dmu_k'.k_k + dmu_v'.v_k
//     dl_ik = w_ik (dw_ik - sum_{k' in S_j} w_ik' dw_ik') + w_ik dlogZ_ij
//     dv_k = sum_i w_ik (dC k_k + dmu_v');  dk_k = sum_i [w_ik (dC^T v_k + dmu_k') + s dl_ik qbar_i]
//     dqbar_i = s sum_k dl_ik k_k
//   centroids   dq_n = dqt_n + (dqbar_i - sum_{n' in i} dqt_n') / |i|
//
// Float32 on the CUDA cores, every sum in a fixed order (no floating-point atomics).
// The forward summaries, C_ij included, are recomputed and materialised in the
// workspace (Cq Ck Dv D floats per problem, twice with dC).  Kernels: means (qbar),
// the forward summaries, rows (per query cluster: softmax backward, dqt and the cluster
// sums), keys (two passes per key cluster: the tilted-moment backward into dk, dv and the
// logit gradients), queries (dqbar and the centroid correction), unsort.
#include <string.h>

#include "internal.h"

namespace muse {
namespace bwd {

struct Geo {
  int N, Cq, Ck;
  float s;
};

// qbar_i = mean of the members of query cluster i (rows in sorted order).
template <typename T, int D>
__global__ void __launch_bounds__(128)
means(Geo g, const T *__restrict__ Q, const int32_t *__restrict__ q_perm,
      const int32_t *__restrict__ q_offsets, float *__restrict__ qbar) {
  const int p = blockIdx.y, i = blockIdx.x;
  const int32_t *off = q_offsets + (int64_t)p * (g.Cq + 1);
  const int r0 = off[i], r1 = off[i + 1];
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int r = r0; r < r1; ++r) acc += ld_elem(Q + ((int64_t)p * g.N + q_perm[(int64_t)p * g.N + r]) * D + d);
    qbar[((int64_t)p * g.Cq + i) * D + d] = r1 > r0 ? acc / (float)(r1 - r0) : 0.f;
  }
}

__device__ __forceinline__ int cluster_of(const int32_t *off, int C, int r) {
  int lo = 0, hi = C - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= r) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Per query cluster i (one CTA of eight warps): the rows of the cluster in passes of
// RP = 32 (four per warp), and for every key cluster j with C_ij, mu_k,ij, mu_v,ij staged in
// shared memory once per pass:
//   pass A: a_nj = logZ_ij + s qt_n.mu_k,ij and dp_nj = dO_n.mu_v,ij + s qt_n.(C_ij^T dO_n)
//           (online softmax statistics; a and dp kept in PA, DA [P][N][Ck], sorted rows);
//   pass B: p_nj, da_nj = p_nj (dp_nj - sum_j' p_nj' dp_nj'), dqt_n += s (da_nj mu_k,ij +
//           p_nj C_ij^T dO_n), and the cluster sums dlogZ_ij, dmu_k,ij, dmu_v,ij and
//           dC_ij = s sum_n p_nj dO_n qt_n^T over the pass's rows (added pass by pass in
//           row order: deterministic).
template <typename T, int D, int DV>
__global__ void __launch_bounds__(256)
rows(Geo g, const T *__restrict__ Q, const T *__restrict__ dO, const int32_t *__restrict__ q_perm,
     const int32_t *__restrict__ q_offsets, const float *__restrict__ qbar,
     const float *__restrict__ logZ, const float *__restrict__ mu_k, const float *__restrict__ mu_v,
     const float *__restrict__ cov, float *__restrict__ PA, float *__restrict__ DA,
     float *__restrict__ dQt, float *__restrict__ dlogZ, float *__restrict__ dmuk,
     float *__restrict__ dmuv, float *__restrict__ dC) {
  constexpr int PD = D / 32, PV = DV / 32, RW = 4, RP = 8 * RW, E = DV * D / 256;
  extern __shared__ float sm_raw[];
  float *Cs = sm_raw;                 // [DV][D]
  float *qt_sh = Cs + DV * D;         // [RP][D]
  float *do_sh = qt_sh + RP * D;      // [RP][DV]
  float *mk = do_sh + RP * DV;        // [D]
  float *mv = mk + D;                 // [DV]
  float *pj_sh = mv + DV;             // [RP]
  float *da_sh = pj_sh + RP;          // [RP]
  const int p = blockIdx.y, i = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t *off = q_offsets + (int64_t)p * (g.Cq + 1);
  const int R0 = off[i], R1 = off[i + 1];
  const int64_t ij0 = ((int64_t)p * g.Cq + i) * g.Ck;
  // C_ij, mu_k, mu_v of cluster j into shared memory (after a barrier of the caller)
  auto stage = [&](int j) {
    const float4 *src = reinterpret_cast<const float4 *>(cov + (ij0 + j) * DV * D);
    for (int e = threadIdx.x; e < DV * D / 4; e += 256) reinterpret_cast<float4 *>(Cs)[e] = src[e];
    if (threadIdx.x < D) mk[threadIdx.x] = mu_k[(ij0 + j) * D + threadIdx.x];
    if (threadIdx.x >= 128 && threadIdx.x - 128 < DV) mv[threadIdx.x - 128] = mu_v[(ij0 + j) * DV + threadIdx.x - 128];
  };
  for (int pr0 = R0; pr0 < R1; pr0 += RP) {
    const int nr = min(RP, R1 - pr0);
    __syncthreads();
    // the pass's residuals and output gradients, float32
    for (int e = threadIdx.x; e < RP * D; e += 256) {
      const int rr = e / D, d = e % D;
      float v = 0.f;
      if (rr < nr) {
        const int n = q_perm[(int64_t)p * g.N + pr0 + rr];
        v = ld_elem(Q + ((int64_t)p * g.N + n) * D + d) - qbar[((int64_t)p * g.Cq + i) * D + d];
      }
      qt_sh[e] = v;
    }
    for (int e = threadIdx.x; e < RP * DV; e += 256) {
      const int rr = e / DV, v = e % DV;
      do_sh[e] = rr < nr ? ld_elem(dO + ((int64_t)p * g.N + q_perm[(int64_t)p * g.N + pr0 + rr]) * DV + v) : 0.f;
    }
    // this warp's rows: pr0 + warp + 8 q, q < RW
    float m[RW], l[RW], sdp[RW];
#pragma unroll
    for (int q = 0; q < RW; ++q) {
      m[q] = -CUDART_INF_F;
      l[q] = 0.f;
      sdp[q] = 0.f;
    }
    // u_q = C^T dO of row q (lane owns coordinates lane + 32 t)
    auto ctdo = [&](float (&u)[RW][PD]) {
#pragma unroll
      for (int q = 0; q < RW; ++q)
#pragma unroll
        for (int t = 0; t < PD; ++t) u[q][t] = 0.f;
      for (int v = 0; v < DV; ++v) {
        float c[PD];
#pragma unroll
        for (int t = 0; t < PD; ++t) c[t] = Cs[v * D + lane + 32 * t];
#pragma unroll
        for (int q = 0; q < RW; ++q) {
          const float dv = do_sh[(warp + 8 * q) * DV + v];
#pragma unroll
          for (int t = 0; t < PD; ++t) u[q][t] = fmaf(c[t], dv, u[q][t]);
        }
      }
    };
    // ---- pass A
    for (int j = 0; j < g.Ck; ++j) {
      const float lz = logZ[ij0 + j];
      if (!(lz > -CUDART_INF_F)) continue;  // uniform
      __syncthreads();
      stage(j);
      __syncthreads();
      float u[RW][PD];
      ctdo(u);
#pragma unroll
      for (int q = 0; q < RW; ++q) {
        const int rr = warp + 8 * q;
        float x = 0.f, y = 0.f, z = 0.f;
#pragma unroll
        for (int t = 0; t < PD; ++t) {
          const float qv = qt_sh[rr * D + lane + 32 * t];
          x = fmaf(qv, mk[lane + 32 * t], x);
          y = fmaf(qv, u[q][t], y);
        }
#pragma unroll
        for (int v = 0; v < PV; ++v) z = fmaf(do_sh[rr * DV + lane + 32 * v], mv[lane + 32 * v], z);
        const float a = lz + g.s * warp_sum(x);
        const float dp = fmaf(g.s, warp_sum(y), warp_sum(z));
        const float mn = fmaxf(m[q], a);
        const float c = expf(m[q] - mn), e = expf(a - mn);
        l[q] = l[q] * c + e;
        sdp[q] = sdp[q] * c + e * dp;
        m[q] = mn;
        if (lane == 0 && rr < nr) {
          PA[((int64_t)p * g.N + pr0 + rr) * g.Ck + j] = a;
          DA[((int64_t)p * g.N + pr0 + rr) * g.Ck + j] = dp;
        }
      }
    }
    float lse[RW], mdp[RW], dq[RW][PD];
#pragma unroll
    for (int q = 0; q < RW; ++q) {
      lse[q] = m[q] + logf(l[q]);
      mdp[q] = sdp[q] / l[q];
#pragma unroll
      for (int t = 0; t < PD; ++t) dq[q][t] = 0.f;
    }
    // ---- pass B
    for (int j = 0; j < g.Ck; ++j) {
      const float lz = logZ[ij0 + j];
      const int64_t ij = ij0 + j;
      if (!(lz > -CUDART_INF_F)) {
        // an empty key cluster: no weight, and zero sums (written once, by the first pass)
        if (pr0 == R0) {
          for (int e = threadIdx.x; e < DV * D; e += 256) dC[ij * DV * D + e] = 0.f;
          if (threadIdx.x < D) dmuk[ij * D + threadIdx.x] = 0.f;
          if (threadIdx.x < DV) dmuv[ij * DV + threadIdx.x] = 0.f;
          if (threadIdx.x == 0) dlogZ[ij] = 0.f;
        }
        if (threadIdx.x < nr) {
          PA[((int64_t)p * g.N + pr0 + threadIdx.x) * g.Ck + j] = 0.f;
          DA[((int64_t)p * g.N + pr0 + threadIdx.x) * g.Ck + j] = 0.f;
        }
        continue;
      }
      __syncthreads();
      stage(j);
      __syncthreads();
      float u[RW][PD];
      ctdo(u);
#pragma unroll
      for (int q = 0; q < RW; ++q) {
        const int rr = warp + 8 * q;
        float pj = 0.f, daj = 0.f;
        if (rr < nr) {
          const int64_t at = ((int64_t)p * g.N + pr0 + rr) * g.Ck + j;
          pj = expf(PA[at] - lse[q]);
          daj = pj * (DA[at] - mdp[q]);
        }
#pragma unroll
        for (int t = 0; t < PD; ++t)
          dq[q][t] = fmaf(g.s, fmaf(daj, mk[lane + 32 * t], pj * u[q][t]), dq[q][t]);
        if (lane == 0) {
          pj_sh[rr] = pj;
          da_sh[rr] = daj;
        }
      }
      __syncthreads();
      // the cluster sums of this pass (rows in order), added to the earlier passes'
      float acc[E];
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = 0.f;
      float amk = 0.f, amv = 0.f, alz = 0.f;
      for (int rr = 0; rr < nr; ++rr) {
        const float pjr = pj_sh[rr], dar = da_sh[rr];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int idx = threadIdx.x + 256 * e;
          acc[e] = fmaf(pjr * do_sh[rr * DV + idx / D], qt_sh[rr * D + idx % D], acc[e]);
        }
        if (threadIdx.x < D) amk = fmaf(dar, qt_sh[rr * D + threadIdx.x], amk);
        if (threadIdx.x >= 128 && threadIdx.x - 128 < DV) amv = fmaf(pjr, do_sh[rr * DV + threadIdx.x - 128], amv);
        if (threadIdx.x == 0) alz += dar;
      }
      const bool first = pr0 == R0;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float *dst = dC + ij * DV * D + threadIdx.x + 256 * e;
        *dst = (first ? 0.f : *dst) + g.s * acc[e];
      }
      if (threadIdx.x < D) {
        float *dst = dmuk + ij * D + threadIdx.x;
        *dst = (first ? 0.f : *dst) + g.s * amk;
      }
      if (threadIdx.x >= 128 && threadIdx.x - 128 < DV) {
        float *dst = dmuv + ij * DV + threadIdx.x - 128;
        *dst = (first ? 0.f : *dst) + amv;
      }
      if (threadIdx.x == 0) dlogZ[ij] = (first ? 0.f : dlogZ[ij]) + alz;
    }
#pragma unroll
    for (int q = 0; q < RW; ++q) {
      const int rr = warp + 8 * q;
      if (rr < nr)
#pragma unroll
        for (int t = 0; t < PD; ++t) dQt[((int64_t)p * g.N + pr0 + rr) * D + lane + 32 * t] = dq[q][t];
    }
  }
  if (R0 == R1) {
    // an empty query cluster: zero cluster sums
    for (int j = 0; j < g.Ck; ++j) {
      const int64_t ij = ij0 + j;
      for (int e = threadIdx.x; e < DV * D; e += 256) dC[ij * DV * D + e] = 0.f;
      if (threadIdx.x < D) dmuk[ij * D + threadIdx.x] = 0.f;
      if (threadIdx.x < DV) dmuv[ij * DV + threadIdx.x] = 0.f;
      if (threadIdx.x == 0) dlogZ[ij] = 0.f;
    }
  }
}

// Per (key cluster j, problem): for every query centroid i, the corrected mean gradients
// dmu_k' = dmu_k - dC^T mu_v, dmu_v' = dmu_v - dC mu_k, then per key of j (one warp per key
// at a time)  dw_ik = v.(dC k) + dmu_k'.k + dmu_v'.v  and R_ij = sum_k w_ik dw_ik
// (R [P][Cq][Ck]).  PASS 1 writes R; PASS 2 recomputes dw and forms
// dl_ik = w_ik (dw_ik - R_ij) + w_ik dlogZ_ij (DL [P][Cq][N]) and accumulates dk, dv of the
// keys over i (dKs, dVs [P][N][*], sorted keys).
template <typename T, int D, int DV, int PASS>
__global__ void __launch_bounds__(256)
keys(Geo g, const T *__restrict__ ks, const T *__restrict__ vs, const int32_t *__restrict__ k_offsets,
     const float *__restrict__ W, int w_stride, const float *__restrict__ qbar,
     const float *__restrict__ mu_k, const float *__restrict__ mu_v, const float *__restrict__ dlogZ,
     const float *__restrict__ dmuk, const float *__restrict__ dmuv, const float *__restrict__ dC,
     float *__restrict__ R, float *__restrict__ DL, float *__restrict__ dKs,
     float *__restrict__ dVs) {
  constexpr int PD = D / 32, PV = DV / 32, KPW = 4;  // keys per warp per chunk
  extern __shared__ float G_raw[];                   // dC_ij [DV][D + 1] (padded rows)
  float(*G)[D + 1] = reinterpret_cast<float(*)[D + 1]>(G_raw);
  __shared__ float mk_t[D], mv_t[DV], qb[D], red[8];
  __shared__ float acc_k[8][KPW][D], acc_v[8][KPW][DV];  // PASS 2: dk, dv of the warp's keys
  const int p = blockIdx.y, j = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t *off = k_offsets + (int64_t)p * (g.Ck + 1);
  const int k0 = off[j], k1 = off[j + 1];
  if (k0 >= k1) return;  // uniform
  const int wl = w_ld(g.N);
  for (int c0 = k0; c0 < k1; c0 += 8 * KPW) {
    // this chunk's keys: warp w takes keys c0 + w + 8 u, u < KPW
    if (PASS == 2) {
      for (int u = 0; u < KPW; ++u) {
        for (int t = lane; t < D; t += 32) acc_k[warp][u][t] = 0.f;
        for (int t = lane; t < DV; t += 32) acc_v[warp][u][t] = 0.f;
      }
    }
    for (int i = 0; i < g.Cq; ++i) {
      const int64_t ij = ((int64_t)p * g.Cq + i) * g.Ck + j;
      __syncthreads();
      for (int e = threadIdx.x; e < DV * D; e += 256) G[e / D][e % D] = dC[ij * DV * D + e];
      if (threadIdx.x < D) qb[threadIdx.x] = qbar[((int64_t)p * g.Cq + i) * D + threadIdx.x];
      __syncthreads();
      // corrected mean gradients (threads over coordinates)
      if (threadIdx.x < D) {
        float a = dmuk[ij * D + threadIdx.x];
        for (int v = 0; v < DV; ++v) a = fmaf(-G[v][threadIdx.x], mu_v[ij * DV + v], a);
        mk_t[threadIdx.x] = a;
      }
      if (threadIdx.x >= 128 && threadIdx.x - 128 < DV) {
        const int v = threadIdx.x - 128;
        float a = dmuv[ij * DV + v];
        for (int d = 0; d < D; ++d) a = fmaf(-G[v][d], mu_k[ij * D + d], a);
        mv_t[v] = a;
      }
      __syncthreads();
      const float *wrow = W + (int64_t)p * w_stride + (int64_t)i * wl;
      float rsum = 0.f;
      const float rij = PASS == 2 ? R[ij] : 0.f, dlz = PASS == 2 ? dlogZ[ij] : 0.f;
#pragma unroll 1
      for (int u = 0; u < KPW; ++u) {
        const int k = c0 + warp + 8 * u;
        if (k >= k1) break;
        const T *krow = ks + ((int64_t)p * g.N + k) * D;
        const T *vrow = vs + ((int64_t)p * g.N + k) * DV;
        // Gk = dC k (lane owns rows v = lane + 32 t), Gv = dC^T v (lane owns columns)
        float Gk[PV];
#pragma unroll
        for (int v = 0; v < PV; ++v) Gk[v] = 0.f;
#pragma unroll 4
        for (int d = 0; d < D; ++d) {
          const float kd = ld_elem(krow + d);
#pragma unroll
          for (int v = 0; v < PV; ++v) Gk[v] = fmaf(G[lane + 32 * v][d], kd, Gk[v]);
        }
        float x = 0.f;
#pragma unroll
        for (int v = 0; v < PV; ++v) x = fmaf(ld_elem(vrow + lane + 32 * v), Gk[v] + mv_t[lane + 32 * v], x);
#pragma unroll
        for (int t = 0; t < PD; ++t) x = fmaf(ld_elem(krow + lane + 32 * t), mk_t[lane + 32 * t], x);
        const float dw = warp_sum(x);
        const float w = wrow[k];
        if (PASS == 1) {
          rsum = fmaf(w, dw, rsum);
        } else {
          float Gv[PD];
#pragma unroll
          for (int t = 0; t < PD; ++t) Gv[t] = 0.f;
#pragma unroll 4
          for (int v = 0; v < DV; ++v) {
            const float vv = ld_elem(vrow + v);
#pragma unroll
            for (int t = 0; t < PD; ++t) Gv[t] = fmaf(G[v][lane + 32 * t], vv, Gv[t]);
          }
          const float dl = w * (dw - rij) + w * dlz;
          if (lane == 0) DL[((int64_t)p * g.Cq + i) * g.N + k] = dl;
#pragma unroll
          for (int t = 0; t < PD; ++t) {
            const int c = lane + 32 * t;
            acc_k[warp][u][c] = fmaf(w, Gv[t] + mk_t[c], fmaf(g.s * dl, qb[c], acc_k[warp][u][c]));
          }
#pragma unroll
          for (int v = 0; v < PV; ++v) {
            const int c = lane + 32 * v;
            acc_v[warp][u][c] = fmaf(w, Gk[v] + mv_t[c], acc_v[warp][u][c]);
          }
        }
      }
      if (PASS == 1) {
        // R_ij accumulates over the chunks in order: chunk partials through shared memory
        if (lane == 0) red[warp] = rsum;
        __syncthreads();
        if (threadIdx.x == 0) {
          float a = c0 == k0 ? 0.f : R[ij];
          for (int w8 = 0; w8 < 8; ++w8) a += red[w8];
          R[ij] = a;
        }
      }
    }
    if (PASS == 2) {
      __syncwarp();
      for (int u = 0; u < KPW; ++u) {
        const int k = c0 + warp + 8 * u;
        if (k >= k1) break;
        for (int t = lane; t < D; t += 32) dKs[((int64_t)p * g.N + k) * D + t] = acc_k[warp][u][t];
        for (int t = lane; t < DV; t += 32) dVs[((int64_t)p * g.N + k) * DV + t] = acc_v[warp][u][t];
      }
    }
  }
}

// dqbar_i = s sum_k dl_ik k_k over every key (sorted order); then every row of cluster i:
// dq_n = dqt_n + (dqbar_i - sum_{n' in i} dqt_n') / |i|, written in token order.
template <typename T, int D>
__global__ void __launch_bounds__(128)
queries(Geo g, const T *__restrict__ ks, const float *__restrict__ DL,
        const int32_t *__restrict__ q_perm, const int32_t *__restrict__ q_offsets,
        const float *__restrict__ dQt, T *__restrict__ dQ) {
  const int p = blockIdx.y, i = blockIdx.x;
  const int32_t *off = q_offsets + (int64_t)p * (g.Cq + 1);
  const int r0 = off[i], r1 = off[i + 1];
  if (r0 >= r1) return;
  const float *dl = DL + ((int64_t)p * g.Cq + i) * g.N;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float a = 0.f;
    for (int k = 0; k < g.N; ++k) a = fmaf(dl[k], ld_elem(ks + ((int64_t)p * g.N + k) * D + d), a);
    float sq = 0.f;
    for (int r = r0; r < r1; ++r) sq += dQt[((int64_t)p * g.N + r) * D + d];
    const float corr = (g.s * a - sq) / (float)(r1 - r0);
    for (int r = r0; r < r1; ++r)
      st_elem(dQ + ((int64_t)p * g.N + q_perm[(int64_t)p * g.N + r]) * D + d,
              dQt[((int64_t)p * g.N + r) * D + d] + corr);
  }
}

// Sorted key rows back to token order, in the output type.
template <typename T>
__global__ void unsort(int N, int width, const int32_t *__restrict__ perm, const float *__restrict__ src,
                       T *__restrict__ dst) {
  const int p = blockIdx.y;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)N * width) return;
  const int r = (int)(e / width), c = (int)(e % width);
  st_elem(dst + ((int64_t)p * N + perm[(int64_t)p * N + r]) * width + c,
          src[((int64_t)p * N + r) * width + c]);
}

struct Ws {
  float *qbar;
  SortedSide ks;
  void *vs;
  StageBufs sb;  // W, logZ, mu_k, mu_v, cov
  float *PA, *DA, *dQt, *dlogZ, *dmuk, *dmuv, *dC, *R, *DL, *dKs, *dVs;
};

struct Bump3 {
  char *base;
  size_t off = 0;
  explicit Bump3(void *b) : base(static_cast<char *>(b)) {}
  template <typename X>
  X *take(size_t count) {
    const size_t o = off;
    off = align_up(off + count * sizeof(X));
    return base ? reinterpret_cast<X *>(base + o) : nullptr;
  }
};

static void plan(Bump3 &bp, const muse_dims &d, int Cq, int Ck, Ws &w) {
  const size_t P = (size_t)d.B * d.H, N = d.N, es = d.dtype == MUSE_F32 ? 4 : 2;
  const size_t z = P * Cq * Ck;
  w.qbar = bp.take<float>(P * Cq * d.D);
  w.ks.rows = bp.take<char>(P * N * d.D * es);
  w.ks.cluster = bp.take<int32_t>(P * N);
  w.vs = bp.take<char>(P * N * d.Dv * es);
  memset(&w.sb, 0, sizeof(w.sb));
  w.sb.W = bp.take<float>(P * Cq * w_ld(d.N));
  w.sb.logZ = bp.take<float>(z);
  w.sb.mu_k = bp.take<float>(z * d.D);
  w.sb.mu_v = bp.take<float>(z * d.Dv);
  w.sb.cov = bp.take<float>(z * d.Dv * d.D);
  w.PA = bp.take<float>(P * N * Ck);
  w.DA = bp.take<float>(P * N * Ck);
  w.dQt = bp.take<float>(P * N * d.D);
  w.dlogZ = bp.take<float>(z);
  w.dmuk = bp.take<float>(z * d.D);
  w.dmuv = bp.take<float>(z * d.Dv);
  w.dC = bp.take<float>(z * d.Dv * d.D);
  w.R = bp.take<float>(z);
  w.DL = bp.take<float>(P * Cq * N);
  w.dKs = bp.take<float>(P * N * d.D);
  w.dVs = bp.take<float>(P * N * d.Dv);
}

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

template <typename T, int D, int DV>
static cudaError_t run_t(const void *Q, const void *K, const void *V, const void *dO,
                         const int32_t *q_perm, const int32_t *q_offsets, const int32_t *k_perm,
                         const int32_t *k_offsets, const muse_dims &d, int Cq, int Ck, void *dQ,
                         void *dK, void *dV, Ws &w, cudaStream_t st) {
  const int P = d.B * d.H, N = d.N;
  Geo g{N, Cq, Ck, d.scale};
  MuseTables mt;
  memset(&mt, 0, sizeof(mt));
  mt.q = whole(N, Cq);
  mt.k = whole(N, Ck);
  mt.in.ninst = 1;
  mt.in.w_stride = Cq * w_ld(N);
  mt.in.z_stride = Cq * Ck;
  mt.in.c_stride = Ck * w_ld(N);
  mt.in.out_stride = N;
  cudaError_t e;
  means<T, D><<<dim3(Cq, P), 128, 0, st>>>(g, (const T *)Q, q_perm, q_offsets, w.qbar);
  if ((e = run_sort_side(K, d.dtype, D, N, mt.k, P, k_perm, k_offsets, nullptr, w.ks, st)) != cudaSuccess)
    return e;
  SortedSide vsd{w.vs, w.ks.cluster};
  if ((e = run_sort_side(V, d.dtype, DV, N, mt.k, P, k_perm, k_offsets, nullptr, vsd, st)) != cudaSuccess)
    return e;
  if ((e = run_summaries(mt, d.dtype, D, DV, P, d.scale, w.qbar, w.ks, w.vs, k_offsets, w.sb, st)) !=
      cudaSuccess)
    return e;
  const size_t rsm = (size_t)(DV * D + 32 * (D + DV) + D + DV + 64) * sizeof(float);
  if ((e = cudaFuncSetAttribute(rows<T, D, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)rsm)) != cudaSuccess)
    return e;
  rows<T, D, DV><<<dim3(Cq, P), 256, rsm, st>>>(g, (const T *)Q, (const T *)dO, q_perm, q_offsets,
                                               w.qbar, w.sb.logZ, w.sb.mu_k, w.sb.mu_v, w.sb.cov,
                                               w.PA, w.DA, w.dQt, w.dlogZ, w.dmuk, w.dmuv, w.dC);
  const size_t gsm = (size_t)DV * (D + 1) * sizeof(float);
  if ((e = cudaFuncSetAttribute(keys<T, D, DV, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)gsm)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(keys<T, D, DV, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)gsm)) != cudaSuccess)
    return e;
  keys<T, D, DV, 1><<<dim3(Ck, P), 256, gsm, st>>>(g, (const T *)w.ks.rows, (const T *)w.vs,
                                                  k_offsets, w.sb.W, mt.in.w_stride, w.qbar,
                                                  w.sb.mu_k, w.sb.mu_v, w.dlogZ, w.dmuk, w.dmuv,
                                                  w.dC, w.R, w.DL, w.dKs, w.dVs);
  keys<T, D, DV, 2><<<dim3(Ck, P), 256, gsm, st>>>(g, (const T *)w.ks.rows, (const T *)w.vs,
                                                  k_offsets, w.sb.W, mt.in.w_stride, w.qbar,
                                                  w.sb.mu_k, w.sb.mu_v, w.dlogZ, w.dmuk, w.dmuv,
                                                  w.dC, w.R, w.DL, w.dKs, w.dVs);
  queries<T, D><<<dim3(Cq, P), 128, 0, st>>>(g, (const T *)w.ks.rows, w.DL, q_perm, q_offsets,
                                            w.dQt, (T *)dQ);
  unsort<T><<<dim3((unsigned)(((int64_t)N * D + 255) / 256), P), 256, 0, st>>>(N, D, k_perm, w.dKs, (T *)dK);
  unsort<T><<<dim3((unsigned)(((int64_t)N * DV + 255) / 256), P), 256, 0, st>>>(N, DV, k_perm, w.dVs, (T *)dV);
  count_launches(7);
  return cudaGetLastError();
}

}  // namespace bwd

size_t muse_backward_ws(const muse_dims &d, int Cq, int Ck) {
  bwd::Bump3 bp(nullptr);
  bwd::Ws w;
  bwd::plan(bp, d, Cq, Ck, w);
  return bp.off;
}

cudaError_t run_backward(const void *Q, const void *K, const void *V, const void *dO,
                         const int32_t *q_perm, const int32_t *q_offsets, const int32_t *k_perm,
                         const int32_t *k_offsets, const muse_dims &d, int Cq, int Ck, void *dQ,
                         void *dK, void *dV, void *ws, cudaStream_t st) {
  bwd::Bump3 bp(ws);
  bwd::Ws w;
  bwd::plan(bp, d, Cq, Ck, w);
#define MUSE_BWD(TT, DD, DDV)                                                                 \
  if (d.D == DD && d.Dv == DDV)                                                               \
    return bwd::run_t<TT, DD, DDV>(Q, K, V, dO, q_perm, q_offsets, k_perm, k_offsets, d, Cq, \
                                   Ck, dQ, dK, dV, w, st);
  if (d.dtype == MUSE_F32) {
    MUSE_BWD(float, 64, 64)
    MUSE_BWD(float, 64, 128)
    MUSE_BWD(float, 128, 64)
    MUSE_BWD(float, 128, 128)
  } else {
    MUSE_BWD(__nv_bfloat16, 64, 64)
    MUSE_BWD(__nv_bfloat16, 64, 128)
    MUSE_BWD(__nv_bfloat16, 128, 64)
    MUSE_BWD(__nv_bfloat16, 128, 128)
  }
#undef MUSE_BWD
  return cudaErrorInvalidValue;
}

}  // namespace muse
