// The partially specialised dipole (an option of the acausal forward pass).
//
// pith.science review of arXiv 2509.10406, "Axioms" ("ad hoc to paper": the covariance
// of a key cluster is taken without the exponential tilt by the query centroid, which
// lowers its cost from O(Cq N D^2) to O(N D^2)), "invented entities" (the dipole
// correction as an aggregated covariance Cov_j(v,k) per query cluster) and the referee
// comment on Algorithm 3 (it is Cov_j(v,k), not the tilted Cov_ij(v,k)).  The
// aggregation weights are not printed; the reading taken here weights key cluster j by
// the monopole softmax at the centroid, pi_ij = softmax_j(logZ_ij):
//   Cov_j  = (1/|S_j|) sum_{k in S_j} (v - vbar_j)(k - kbar_j)^T           [Dv x D]
//   Cbar_i = sum_j pi_ij Cov_j
//   O_n   += s Cbar_i qt_n        (on top of the monopole-only refinement, whose
//                                   coefficients are c0 = p, c1 = 0)
// Three CUDA-core kernels; the work is O(N D Dv + Cq Ck D Dv) per problem, small next
// to the refinement.  Single-instance (acausal) tables only.
#include "internal.h"

namespace muse {
namespace pdp {

// Cov_j for every key cluster: CTA per (j, problem); thread (dv, d) pairs tid + 256 u.
template <typename T, int D, int DV>
__global__ void __launch_bounds__(256)
pd_cov(MuseTables mt, int N, const T *__restrict__ ks, const T *__restrict__ V,
       const int32_t *__restrict__ k_perm, const int32_t *__restrict__ k_offsets,
       float *__restrict__ cov) {
  constexpr int NO = DV * D / 256;  // outputs per thread
  const int p = blockIdx.y, j = blockIdx.x;
  const Task k = make_task(mt.k, p * mt.k.nseg);
  if (j >= k.C) return;  // uniform
  const int b = k_offsets[k.off + j], e = k_offsets[k.off + j + 1], n = e - b;
  __shared__ float Ks[32][D + 1], Vs[32][DV + 1], kbar[D], vbar[DV];
  const int tid = threadIdx.x;
  const T *vrow0 = V + (int64_t)p * N * DV;
  // member means, summed in sorted order
  for (int x = tid; x < D + DV; x += 256) {
    float acc = 0.f;
    if (x < D) {
      for (int pos = b; pos < e; ++pos) acc += ld_elem(ks + (k.lab + pos) * D + x);
      kbar[x] = n ? acc / (float)n : 0.f;
    } else {
      const int dv = x - D;
      for (int pos = b; pos < e; ++pos)
        acc += ld_elem(vrow0 + (int64_t)k_perm[k.lab + pos] * DV + dv);
      vbar[dv] = n ? acc / (float)n : 0.f;
    }
  }
  float acc[NO];
#pragma unroll
  for (int u = 0; u < NO; ++u) acc[u] = 0.f;
  for (int pc = b; pc < e; pc += 32) {
    const int pt = min(32, e - pc);
    __syncthreads();  // the means are ready; the previous rows are consumed
    for (int x = tid; x < pt * D; x += 256) {
      const int rr = x / D, d = x % D;
      Ks[rr][d] = ld_elem(ks + (k.lab + pc + rr) * D + d) - kbar[d];
    }
    for (int x = tid; x < pt * DV; x += 256) {
      const int rr = x / DV, dv = x % DV;
      Vs[rr][dv] = ld_elem(vrow0 + (int64_t)k_perm[k.lab + pc + rr] * DV + dv) - vbar[dv];
    }
    __syncthreads();
    for (int rr = 0; rr < pt; ++rr) {
#pragma unroll
      for (int u = 0; u < NO; ++u) {
        const int e2 = tid + 256 * u;
        acc[u] = fmaf(Vs[rr][e2 / D], Ks[rr][e2 % D], acc[u]);
      }
    }
  }
  float *out = cov + ((int64_t)p * k.C + j) * DV * D;
  const float inv = n ? 1.f / (float)n : 0.f;
#pragma unroll
  for (int u = 0; u < NO; ++u) out[tid + 256 * u] = acc[u] * inv;
}

// Cbar_i = sum_j softmax_j(logZ_ij) Cov_j: CTA per (i, problem).
template <int D, int DV>
__global__ void __launch_bounds__(256)
pd_aggregate(MuseTables mt, const float *__restrict__ logZ, const float *__restrict__ cov,
             float *__restrict__ cbar) {
  constexpr int NO = DV * D / 256;
  const int p = blockIdx.y, i = blockIdx.x;
  const Task q = make_task(mt.q, p * mt.q.nseg), k = make_task(mt.k, p * mt.k.nseg);
  if (i >= q.C) return;  // uniform
  const int Ck = k.C;
  __shared__ float pi[kMaxClusters];
  __shared__ float red[2];
  const float *lz = logZ + (int64_t)p * mt.in.z_stride + mt.in.z0[0] + (int64_t)i * Ck;
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid < 32) {
    float m = -CUDART_INF_F;
    for (int j = lane; j < Ck; j += 32) m = fmaxf(m, lz[j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < Ck; j += 32) l += lz[j] > -CUDART_INF_F ? expf(lz[j] - m) : 0.f;
    l = warp_sum(l);
    if (lane == 0) {
      red[0] = m;
      red[1] = l;
    }
  }
  __syncthreads();
  for (int j = tid; j < Ck; j += 256)
    pi[j] = lz[j] > -CUDART_INF_F ? expf(lz[j] - red[0]) / red[1] : 0.f;
  __syncthreads();
  float acc[NO];
#pragma unroll
  for (int u = 0; u < NO; ++u) acc[u] = 0.f;
  const float *cv = cov + (int64_t)p * Ck * DV * D;
  for (int j = 0; j < Ck; ++j) {
    const float w = pi[j];
#pragma unroll
    for (int u = 0; u < NO; ++u) acc[u] = fmaf(w, cv[(int64_t)j * DV * D + tid + 256 * u], acc[u]);
  }
  float *out = cbar + ((int64_t)p * q.C + i) * DV * D;
#pragma unroll
  for (int u = 0; u < NO; ++u) out[tid + 256 * u] = acc[u];
}

// O[row] += s Cbar_i qt for every query: four threads per sorted query position, each
// a quarter of the Dv outputs.
template <typename T, int D, int DV>
__global__ void __launch_bounds__(256)
pd_correct(MuseTables mt, int N, float scale, const T *__restrict__ qt_rows,
           const int32_t *__restrict__ q_cluster, const int32_t *__restrict__ q_perm,
           const float *__restrict__ cbar, T *__restrict__ O) {
  constexpr int QV = DV / 4;
  const int p = blockIdx.y;
  const Task q = make_task(mt.q, p * mt.q.nseg);
  const int pos = blockIdx.x * 64 + (threadIdx.x >> 2), part = threadIdx.x & 3;
  if (pos >= q.n) return;  // no barriers below
  const int i = q_cluster[q.lab + pos];
  const int row = q_perm[q.lab + pos];
  float qt[D];
#pragma unroll
  for (int d = 0; d < D; ++d) qt[d] = ld_elem(qt_rows + (q.lab + pos) * D + d);
  const float *cb = cbar + ((int64_t)p * q.C + i) * DV * D;
  T *o = O + ((int64_t)p * N + row) * DV + part * QV;
  for (int dv = 0; dv < QV; ++dv) {
    const float4 *c4 = reinterpret_cast<const float4 *>(cb + (int64_t)(part * QV + dv) * D);
    float acc = 0.f;
#pragma unroll
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 c = __ldg(c4 + d4);
      acc = fmaf(c.x, qt[4 * d4], acc);
      acc = fmaf(c.y, qt[4 * d4 + 1], acc);
      acc = fmaf(c.z, qt[4 * d4 + 2], acc);
      acc = fmaf(c.w, qt[4 * d4 + 3], acc);
    }
    o[dv] = T(ld_elem(o + dv) + scale * acc);
  }
}

// O == nullptr: Cov_j and Cbar_i only (the summary-form output applies the correction).
template <typename T, int D, int DV>
static cudaError_t run_t(const MuseTables &mt, int N, int P, float scale, SortedSide qs,
                         const int32_t *q_perm, SortedSide ks, const void *V,
                         const int32_t *k_perm, const int32_t *k_offsets, const float *logZ,
                         float *cov, float *cbar, void *O, cudaStream_t st) {
  pd_cov<T, D, DV><<<dim3(mt.k.max_C, P), 256, 0, st>>>(mt, N, (const T *)ks.rows, (const T *)V,
                                                        k_perm, k_offsets, cov);
  pd_aggregate<D, DV><<<dim3(mt.q.max_C, P), 256, 0, st>>>(mt, logZ, cov, cbar);
  count_launches(2);
  if (O) {
    pd_correct<T, D, DV><<<dim3((mt.q.max_rows + 63) / 64, P), 256, 0, st>>>(
        mt, N, scale, (const T *)qs.rows, qs.cluster, q_perm, cbar, (T *)O);
    count_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace pdp

size_t partial_dipole_ws_floats(int P, int Cq, int Ck, int D, int Dv) {
  return (size_t)P * (size_t)(Cq + Ck) * (size_t)D * (size_t)Dv;
}

float *partial_dipole_cbar(float *ws, int P, int maxCk, int D, int Dv) {
  return ws + (size_t)P * maxCk * D * Dv;
}

cudaError_t run_partial_dipole(const MuseTables &mt, int dtype, int D, int Dv, int N, int P,
                               float scale, SortedSide qs, const int32_t *q_perm, SortedSide ks,
                               const void *V, const int32_t *k_perm, const int32_t *k_offsets,
                               const float *logZ, float *ws, void *O, cudaStream_t st) {
  if (mt.in.ninst != 1) return cudaErrorInvalidValue;
  float *cov = ws;
  float *cbar = partial_dipole_cbar(ws, P, mt.k.max_C, D, Dv);
  using namespace pdp;
#define PD_CASE(TT, DD, DVV)                                                                    \
  if (D == DD && Dv == DVV)                                                                     \
    return run_t<TT, DD, DVV>(mt, N, P, scale, qs, q_perm, ks, V, k_perm, k_offsets, logZ, cov, \
                              cbar, O, st);
  if (dtype == MUSE_F32) {
    PD_CASE(float, 64, 64)
    PD_CASE(float, 64, 128)
    PD_CASE(float, 128, 64)
    PD_CASE(float, 128, 128)
  } else {
    PD_CASE(__nv_bfloat16, 64, 64)
    PD_CASE(__nv_bfloat16, 64, 128)
    PD_CASE(__nv_bfloat16, 128, 64)
    PD_CASE(__nv_bfloat16, 128, 128)
  }
#undef PD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace muse
