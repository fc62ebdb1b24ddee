// The refinement from materialised summaries: muse_dipole_refine with mu_v and cov
// given by the caller (teacher forcing of the tilted dipole, or summaries computed
// elsewhere).  CUDA cores, float32.
//
// pith.science review of arXiv 2509.10406, "What carries the argument" (the query
// residual refines the tilted summaries; only the qt.kt term is dropped); gist.science
// "Kernmechanismen" items 1-2.  For query n in cluster i with qt = q_n - qbar_i:
//     a_j = log Z_ij + s qt.mu_k,ij;   p = softmax_j(a);
//     O_n = sum_j p_j (mu_v,ij + s C_ij qt)
// evaluated as written, against the stacked per-cluster summaries [mu_k | mu_v | C_ij]
// of the row's query cluster, with an online softmax over j.
//
// One warp per query row; a CTA takes 8 consecutive rows of the query-cluster order
// (mostly one cluster, so its summaries are read once into L1 and reused).  Lanes split
// the D coordinates for the logits and the Dv outputs for the dipole products; the
// residual is formed in float32 from Q and the centroid.
#include "internal.h"

namespace muse {
namespace rsum {

template <typename T, int D, int DV>
__global__ void __launch_bounds__(256)
refine_summaries(int N, int Cq, int Ck, float scale, const T *__restrict__ Q,
                 const float *__restrict__ qcen, const int32_t *__restrict__ q_perm,
                 const int32_t *__restrict__ q_offsets, const int32_t *__restrict__ q_labels,
                 const float *__restrict__ logZ, const float *__restrict__ mu_k,
                 const float *__restrict__ mu_v, const float *__restrict__ cov, T *__restrict__ O,
                 int *status) {
  constexpr int PD = D / 32, PV = DV / 32;
  __shared__ float qt_sh[8][D];
  const int p = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;  // sorted query row
  if (r >= N) return;                   // whole warps only: no CTA barrier below
  const int32_t *off = q_offsets + (int64_t)p * (Cq + 1);
  // the row's cluster: the last i with off[i] <= r
  int lo = 0, hi = Cq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= r) lo = mid;
    else hi = mid - 1;
  }
  const int i = lo;
  const int n = q_perm[(int64_t)p * N + r];
  if (q_labels && q_labels[(int64_t)p * N + n] != i) {
    if (lane == 0) report(status, MUSE_ERR_DEVICE);  // labels disagree with perm/offsets
    return;
  }
  const T *qrow = Q + ((int64_t)p * N + n) * D;
  const float *c = qcen + ((int64_t)p * Cq + i) * D;
  float qt[PD];
#pragma unroll
  for (int t = 0; t < PD; ++t) {
    qt[t] = ld_elem(qrow + lane + 32 * t) - c[lane + 32 * t];
    qt_sh[warp][lane + 32 * t] = qt[t];
  }
  __syncwarp();
  const int64_t ij0 = ((int64_t)p * Cq + i) * Ck;
  float m = -CUDART_INF_F, l = 0.f, o[PV];
#pragma unroll
  for (int v = 0; v < PV; ++v) o[v] = 0.f;
  for (int j = 0; j < Ck; ++j) {
    const float lz = logZ[ij0 + j];
    if (!(lz > -CUDART_INF_F)) continue;  // empty key cluster
    const float *mk = mu_k + (ij0 + j) * D;
    float dot = 0.f;
#pragma unroll
    for (int t = 0; t < PD; ++t) dot = fmaf(qt[t], mk[lane + 32 * t], dot);
    const float a = lz + scale * warp_sum(dot);
    const float mn = fmaxf(m, a);
    const float corr = expf(m - mn), pj = expf(a - mn);
    l = l * corr + pj;
    m = mn;
    const float *mv = mu_v + (ij0 + j) * DV;
    const float *cj = cov + (ij0 + j) * DV * D;
#pragma unroll
    for (int v = 0; v < PV; ++v) {
      const float *crow = cj + (int64_t)(lane + 32 * v) * D;
      float cq = 0.f;
      for (int d = 0; d < D; d += 4) {
        const float4 c4 = *reinterpret_cast<const float4 *>(crow + d);
        cq = fmaf(c4.x, qt_sh[warp][d], cq);
        cq = fmaf(c4.y, qt_sh[warp][d + 1], cq);
        cq = fmaf(c4.z, qt_sh[warp][d + 2], cq);
        cq = fmaf(c4.w, qt_sh[warp][d + 3], cq);
      }
      o[v] = fmaf(pj, fmaf(scale, cq, mv[lane + 32 * v]), o[v] * corr);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  T *orow = O + ((int64_t)p * N + n) * DV;
#pragma unroll
  for (int v = 0; v < PV; ++v) st_elem(orow + lane + 32 * v, o[v] * inv);
}

template <typename T, int D, int DV>
static cudaError_t launch(int N, int P, int Cq, int Ck, float scale, const void *Q,
                          const float *qcen, const int32_t *q_perm, const int32_t *q_offsets,
                          const int32_t *q_labels, const float *logZ, const float *mu_k,
                          const float *mu_v, const float *cov, void *O, int *status,
                          cudaStream_t st) {
  refine_summaries<T, D, DV><<<dim3((N + 7) / 8, P), 256, 0, st>>>(
      N, Cq, Ck, scale, (const T *)Q, qcen, q_perm, q_offsets, q_labels, logZ, mu_k, mu_v, cov,
      (T *)O, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace rsum

cudaError_t run_refine_summaries(int dtype, int D, int Dv, int N, int P, int Cq, int Ck,
                                 float scale, const void *Q, const float *q_centroids,
                                 const int32_t *q_perm, const int32_t *q_offsets,
                                 const int32_t *q_labels, const float *logZ, const float *mu_k,
                                 const float *mu_v, const float *cov, void *O, int *status,
                                 cudaStream_t st) {
#define MUSE_RSUM(TT, DD, DDV)                                                                  \
  if (D == DD && Dv == DDV)                                                                     \
    return rsum::launch<TT, DD, DDV>(N, P, Cq, Ck, scale, Q, q_centroids, q_perm, q_offsets,  \
                                     q_labels, logZ, mu_k, mu_v, cov, O, status, st);
  if (dtype == MUSE_F32) {
    MUSE_RSUM(float, 64, 64)
    MUSE_RSUM(float, 64, 128)
    MUSE_RSUM(float, 128, 64)
    MUSE_RSUM(float, 128, 128)
  } else {
    MUSE_RSUM(__nv_bfloat16, 64, 64)
    MUSE_RSUM(__nv_bfloat16, 64, 128)
    MUSE_RSUM(__nv_bfloat16, 128, 64)
    MUSE_RSUM(__nv_bfloat16, 128, 128)
  }
#undef MUSE_RSUM
  return cudaErrorInvalidValue;
}

}  // namespace muse
