// Host-side declarations shared by the libmuse translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace muse {

inline size_t align_up(size_t b) { return (b + 255) & ~(size_t)255; }

// Host-side count of enqueued kernels (muse_launch_counter).
void count_launches(int n);

// Device address of the current device's status word (NULL if unavailable).
int *device_status_word();

// Records a CUDA error for muse_last_error_detail (this thread) and returns MUSE_ERR_CUDA.
muse_status cuda_fail(cudaError_t e);

// Records the event set by muse_set_profile_events before (start) or after the dominant
// kernel of a call, when events are set; cudaSuccess otherwise.
cudaError_t profile_mark(bool start, cudaStream_t st);

// Per-instance offsets of the stage buffers.  An instance pairs query segment s
// with key segment s (acausal: the one whole-sequence segment; causal: one square).
struct InstTable {
  int ninst;
  int w_stride;   // per problem: floats of W (sum over instances of Cq_s * nk_s)
  int z_stride;   // per problem: entries of logZ (sum of Cq_s * Ck_s)
  int c_stride;   // per problem: floats of each coefficient array (sum of Ck_s * nq_s)
  int out_stride; // per problem: rows of the output / partial arrays
  int w0[kMaxSeg], z0[kMaxSeg], cc0[kMaxSeg], out0[kMaxSeg];
};

struct MuseTables {
  SegTable q, k;
  InstTable in;
};

struct KmeansOut {
  int32_t *labels;
  float *centroids;
  int32_t *perm;
  int32_t *offsets;
};

size_t kmeans_ws_bytes(const SegTable &t, int P, int D);
size_t kmeans_pair_ws_bytes(const SegTable *tq, const SegTable *tk, int P, int D);
cudaError_t run_kmeans(const void *X, int dtype, int D, int N, const SegTable &tab, int P,
                       int iters, const KmeansOut &o, char *ws, int *status, cudaStream_t st);
// Queries and keys clustered in the same launches.
cudaError_t run_kmeans_pair(const void *Xq, const SegTable &tq, const KmeansOut &oq,
                            const void *Xk, const SegTable &tk, const KmeansOut &ok, int dtype,
                            int D, int N, int P, int iters, char *ws, int *status,
                            cudaStream_t st);
// Every round of K-means in one launch (kmeans_fused.cu): bfloat16, D = 64, C <= 128.
bool kmeans_fused_supported(int dtype, int D, const SegTable &t);
cudaError_t run_kmeans_fused(int njobs, const void *const *X, const SegTable *const *tabs,
                             const KmeansOut *outs, int N, int P, int iters, int *status,
                             cudaStream_t st);

// Sorted working copies of one side (rows in cluster order).
struct SortedSide {
  void *rows;        // [P][row_stride][width] in the input dtype (queries: residuals q - qbar)
  int32_t *cluster;  // [P][row_stride] cluster of each sorted position
};

// Stage buffers for the summaries + refinement of every instance.
struct StageBufs {
  float *W;        // [P][w_stride]  tilt logits, then tilt weights w_ik
  float *logZ;     // [P][z_stride]
  float *mu_k;     // [P][z_stride][D]
  float *mu_v;     // [P][z_stride][Dv] (optional)
  float *cov;      // [P][z_stride][Dv][D] (optional)
  float *c0, *c1;  // [P][c_stride]
  float *lse;      // [P][q.row_stride] logsumexp_j a_j per sorted query position
  float *opart;    // [kSplitCtas][128][Dv] partial outputs of the refinement's split last wave
};
// The tensor-core refinement splits at most this many CTAs' key ranges (half an SM count).
constexpr int kSplitCtas = 256;

cudaError_t run_sort_side(const void *X, int dtype, int width, int N, const SegTable &tab, int P,
                          const int32_t *perm, const int32_t *offsets, const float *centroids,
                          SortedSide out, cudaStream_t st);
// Transposed sorted copy (keys innermost) for the tensor-core refinement.
cudaError_t run_sort_side_t(const void *X, int dtype, int width, int N, const SegTable &tab,
                            int P, const int32_t *perm, void *vt, cudaStream_t st);
cudaError_t run_summaries(const MuseTables &mt, int dtype, int D, int Dv, int P, float scale,
                          const float *q_centroids, SortedSide ks, const void *vs_rows,
                          const int32_t *k_offsets, StageBufs b, cudaStream_t st);
// W = exp(s qbar_i.k - logZ_ij) for given logZ (the refinement's tilt weights).
cudaError_t run_tilt_weights(const MuseTables &mt, int dtype, int D, int P, float scale,
                             const float *q_centroids, SortedSide ks, const float *logZ, float *W,
                             cudaStream_t st);
// mu_v[i][j] = sum_{k in S_j} w_ik v_k from the tilt weights W and the cluster-sorted
// values (row-major).
cudaError_t run_tilt_values(const MuseTables &mt, int dtype, int Dv, int P, const int32_t *k_offsets,
                            const float *W, const void *vs_rows, float *mu_v, cudaStream_t st);
// Partially specialised dipole (acausal tables): Cov_j per key cluster, Cbar_i per query
// cluster, O += s Cbar_i qt.  ws holds P (Cq + Ck) D Dv floats; with O == nullptr only
// Cov_j and Cbar_i ([P][Cq][Dv][D], at partial_dipole_cbar(ws, ...)) are computed.
size_t partial_dipole_ws_floats(int P, int Cq, int Ck, int D, int Dv);
float *partial_dipole_cbar(float *ws, int P, int maxCk, int D, int Dv);
cudaError_t run_partial_dipole(const MuseTables &mt, int dtype, int D, int Dv, int N, int P,
                               float scale, SortedSide qs, const int32_t *q_perm, SortedSide ks,
                               const void *V, const int32_t *k_perm, const int32_t *k_offsets,
                               const float *logZ, float *ws, void *O, cudaStream_t st);
// Tilt logits s qbar_i . k of every instance on the tensor cores (logits_tc.cu), written
// into W for the tilt stage: bfloat16, D = 64 or 128.
bool logits_tc_supported(int dtype, int D);
cudaError_t run_logits_tc(const MuseTables &mt, int D, int P, float scale, const float *q_centroids,
                          const void *ks_rows, float *W, int *status, cudaStream_t st);
// Instances a kernel leaves to another one (bit s: instance s).
struct InstMask {
  uint32_t w[kMaxSeg / 32];
};
// The coefficients on the tensor cores (coef_tc.cu): bfloat16, D = 64 or 128, Ck <= 256;
// the instances in `skip` are left out.
bool coef_tc_supported(int dtype, int D, int maxCk);
cudaError_t run_coef_tc(const MuseTables &mt, int D, int P, float scale, const void *qs_rows,
                        const int32_t *q_offsets, const StageBufs &b, const InstMask &skip,
                        float sdip, int *status, cudaStream_t st);
// The monopole-only method (cbar == nullptr) and the partially specialised dipole in
// summary form (coef_tc.cu): O_n = sum_j p_j mu_v,ij (+ s Cbar_i qt_n) with b.mu_v given;
// bfloat16, D = Dv, no O(N^2) contraction.
bool coef_out_supported(int dtype, int D, int Dv, int maxCk);
cudaError_t run_coef_out(const MuseTables &mt, int D, int N, int P, float scale, const void *qs_rows,
                         const int32_t *q_perm, const int32_t *q_offsets, const StageBufs &b,
                         const float *cbar, void *O, int *status, cudaStream_t st);
// sdip: the factor of the dipole terms (the logit scale, or 0 for the monopole only).
cudaError_t run_coeffs(const MuseTables &mt, int dtype, int D, int P, float scale,
                       SortedSide qs, const int32_t *q_offsets, StageBufs b, float sdip,
                       cudaStream_t st);
// Refinement: acausal writes O[p][row][:] (row = sequence row); partial mode writes
// part_o[p][out0 + row][:] (float32) and part_lse[p][out0 + row].
cudaError_t run_refine(const MuseTables &mt, int dtype, int D, int Dv, int N, int P,
                       SortedSide qs, const int32_t *q_perm, SortedSide ks, const void *vs_rows,
                       StageBufs b, void *O, float *part_o, float *part_lse, cudaStream_t st);
// The refinement in summary form on the tensor cores (refine_sf.cu): O_n = sum_j c0_nj
// mu_v,ij + sum_j c1_nj C'_ij qt_n with C'_ij = sum_{k in S_j} w_ik v_k k^T formed on chip per
// query cluster; bfloat16, D = Dv = 128, one instance (acausal), Ck <= 256.  vt: the
// transposed sorted values (run_sort_side_t).
bool refine_sf_supported(int dtype, int D, int Dv, const MuseTables &mt);
cudaError_t run_refine_sf(const MuseTables &mt, int N, int P, const void *qs_rows,
                          const int32_t *q_perm, const int32_t *q_offsets, const void *ks_rows,
                          const int32_t *k_offsets, const void *vt, const StageBufs &b, void *O,
                          int *status, cudaStream_t st);
// The refinement from materialised summaries (refine_summaries.cu): O_n = sum_j p_j
// (mu_v,ij + s C_ij qt) with p = softmax_j(logZ_ij + s qt.mu_k,ij), float32 on the CUDA
// cores.  q_labels (natural order) is optional; a row whose label disagrees with
// q_perm / q_offsets is reported as MUSE_ERR_DEVICE.
cudaError_t run_refine_summaries(int dtype, int D, int Dv, int N, int P, int Cq, int Ck,
                                 float scale, const void *Q, const float *q_centroids,
                                 const int32_t *q_perm, const int32_t *q_offsets,
                                 const int32_t *q_labels, const float *logZ, const float *mu_k,
                                 const float *mu_v, const float *cov, void *O, int *status,
                                 cudaStream_t st);
// Backward pass (backward.cu): dQ, dK, dV of sum(O * dO), clusterings fixed.
size_t muse_backward_ws(const muse_dims &d, int Cq, int Ck);
cudaError_t run_backward(const void *Q, const void *K, const void *V, const void *dO,
                         const int32_t *q_perm, const int32_t *q_offsets, const int32_t *k_perm,
                         const int32_t *k_offsets, const muse_dims &d, int Cq, int Ck, void *dQ,
                         void *dK, void *dV, void *ws, cudaStream_t st);
size_t muse_retrieval_ws(const muse_dims &d, int block, int Cq, int Ck, int k1, int k2);
// The exact diagonal on the tensor cores (diag_tc.cu): bf16, D = Dv = 64, block a
// multiple of 128.  levels > 0: the causal decomposition's level partials
// part_*[P][levels][N] (level l merged into the rows of blocks whose bit l-1 is set);
// levels < 0: one partial array part_*[P][N] merged into every row (retrieval).
bool diag_tc_supported(int dtype, int D, int Dv, int N, int block);
cudaError_t run_diag_tc(const void *Q, const void *K, const void *V, int N, int P, int block,
                        int levels, float scale, const float *part_o, const float *part_lse,
                        void *O, int *status, cudaStream_t st);
cudaError_t run_diag_merge(const void *Q, const void *K, const void *V, int dtype, int D, int Dv,
                           int N, int P, int block, int levels, float scale,
                           const float *part_o, const float *part_lse, void *O, cudaStream_t st);

}  // namespace muse
