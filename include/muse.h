/*
 * muse.h - C ABI of libmuse.so, the sm_100a (B200) forward pass of Multipole
 * Semantic Attention (MuSe).
 *
 * Method (pith.science review of arXiv 2509.10406, "Multipole Semantic Attention:
 * A Fast Approximation of Softmax Attention for Pretraining", section "What carries
 * the argument"; gist.science "Technische Samenvatting", "Kernmechanismen"):
 * per (batch, head), queries and keys are clustered separately with K-means; every
 * query centroid qbar_i attends every key cluster S_j through exponentially tilted
 * summaries (log Z_ij, tilted key mean mu_k,ij, tilted value mean mu_v,ij) and the
 * tilted value-key covariance C_ij (the dipole); every query then refines with its
 * residual qt = q - qbar_i:
 *
 *     out(q) = sum_j softmax_j(log Z_ij + s qt.mu_k,ij) (mu_v,ij + s C_ij qt)
 *
 * dropping only the qt.kt term.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major, innermost dimension last: Q, K [B,H,N,D],
 *    V [B,H,N,Dv], O [B,H,N,Dv].  One (b,h) pair is one "problem" p = b*H + h.
 *  - Q, K, V and O have the element type muse_dims.dtype (float32 or bfloat16).
 *    Arithmetic is float32; the bfloat16 path feeds bfloat16 operands to the
 *    tensor cores with float32 accumulation.
 *  - muse_dims.scale is the logit scale s in exp(s q.k).  Clustering always runs
 *    on the unscaled Q and K.
 *  - D and Dv must be 64 or 128; 1 <= C <= min(N, 1024) for every clustering.
 *  - Every pointer is a DEVICE pointer, 16-byte aligned, owned by the caller.
 *    The library allocates nothing and keeps no pointer after a call returns.
 *    Scratch memory is the caller's workspace `ws` of `ws_bytes` bytes; its
 *    required size comes from muse_workspace_size().
 *  - Calls are asynchronous on stream `st` (NULL = the legacy default stream).
 *    Arguments are validated before anything is enqueued: a rejected call
 *    returns INVALID_ARG / SHAPE / DTYPE / WORKSPACE and enqueues nothing.  A
 *    launch failure returns MUSE_ERR_CUDA.  Problems found on the device
 *    (a bounded wait that gave up, a bounds check) set a device status word that
 *    muse_last_device_status() reads.
 *  - Results are deterministic: no floating-point atomics anywhere.
 */
#ifndef MUSE_H
#define MUSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *muse_stream_t; /* a cudaStream_t */

typedef enum {
  MUSE_OK = 0,
  MUSE_ERR_INVALID_ARG = 1, /* null pointer, misaligned pointer, C/iters/k out of range */
  MUSE_ERR_SHAPE = 2,       /* D/Dv not 64/128, N not a multiple of the block, sizes <= 0 */
  MUSE_ERR_DTYPE = 3,       /* dtype not MUSE_F32 / MUSE_BF16 */
  MUSE_ERR_WORKSPACE = 4,   /* ws NULL or ws_bytes below muse_workspace_size() */
  MUSE_ERR_CUDA = 5,        /* a kernel launch failed (cudaGetLastError) */
  MUSE_ERR_TIMEOUT = 6,     /* device: a bounded wait ran out */
  MUSE_ERR_DEVICE = 7       /* device: a bounds check fired */
} muse_status;

typedef enum { MUSE_F32 = 0, MUSE_BF16 = 1 } muse_dtype;

typedef struct {
  int B, H, N; /* batch, heads, sequence length */
  int D, Dv;   /* query/key width, value width (64 or 128 each) */
  int dtype;   /* muse_dtype of Q, K, V, O */
  float scale; /* logit scale s */
} muse_dims;

/*
 * muse_kmeans - Lloyd K-means of every problem's N rows of X [B,H,N,D] into C
 * clusters (one call clusters one tensor: queries or keys).
 *   Start: centroids = the first C rows.  Then `iters` rounds of
 *   (assign every row to its nearest centroid by squared Euclidean distance,
 *   ties to the lowest index; replace every non-empty cluster's centroid by the
 *   mean of its members, an empty cluster keeping its centroid).
 *   Source: pith.science review, "What carries the argument" / "Core claim"
 *   (separate K-means over queries and keys); gist.science "Kernmechanismen" 1.
 * Outputs (device, caller-owned):
 *   labels    int32 [B,H,N]   cluster of every row after the last round
 *   centroids f32   [B,H,C,D] centroids after the last round's update
 *   perm      int32 [B,H,N]   rows sorted by cluster, stable (row order kept
 *                             inside a cluster); values are row indices 0..N-1
 *   offsets   int32 [B,H,C+1] cluster c occupies perm[offsets[c] .. offsets[c+1])
 * d.Dv is ignored.  1 <= iters <= 1000.
 */
muse_status muse_kmeans(const void *X, muse_dims d, int C, int iters, int32_t *labels,
                        float *centroids, int32_t *perm, int32_t *offsets, void *ws,
                        size_t ws_bytes, muse_stream_t st);

/*
 * muse_kmeans_noalloc - muse_kmeans for callers that cannot allocate device memory
 * and so cannot hand over a workspace: code running inside another runtime's memory
 * pool that offers no allocation hook, code called while a global-mode stream
 * capture is active (cudaMalloc is an error there), latency-critical loops that
 * cannot pay for cudaMalloc's synchronisation.  The paper has no counterpart: this
 * is a deployment variant of the same computation, with identical results.
 *   Same arguments and outputs as muse_kmeans, minus the workspace.  Its scratch is
 *   a static device array of MUSE_NOALLOC_SCRATCH_BYTES (16 MiB) inside the library,
 *   held by every GPU that loads it until the process exits.  Problems that take the
 *   multi-launch kernels (float32 inputs, D = 128 or C > 128) use that scratch: one
 *   whose need (muse_workspace_size("muse_kmeans", ...)) exceeds the array returns
 *   MUSE_ERR_WORKSPACE before anything is enqueued; e.g. B*H = 8, N = 8192, C = 256,
 *   D = 128 needs about 1 MiB.  The one-launch kernel (bfloat16, D = 64, C <= 128)
 *   uses no scratch and has no size limit beyond muse_kmeans's.
 *   The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture.  The library
 *   allocates nothing and calls no allocating routine.  Every call shares the one
 *   array and leaves its contents behind: calls that overlap on the GPU (several
 *   streams, or several threads) race on it and must be serialised by the caller.
 */
#define MUSE_NOALLOC_SCRATCH_BYTES (16u << 20)
muse_status muse_kmeans_noalloc(const void *X, muse_dims d, int C, int iters, int32_t *labels,
                                float *centroids, int32_t *perm, int32_t *offsets,
                                muse_stream_t st);

/*
 * muse_tilted_summaries - stage 1: for every query centroid i and key cluster j
 *     l_k = s qbar_i.k (k in S_j);  log Z_ij = log sum_k exp(l_k);
 *     w_k = exp(l_k - log Z_ij);    mu_k,ij = sum_k w_k k;  mu_v,ij = sum_k w_k v;
 *     C_ij = sum_k w_k (v - mu_v,ij)(k - mu_k,ij)^T   (Dv x D)
 *   Source: pith.science review, "What carries the argument" (tilted monopole and
 *   dipole from the cumulant generating function), "Assumptions & free
 *   parameters" (M_j(q) = E exp(q.k)), referee minor comment on Algorithm 3
 *   (the dipole of Eq. (6) is the tilted Cov_ij(v,k)).
 * Inputs:  q_centroids f32 [B,H,Cq,D]; K [B,H,N,D]; V [B,H,N,Dv] (may be NULL when
 *          mu_v and cov are NULL); k_perm, k_offsets from muse_kmeans on K.
 * Outputs: logZ f32 [B,H,Cq,Ck] (required; -inf for an empty key cluster);
 *          mu_k f32 [B,H,Cq,Ck,D], mu_v f32 [B,H,Cq,Ck,Dv],
 *          cov f32 [B,H,Cq,Ck,Dv,D] - each optional (NULL = not computed).
 *          cov is materialised only on request (inspection, tests): the forward
 *          pass never writes it to memory.
 */
muse_status muse_tilted_summaries(const float *q_centroids, const void *K, const void *V,
                                  const int32_t *k_perm, const int32_t *k_offsets,
                                  muse_dims d, int Cq, int Ck, float *logZ, float *mu_k,
                                  float *mu_v, float *cov, void *ws, size_t ws_bytes,
                                  muse_stream_t st);

/*
 * muse_dipole_refine - stage 2: for query n in cluster i with qt = q_n - qbar_i,
 *     a_j = log Z_ij + s qt.mu_k,ij;   p = softmax_j(a);
 *     O_n = sum_j p_j (mu_v,ij + s C_ij qt)
 *   Source: pith.science review, "What carries the argument" (drop only qt.kt);
 *   gist.science "Kernmechanismen" 1-2.
 *   Two ways to evaluate it:
 *   - mu_v = cov = NULL (the forward pass): C_ij is never materialised; with
 *     u_j = qt.mu_k,ij the output is computed as
 *       O_n = sum_j sum_{k in S_j} w_ik p_j (1 - s u_j + s qt.k) v_k,
 *     an identity of the definition (sum_k w_ik (k - mu_k,ij) = 0), on the tensor
 *     cores for bfloat16 inputs; the tilt weights w_ik are recomputed from logZ.  That
 *     sum is taken over all keys (the pair form) or, grouped by key cluster, against
 *     the uncentred summaries C'_ij = sum_{k in S_j} w_ik v_k k^T formed on chip (the
 *     summary form), as MUSE_FLAG_REFINE_SUMMARY below describes, by the same rule
 *     as muse_forward with no flags.
 *   - mu_v and cov given: the formula above is evaluated as written from the
 *     caller's materialised summaries (float32, CUDA cores; teacher forcing of the
 *     dipole, or summaries from elsewhere).
 * Inputs:  Q, K, V; q_labels int32 [B,H,N] (optional, may be NULL; when given, a row
 *          whose label disagrees with q_perm/q_offsets sets MUSE_ERR_DEVICE in the
 *          device status word); q_centroids/q_perm/q_offsets from muse_kmeans on Q
 *          (Cq clusters); k_perm/k_offsets from muse_kmeans on K (Ck clusters); logZ
 *          and mu_k from muse_tilted_summaries; mu_v f32 [B,H,Cq,Ck,Dv] and cov f32
 *          [B,H,Cq,Ck,Dv,D] both NULL or both given (else MUSE_ERR_INVALID_ARG).  Any
 *          values of the right shape are accepted, so the refinement can be fed
 *          reference summaries.
 * Output:  O [B,H,N,Dv] in d.dtype.
 */
muse_status muse_dipole_refine(const void *Q, const void *K, const void *V,
                               const int32_t *q_labels, const float *q_centroids,
                               const int32_t *q_perm, const int32_t *q_offsets,
                               const int32_t *k_perm, const int32_t *k_offsets,
                               const float *logZ, const float *mu_k, const float *mu_v,
                               const float *cov, muse_dims d, int Cq, int Ck, void *O,
                               void *ws, size_t ws_bytes, muse_stream_t st);

/*
 * muse_forward - the whole acausal forward pass: muse_kmeans on Q (Cq) and on K
 * (Ck), muse_tilted_summaries (logZ, mu_k), muse_dipole_refine.  O [B,H,N,Dv].
 */
muse_status muse_forward(const void *Q, const void *K, const void *V, muse_dims d, int Cq,
                         int Ck, int iters, void *O, void *ws, size_t ws_bytes,
                         muse_stream_t st);

/*
 * muse_forward_ex - muse_forward with option flags (0 = muse_forward).
 *   MUSE_FLAG_MONOPOLE: the monopole-only ablation - the dipole term s C_ij qt is
 *   dropped and O_n = sum_j p_j mu_v,ij with the same weights p_j = softmax_j(logZ_ij +
 *   s qt.mu_k,ij) (pith.science review of arXiv 2509.10406, "invented entities": the
 *   dipole correction, whose removal the paper's Table 3 measures).
 *   MUSE_FLAG_PARTIAL_DIPOLE: the partially specialised dipole - the tilted C_ij is
 *   replaced by the untilted covariance of each key cluster, Cov_j = mean over S_j of
 *   (v - vbar_j)(k - kbar_j)^T, aggregated per query cluster with the weights
 *   softmax_j(logZ_ij): O_n = sum_j p_j mu_v,ij + s (sum_j softmax_j(logZ_ij) Cov_j) qt_n
 *   (same review: "Axioms", the covariance taken without the tilt by the query
 *   centroid; "invented entities", an aggregated covariance per query cluster; the
 *   weights are not printed, this is the reading taken).
 * Both ablations need only the summaries: for bfloat16 with Dv = 64 (D = 64 with
 * Ck <= 256, D = 128 with Ck <= 128) they are evaluated in that form, O_n = sum_j p_j mu_v,ij (+ s Cbar_i qt_n),
 * with the tilted value means mu_v and no contraction over all N keys; other shapes run
 * the pair form of muse_forward with the dipole coefficient set to zero (plus the
 * covariance correction).
 * Same arguments, layouts and ownership as muse_forward.  Workspace: that of
 * muse_forward, plus B*H*(Cq + Ck)*D*Dv floats and 256 bytes with
 * MUSE_FLAG_PARTIAL_DIPOLE, plus B*H*Cq*Ck*Dv floats and 256 bytes in summary form;
 * muse_workspace_size("muse_forward_ex", ...) returns the largest of these sizes.  Unknown flag bits, or both ablation flags at once, return
 * MUSE_ERR_INVALID_ARG before anything is enqueued.
 */
#define MUSE_FLAG_MONOPOLE 1u
#define MUSE_FLAG_PARTIAL_DIPOLE 2u
/*
 * The form of the full method's refinement (muse_forward, muse_dipole_refine evaluate
 * the same sum either way; pith.science review of arXiv 2509.10406, "What carries the
 * argument"):
 *   pair form: O_n = sum_k w_ik (c0_nj + c1_nj qt_n.k) v_k over all keys, 2 N^2 (D + Dv)
 *   tensor flops per problem;
 *   summary form: O_n = sum_j c0_nj mu_v,ij + sum_j c1_nj C'_ij qt_n with
 *   C'_ij = sum_{k in S_j} w_ik v_k k^T formed on chip for each query cluster and never
 *   stored, about 2 Dv D N (N / 224 + Cq / 2) + 2 Dv (D + 16) Ck N flops; bfloat16 with
 *   D = Dv = 128 and Ck <= 256 only.
 * With neither flag the summary form is taken where it is supported and needs under three
 * quarters of the pair form's flops; MUSE_FLAG_REFINE_SUMMARY takes it wherever it is
 * supported, MUSE_FLAG_REFINE_PAIR never.  Both at once, or either with an ablation flag,
 * return MUSE_ERR_INVALID_ARG.
 */
#define MUSE_FLAG_REFINE_SUMMARY 4u
#define MUSE_FLAG_REFINE_PAIR 8u

/*
 * muse_refine_form - the form in which muse_forward_ex (with these flags, 0 or one of the
 * two form flags) and muse_dipole_refine (flags 0) evaluate the full method's
 * refinement for these sizes: 1 = summary form, 0 = pair form, -1 = invalid dims, cluster
 * counts or flags.  Host only (enqueues nothing, needs no device).
 */
int muse_refine_form(muse_dims d, int Cq, int Ck, unsigned flags);
muse_status muse_forward_ex(const void *Q, const void *K, const void *V, muse_dims d, int Cq,
                            int Ck, int iters, unsigned flags, void *O, void *ws,
                            size_t ws_bytes, muse_stream_t st);

/*
 * muse_causal_levels - number of levels L of the causal decomposition of N rows
 * into blocks of `block` rows (levels with side block*2^(l-1) < N).
 */
int muse_causal_levels(int N, int block);

/*
 * muse_causal_blocks - causal MuSe with the hierarchical block decomposition.
 *   Exact causal attention inside every diagonal block of `block` rows; below the
 *   diagonal, level l = 1..L (side s_l = block*2^(l-1)) holds the squares with
 *   queries [r s_l, (r+1) s_l) and keys [(r-1) s_l, r s_l) for odd r: each square is
 *   an acausal MuSe instance with its own K-means (C_eff = min(C, s_l)).  Every
 *   query's diagonal and square terms share one softmax normaliser.
 *   Source: pith.science review, Figure 2 caption (diagonal blocks exact, blocks
 *   below the diagonal MuSe), "Assumptions & free parameters" (hierarchical block
 *   decomposition); fugumt.com v2 abstract (O(NCD log N)).
 * Optional outputs (NULL = skip): q_labels_out, k_labels_out int32 [B,H,L,N]:
 *   the square-level cluster of every query / key row (-1 where the row is in no
 *   square of that level).  N % block == 0, block >= 64 and a multiple of 64.
 */
muse_status muse_causal_blocks(const void *Q, const void *K, const void *V, muse_dims d,
                               int block, int Cq, int Ck, int iters, void *O,
                               int32_t *q_labels_out, int32_t *k_labels_out, void *ws,
                               size_t ws_bytes, muse_stream_t st);

/*
 * muse_retrieve_exact - causal MuSe with retrieval (global clusters).
 *   For query cluster i and query block b: sigma_ij = logsumexp_{b'<b} log Z_{i,j,b'}
 *   (log Z over the keys of cluster j in block b'); the k1 largest sigma_ij pick
 *   the clusters, and inside each the k2 largest log Z_{i,j,b'} (b' < b) pick the
 *   blocks (ties to the lower index).  Exact attention over the keys of every
 *   selected (cluster, block) pair and over the diagonal keys [bS, n]; for every
 *   key cluster, a tilted monopole+dipole summary (tilt qbar_i) of its remaining
 *   keys in blocks < b.  One softmax normaliser over all terms.
 *   Source: gist.science "Kernmechanismen" 3 (causal accumulation over spatial
 *   blocks) and 4 (top-k1 clusters, top-k2 blocks, exact on retrieved pairs plus
 *   the local diagonal, summaries for the rest).
 * Optional outputs: q_labels_out, k_labels_out int32 [B,H,N];
 *   selected_pairs int32 [B,H,Cq,N/block,max(1,k1*k2),2]: (cluster, block) of slot
 *   t*k2+u = the u-th block of the t-th cluster, (-1,-1) when unused.
 * N % block == 0, block a multiple of 64, N/block <= 1024; 0 <= k1 <= Ck;
 * 0 <= k2 <= N/block; k1*k2 <= 64.  Runs on the CUDA cores (float32 arithmetic).
 */
muse_status muse_retrieve_exact(const void *Q, const void *K, const void *V, muse_dims d,
                                int block, int Cq, int Ck, int iters, int k1, int k2,
                                int32_t *q_labels_out, int32_t *k_labels_out,
                                int32_t *selected_pairs, void *O, void *ws, size_t ws_bytes,
                                muse_stream_t st);

/*
 * muse_backward - gradients of the acausal forward pass: dQ, dK, dV of sum(O * dO) for
 *   O = muse_forward's output, with the clusterings held fixed (K-means assignments are
 *   discrete) and each query centroid the mean of its members, so gradients reach Q
 *   through both the centroid and the residual.
 *   Source: pith.science review of arXiv 2509.10406, referee report (the approximation
 *   is used for pretraining, i.e. differentiated; the pages never measure it) and
 *   "What carries the argument" (the quantities differentiated).
 * Inputs:  Q, K, V, dO [B,H,N,*] (d.dtype); q_perm/q_offsets (Cq clusters) and
 *          k_perm/k_offsets (Ck clusters): the clusterings of the forward pass, from
 *          muse_kmeans.
 * Outputs: dQ, dK [B,H,N,D], dV [B,H,N,Dv] in d.dtype.
 * Float32 arithmetic on the CUDA cores, deterministic.  The forward summaries are
 * recomputed; the workspace (muse_workspace_size("muse_backward", ...)) holds the
 * materialised C_ij and its gradient, 8 B*H*Cq*Ck*Dv*D bytes among the rest.
 */
muse_status muse_backward(const void *Q, const void *K, const void *V, const void *dO,
                          const int32_t *q_perm, const int32_t *q_offsets, const int32_t *k_perm,
                          const int32_t *k_offsets, muse_dims d, int Cq, int Ck, void *dQ,
                          void *dK, void *dV, void *ws, size_t ws_bytes, muse_stream_t st);

/*
 * muse_workspace_size - bytes of workspace `entry` needs ("muse_kmeans" with C = Cq,
 * "muse_tilted_summaries", "muse_dipole_refine", "muse_forward", "muse_forward_ex",
 * "muse_causal_blocks", "muse_retrieve_exact", "muse_backward").  Arguments an entry does not
 * use are ignored.  Returns 0 for an unknown entry or invalid sizes.
 */
size_t muse_workspace_size(const char *entry, muse_dims d, int Cq, int Ck, int block, int k1,
                           int k2);

/* muse_status_string - static, human-readable name of a status code. */
const char *muse_status_string(muse_status s);

/*
 * muse_last_error_detail - the CUDA runtime's description of the error behind the
 * calling thread's most recent MUSE_ERR_CUDA ("" if none); valid until the next call
 * into the library on this thread.
 */
const char *muse_last_error_detail(void);

/*
 * muse_last_device_status - synchronises `st`, returns and clears the device status
 * word of the current device (MUSE_OK, MUSE_ERR_TIMEOUT or MUSE_ERR_DEVICE), or
 * MUSE_ERR_CUDA if the synchronisation itself failed.  The word is shared by every
 * call on the device.
 */
muse_status muse_last_device_status(muse_stream_t st);

/*
 * muse_set_test_hooks - failure-path testing aid (no counterpart in the method).
 *   Every wait inside the library's tensor-core kernels is bounded: when it runs out
 *   the kernel records MUSE_ERR_TIMEOUT in the device status word, every warp of the
 *   block winds down (copies and tensor-core work in flight are drained, tensor memory
 *   is freed) and the kernel returns, leaving the context usable.  This call lets a
 *   test make such a wait run out without any fault:
 *     hooks = MUSE_TEST_WITHHOLD_VALUES: the refinement kernel (the tensor-core path of
 *       muse_dipole_refine, muse_forward, muse_causal_blocks) never loads its value
 *       tiles, so the waits for them can only run out;
 *     wait_limit_ns > 0: the limit of the refinement kernel's waits (default 2 s when 0).
 *   The outputs of a call that timed out are undefined.  hooks = 0, wait_limit_ns = 0
 *   restores normal operation.  Applies to the current device, synchronises it first,
 *   and is process-wide: not for use while other work runs on the device.  Unknown hook
 *   bits return MUSE_ERR_INVALID_ARG.
 */
#define MUSE_TEST_WITHHOLD_VALUES 1u
muse_status muse_set_test_hooks(unsigned hooks, uint64_t wait_limit_ns);

/*
 * Instrumentation (no counterpart in the method; used by the benchmark).
 *
 * muse_launch_counter - number of kernels this process has enqueued through the
 *   library so far (host-side count; CUDA-graph replays do not add to it).
 * muse_set_profile_events - when both are non-NULL, every later call records
 *   `start` (a cudaEvent_t) on its stream just before the refinement kernel (the
 *   dominant kernel of every path) and `stop` just after it; NULL, NULL turns it
 *   off.  A process-wide setting: not for concurrent use from several threads.
 */
uint64_t muse_launch_counter(void);
void muse_set_profile_events(void *start, void *stop);

#ifdef __cplusplus
}
#endif

#endif /* MUSE_H */
