// Lloyd K-means over the segments of a SegTable, batched over (problem, segment).
//
// Separate K-means over queries and over keys: pith.science review of arXiv
// 2509.10406, "What carries the argument" / "Core claim"; gist.science
// "Technische Samenvatting", "Kernmechanismen" item 1.
//
// One round = assign (nearest centroid, ties to the lowest index) + update (mean of
// the members, an empty cluster keeps its centroid).  The update is a stable
// counting sort of the rows by label (perm/offsets, the CSR layout every later
// stage reads) followed by per-cluster sums taken over the sorted members in row
// order: no floating-point atomics, bitwise reproducible.
//
// Per round: km_assign_count (distances, argmin, per-chunk label histogram and
// in-chunk stable rank), km_scan (per-cluster chunk bases, offsets), km_scatter
// (perm), km_centroid (means).
#include "internal.h"

namespace muse {

constexpr int kChunk = 256;   // rows per assign CTA (= rows per counting-sort chunk)
constexpr int kCTile = 64;    // centroids staged in shared memory at a time

template <typename T, int D>
__global__ void km_init(const T *__restrict__ X, int N, SegTable tab,
                        float *__restrict__ centroids) {
  Task tk = make_task(tab, blockIdx.x);
  const T *x = X + ((int64_t)tk.p * N + tk.row0) * D;
  float *c = centroids + tk.cen * D;
  for (int e = threadIdx.x; e < tk.C * D; e += blockDim.x) c[e] = ld_elem(x + e);
}

template <typename T, int D>
__global__ void __launch_bounds__(kChunk)
km_assign_count(const T *__restrict__ X, int N, SegTable tab, const float *__restrict__ centroids,
                int32_t *__restrict__ labels, int32_t *__restrict__ counts,
                int32_t *__restrict__ lrank, int nchunks_max) {
  extern __shared__ float smem[];
  float *cs = smem;                                // [kCTile][D]
  int *cnt = reinterpret_cast<int *>(smem + kCTile * D);  // [8][C]
  const Task tk = make_task(tab, blockIdx.y);
  const int chunk = blockIdx.x;
  if (chunk * kChunk >= tk.n) return;  // uniform over the CTA
  const int r = chunk * kChunk + threadIdx.x;
  const bool valid = r < tk.n;

  float x[D];
  if (valid) {
    const T *xr = X + ((int64_t)tk.p * N + tk.row0 + r) * D;
#pragma unroll
    for (int d = 0; d < D; ++d) x[d] = ld_elem(xr + d);
  }
  float best = CUDART_INF_F;
  int bi = 0;
  const float *cg = centroids + tk.cen * D;
  for (int c0 = 0; c0 < tk.C; c0 += kCTile) {
    const int ct = min(kCTile, tk.C - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < ct * D; e += blockDim.x) cs[e] = cg[(int64_t)c0 * D + e];
    __syncthreads();
    if (valid) {
      for (int c = 0; c < ct; ++c) {
        const float *cc = cs + c * D;
        float d2 = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          const float t = x[d] - cc[d];
          d2 = fmaf(t, t, d2);
        }
        if (d2 < best) {  // strict: the lowest index wins a tie
          best = d2;
          bi = c0 + c;
        }
      }
    }
  }
  const int L = valid ? bi : -1;
  if (valid) labels[tk.lab + r] = L;

  // per-chunk histogram and stable in-chunk rank
  for (int e = threadIdx.x; e < 8 * tk.C; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const unsigned peers = __match_any_sync(0xffffffffu, L);
  const int wrank = __popc(peers & ((1u << lane) - 1u));
  if (valid && wrank == 0) cnt[w * tk.C + L] = __popc(peers);
  __syncthreads();
  if (valid) {
    int before = 0;
    for (int w2 = 0; w2 < w; ++w2) before += cnt[w2 * tk.C + L];
    lrank[tk.lab + r] = before + wrank;
  }
  int32_t *out = counts + ((int64_t)blockIdx.y * nchunks_max + chunk) * tab.max_C;
  for (int c = threadIdx.x; c < tk.C; c += blockDim.x) {
    int s = 0;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) s += cnt[w2 * tk.C + c];
    out[c] = s;
  }
}

// One CTA of 1024 threads per task: thread c walks the chunks in order.
__global__ void __launch_bounds__(1024)
km_scan(SegTable tab, const int32_t *__restrict__ counts, int32_t *__restrict__ base,
        int32_t *__restrict__ offsets, int nchunks_max) {
  __shared__ int tot[kMaxClusters];
  const Task tk = make_task(tab, blockIdx.x);
  const int nch = (tk.n + kChunk - 1) / kChunk;
  const int c = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * nchunks_max * tab.max_C;
  int run = 0;
  if (c < tk.C) {
    for (int ch = 0; ch < nch; ++ch) {
      base[t0 + (int64_t)ch * tab.max_C + c] = run;
      run += counts[t0 + (int64_t)ch * tab.max_C + c];
    }
  }
  tot[c] = (c < tk.C) ? run : 0;
  __syncthreads();
  // inclusive Hillis-Steele scan over 1024 entries
  for (int o = 1; o < kMaxClusters; o <<= 1) {
    const int v = (c >= o) ? tot[c - o] : 0;
    __syncthreads();
    tot[c] += v;
    __syncthreads();
  }
  const int excl = tot[c] - run;
  if (c < tk.C) {
    offsets[tk.off + c] = excl;
    for (int ch = 0; ch < nch; ++ch) base[t0 + (int64_t)ch * tab.max_C + c] += excl;
  }
  if (c == 0) offsets[tk.off + tk.C] = tk.n;
}

__global__ void __launch_bounds__(kChunk)
km_scatter(SegTable tab, const int32_t *__restrict__ labels, const int32_t *__restrict__ lrank,
           const int32_t *__restrict__ base, int32_t *__restrict__ perm, int nchunks_max,
           int *status) {
  const Task tk = make_task(tab, blockIdx.y);
  const int chunk = blockIdx.x;
  const int r = chunk * kChunk + threadIdx.x;
  if (r >= tk.n) return;
  const int L = labels[tk.lab + r];
  const int pos = base[((int64_t)blockIdx.y * nchunks_max + chunk) * tab.max_C + L] +
                  lrank[tk.lab + r];
  if (pos < 0 || pos >= tk.n) {
    report(status, MUSE_ERR_DEVICE);
    return;
  }
  perm[tk.lab + pos] = tk.row0 + r;  // sequence row index
}

// One CTA per (cluster, task); thread d sums coordinate d over the members in row order.
template <typename T, int D>
__global__ void km_centroid(const T *__restrict__ X, int N, SegTable tab,
                            const int32_t *__restrict__ perm, const int32_t *__restrict__ offsets,
                            float *__restrict__ centroids) {
  const Task tk = make_task(tab, blockIdx.y);
  const int c = blockIdx.x;
  if (c >= tk.C) return;
  const int b = offsets[tk.off + c], e = offsets[tk.off + c + 1];
  if (e <= b) return;  // empty: keep the previous centroid
  const T *xp = X + (int64_t)tk.p * N * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float s = 0.f;
    for (int m = b; m < e; ++m) s += ld_elem(xp + (int64_t)perm[tk.lab + m] * D + d);
    centroids[(tk.cen + c) * D + d] = s / (float)(e - b);
  }
}

size_t kmeans_ws_bytes(const SegTable &t, int P) {
  const int64_t tasks = (int64_t)P * t.nseg;
  const int64_t nch = (t.max_rows + kChunk - 1) / kChunk;
  const size_t cnt = (size_t)(tasks * nch * t.max_C) * sizeof(int32_t);
  const size_t lr = (size_t)P * t.row_stride * sizeof(int32_t);
  return align_up(cnt) * 2 + align_up(lr);
}

template <typename T, int D>
static cudaError_t run_kmeans_t(const T *X, int N, const SegTable &tab, int P, int iters,
                                const KmeansOut &o, char *ws, int *status, cudaStream_t st) {
  const int tasks = P * tab.nseg;
  const int nch = (tab.max_rows + kChunk - 1) / kChunk;
  const size_t cnt_bytes = align_up((size_t)tasks * nch * tab.max_C * sizeof(int32_t));
  int32_t *counts = reinterpret_cast<int32_t *>(ws);
  int32_t *base = reinterpret_cast<int32_t *>(ws + cnt_bytes);
  int32_t *lrank = reinterpret_cast<int32_t *>(ws + 2 * cnt_bytes);
  const size_t smem = (size_t)kCTile * D * sizeof(float) + 8 * (size_t)tab.max_C * sizeof(int);
  cudaError_t err = cudaFuncSetAttribute(km_assign_count<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  km_init<T, D><<<tasks, 256, 0, st>>>(X, N, tab, o.centroids);
  count_launches(1 + 4 * iters);
  for (int it = 0; it < iters; ++it) {
    km_assign_count<T, D><<<dim3(nch, tasks), kChunk, smem, st>>>(X, N, tab, o.centroids, o.labels,
                                                                   counts, lrank, nch);
    km_scan<<<tasks, 1024, 0, st>>>(tab, counts, base, o.offsets, nch);
    km_scatter<<<dim3(nch, tasks), kChunk, 0, st>>>(tab, o.labels, lrank, base, o.perm, nch,
                                                     status);
    km_centroid<T, D><<<dim3(tab.max_C, tasks), D, 0, st>>>(X, N, tab, o.perm, o.offsets,
                                                             o.centroids);
  }
  return cudaGetLastError();
}

cudaError_t run_kmeans(const void *X, int dtype, int D, int N, const SegTable &tab, int P,
                       int iters, const KmeansOut &o, char *ws, int *status, cudaStream_t st) {
  if (dtype == MUSE_F32) {
    if (D == 64) return run_kmeans_t<float, 64>((const float *)X, N, tab, P, iters, o, ws, status, st);
    return run_kmeans_t<float, 128>((const float *)X, N, tab, P, iters, o, ws, status, st);
  }
  if (D == 64)
    return run_kmeans_t<__nv_bfloat16, 64>((const __nv_bfloat16 *)X, N, tab, P, iters, o, ws, status, st);
  return run_kmeans_t<__nv_bfloat16, 128>((const __nv_bfloat16 *)X, N, tab, P, iters, o, ws, status, st);
}

}  // namespace muse
