// muse_kmeans_noalloc: the K-means entry point for callers that cannot allocate
// device memory and so cannot provide a workspace.  Examples: code that runs
// inside another runtime's memory pool (which owns every device byte and offers
// no allocation hook), code called while a stream capture in global mode is
// active (cudaMalloc is an error there), and latency-critical loops that cannot
// pay for cudaMalloc's implicit synchronisation.  Its scratch is a file-scope
// device array of MUSE_NOALLOC_SCRATCH_BYTES that every GPU loading the library
// holds until the process exits.
#include <mutex>
#include <string.h>

#include "internal.h"

namespace muse {

static __device__ __align__(256) unsigned char g_kmeans_scratch[MUSE_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so its address is looked up once per
// device (with that device current) and cached.
static cudaError_t kmeans_scratch_address(char **out) {
  static std::mutex mu;
  static char *addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_kmeans_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<char *>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace muse

using namespace muse;

extern "C" muse_status muse_kmeans_noalloc(const void *X, muse_dims d, int C, int iters,
                                           int32_t *labels, float *centroids, int32_t *perm,
                                           int32_t *offsets, muse_stream_t st) {
  if (d.dtype != MUSE_F32 && d.dtype != MUSE_BF16) return MUSE_ERR_DTYPE;
  if (d.B <= 0 || d.H <= 0 || d.N <= 0 || (d.D != 64 && d.D != 128)) return MUSE_ERR_SHAPE;
  if ((int64_t)d.B * d.H > 65535 || (int64_t)d.N * 128 > ((int64_t)1 << 31)) return MUSE_ERR_SHAPE;
  if (!X || !labels || !centroids || !perm || !offsets) return MUSE_ERR_INVALID_ARG;
  for (const void *p : {X, (const void *)labels, (const void *)centroids, (const void *)perm,
                        (const void *)offsets})
    if (reinterpret_cast<uintptr_t>(p) & 15u) return MUSE_ERR_INVALID_ARG;
  if (C < 1 || C > d.N || C > kMaxClusters || iters < 1 || iters > 1000)
    return MUSE_ERR_INVALID_ARG;

  SegTable t;
  memset(&t, 0, sizeof(t));
  t.nseg = 1;
  t.row_stride = d.N;
  t.cen_stride = C;
  t.off_stride = C + 1;
  t.max_rows = d.N;
  t.max_C = C;
  t.nrow[0] = d.N;
  t.C[0] = C;
  const int P = d.B * d.H;
  // The multi-launch kernels keep per-chunk label counts, chunk bases and in-chunk ranks
  // in the scratch; a problem of theirs needing more than the array holds is refused
  // before anything runs.  The one-launch kernel (bfloat16, D = 64, C <= 128) keeps all
  // of its state on chip and uses no scratch, so no size limit applies to it.
  if (!kmeans_fused_supported(d.dtype, d.D, t) &&
      kmeans_ws_bytes(t, P, d.D) > (size_t)MUSE_NOALLOC_SCRATCH_BYTES)
    return MUSE_ERR_WORKSPACE;

  char *scratch = nullptr;
  if (kmeans_scratch_address(&scratch) != cudaSuccess) return MUSE_ERR_CUDA;
  // Nothing in the scratch has to start at zero: every word a call reads was written
  // earlier in the same call.
  KmeansOut o{labels, centroids, perm, offsets};
  if (run_kmeans(X, d.dtype, d.D, d.N, t, P, iters, o, scratch, device_status_word(),
                 (cudaStream_t)st) != cudaSuccess)
    return MUSE_ERR_CUDA;
  return MUSE_OK;
}
