// Shared device helpers for libmuse (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "../../include/muse.h"

namespace muse {

// ---------------------------------------------------------------------------
// Element I/O: inputs are float32 or bfloat16; arithmetic is float32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ld_elem(const float *p) { return *p; }
__device__ __forceinline__ float ld_elem(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_elem(float *p, float v) { *p = v; }
__device__ __forceinline__ void st_elem(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// Segment table: the row ranges of the sequence axis that are clustered
// separately.  The same table applies to every (b,h) problem.
//   acausal / retrieval: one segment covering [0, N)
//   causal: one segment per below-diagonal square (its query range on the query
//           side, its key range on the key side)
// Per problem p and segment s:
//   row-indexed arrays (labels, perm, sorted copies) start at p*row_stride + lab0[s]
//   cluster-indexed arrays (centroids, counts)       start at p*cen_stride + cen0[s]
//   offsets arrays (C+1 entries)                      start at p*off_stride + off0[s]
// ---------------------------------------------------------------------------
constexpr int kMaxSeg = 128;
constexpr int kMaxClusters = 1024;

struct SegTable {
  int nseg;
  int row_stride, cen_stride, off_stride;
  int max_rows, max_C;
  int row0[kMaxSeg];
  int nrow[kMaxSeg];
  int C[kMaxSeg];
  int lab0[kMaxSeg];
  int cen0[kMaxSeg];
  int off0[kMaxSeg];
};

// Row stride of the tilt-weight matrix W of an instance with nk sorted keys: padded
// to 8 floats so every row starts 32-byte aligned.
__host__ __device__ __forceinline__ int w_ld(int nk) { return (nk + 7) & ~7; }
// Row stride of the transposed sorted values (keys innermost): 8 elements (16 bytes).
__host__ __device__ __forceinline__ int vt_ld(int row_stride) { return (row_stride + 7) & ~7; }

// A task is one (problem, segment) pair.
struct Task {
  int p, s;
  int row0, n, C;
  int64_t lab, cen, off;  // absolute element offsets of the task's arrays
};

__host__ __device__ __forceinline__ Task make_task(const SegTable &t, int task) {
  Task k;
  k.p = task / t.nseg;
  k.s = task - k.p * t.nseg;
  k.row0 = t.row0[k.s];
  k.n = t.nrow[k.s];
  k.C = t.C[k.s];
  k.lab = (int64_t)k.p * t.row_stride + t.lab0[k.s];
  k.cen = (int64_t)k.p * t.cen_stride + t.cen0[k.s];
  k.off = (int64_t)k.p * t.off_stride + t.off0[k.s];
  return k;
}

// Blocks of `rows` consecutive rows of every segment of a table, numbered segment
// after segment: a compact grid (no block lies past its segment's rows, which matters
// when the segments differ in size, as the squares of the causal decomposition do).
struct BlockMap {
  int total;
  int pre[kMaxSeg + 1];  // first block of segment s; pre[nseg] = total
};
inline BlockMap make_block_map(const SegTable &t, int rows) {
  BlockMap m;
  m.pre[0] = 0;
  for (int s = 0; s < t.nseg; ++s) m.pre[s + 1] = m.pre[s] + (t.nrow[s] + rows - 1) / rows;
  for (int s = t.nseg + 1; s <= kMaxSeg; ++s) m.pre[s] = m.pre[t.nseg];
  m.total = m.pre[t.nseg];
  return m;
}
// Segment of block b (the last segment whose first block is <= b) and its first block.
__device__ __forceinline__ int map_block(const BlockMap &m, int nseg, int b, int &first) {
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (m.pre[mid] <= b) lo = mid;
    else hi = mid - 1;
  }
  first = m.pre[lo];
  return lo;
}

// ---------------------------------------------------------------------------
// Device status block, one per device.  Kernels get its address as a parameter.
//   [0]    status word (MUSE_OK / MUSE_ERR_TIMEOUT / MUSE_ERR_DEVICE); first error wins
//   [1]    test hooks (MUSE_TEST_* bits of muse_set_test_hooks; 0 in normal use)
//   [2..3] wait limit in nanoseconds for the kernels that honour it (0 = default)
// ---------------------------------------------------------------------------
constexpr int kStatusInts = 4;
__device__ __forceinline__ unsigned test_hooks(const int *status) {
  return status ? (unsigned)*reinterpret_cast<const volatile int *>(status + 1) : 0u;
}
__device__ __forceinline__ void report(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace muse
