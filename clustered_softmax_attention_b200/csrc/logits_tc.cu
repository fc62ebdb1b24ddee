// Tilt logits on the tensor cores (bfloat16 keys, D = 64 or 128):
//   L[i][pos] = s qbar_i . k_pos
// for every query centroid i and sorted key position pos of an instance, written into the
// tilt-weight array W, where the tilt stage (tilt_fused in stages.cu) turns them into
// log-normalisers, weights and tilted key means (pith.science review of arXiv 2509.10406,
// "Assumptions & free parameters": log M_j(q) = log E exp(q . k) of a key cluster).
//
// One CTA = 128 query centroids (TMEM lanes, thread t owns centroid i0 + t) and up to
// kTiles consecutive 128-key tiles of one instance.  The centroids enter the product as
// three bfloat16 parts (qbar = c0 + c1 + c2, 24 significant bits), so the logits keep
// float32 accuracy against the float32 centroids; the keys are the bfloat16 inputs.
//   L = qbar . K_tile^T    tcgen05.mma, M = 128, N = 128, K = D, fp32 in TMEM (two buffers)
// Key tiles arrive by TMA two ahead; the product of tile t + 1 is issued before tile t is
// read out, so the read-out (TMEM -> registers -> 16-byte stores of each centroid's row)
// overlaps the next product.  Thread 0 issues the copies and the products; every wait is
// bounded.
#include "internal.h"
#include "tc_ptx.cuh"

namespace muse {
namespace ltc {

using namespace ptx;

constexpr int TM = 128;     // centroids per CTA, keys per tile
constexpr int kTiles = 2;   // key tiles per CTA (at most): 256 CTAs at N = 8k, 8 heads

template <int D> struct __align__(1024) Smem {
  __nv_bfloat16 c[3][D / 64][TM * 64];  // centroid parts, K-major, 128-byte swizzle
  __nv_bfloat16 k[2][D / 64][TM * 64];  // key tiles (TMA, same layout)
  uint64_t lbar[2], mbar[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(TM)
logits_tc(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ MuseTables mt,
          float scale, const float *__restrict__ qcen, float *__restrict__ W,
          const __grid_constant__ BlockMap bm, int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem<D> &sm = *reinterpret_cast<Smem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const int t = threadIdx.x, warp = t >> 5;
  int bfirst;
  const int p = blockIdx.z, s = map_block(bm, mt.in.ninst, blockIdx.x, bfirst);
  const Task q = make_task(mt.q, p * mt.q.nseg + s), k = make_task(mt.k, p * mt.k.nseg + s);
  const int Cq = q.C, nk = k.n, i0 = blockIdx.y * TM;
  const int tile0 = ((int)blockIdx.x - bfirst) * kTiles;
  const int ntile = min(kTiles, (nk + TM - 1) / TM - tile0);
  if (ntile <= 0 || i0 >= Cq) return;  // uniform
  volatile int *abort_flag = &sm.abort_flag;

  if (t == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.lbar[b], 1);
      mbar_init(&sm.mbar[b], 1);
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(&sm.tmem_base)),
                 "r"(2u * TM)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // the centroids in three bfloat16 parts: 8 consecutive coordinates per item
  for (int u = t; u < TM * (D / 8); u += TM) {
    const int r = u / (D / 8), c = u % (D / 8);
    float v[8];
    if (i0 + r < Cq) {
      const float4 *src = reinterpret_cast<const float4 *>(qcen + (q.cen + i0 + r) * D + 8 * c);
      const float4 x = __ldg(src), y = __ldg(src + 1);
      v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
      v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
    } else {
#pragma unroll
      for (int x = 0; x < 8; ++x) v[x] = 0.f;
    }
    const int kb = c >> 3, off = r * 64 + (((c & 7) ^ (r & 7)) << 3);
#pragma unroll
    for (int part = 0; part < 3; ++part) {
      uint32_t w4[4];
#pragma unroll
      for (int x = 0; x < 8; x += 2) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[x], v[x + 1]);
        const float2 hf = __bfloat1622float2(h);
        v[x] -= hf.x;
        v[x + 1] -= hf.y;
        w4[x >> 1] = *reinterpret_cast<const uint32_t *>(&h);
      }
      *reinterpret_cast<uint4 *>(&sm.c[part][kb][off]) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // centroid parts -> tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  auto load = [&](int tt) {  // thread 0: key tile tt into buffer tt & 1
    const int b = tt & 1;
    mbar_expect_tx(&sm.lbar[b], (uint32_t)(D / 64) * TM * 128);
    for (int kb = 0; kb < D / 64; ++kb)
      tma_load_2d(sm.k[b][kb], &map_k, kb * 64, (int)(k.lab + (int64_t)(tile0 + tt) * TM), &sm.lbar[b]);
  };
  auto product = [&](int tt) {  // thread 0, after the tile's keys have landed
    const int b = tt & 1;
    tc_fence_after();
    constexpr uint32_t id = idesc(TM, TM);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t bd = sdesc(sm.k[b][kk >> 2] + (kk & 3) * 16);
#pragma unroll
      for (int part = 0; part < 3; ++part)
        tc_mma(tmem + b * TM, sdesc(sm.c[part][kk >> 2] + (kk & 3) * 16), bd, id,
               (kk > 0 || part > 0) ? 1u : 0u);
    }
    tc_commit(&sm.mbar[b]);
  };
  // loads issued per buffer, products committed per buffer (thread 0; for the teardown)
  int nl[2] = {0, 0}, nm[2] = {0, 0};
  bool ok = true;
  if (t == 0) {
    load(0);
    ++nl[0];
    if (ntile > 1) {
      load(1);
      ++nl[1];
    }
    ok = mbar_wait(&sm.lbar[0], 0, abort_flag, status);
    if (ok) {
      product(0);
      ++nm[0];
    }
  }
  ok = __syncthreads_and(ok);
  const int i = i0 + t;
  const int wl = w_ld(nk);
  float *wrow = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s] + (int64_t)i * wl;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  for (int tt = 0; ok && tt < ntile; ++tt) {
    const int b = tt & 1;
    // tile tt's logits (its keys are consumed: the buffer takes tile tt + 2)
    bool r = mbar_wait(&sm.mbar[b], (tt >> 1) & 1, abort_flag, status);
    tc_fence_after();
    if (t == 0 && r) {
      if (tt + 2 < ntile) {
        load(tt + 2);
        ++nl[b];
      }
      if (tt + 1 < ntile) {  // the next product, into the other buffer (read out last step)
        r = mbar_wait(&sm.lbar[b ^ 1], ((tt + 1) >> 1) & 1, abort_flag, status);
        if (r) {
          product(tt + 1);
          ++nm[b ^ 1];
        }
      }
    }
    if (!(ok = __syncthreads_and(r))) break;
    // read-out: scale and store the row's valid keys, 16-byte stores (rows start on
    // 8-float boundaries, tiles on 128-key boundaries)
    const int pos0 = (tile0 + tt) * TM;
    const int nv = min(TM, nk - pos0);
    for (int cb = 0; cb < TM; cb += 16) {
      float x[16];
      tmem_ld16(tmem + lane_base + b * TM + cb, x);
      if (i < Cq) {
        float4 *dst = reinterpret_cast<float4 *>(wrow + pos0 + cb);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int col = cb + 4 * u;
          if (col + 3 < nv) {
            dst[u] = make_float4(scale * x[4 * u], scale * x[4 * u + 1], scale * x[4 * u + 2],
                                 scale * x[4 * u + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (col + e < nv) wrow[pos0 + col + e] = scale * x[4 * u + e];
          }
        }
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok);  // buffer b is read: the product of tile tt + 2 may overwrite it
  }
  // copies and products still in flight land before the CTA releases its memory
  if (t == 0) {
    for (int b = 0; b < 2; ++b) {
      if (nl[b] > 0) mbar_drain(&sm.lbar[b], (nl[b] - 1) & 1, status);
      if (nm[b] > 0) mbar_drain(&sm.mbar[b], (nm[b] - 1) & 1, status);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2u * TM)
                 : "memory");
  }
}

template <int D>
static cudaError_t launch(const MuseTables &mt, int P, float scale, const float *qcen,
                          const void *ks_rows, float *W, int *status, cudaStream_t st) {
  BlockMap bm;  // ceil(tiles / kTiles) blocks per instance
  bm.pre[0] = 0;
  for (int si = 0; si < mt.in.ninst; ++si) {
    const int tiles = (mt.k.nrow[si] + TM - 1) / TM;
    bm.pre[si + 1] = bm.pre[si] + (tiles + kTiles - 1) / kTiles;
  }
  for (int si = mt.in.ninst + 1; si <= kMaxSeg; ++si) bm.pre[si] = bm.pre[mt.in.ninst];
  bm.total = bm.pre[mt.in.ninst];
  if (bm.total == 0) return cudaSuccess;
  CUtensorMap mk;
  if (!make_map(&mk, ks_rows, D, (uint64_t)P * mt.k.row_stride, D, TM)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem<D>) + 1024;
  auto kern = logits_tc<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(bm.total, (mt.q.max_C + TM - 1) / TM, P), TM, smem, st>>>(mk, mt, scale, qcen, W,
                                                                         bm, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ltc

bool logits_tc_supported(int dtype, int D) { return dtype == MUSE_BF16 && (D == 64 || D == 128); }

cudaError_t run_logits_tc(const MuseTables &mt, int D, int P, float scale, const float *q_centroids,
                          const void *ks_rows, float *W, int *status, cudaStream_t st) {
  return D == 64 ? ltc::launch<64>(mt, P, scale, q_centroids, ks_rows, W, status, st)
                 : ltc::launch<128>(mt, P, scale, q_centroids, ks_rows, W, status, st);
}

}  // namespace muse
