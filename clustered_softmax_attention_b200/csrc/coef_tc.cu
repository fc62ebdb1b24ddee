// Refinement coefficients on the tensor cores (bfloat16 residuals, D = 64 or 128,
// Ck <= 256).  Same result as refine_coeffs_tiled in stages.cu:
//   a_j = logZ_ij + s u_j,  u_j = qt_n . mu_k,ij;  p = softmax_j(a);
//   c0[j][n] = p_j (1 - sd u_j),  c1[j][n] = sd p_j,  lse[n] = logsumexp_j a_j
// (pith.science review of arXiv 2509.10406, "What carries the argument": the residual
// refines the tilted summaries through qt.mu_k; gist.science "Kernmechanismen" 1-2).
//
// One CTA = one query cluster i and up to 128 of its sorted rows.  The projections
// U = Qt . mu_k,i^T are one tcgen05 product: M = 128 rows (TMA tile of the sorted
// residuals, rows of other clusters included and ignored), N = the Ck key clusters
// (padded to CK), K = D.  The float32 means enter as a split mu = mu_hi + mu_lo of two
// bfloat16 parts (two accumulating products), so u keeps about 16 bits of the means;
// the residual rows are the same bfloat16 rows the refinement contracts.  Thread t owns
// row t (TMEM lane t): one pass over its CK columns for the maximum and the sum of the
// softmax, a second one for the coefficients, stored column by column (each warp writes
// 32 consecutive rows of c0[j], c1[j]: coalesced).  Thread 0 issues the copy and the
// products; every wait is bounded.
#include <algorithm>

#include "internal.h"
#include "tc_ptx.cuh"

namespace muse {
namespace ctc {

using namespace ptx;

constexpr int TM = 128;  // rows per CTA

// Packed float32 pairs in 64-bit registers (low word = first element).
__device__ __forceinline__ unsigned long long pack2(float a, float b) {
  unsigned long long v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(a), "f"(b));
  return v;
}
__device__ __forceinline__ void unpack2(unsigned long long v, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ void ffma2(unsigned long long &acc, unsigned long long a, unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// Output mode: the monopole-only method and the partially specialised dipole evaluated
// in summary form, O_n = sum_j p_j mu_v,ij (+ s Cbar_i qt_n), Dv = 64, on the tensor cores:
//   O  = Qt . (s Cbar_i)^T        (partial dipole; B = split s Cbar_i, K-major [dv][d])
//   O += P . mu_v,i               (A = P, bf16, from TMEM; B = split mu_v,i as stored,
//                                  [j][dv] with dv innermost: an MN-major operand)
// with P = softmax_j(logZ_ij + s u_j) of each row, u from the first product as above.
constexpr int OV = 64;  // Dv of the output mode
struct CoefOut {
  const float *mu_v;      // [P][z_stride][OV] tilted value means
  const float *cbar;      // [P][Cq][OV][D] aggregated covariances, or null (monopole only)
  const int32_t *q_perm;  // sorted position -> sequence row
  __nv_bfloat16 *O;       // [P][N][OV]
  int N;
  float s;                // factor of the covariance term
};

template <int D, int CK, bool OUT> struct __align__(1024) Smem {
  __nv_bfloat16 q[D / 64][TM * 64];          // residual rows, K-major SW128 (TMA)
  __nv_bfloat16 hi[D / 64][CK * 64];         // mu_k split, same layout
  __nv_bfloat16 lo[D / 64][CK * 64];
  __nv_bfloat16 vh[OUT ? CK * 64 : 64];      // output mode: mu_v split, MN-major SW128
  __nv_bfloat16 vl[OUT ? CK * 64 : 64];
  __nv_bfloat16 ch[OUT ? D / 64 : 1][OUT ? OV * 64 : 64];  // output mode: s Cbar split, K-major
  __nv_bfloat16 cl[OUT ? D / 64 : 1][OUT ? OV * 64 : 64];
  float lz[CK];
  float2 ml[2][TM];                          // per half: running maximum and sum of each row
  uint64_t lbar, mbar;
  uint32_t tmem_base;
  int abort_flag;
  int s_i, s_r0;
};

// bfloat16 split x = hi + lo of 8 values, as two 16-byte units
__device__ __forceinline__ void split8(const float (&v)[8], uint4 &hi, uint4 &lo) {
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int x = 0; x < 8; x += 2) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[x], v[x + 1]);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(v[x] - hf.x, v[x + 1] - hf.y);
    hw[x >> 1] = *reinterpret_cast<const uint32_t *>(&h);
    lw[x >> 1] = *reinterpret_cast<const uint32_t *>(&l);
  }
  hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// Shared-memory descriptor of an MN-major operand, 128-byte swizzle, one 64-element
// block along N (rows of 128 B, one per K index; 8 K-rows per 1024-B atom).
__device__ __forceinline__ uint64_t sdesc_mn64(const void *p) {
  const uint32_t a = saddr(p);
  uint64_t d = 0;
  d |= (uint64_t)((a & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

template <int D, int CK, bool OUT>
__global__ void __launch_bounds__(2 * TM)
coef_tc(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ MuseTables mt,
        float scale, const int32_t *__restrict__ q_offsets, const float *__restrict__ logZ,
        const float *__restrict__ mu_k, float *__restrict__ c0, float *__restrict__ c1,
        float *__restrict__ lse, const __grid_constant__ InstMask skip, float sdip,
        const __grid_constant__ CoefOut oa, const __grid_constant__ BlockMap bm, int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem<D, CK, OUT> &sm = *reinterpret_cast<Smem<D, CK, OUT> *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  // blockIdx.x: a chunk slot of one instance (compact grid over this kernel's instances),
  // blockIdx.y: the problem
  int bfirst;
  const int p = blockIdx.y, s = map_block(bm, mt.in.ninst, blockIdx.x, bfirst);
  const int chunk = (int)blockIdx.x - bfirst;
  if ((skip.w[s >> 5] >> (s & 31)) & 1u) return;  // uniform: another kernel's instance
  const Task q = make_task(mt.q, p * mt.q.nseg + s), k = make_task(mt.k, p * mt.k.nseg + s);
  // this CTA's chunk of the instance, counting ceil(rows / 128) chunks
  // per query cluster in cluster order
  if (warp == 0) {
    int run = 0, found = -1, fr0 = 0;
    for (int cb = 0; cb < q.C && found < 0; cb += 32) {
      const int c = cb + lane;
      int nch = 0, bb = 0;
      if (c < q.C) {
        bb = q_offsets[q.off + c];
        nch = (q_offsets[q.off + c + 1] - bb + TM - 1) / TM;
      }
      int inc = nch;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const int first = run + inc - nch;
      const bool mine = chunk >= first && chunk < first + nch;
      const unsigned bal = __ballot_sync(0xffffffffu, mine);
      if (bal) {
        const int src = __ffs(bal) - 1;
        found = __shfl_sync(0xffffffffu, c, src);
        fr0 = __shfl_sync(0xffffffffu, bb + TM * (chunk - first), src);
      }
      run += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) {
      sm.s_i = found;
      sm.s_r0 = fr0;
    }
  }
  __syncthreads();
  const int i = sm.s_i;
  if (i < 0) return;  // uniform: past the instance's last chunk
  const int r0 = sm.s_r0, Ck = k.C;
  const int e = q_offsets[q.off + i + 1];
  volatile int *abort_flag = &sm.abort_flag;

  if (t == 0) {
    mbar_init(&sm.lbar, 1);
    mbar_init(&sm.mbar, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // TMEM columns: U [0, CK); output mode: O [CK, CK + OV), P (packed) [CK + OV, CK + OV + CK / 2)
  constexpr uint32_t kCols = OUT ? (CK > 128 ? 512u : 256u) : (uint32_t)CK;
  constexpr uint32_t kO = CK, kP = CK + OV;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(&sm.tmem_base)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (t == 0) {
    mbar_expect_tx(&sm.lbar, (uint32_t)(D / 64) * TM * 128);
    for (int kb = 0; kb < D / 64; ++kb)
      tma_load_2d(sm.q[kb], &map_q, kb * 64, (int)(q.lab + r0), &sm.lbar);
  }
  // the split means of cluster i: 8 consecutive coordinates per item (zero past Ck)
  const int64_t zrow = (int64_t)p * mt.in.z_stride + mt.in.z0[s] + (int64_t)i * Ck;
  for (int u = t; u < CK * (D / 8); u += 2 * TM) {
    const int j = u / (D / 8), c = u % (D / 8);
    float v[8];
    if (j < Ck) {
      const float4 *src = reinterpret_cast<const float4 *>(mu_k + (zrow + j) * D + 8 * c);
      const float4 x = __ldg(src), y = __ldg(src + 1);
      v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
      v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
    } else {
#pragma unroll
      for (int x = 0; x < 8; ++x) v[x] = 0.f;
    }
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int x = 0; x < 8; x += 2) {
      const __nv_bfloat162 hh = __floats2bfloat162_rn(v[x], v[x + 1]);
      const float2 hf = __bfloat1622float2(hh);
      const __nv_bfloat162 ll = __floats2bfloat162_rn(v[x] - hf.x, v[x + 1] - hf.y);
      hw[x >> 1] = *reinterpret_cast<const uint32_t *>(&hh);
      lw[x >> 1] = *reinterpret_cast<const uint32_t *>(&ll);
    }
    const int kb = c >> 3, off = j * 64 + (((c & 7) ^ (j & 7)) << 3);
    *reinterpret_cast<uint4 *>(&sm.hi[kb][off]) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4 *>(&sm.lo[kb][off]) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
  for (int j = t; j < CK; j += 2 * TM) sm.lz[j] = j < Ck ? logZ[zrow + j] : -CUDART_INF_F;
  if constexpr (OUT) {
    // mu_v,i split, rows j (zero past Ck) of 64 values, 16-byte unit c at c ^ (j & 7)
    for (int u = t; u < CK * (OV / 8); u += 2 * TM) {
      const int j = u / (OV / 8), c = u % (OV / 8);
      float v[8];
      if (j < Ck) {
        const float4 *src = reinterpret_cast<const float4 *>(oa.mu_v + (zrow + j) * OV + 8 * c);
        const float4 x = __ldg(src), y = __ldg(src + 1);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
      } else {
#pragma unroll
        for (int x = 0; x < 8; ++x) v[x] = 0.f;
      }
      uint4 h4, l4;
      split8(v, h4, l4);
      const int off = j * 64 + ((c ^ (j & 7)) << 3);
      *reinterpret_cast<uint4 *>(&sm.vh[off]) = h4;
      *reinterpret_cast<uint4 *>(&sm.vl[off]) = l4;
    }
    // s Cbar_i split, rows dv of D values (K-major, blocks of 64)
    if (oa.cbar) {
      const float *cbi = oa.cbar + ((int64_t)p * q.C + i) * OV * D;
      for (int u = t; u < OV * (D / 8); u += 2 * TM) {
        const int dv = u / (D / 8), c = u % (D / 8);
        const float4 *src = reinterpret_cast<const float4 *>(cbi + (int64_t)dv * D + 8 * c);
        const float4 x = __ldg(src), y = __ldg(src + 1);
        float v[8] = {oa.s * x.x, oa.s * x.y, oa.s * x.z, oa.s * x.w,
                      oa.s * y.x, oa.s * y.y, oa.s * y.z, oa.s * y.w};
        uint4 h4, l4;
        split8(v, h4, l4);
        const int off = dv * 64 + (((c & 7) ^ (dv & 7)) << 3);
        *reinterpret_cast<uint4 *>(&sm.ch[c >> 3][off]) = h4;
        *reinterpret_cast<uint4 *>(&sm.cl[c >> 3][off]) = l4;
      }
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // split means -> tensor cores
  __syncthreads();
  bool ok = true;
  if (t == 0) {
    ok = mbar_wait(&sm.lbar, 0, abort_flag, status);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t id = idesc(TM, CK);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t a = sdesc(sm.q[kk >> 2] + (kk & 3) * 16);
        tc_mma(tmem, a, sdesc(sm.hi[kk >> 2] + (kk & 3) * 16), id, kk > 0 ? 1u : 0u);
        tc_mma(tmem, a, sdesc(sm.lo[kk >> 2] + (kk & 3) * 16), id, 1u);
      }
      if constexpr (OUT) {
        if (oa.cbar) {  // O = Qt . (s Cbar_i)^T
          constexpr uint32_t io = idesc(TM, OV);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sdesc(sm.q[kk >> 2] + (kk & 3) * 16);
            tc_mma(tmem + kO, a, sdesc(sm.ch[kk >> 2] + (kk & 3) * 16), io, kk > 0 ? 1u : 0u);
            tc_mma(tmem + kO, a, sdesc(sm.cl[kk >> 2] + (kk & 3) * 16), io, 1u);
          }
        }
      }
    }
    tc_commit(&sm.mbar);  // also when the load gave up: the drain below waits for it
  }
  ok = __syncthreads_and(ok);
  if (ok) ok = __syncthreads_and(mbar_wait(&sm.mbar, 0, abort_flag, status));
  tc_fence_after();
  // two threads per row (warps w and w + 4 read the same TMEM lanes), each taking half of
  // the CK columns; their softmax partials meet in shared memory
  const int rr = t % TM, hh = t / TM;
  const int n = r0 + rr;  // the thread's sorted row within the instance
  bool second = false;    // thread 0: the output product was committed (phase 1)
  const bool mine = n < e;
  constexpr int HC = CK / 2;
  if (ok) {  // CTA-uniform: the TMEM loads are warp-collective
    const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16) + hh * HC;
    const float *lzh = sm.lz + hh * HC;
    float m = -CUDART_INF_F, l = 0.f;
    for (int cb = 0; cb < HC; cb += 16) {
      float x[16];
      tmem_ld16(ta + cb, x);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float a = fmaf(scale, x[c], lzh[cb + c]);
        if (a > m) {
          l = l * __expf(m - a) + 1.f;
          m = a;
        } else if (a > -CUDART_INF_F) {
          l += __expf(a - m);
        }
      }
    }
    sm.ml[hh][rr] = make_float2(m, l);
    __syncthreads();
    {
      const float2 o = sm.ml[hh ^ 1][rr];
      const float mm = fmaxf(m, o.x);
      l = (m > -CUDART_INF_F ? l * __expf(m - mm) : 0.f) + (o.x > -CUDART_INF_F ? o.y * __expf(o.x - mm) : 0.f);
      m = mm;
    }
    const float inv = 1.f / l;
    if constexpr (OUT) {
      // P (bfloat16, packed two per column) for this thread's half of the key clusters
      for (int cb = 0; cb < HC; cb += 16) {
        float x[16];
        tmem_ld16(ta + cb, x);
        uint32_t pk[8];
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          const float a0 = fmaf(scale, x[c], lzh[cb + c]), a1 = fmaf(scale, x[c + 1], lzh[cb + c + 1]);
          const float p0 = a0 > -CUDART_INF_F ? __expf(a0 - m) * inv : 0.f;
          const float p1 = a1 > -CUDART_INF_F ? __expf(a1 - m) * inv : 0.f;
          __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          pk[c >> 1] = *reinterpret_cast<uint32_t *>(&h2);
        }
        tmem_st8(tmem + ((uint32_t)((warp & 3) * 32) << 16) + kP + (hh * HC + cb) / 2, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncthreads();  // P complete
      bool r3 = true;
      if (t == 0) {  // O (+)= P . mu_v,i
        second = true;
        tc_fence_after();
        constexpr uint32_t iv = idesc(TM, OV) | (1u << 16);  // B MN-major
#pragma unroll
        for (int kk = 0; kk < CK / 16; ++kk) {
          const uint32_t acc0 = (kk > 0 || oa.cbar) ? 1u : 0u;
          tc_mma_ts(tmem + kO, tmem + kP + kk * 8, sdesc_mn64(sm.vh + kk * 16 * 64), iv, acc0);
          tc_mma_ts(tmem + kO, tmem + kP + kk * 8, sdesc_mn64(sm.vl + kk * 16 * 64), iv, 1u);
        }
        tc_commit(&sm.mbar);
      }
      r3 = mbar_wait(&sm.mbar, 1, abort_flag, status);
      tc_fence_after();
      if (__syncthreads_and(r3)) {
        constexpr int DH = OV / 2;
        float o[DH];
        const uint32_t to = tmem + ((uint32_t)((warp & 3) * 32) << 16) + kO + hh * DH;
#pragma unroll
        for (int c = 0; c < DH; c += 16) {
          float x[16];
          tmem_ld16(to + c, x);
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) o[c + e2] = x[e2];
        }
        if (mine) {
          const int row = oa.q_perm[q.lab + n];
          uint4 *dst = reinterpret_cast<uint4 *>(oa.O + ((int64_t)p * oa.N + row) * OV + hh * DH);
#pragma unroll
          for (int u = 0; u < DH / 8; ++u) {
            uint32_t w[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(o[8 * u + 2 * e2], o[8 * u + 2 * e2 + 1]);
              w[e2] = *reinterpret_cast<uint32_t *>(&b2);
            }
            dst[u] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    } else {
    const int64_t cl = w_ld(q.n);
    const int64_t cbase = (int64_t)p * mt.in.c_stride + mt.in.cc0[s] + n + hh * HC * cl;
    float *C0 = c0 + cbase, *C1 = c1 + cbase;
    const int jn = min(HC, Ck - hh * HC);  // this half's key clusters
    for (int cb = 0; cb < HC; cb += 16) {
      float x[16];
      tmem_ld16(ta + cb, x);
      if (mine) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          if (cb + c < jn) {
            const float a = fmaf(scale, x[c], lzh[cb + c]);
            const float pj = a > -CUDART_INF_F ? __expf(a - m) * inv : 0.f;
            C0[(cb + c) * cl] = pj * (1.f - sdip * x[c]);
            C1[(cb + c) * cl] = sdip * pj;
          }
        }
      }
    }
    if (mine && hh == 0) lse[q.lab + n] = m + logf(l);
    }
  }
  if (t == 0) {
    mbar_drain(&sm.lbar, 0, status);
    // the last phase committed: after two completed phases the parity of phase 0 is also
    // that of the open phase 2, so phase 0 is drained only when it is the last one
    // (the output product is committed only after phase 0 completed)
    mbar_drain(&sm.mbar, (OUT && second) ? 1u : 0u, status);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols)
                 : "memory");
  }
}

template <int D, int CK, bool OUT>
static cudaError_t launch(const MuseTables &mt, int P, float scale, const void *qs_rows,
                          const int32_t *q_offsets, const StageBufs &b, const InstMask &skip,
                          float sdip, const CoefOut &oa, int *status, cudaStream_t st) {
  CUtensorMap mq;
  if (!make_map(&mq, qs_rows, D, (uint64_t)P * mt.q.row_stride, D, TM)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem<D, CK, OUT>) + 1024;
  auto kern = coef_tc<D, CK, OUT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // chunk slots of an instance (none for the skipped ones): at most ceil(rows / 128) + one
  // partial chunk per cluster
  BlockMap bm;
  bm.pre[0] = 0;
  for (int si = 0; si < mt.in.ninst; ++si) {
    const bool mine = !((skip.w[si >> 5] >> (si & 31)) & 1u);
    const int n = mt.q.nrow[si];
    bm.pre[si + 1] = bm.pre[si] + (mine ? (n + TM - 1) / TM + std::min(mt.q.C[si], n) : 0);
  }
  for (int si = mt.in.ninst + 1; si <= kMaxSeg; ++si) bm.pre[si] = bm.pre[mt.in.ninst];
  bm.total = bm.pre[mt.in.ninst];
  if (bm.total == 0) return cudaSuccess;
  kern<<<dim3(bm.total, P), 2 * TM, smem, st>>>(mq, mt, scale, q_offsets, b.logZ, b.mu_k, b.c0, b.c1,
                                                b.lse, skip, sdip, oa, bm, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ctc

bool coef_tc_supported(int dtype, int D, int maxCk) {
  return dtype == MUSE_BF16 && (D == 64 || D == 128) && maxCk <= 256;
}

cudaError_t run_coef_tc(const MuseTables &mt, int D, int P, float scale, const void *qs_rows,
                        const int32_t *q_offsets, const StageBufs &b, const InstMask &skip,
                        float sdip, int *status, cudaStream_t st) {
  const int ck = mt.k.max_C;
  const ctc::CoefOut none{};
#define MUSE_COEF(DD, CC)                                                                   \
  return ctc::launch<DD, CC, false>(mt, P, scale, qs_rows, q_offsets, b, skip, sdip, none, \
                                    status, st)
  if (D == 64) {
    if (ck <= 64) MUSE_COEF(64, 64);
    if (ck <= 128) MUSE_COEF(64, 128);
    MUSE_COEF(64, 256);
  }
  if (ck <= 64) MUSE_COEF(128, 64);
  if (ck <= 128) MUSE_COEF(128, 128);
  MUSE_COEF(128, 256);
#undef MUSE_COEF
}

bool coef_out_supported(int dtype, int D, int Dv, int maxCk) {
  return dtype == MUSE_BF16 && Dv == ctc::OV && ((D == 64 && maxCk <= 256) || (D == 128 && maxCk <= 128));
}

cudaError_t run_coef_out(const MuseTables &mt, int D, int N, int P, float scale, const void *qs_rows,
                         const int32_t *q_perm, const int32_t *q_offsets, const StageBufs &b,
                         const float *cbar, void *O, int *status, cudaStream_t st) {
  const ctc::CoefOut oa{b.mu_v, cbar, q_perm, (__nv_bfloat16 *)O, N, scale};
  const InstMask all{};
  const int ck = mt.k.max_C;
#define MUSE_OUT(DD, CC) \
  return ctc::launch<DD, CC, true>(mt, P, scale, qs_rows, q_offsets, b, all, 0.f, oa, status, st)
  if (D == 64) {
    if (ck <= 64) MUSE_OUT(64, 64);
    if (ck <= 128) MUSE_OUT(64, 128);
    MUSE_OUT(64, 256);
  }
  if (ck <= 64) MUSE_OUT(128, 64);
  MUSE_OUT(128, 128);
#undef MUSE_OUT
}

}  // namespace muse
