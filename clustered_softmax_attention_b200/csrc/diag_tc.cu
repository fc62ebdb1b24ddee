// Causal MuSe: the exact diagonal block on the tensor cores, merged with the level
// partials of the squares below the diagonal (bfloat16, D = Dv = 64).
//
// pith.science review of arXiv 2509.10406, Figure 2 caption and "Assumptions & free
// parameters" (the hierarchical decomposition: exact attention on the block diagonal,
// summaries for everything below it).  Same result as diag_merge in stages.cu: for
// query row n of block b, exact attention over the keys [b S, n] combined in one
// softmax with the partials (log-normaliser, normalised output) of every level whose
// square holds the row.
//
// One CTA = 128 query rows inside one block (block a multiple of 128); it attends the
// key tiles t = 0 .. qt of its block (qt = the query tile's index in the block; tile qt
// is the diagonal one, masked k <= n).  TMA brings the residual-free query tile and, when
// at most four key tiles are attended, all key and value tiles at once; otherwise the
// key tiles (pass 1) and the key and value tiles (pass 2) come in groups of four.  Two
// passes over the key tiles:
//   pass 1: S = Q . K_t^T (tcgen05, fp32 in TMEM) -> running row maximum of s S
//   pass 2: S again; P = exp(s S - m) (bf16, TMEM); l += sum P; O += P . V_t
//           (tcgen05, A = P from TMEM, B = V_t as stored: keys x Dv, Dv innermost)
// then the merge with the level partials and the bf16 store.  Thread t owns row t
// (TMEM lane t); thread 0 issues the copies and the MMAs.  Every wait is bounded.
#include "internal.h"
#include "tc_ptx.cuh"

namespace muse {
namespace dtc {

constexpr int TM = 128;       // query rows per CTA and keys per tile
constexpr int D = 64;
constexpr int MAXT = 4;       // key and value tiles resident at once
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kS = 0, kP = 128, kO = 192;  // TMEM columns: S, P (packed bf16), O

struct __align__(1024) Smem {
  __nv_bfloat16 q[TM * 64];
  __nv_bfloat16 k[MAXT][TM * 64];
  __nv_bfloat16 v[MAXT][TM * 64];
  uint64_t lbar, mbar;
  uint32_t tmem_base;
  int abort_flag;
};

using namespace ptx;

// Shared-memory descriptor of an MN-major operand with 128-byte swizzle (rows of
// 128 B hold 64 consecutive N elements of one K index; 8 K-rows per 1024-B atom).
__device__ __forceinline__ uint64_t sdesc_mn(const void *p) {
  const uint32_t a = saddr(p);
  uint64_t d = 0;
  d |= (uint64_t)((a & 0x3FFFFu) >> 4);
  d |= (uint64_t)((16384u >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__global__ void __launch_bounds__(TM, 1)
diag_tc(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
        const __grid_constant__ CUtensorMap map_v, int N, int block, int levels, float scale,
        const float *__restrict__ part_o, const float *__restrict__ part_lse,
        __nv_bfloat16 *__restrict__ O, int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~(uintptr_t)1023);
  const int t = threadIdx.x, warp = t >> 5;
  volatile int *abort_flag = &sm.abort_flag;
  const int p = blockIdx.y;
  const int n0 = blockIdx.x * TM;              // first query row of the tile
  const int bidx = n0 / block;                 // its diagonal block
  const int ks0 = bidx * block;                // the block's first key
  const int qt = (n0 - ks0) / TM;              // key tiles 0 .. qt
  const int64_t row0 = (int64_t)p * N;         // first row of problem p in Q, K, V

  if (t == 0) {
    mbar_init(&sm.lbar, 1);
    mbar_init(&sm.mbar, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(&sm.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  const bool one = qt < MAXT;  // every key and value tile resident from the start
  if (t == 0) {
    const int nk = one ? qt + 1 : MAXT;
    mbar_expect_tx(&sm.lbar, (uint32_t)(1 + (one ? 2 : 1) * nk) * TM * 128);
    tma_load_2d(sm.q, &map_q, 0, (int)(row0 + n0), &sm.lbar);
    for (int kt = 0; kt < nk; ++kt) {
      tma_load_2d(sm.k[kt], &map_k, 0, (int)(row0 + ks0 + kt * TM), &sm.lbar);
      if (one) tma_load_2d(sm.v[kt], &map_v, 0, (int)(row0 + ks0 + kt * TM), &sm.lbar);
    }
  }
  // (every decision to go on is made CTA-wide: a wait that gives up in one thread stops
  // all of them at the next barrier)
  bool ok = __syncthreads_and(mbar_wait(&sm.lbar, 0, abort_flag, status));
  uint32_t lph = 1;  // loads issued on lbar (each one phase)
  // key tiles g0 .. g0 + cnt - 1 (and their value tiles) into slots 0 .. cnt - 1; called
  // by every thread after a CTA barrier that follows the last MMA reading the slots
  auto load_group = [&](int g0, bool withv) -> bool {
    const int cnt = min(MAXT, qt + 1 - g0);
    if (t == 0) {
      mbar_expect_tx(&sm.lbar, (uint32_t)((withv ? 2 : 1) * cnt) * TM * 128);
      for (int i = 0; i < cnt; ++i) {
        tma_load_2d(sm.k[i], &map_k, 0, (int)(row0 + ks0 + (g0 + i) * TM), &sm.lbar);
        if (withv) tma_load_2d(sm.v[i], &map_v, 0, (int)(row0 + ks0 + (g0 + i) * TM), &sm.lbar);
      }
    }
    const bool r = mbar_wait(&sm.lbar, lph & 1, abort_flag, status);
    ++lph;
    return __syncthreads_and(r);
  };
  uint32_t mph = 0;  // phase of the MMA barrier
  // S = Q . K_kt^T into TMEM columns [kS, kS + 128); every thread waits for it
  auto qk = [&](int kt) -> bool {
    if (t == 0) {
      tc_fence_after();
      const uint32_t id = idesc(TM, TM);
      for (int kk = 0; kk < D / 16; ++kk)
        tc_mma(tmem + kS, sdesc(sm.q + kk * 16), sdesc(sm.k[kt % MAXT] + kk * 16), id, kk > 0 ? 1u : 0u);
      tc_commit(&sm.mbar);
    }
    const bool r = mbar_wait(&sm.mbar, mph & 1, abort_flag, status);
    ++mph;
    tc_fence_after();
    return r;
  };
  const float c = scale * 1.4426950408889634f;  // s log2(e): exp(s S - m) = 2^(c S - m')
  const int n = n0 + t;
  float m2 = -CUDART_INF_F;  // running maximum of c S over the valid keys of the row
  // ------------------------------------------------ pass 1: row maxima
  for (int kt = 0; ok && kt <= qt; ++kt) {
    if (kt > 0 && kt % MAXT == 0 && !(ok = load_group(kt, false))) break;
    const bool r = qk(kt);
    const int lim = kt < qt ? TM : t + 1;  // valid columns of this row
    for (int cb = 0; r && cb < TM / 16; ++cb) {
      float x[16];
      tmem_ld16(tmem + lane_base + kS + cb * 16, x);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (cb * 16 + e < lim) m2 = fmaxf(m2, c * x[e]);
    }
    tc_fence_before();
    ok = __syncthreads_and(r);  // S is read before the next MMA overwrites it
  }
  // ------------------------------------------------ pass 2: P, l and O += P V
  float l = 0.f;
  for (int kt = 0; ok && kt <= qt; ++kt) {
    if (!one && kt % MAXT == 0 && !(ok = load_group(kt, true))) break;
    const bool r = qk(kt);
    const int lim = kt < qt ? TM : t + 1;
    for (int cb = 0; r && cb < TM / 16; ++cb) {
      float x[16];
      tmem_ld16(tmem + lane_base + kS + cb * 16, x);
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        const float p0 = cb * 16 + e < lim ? exp2f(fmaf(c, x[e], -m2)) : 0.f;
        const float p1 = cb * 16 + e + 1 < lim ? exp2f(fmaf(c, x[e + 1], -m2)) : 0.f;
        l += p0 + p1;
        __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
        pk[e >> 1] = *reinterpret_cast<uint32_t *>(&h);
      }
      tmem_st8(tmem + lane_base + kP + cb * 8, pk);
    }
    tmem_st_wait();
    tc_fence_before();
    if (!(ok = __syncthreads_and(r))) break;  // P complete in TMEM, S read
    if (t == 0) {
      tc_fence_after();
      // B = V_kt as stored (keys x Dv, Dv innermost): MN-major operand
      const uint32_t id = idesc(TM, D) | (1u << 16);
      for (int kk = 0; kk < TM / 16; ++kk)
        tc_mma_ts(tmem + kO, tmem + kP + kk * 8, sdesc_mn(sm.v[kt % MAXT] + kk * 16 * 64), id,
                  (kt > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&sm.mbar);
    }
    const bool w = mbar_wait(&sm.mbar, mph & 1, abort_flag, status);  // P and S are reused next
    ++mph;
    tc_fence_after();
    ok = __syncthreads_and(w);
  }
  // ------------------------------------------------ merge with the level partials
  if (ok) {
    float acc[D];
#pragma unroll
    for (int cb = 0; cb < D / 16; ++cb) {
      float x[16];
      tmem_ld16(tmem + lane_base + kO + cb * 16, x);
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[cb * 16 + e] = x[e];
    }
    // natural-log units from here: m = m2 / log2(e)
    float m = m2 * 0.6931471805599453f;
    if (n < N) {
      // levels < 0: a single partial array, merged into every row
      const int nlev = levels < 0 ? 1 : levels;
      for (int lev = 1; lev <= nlev; ++lev) {
        if (levels > 0 && !((bidx >> (lev - 1)) & 1)) continue;
        const int64_t r = ((int64_t)p * nlev + (lev - 1)) * N + n;
        const float L = part_lse[r];
        if (!(L > -CUDART_INF_F)) continue;
        const float mn = fmaxf(m, L);
        const float ca = expf(m - mn), cb = expf(L - mn);
        l = l * ca + cb;
        const float4 *po = reinterpret_cast<const float4 *>(part_o + r * D);
#pragma unroll
        for (int u = 0; u < D / 4; ++u) {
          const float4 v = po[u];
          acc[4 * u] = acc[4 * u] * ca + cb * v.x;
          acc[4 * u + 1] = acc[4 * u + 1] * ca + cb * v.y;
          acc[4 * u + 2] = acc[4 * u + 2] * ca + cb * v.z;
          acc[4 * u + 3] = acc[4 * u + 3] * ca + cb * v.w;
        }
        m = mn;
      }
      const float inv = 1.f / l;
      uint4 *dst = reinterpret_cast<uint4 *>(O + (row0 + n) * D);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[8 * u + 2 * h] * inv, acc[8 * u + 2 * h + 1] * inv);
          w[h] = *reinterpret_cast<uint32_t *>(&b2);
        }
        dst[u] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  // copies and MMAs still in flight land before the CTA releases its memory
  if (t == 0) {
    mbar_drain(&sm.lbar, (lph - 1) & 1, status);  // the last load issued
    // A wait that gave up may leave MMA phase mph - 1 incomplete: drain it before the final
    // commit (once that commit has landed, the parity of phase mph - 1 is also that of the
    // open phase mph + 1, and the probe would wait for good).  On the normal path phase
    // mph - 1 is complete and the probe returns at once.  Then the final commit's phase,
    // which tracks every MMA issued.
    if (mph > 0) mbar_drain(&sm.mbar, (mph - 1) & 1, status);
    tc_commit(&sm.mbar);
    mbar_drain(&sm.mbar, mph & 1, status);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace dtc

bool diag_tc_supported(int dtype, int D, int Dv, int N, int block) {
  return dtype == MUSE_BF16 && D == dtc::D && Dv == dtc::D && block % dtc::TM == 0 && N % block == 0;
}

cudaError_t run_diag_tc(const void *Q, const void *K, const void *V, int N, int P, int block,
                        int levels, float scale, const float *part_o, const float *part_lse,
                        void *O, int *status, cudaStream_t st) {
  using namespace dtc;
  CUtensorMap mq, mk, mv;
  if (!ptx::make_map(&mq, Q, D, (uint64_t)P * N, D, TM) ||
      !ptx::make_map(&mk, K, D, (uint64_t)P * N, D, TM) ||
      !ptx::make_map(&mv, V, D, (uint64_t)P * N, D, TM))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(diag_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  diag_tc<<<dim3(N / TM, P), TM, smem, st>>>(mq, mk, mv, N, block, levels, scale, part_o, part_lse,
                                             (__nv_bfloat16 *)O, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace muse
