// Refinement in summary form on the tensor cores (bfloat16, D = Dv = 128): for each query
// tile, one product against the stacked summaries of its query cluster i,
//   O_n = sum_j c0_nj mu_v,ij + sum_j c1_nj C'_ij qt_n,
//   C'_ij = sum_{k in S_j} w_ik v_k k^T,   mu_v,ij = sum_{k in S_j} w_ik v_k,
// with the coefficients of the pair form, c0 = p_j (1 - s qt.mu_k,ij) and c1 = s p_j
// (pith.science review of arXiv 2509.10406, "What carries the argument": out(q) =
// sum_j softmax_j(log Z_ij + s qt.mu_k,ij) (mu_v,ij + s C_ij qt), C_ij the tilted
// covariance; C_ij qt = C'_ij qt - mu_v,ij (mu_k,ij . qt) moves the centring into c0).
// Grouping the pair form's sum over keys by key cluster gives the same result:
// sum_k w_ik (c0 + c1 qt.k) v_k.  The tensor work per query cluster is
// 2 Dv D nk (the summaries) + 2 Dv (D + 16) Ck nq (the product), against the pair form's
// 2 nq nk (D + Dv): the smaller one at long context (N >> Ck D).
//
// One CTA = one query cluster i and up to 224 of its sorted rows (a unit).  For every
// non-empty key cluster j, in order:
//   (a) [C'_ij | mu_v,ij] (fp32, TMEM, M = Dv lanes, N = D + 16 columns) =
//       (w .* V_j)^T . [K_j | 1] over key tiles of 64: the value tile (transposed, TMA) is
//       scaled in place by the tilt weights of cluster i (zero outside S_j: the tile starts
//       8-aligned before S_j); the key tile (TMA, rows of 64 coordinates) is an MN-major B
//       operand, and a constant tile of ones gives the 16 columns of mu_v,ij.
//   (b) C'_ij is copied as bfloat16 pairs into one of two packed buffers, followed by the
//       K columns [mu_hi, mu_lo, mu_hi, 0 ...] (the A operand of (c), in TMEM); the
//       float32 buffer is then free for (a) of the next cluster.
//   (c) O^T (fp32, TMEM, M = Dv lanes, N = unit rows) += [C'_ij | aux] . [c1 qt_n | c0_hi,
//       c0_hi, c0_lo, 0 ...]^T, B built per row from the residual (held in registers)
//       and the coefficients.
// TMEM columns: C' and mu_v [0, 144), packed buffers [144, 216) and [216, 288), O^T
// [288, 512).
// The tensor cores run (a) of cluster j + 1 while (b) of cluster j is copied and the rows
// of (c) are built; (c) of cluster j follows (a) of cluster j + 1.
// Warp roles: 0 = TMA producer, 1 = MMA issuer (+ TMEM owner), 2-5 = scaling, 6-13 =
// rows: each thread builds one query row of the B operand of (c), and each warp copies
// (b) one half of C' in its TMEM lane quadrant (warp % 4); the same warps store O.  Every
// wait on an mbarrier is bounded: past the limit the kernel records MUSE_ERR_TIMEOUT and
// winds down.
#include <algorithm>

#include "internal.h"
#include "tc_ptx.cuh"

namespace muse {
namespace rsf {

using namespace ptx;

constexpr int D = 128, DV = 128;
constexpr int BN = 64;       // keys per tile
constexpr int NST = 4;       // tile stages
constexpr int UR = 224;      // query rows per unit (N of the product (c))
constexpr int kMaxCk = 256;  // key clusters (offsets staged in shared memory)
constexpr int kScale0 = 2, kRow0 = 6;                // first warp of each role
constexpr int kRowWarps = 8;                         // 256 threads: rows UR.. are idle
constexpr int kThreads = 32 * (kRow0 + kRowWarps);   // 448
constexpr int KA = D / 16 + 1;                       // K steps of (c): D + the aux step
constexpr uint32_t kPcol = D + 16, kPstride = D / 2 + 8;  // packed buffers: 72 columns each
constexpr uint32_t kOcol = kPcol + 2 * kPstride;          // O^T: 224 columns

struct __align__(1024) Smem {
  __nv_bfloat16 k[NST][D / 64][BN * 64];  // key tiles: a row per key, 64 coordinates per block
  __nv_bfloat16 vt[NST][DV * 64];         // value tiles: a row per value coordinate, 64 keys
  __nv_bfloat16 bq[D / 64 + 1][UR * 64];  // B of (c): a row per query row, K-major SW128
  float w[NST][BN];                       // tilt weights of cluster i over each tile's keys
  __nv_bfloat16 ones[16 * 64];            // B of the mu_v columns: 16 K-rows of ones
  int koff[kMaxCk + 1];                   // the key-cluster offsets
  uint64_t full[NST], scaled[NST], empty[NST];
  uint64_t cfull, cfree, pready[2], bqready, bdone;
  uint32_t tmem_base;
  int abort_flag;
  int s_i, s_r0, s_nr;
};

// Shared-memory descriptor of an MN-major operand, 128-byte swizzle, as the key tiles
// arrive from TMA: blocks of 64 elements along N (rows of 128 B, one per K index; 8 K-rows
// per 1024-B atom), consecutive N blocks lbo bytes apart.
__device__ __forceinline__ uint64_t sdesc_mn(const void *p, uint32_t lbo) {
  const uint32_t a = saddr(p);
  uint64_t d = 0;
  d |= (uint64_t)((a & 0x3FFFFu) >> 4);
  d |= (uint64_t)(lbo >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Untiled bulk copy global -> shared (16-byte aligned, a multiple of 16 bytes) on an
// mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(saddr(dst)), "l"(src), "r"(bytes), "r"(saddr(bar))
               : "memory");
}
// Every lane waits (each gets the acquire), the warp agrees on the outcome.
__device__ __forceinline__ bool wait_all(uint64_t *b, uint32_t parity, volatile int *abort_flag,
                                         int *status) {
  return __all_sync(0xffffffffu, mbar_wait<true>(b, parity, abort_flag, status));
}
// 8 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(r[e]);
}
// Store 4 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&v)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3])
               : "memory");
}
__device__ __forceinline__ void add2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(kThreads, 1)
refine_sf(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_vt,
          const __grid_constant__ MuseTables mt, int N, const __nv_bfloat16 *__restrict__ qs,
          const int32_t *__restrict__ q_perm, const int32_t *__restrict__ q_offsets,
          const int32_t *__restrict__ k_offsets, const float *__restrict__ W,
          const float *__restrict__ c0g, const float *__restrict__ c1g,
          __nv_bfloat16 *__restrict__ O, int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~(uintptr_t)1023);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int p = blockIdx.y, unit = blockIdx.x;
  const Task q = make_task(mt.q, p * mt.q.nseg), k = make_task(mt.k, p * mt.k.nseg);
  const int Ck = k.C;
  // the unit: counting ceil(rows / UR) units per query cluster, in cluster order
  if (warp == 0) {
    int run = 0, found = -1, fr0 = 0, fnr = 0;
    for (int cb = 0; cb < q.C && found < 0; cb += 32) {
      const int c = cb + lane;
      int nch = 0, bb = 0, ee = 0;
      if (c < q.C) {
        bb = q_offsets[q.off + c];
        ee = q_offsets[q.off + c + 1];
        nch = (ee - bb + UR - 1) / UR;
      }
      int inc = nch;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const int first = run + inc - nch;
      const bool mine = unit >= first && unit < first + nch;
      const unsigned bal = __ballot_sync(0xffffffffu, mine);
      if (bal) {
        const int src = __ffs(bal) - 1;
        const int r0 = bb + UR * (unit - first);
        found = __shfl_sync(0xffffffffu, c, src);
        fr0 = __shfl_sync(0xffffffffu, r0, src);
        fnr = __shfl_sync(0xffffffffu, min(UR, ee - r0), src);
      }
      run += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) {
      sm.s_i = found;
      sm.s_r0 = fr0;
      sm.s_nr = fnr;
    }
  }
  for (int j = t; j <= Ck; j += kThreads) sm.koff[j] = k_offsets[k.off + j];
  __syncthreads();
  const int i = sm.s_i;
  if (i < 0) return;  // uniform: past the problem's last unit
  const int r0 = sm.s_r0, nr = sm.s_nr;
  const int NU = (nr + 15) & ~15;  // N of the output product (<= UR)
  volatile int *abort_flag = &sm.abort_flag;

  if (t == 0) {
    for (int st = 0; st < NST; ++st) {
      mbar_init(&sm.full[st], 1);
      mbar_init(&sm.scaled[st], 4);
      mbar_init(&sm.empty[st], 1);
    }
    mbar_init(&sm.cfull, 1);
    mbar_init(&sm.cfree, kRowWarps);
    for (int b = 0; b < 2; ++b) mbar_init(&sm.pready[b], kRowWarps);
    mbar_init(&sm.bqready, kRowWarps);
    mbar_init(&sm.bdone, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int u = t; u < 16 * 64 / 8; u += kThreads)  // bfloat16 1.0 = 0x3F80
    reinterpret_cast<uint4 *>(sm.ones)[u] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // ones -> tensor cores
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(&sm.tmem_base)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int *koff = sm.koff;
  const int kcol0 = (int)(k.lab - (int64_t)p * mt.k.row_stride);  // first key column of the problem

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int wl = w_ld(k.n);
      const float *Wi = W + (int64_t)p * mt.in.w_stride + mt.in.w0[0] + (int64_t)i * wl;
      int g = 0;
      bool ok = true;
      for (int j = 0; ok && j < Ck; ++j) {
        const int b0 = koff[j], e0 = koff[j + 1];
        for (int x0 = b0 & ~7; b0 < e0 && x0 < e0; x0 += BN, ++g) {
          const int st = g % NST;
          if (g >= NST && !(ok = mbar_wait<true>(&sm.empty[st], ((g / NST) - 1) & 1, abort_flag, status)))
            break;
          // the weights of keys x0.. up to the end of W's row (x0 and w_ld(nk) are
          // multiples of 8: 32-byte aligned, a multiple of 32 bytes)
          const uint32_t wbytes = (uint32_t)min(BN, wl - x0) * 4u;
          mbar_expect_tx(&sm.full[st], (uint32_t)(D / 64) * BN * 128 + DV * 128 + wbytes);
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_2d(sm.k[st][kb], &map_k, kb * 64, (int)(k.lab + x0), &sm.full[st]);
          tma_load_2d(sm.vt[st], &map_vt, kcol0 + x0, p * DV, &sm.full[st]);
          bulk_load(sm.w[st], Wi + x0, wbytes, &sm.full[st]);
        }
      }
      // copies still in flight land before the CTA may exit
      for (int u = max(0, g - NST); u < g; ++u) mbar_drain(&sm.full[u % NST], (u / NST) & 1, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint64_t *lastbar = nullptr;  // the last commit (its completion implies all earlier ones)
      uint32_t lastpar = 0;
      int nb = 0;  // output products committed
      // (c) for the x-th non-empty key cluster
      auto out_product = [&](int x) -> bool {
        const int b = x & 1;
        if (!mbar_wait<true>(&sm.pready[b], (x >> 1) & 1, abort_flag, status)) return false;
        if (!mbar_wait<true>(&sm.bqready, x & 1, abort_flag, status)) return false;
        tc_fence_after();
        const uint32_t ib = idesc(128, NU);
#pragma unroll
        for (int kk = 0; kk < KA; ++kk)
          tc_mma_ts(tmem + kOcol, tmem + kPcol + b * kPstride + kk * 8,
                    sdesc(sm.bq[kk >> 2] + (kk & 3) * 16), ib, (x > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&sm.bdone);
        lastbar = &sm.bdone;
        lastpar = nb & 1;
        ++nb;
        return true;
      };
      int g = 0, jj = 0;
      bool ok = true;
      constexpr uint32_t ia = idesc(128, D) | (1u << 16);  // B (the key tile) MN-major
      constexpr uint32_t i1 = idesc(128, 16) | (1u << 16);  // B: 16 columns of ones
      for (int j = 0; ok && j < Ck; ++j) {
        const int b0 = koff[j], e0 = koff[j + 1];
        if (b0 == e0) continue;
        // the float32 buffer is free once (b) of the previous cluster has read it
        if (jj >= 1 && !(ok = mbar_wait<true>(&sm.cfree, (jj - 1) & 1, abort_flag, status))) break;
        tc_fence_after();
        int tl = 0;
        for (int x0 = b0 & ~7; x0 < e0; x0 += BN, ++g, ++tl) {
          const int st = g % NST;
          if (!(ok = mbar_wait<true>(&sm.scaled[st], (g / NST) & 1, abort_flag, status))) break;
          tc_fence_after();
          const int nks = (min(BN, e0 - x0) + 15) / 16;
          for (int kk = 0; kk < nks; ++kk) {  // the D/64 blocks of the key tile: BN*128 B apart
            const uint64_t a = sdesc(sm.vt[st] + kk * 16);
            const uint32_t acc = (tl > 0 || kk > 0) ? 1u : 0u;
            tc_mma(tmem, a, sdesc_mn(sm.k[st][0] + kk * 16 * 64, BN * 128), ia, acc);
            tc_mma(tmem + D, a, sdesc_mn(sm.ones, 1024), i1, acc);  // mu_v in all 16 columns
          }
          tc_commit(&sm.empty[st]);
          lastbar = &sm.empty[st];
          lastpar = (g / NST) & 1;
        }
        if (!ok) break;
        tc_commit(&sm.cfull);
        lastbar = &sm.cfull;
        lastpar = jj & 1;
        if (jj >= 1 && !(ok = out_product(jj - 1))) break;
        ++jj;
      }
      if (ok && jj >= 1) ok = out_product(jj - 1);
      if (ok && jj == 0) report(status, MUSE_ERR_DEVICE);  // no keys: cannot occur
      if (lastbar) mbar_drain(lastbar, lastpar, status);
    }
  } else if (warp < kRow0) {
    // ------------------------------------------------------------ scaling
    const int ts = t - 32 * kScale0;
    const int c = ts & 7, rb = ts >> 3;  // 8 keys of the tile; rows rb + 16 m
    int g = 0;
    bool ok = true;
    for (int j = 0; ok && j < Ck; ++j) {
      const int b0 = koff[j], e0 = koff[j + 1];
      for (int x0 = b0 & ~7; b0 < e0 && x0 < e0; x0 += BN, ++g) {
        const int st = g % NST;
        const int pos = x0 + 8 * c;
        unsigned in = 0;  // bit e: key pos + e lies in S_j
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (pos + e >= b0 && pos + e < e0) in |= 1u << e;
        uint32_t keep[4];  // per pair: the halves that lie in S_j
#pragma unroll
        for (int e = 0; e < 4; ++e)
          keep[e] = (((in >> (2 * e)) & 1u) ? 0x0000ffffu : 0u) | (((in >> (2 * e + 1)) & 1u) ? 0xffff0000u : 0u);
        if (!(ok = wait_all(&sm.full[st], (g / NST) & 1, abort_flag, status))) break;
        // (weights past the end of W's row are not copied: they lie outside S_j)
        const float4 wa = *reinterpret_cast<const float4 *>(&sm.w[st][8 * c]);
        const float4 wb = *reinterpret_cast<const float4 *>(&sm.w[st][8 * c + 4]);
        const __nv_bfloat162 w2[4] = {__floats2bfloat162_rn(wa.x, wa.y), __floats2bfloat162_rn(wa.z, wa.w),
                                      __floats2bfloat162_rn(wb.x, wb.y), __floats2bfloat162_rn(wb.z, wb.w)};
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int v = rb + 16 * m;
          uint4 *ptr = reinterpret_cast<uint4 *>(sm.vt[st] + v * 64 + ((c ^ (v & 7)) << 3));
          uint4 x = *ptr;
          uint32_t *xs = reinterpret_cast<uint32_t *>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 pr = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&xs[e]), w2[e]);
            // keys outside S_j (and padding, which may hold anything) become zero
            xs[e] = *reinterpret_cast<const uint32_t *>(&pr) & keep[e];
          }
          *ptr = x;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // scaled tile -> tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.scaled[st]);
      }
    }
  } else {
    // ------------------------------------------------------------ rows: (b), B of (c), O
    const int h = (warp - kRow0) >> 2, qd = warp & 3;
    const int v = qd * 32 + lane;
    const uint32_t lb = (uint32_t)(qd * 32) << 16;
    const int r = t - 32 * kRow0;  // the unit's row built by this thread
    const bool builds = r < UR;    // rows UR.. take part in the warps' TMEM work only
    const bool valid = r < nr;
    const int n = r0 + r;          // sorted row within the problem
    const int cl = w_ld(q.n);
    const float *C0 = c0g + (int64_t)p * mt.in.c_stride + mt.in.cc0[0] + n;
    const float *C1 = c1g + (int64_t)p * mt.in.c_stride + mt.in.cc0[0] + n;
    uint32_t qh[D / 2];  // the residual row, bfloat16 pairs
    {
      const uint4 *src = reinterpret_cast<const uint4 *>(qs + (q.lab + (valid ? n : 0)) * D);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) {
        const uint4 x = valid ? src[u] : make_uint4(0u, 0u, 0u, 0u);
        qh[4 * u] = x.x;
        qh[4 * u + 1] = x.y;
        qh[4 * u + 2] = x.z;
        qh[4 * u + 3] = x.w;
      }
    }
    const int sw = r & 7;
    __nv_bfloat16 *row = &sm.bq[0][(builds ? r : 0) * 64];
    __nv_bfloat16 *aux = &sm.bq[D / 64][(builds ? r : 0) * 64];
    if (builds) *reinterpret_cast<uint4 *>(aux + ((1 ^ sw) << 3)) = make_uint4(0u, 0u, 0u, 0u);
    int jj = 0;
    bool ok = true;
    for (int j = 0; ok && j < Ck; ++j) {
      if (koff[j] == koff[j + 1]) continue;
      const int b = jj & 1;
      const float c0 = valid ? C0[(int64_t)j * cl] : 0.f, c1 = valid ? C1[(int64_t)j * cl] : 0.f;
      // (b) this warp's half of C' (columns [64 h, 64 h + 64)) as bfloat16 pairs into
      // packed columns [32 h, 32 h + 32) of buffer b; once mu_v is read too, the float32
      // buffer is released
      const uint32_t src = tmem + lb + h * 64;
      const uint32_t dst = tmem + lb + kPcol + b * kPstride + h * 32;
      if (!(ok = wait_all(&sm.cfull, jj & 1, abort_flag, status))) break;
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        float x[8];
        tmem_ld8(src + 8 * ch, x);
        const uint32_t pk[4] = {pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                                pack_bf16(x[6], x[7])};
        tmem_st4(dst + 4 * ch, pk);
      }
      float mu = 0.f;  // h = 1: mu_v,ij of row v (column D; its 16 columns are equal)
      if (h == 1) {
        float xm[8];
        tmem_ld8(tmem + lb + D, xm);
        mu = xm[0];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.cfree);
      if (h == 1) {  // the aux step [mu_hi, mu_lo, mu_hi, 0 ...]
        const float mh = __bfloat162float(__float2bfloat16_rn(mu));
        const uint32_t ax[8] = {pack_bf16(mh, mu - mh), pack_bf16(mh, 0.f), 0u, 0u, 0u, 0u, 0u, 0u};
        tmem_st8(dst + 32, ax);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.pready[b]);
      // B rows of (c): the previous cluster's product has read them
      if (jj >= 1 && !(ok = wait_all(&sm.bdone, (jj - 1) & 1, abort_flag, status))) break;
      const __nv_bfloat162 s2 = __float2bfloat162_rn(c1);
#pragma unroll
      for (int kb = 0; kb < (builds ? D / 64 : 0); ++kb)
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t y[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 xq = *reinterpret_cast<const __nv_bfloat162 *>(&qh[kb * 32 + 4 * cc + e]);
            const __nv_bfloat162 pr = __hmul2(xq, s2);
            y[e] = *reinterpret_cast<const uint32_t *>(&pr);
          }
          *reinterpret_cast<uint4 *>(row + kb * (UR * 64) + ((cc ^ sw) << 3)) = make_uint4(y[0], y[1], y[2], y[3]);
        }
      const float ch = __bfloat162float(__float2bfloat16_rn(c0));
      if (builds)
        *reinterpret_cast<uint4 *>(aux + (sw << 3)) =
            make_uint4(pack_bf16(ch, ch), pack_bf16(c0 - ch, 0.f), 0u, 0u);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // rows -> tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bqready);
      ++jj;
    }
    // O: this warp's lane quadrant, columns (unit rows) [128 h, 128 h + 128) below NU
    if (ok && jj > 0 && wait_all(&sm.bdone, (jj - 1) & 1, abort_flag, status)) {
      tc_fence_after();
      const int32_t *perm = q_perm + q.lab + r0;
      for (int cb2 = 128 * h; cb2 < min(NU, 128 * h + 128); cb2 += 16) {
        float x[16];
        tmem_ld16(tmem + lb + kOcol + cb2, x);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int m = cb2 + e;
          if (m < nr) O[((int64_t)p * N + perm[m]) * DV + v] = __float2bfloat16_rn(x[e]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

}  // namespace rsf

bool refine_sf_supported(int dtype, int D, int Dv, const MuseTables &mt) {
  return dtype == MUSE_BF16 && D == rsf::D && Dv == rsf::DV && mt.in.ninst == 1 &&
         mt.q.nseg == 1 && mt.k.nseg == 1 && mt.k.lab0[0] == 0 && mt.k.C[0] <= rsf::kMaxCk;
}

cudaError_t run_refine_sf(const MuseTables &mt, int N, int P, const void *qs_rows,
                          const int32_t *q_perm, const int32_t *q_offsets, const void *ks_rows,
                          const int32_t *k_offsets, const void *vt, const StageBufs &b, void *O,
                          int *status, cudaStream_t st) {
  using namespace rsf;
  CUtensorMap mk, mv;
  const int ldv = vt_ld(mt.k.row_stride);
  if (!make_map(&mk, ks_rows, D, (uint64_t)P * mt.k.row_stride, D, BN) ||
      !make_map(&mv, vt, ldv, (uint64_t)P * DV, ldv, DV))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(refine_sf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // units: at most ceil(rows / UR) plus one partial unit per query cluster
  const int nq = mt.q.nrow[0];
  const int units = (nq + UR - 1) / UR + std::min(mt.q.C[0], nq);
  refine_sf<<<dim3(units, P), kThreads, smem, st>>>(mk, mv, mt, N, (const __nv_bfloat16 *)qs_rows, q_perm,
                                                    q_offsets, k_offsets, b.W, b.c0, b.c1,
                                                    (__nv_bfloat16 *)O, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace muse
