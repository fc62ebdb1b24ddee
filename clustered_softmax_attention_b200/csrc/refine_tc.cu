// Refinement on the 5th-generation tensor cores (sm_100a): tcgen05.mma with TMEM
// accumulators, operands staged by TMA, warp-specialised.
//
// Stage 2 of MuSe (pith.science review of arXiv 2509.10406, "What carries the
// argument": the two-stage scheme drops only the residual-residual term qt.kt;
// gist.science "Technische Samenvatting", "Kernmechanismen" 1-2) evaluated as
//   O_n = sum_k w_{i(n),k} (c0_{n,j(k)} + c1_{n,j(k)} qt_n.k) v_k
// over the cluster-sorted keys (the identity is derived in stages.cu).
//
// One CTA = 128 consecutive sorted query rows of one instance (their residuals are
// the A operand of the first contraction, resident in shared memory).  The CTA walks
// the cluster-sorted keys in windows of BN keys (8-key-aligned starts, so the
// transposed values can be fetched by TMA); a window holds up to 8 key clusters or
// parts of them, and columns outside it are masked to zero.  With every
// key/value tile the producer also stages, by cp.async into the same stage, the tile's
// tilt weights for up to 8 query clusters of the CTA and the tile's coefficients
// c0, c1 for the CTA's 128 rows.
//   S  = Qt . K_tile^T            (tcgen05, 128 x npad, fp32 in TMEM, three buffers)
//   P  = w .* (c0 + c1 .* S)      (epilogue warps: TMEM -> registers -> bf16 TMEM, written
//                                  over S(t) in its own buffer, two per column)
//   O += P . V_tile               (tcgen05, A = P from TMEM, 128 x Dv, fp32 in TMEM)
// TMEM columns: S/P buffers [0, 3 BN) (tile t uses buffer t % 3; it takes S(t + 3) once
// O += P(t) V has completed), O [3 BN, 3 BN + Dv).
// Warp roles: warp 0 = TMA producer of the key tiles, warp 12 = of the value tiles
// (each stage released as soon as its MMA has consumed it), warp 1 = MMA issuer
// (+ TMEM owner), warps 2-9 = epilogue
// in two groups of four (TMEM lane quadrant = warp % 4): group g takes the tiles of
// parity g, so the groups overlap; warps 10-11 = cp.async producers
// of the epilogue data (tiles of parity 0 and 1).  Every wait on an mbarrier is
// bounded: past the limit the kernel records MUSE_ERR_TIMEOUT and winds down.
//
// Retrieval mode (RET): the remainder of causal accumulation with retrieval
// (gist.science "Kernmechanismen" items 3-4) has the same pair form over the global
// clusters, restricted per query: query n (block b, cluster i) takes the keys of every
// cluster in blocks b' < b, minus the (cluster, block) pairs selected for (i, b), which
// are attended exactly elsewhere; c0, c1 then carry the remainder coefficients.  The
// keys of a cluster are in token order, so for the CTA's latest query block b_hi each
// cluster contributes a prefix of its sorted keys; the tiles walk those prefixes only.
// Per element the epilogue masks key blocks b' >= b (a per-chunk block range decides
// most chunks at once) and, for the few tiles holding a selected cluster of the row,
// the selected blocks.
#include <cuda.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace muse {
namespace tcr {

constexpr int BM = 128;      // query rows per CTA
constexpr int NST = 4;       // K / V^T stages
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps + 96;  // + two epilogue-data producers, value loader
constexpr int kEWarp = 2 + kEpiWarps;               // first epilogue-data producer (parity 0)
constexpr int kVWarp = kEWarp + 2;                  // value-tile TMA producer
constexpr int kSlots = 8;    // query clusters per CTA whose tilt weights are staged
constexpr int kTileSegs = 8; // key clusters packed into one tile at most
constexpr int kComplex = 1 << 13;  // chunk code flag: more than two key clusters in 16 columns
constexpr int kSBuf = 3;     // S buffers (tile t uses t % 3); P(t) is written over S(t) in place
constexpr int kSplitSlots = kSplitCtas;  // key-range split: CTAs of half units at most

// Widest key tile: 128 keys when D = Dv = 64, else 64 (shared memory budget).
template <int D, int DV>
struct TileCfg {
  static constexpr int BN = (D == 64 && DV == 64) ? 128 : 64;
};

template <int D, int DV>
struct __align__(1024) Smem {
  static constexpr int BN = TileCfg<D, DV>::BN;
  __nv_bfloat16 q[D / 64][BM * 64];            // residual tile, K-major SW128 blocks
  __nv_bfloat16 k[NST][D / 64][BN * 64];       // key tiles
  __nv_bfloat16 vt[NST][BN / 64][DV * 64];     // transposed value tiles
  float w[NST][kSlots][BN];                    // tilt weights of the CTA's query clusters
  float c0[NST][kTileSegs][BM];                // coefficients of the tile's key clusters
  float c1[NST][kTileSegs][BM];
  unsigned char seg[NST][BN];                  // column -> cluster of the tile (0xFF: masked)
  int chunk[NST][BN / 16];                     // per 16 columns: mask, clusters, split (or kComplex)
  int koff[kMaxClusters + 1];                  // the instance's key-cluster offsets
  int kend[kMaxClusters];                      // RET: end of each cluster's causal prefix
  alignas(16) unsigned short kblk[NST][BN];    // RET: key block of every column (cp.async)
  int kgrp[NST][BN / 8];                       // RET: min | max << 16 key block per 8 columns
  int wbhi[BM / 32];                           // RET: latest query block per row warp
  int xblk[BM][17];                            // RET: each row's selected blocks (k1 k2 <= 16)
  int tnpad[4];                                // padded width of the tiles in flight (MMA issuer)
  // per stage: key tile (consumed by the first MMA), values (second MMA), epilogue
  // data (tilt weights, coefficients, segment map; consumed by the epilogue)
  uint64_t fullk[NST], emptyk[NST], fullv[NST], emptyv[NST], fulle[NST], emptye[NST];
  // S(t) in TMEM; P(t) over it; O += P(t) V done (the buffer is free again)
  uint64_t sfull[kSBuf], pready[kSBuf], spfree[kSBuf], qbar, obar;
  uint32_t tmem_base;
  int abort_flag;
};

using namespace ptx;

struct F16 {
  float v[16];
};
struct P8 {
  uint32_t v[8];
};

// P for a 16-column chunk whose valid columns belong to more than two key clusters, or
// for a warp with a row whose tilt weights are not staged: per-column cluster lookup.
// Rare, so kept out of line (the hot loop stays small).
template <int D, int DV>
static __device__ __noinline__ P8 mixed_chunk(const Smem<D, DV> &sm, int st, int cb, int r,
                                              const float *wp, F16 x) {
  P8 out;
  const int col0 = cb * 16;
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    float pv[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = col0 + e + h;
      const int g = sm.seg[st][col];
      pv[h] = g == 0xFF ? 0.f : wp[col] * fmaf(sm.c1[st][g][r], x.v[e + h], sm.c0[st][g][r]);
    }
    __nv_bfloat162 hh = __floats2bfloat162_rn(pv[0], pv[1]);
    out.v[e >> 1] = *reinterpret_cast<uint32_t *>(&hh);
  }
  return out;
}

// Key tiles of an instance: windows of at most BN consecutive sorted keys [c, c+n),
// starting 8-key aligned at x0 = c & ~7 (so the transposed values can be fetched by TMA)
// and padded to npad columns (multiple of 16).  A window spans the key clusters
// j .. j+nseg-1 (at most kTileSegs; it ends early at the start of cluster j+kTileSegs)
// and may start or end inside a cluster, whose keys then fall in two tiles.
struct KTile {
  int j, nseg, c, n, x0, npad;
};
// With `live` (retrieval mode) only the first live[j] - off[j] keys of cluster j are
// walked: a window ends where a cluster's live keys end before the cluster does.
template <int BN>
struct TileIter {
  const int32_t *off;
  const int32_t *live;
  int C;
  int khi;  // keys from khi on are left to another CTA (a split key range)
  KTile t;
  __device__ void begin(const int32_t *o, int Ck, const int32_t *lv = nullptr, int klo = -1,
                        int khi_ = 0x7fffffff) {
    off = o;
    live = lv;
    C = Ck;
    khi = khi_;
    make(0, klo >= 0 ? klo : off[0]);
  }
  // The window starting at key c, which lies in cluster j or a later one.
  __device__ void make(int j, int c) {
    if (live) {
      while (j < C) {
        if (c < off[j]) c = off[j];
        if (c < live[j]) break;
        ++j;
      }
    } else {
      while (j < C && c >= off[j + 1]) ++j;
    }
    t.j = j;
    t.c = c;
    if (j >= C) return;
    if (c >= khi) {  // the range is done
      t.j = C;
      return;
    }
    t.x0 = c & ~7;
    int end = min(min(t.x0 + BN, off[C]), khi);
    if (j + kTileSegs < C) end = min(end, off[j + kTileSegs]);
    int last = j;  // cluster holding key end-1
    if (live) {
      while (true) {
        if (live[last] < off[last + 1]) {  // dead keys follow: the window stops there
          end = min(end, live[last]);
          break;
        }
        if (last + 1 >= C || off[last + 1] >= end) break;
        ++last;
      }
    } else {
      while (last + 1 < C && off[last + 1] < end) ++last;
    }
    t.nseg = last - j + 1;
    t.n = end - c;
    t.npad = ((end - t.x0) + 15) & ~15;
  }
  __device__ bool done() const { return t.j >= C; }
  __device__ KTile get() const { return t; }
  __device__ void next() { make(t.j + t.nseg - 1, t.c + t.n); }
};

// Retrieval-mode arguments (unused by the plain refinement).
struct RetArgs {
  const unsigned short *kblk;  // [P][N] block of every sorted key
  const int *kgrp;             // [P][N / 8] min | max << 16 block of every 8 sorted keys
  const int32_t *pend;         // [P][Ck][nb + 1] keys of cluster j in blocks < b'
  const int32_t *sel;          // [P][Cq][nb][K12][2] (cluster, block) pairs selected per (i, b)
  int S, nb, k1, k2, K12, Cq;
};

// The last wave's key-range split (single-instance output mode).  With tpp > 0 the grid
// is one-dimensional over units (problem, 128-row tile), unit = p * tpp + tile: CTAs below
// `full` take a whole unit; the 2 (units - full) CTAs after them take one half of the keys
// of a unit each, writing float32 partial outputs to opart[slot][row][:] (slot = CTA -
// full), which refine_halves adds (the pair form is a plain sum over the keys).
struct SplitArgs {
  int tpp, full;
  float *opart;
};

// RET: columns of chunk cb whose key block precedes the row's block brow (the chunk's
// block range was not enough to decide).
template <int D, int DV>
static __device__ __noinline__ uint32_t causal_bits(const Smem<D, DV> &sm, int st, int cb, int brow) {
  uint32_t keep = 0;
#pragma unroll
  for (int e = 0; e < 16; ++e) keep |= (sm.kblk[st][cb * 16 + e] < brow ? 1u : 0u) << e;
  return keep;
}
// RET: columns of chunk cb that are not in a (cluster, block) pair selected for the row
// (so, its k1 x k2 slots; xseg: the tile segments whose cluster the row selected).
template <int D, int DV>
static __device__ __noinline__ uint32_t excl_bits(const Smem<D, DV> &sm, int st, int cb,
                                                  uint32_t xseg, int tj, const int32_t *so,
                                                  int k1, int k2) {
  uint32_t keep = 0xFFFFu;
  for (int e = 0; e < 16; ++e) {
    const int col = cb * 16 + e;
    const int g = sm.seg[st][col];
    if (g == 0xFF || !((xseg >> g) & 1u)) continue;
    const int j = tj + g, b = sm.kblk[st][col];
    for (int t = 0; t < k1; ++t) {
      if (so[2 * t * k2] != j) continue;
      for (int u = 0; u < k2; ++u)
        if (so[2 * (t * k2 + u) + 1] == b) keep &= ~(1u << e);
    }
  }
  return keep;
}

// RET: bit e set where the 16-bit block of column e (two per word, low half first) is
// below `lim` (pair = lim in both halves).
__device__ __forceinline__ uint32_t lt_bits16(const uint4 &a, const uint4 &b, uint32_t pair) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t m = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t c = __vcmpltu2(w[k], pair);  // 0xFFFF per half where below
    m |= ((c & 1u) | ((c >> 15) & 2u)) << (2 * k);
  }
  return m;
}
// RET: bit e set where the block of column e equals `pair`'s.
__device__ __forceinline__ uint32_t eq_bits16(const uint4 &a, const uint4 &b, uint32_t pair) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t m = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t c = __vcmpeq2(w[k], pair);
    m |= ((c & 1u) | ((c >> 15) & 2u)) << (2 * k);
  }
  return m;
}

// RET: columns of a chunk (at most two key clusters: glo over columns [0, split), ghi over
// [split, 16)) that are not in a block the row selected for their cluster; xb: the row's
// selected blocks, slot t * k2 + u; tmap: 4 bits per tile segment, its slot (15: none).
// Out of line: only chunks of a selected cluster come here.
static __device__ __noinline__ uint32_t excl_fast(uint4 ka, uint4 kb, int code, uint32_t tmap,
                                                  const int *xb, int k2) {
  const int glo = code & 15, ghi = (code >> 4) & 15, split = (code >> 8) & 31;
  const uint32_t lomask = split >= 16 ? 0xFFFFu : ((1u << split) - 1u);
  uint32_t keep = 0xFFFFu;
  for (int h = 0; h < 2; ++h) {
    const int sg = h ? ghi : glo;
    if (h && ghi == glo) break;
    const uint32_t tt = (tmap >> (4 * sg)) & 15u;
    if (tt == 15u) continue;
    uint32_t ex = 0;
    for (int u = 0; u < k2; ++u) {
      const int bb = xb[tt * k2 + u];
      if (bb >= 0) ex |= eq_bits16(ka, kb, (uint32_t)bb * 0x10001u);
    }
    keep &= ~(ex & (h ? ~lomask & 0xFFFFu : lomask));
  }
  return keep;
}

template <int D, int DV, bool RET>
__device__ __forceinline__ void
refine_tc_body(const CUtensorMap &map_q, const CUtensorMap &map_k, const CUtensorMap &map_vt,
               const MuseTables &mt, int N, const int32_t *__restrict__ q_perm,
               const int32_t *__restrict__ q_cluster, const int32_t *__restrict__ k_offsets,
               const float *__restrict__ W, const float *__restrict__ c0g,
               const float *__restrict__ c1g, const float *__restrict__ lse,
               __nv_bfloat16 *__restrict__ O, float *__restrict__ part_o,
               float *__restrict__ part_lse, int *status, const BlockMap &bm, const RetArgs &ra,
               const SplitArgs &sp) {
  constexpr int BN = TileCfg<D, DV>::BN;
  // blockIdx.x: a 128-row block of one instance (compact grid), blockIdx.y: the problem;
  // or, with the key-range split, a unit or half a unit (SplitArgs)
  int p, s, r0, half = -1, pslot = 0;  // pslot: this CTA's slot of partial outputs
  if (sp.tpp > 0) {
    const int cta = (int)blockIdx.x;
    int unit = cta;
    if (cta >= sp.full) {
      pslot = cta - sp.full;
      unit = sp.full + (pslot >> 1);
      half = pslot & 1;
    }
    p = unit / sp.tpp;
    s = 0;
    r0 = (unit % sp.tpp) * BM;
  } else {
    int bfirst;
    p = blockIdx.y;
    s = map_block(bm, mt.in.ninst, blockIdx.x, bfirst);
    r0 = ((int)blockIdx.x - bfirst) * BM;
  }
  const Task q = make_task(mt.q, p * mt.q.nseg + s);
  const Task k = make_task(mt.k, p * mt.k.nseg + s);
  if (r0 >= q.n) return;  // uniform: nothing allocated yet
  // this CTA's keys: all, or one half of the instance's sorted keys
  const int kmid = (k.n / 2) & ~7;
  const int klo = half == 1 ? kmid : -1, khi = half == 0 ? kmid : 0x7fffffff;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem<D, DV> &sm = *reinterpret_cast<Smem<D, DV> *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&sm.fullk[i], 1);
      mbar_init(&sm.emptyk[i], 1);
      mbar_init(&sm.fullv[i], 1);
      mbar_init(&sm.emptyv[i], 1);
      mbar_init(&sm.fulle[i], 1 + 32);  // lane 0 arrive + one cp.async arrival per lane
      mbar_init(&sm.emptye[i], kEpiWarps / 2);
    }
    for (int i = 0; i < kSBuf; ++i) {
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.pready[i], kEpiWarps / 2);  // the four warps of the tile's group
      mbar_init(&sm.spfree[i], 1);
    }
    mbar_init(&sm.qbar, 1);
    mbar_init(&sm.obar, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(&sm.tmem_base)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  for (int j = threadIdx.x; j <= k.C; j += blockDim.x) sm.koff[j] = k_offsets[k.off + j];
  if constexpr (RET) {
    // the CTA's latest query block b_hi: each key cluster takes the keys of blocks < b_hi
    if (warp < BM / 32) {
      const int n = r0 + threadIdx.x;
      int b = n < q.n ? q_perm[q.lab + n] / ra.S : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
      if (lane == 0) sm.wbhi[warp] = b;
    }
    __syncthreads();
    int bhi = 0;
#pragma unroll
    for (int w = 0; w < BM / 32; ++w) bhi = max(bhi, sm.wbhi[w]);
    const int32_t *pe = ra.pend + (int64_t)p * k.C * (ra.nb + 1) + bhi;
    for (int j = threadIdx.x; j < k.C; j += blockDim.x) sm.kend[j] = sm.koff[j] + pe[(int64_t)j * (ra.nb + 1)];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tmem_o = tmem + kSBuf * BN;
  auto s_col = [](int buf) { return (uint32_t)(buf * BN); };  // S(t) and, over it, P(t)
  const int32_t *koff = sm.koff;
  const int32_t *kend = RET ? sm.kend : nullptr;
  const int kcol0 = (int)(k.lab - (int64_t)p * mt.k.row_stride);  // instance's first key column
  const int wl = w_ld(k.n), cl = w_ld(q.n);
  const float *Wi = W + (int64_t)p * mt.in.w_stride + mt.in.w0[s];      // row i: Wi + i*wl
  const float *C0 = c0g + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];   // row j: C0 + j*cl
  const float *C1 = c1g + (int64_t)p * mt.in.c_stride + mt.in.cc0[s];
  const int i_first = q_cluster[q.lab + r0];  // query clusters i_first.. get staged weights
  const int nslots = min(kSlots, q_cluster[q.lab + min(r0 + BM, q.n) - 1] - i_first + 1);

  if (warp == 0 || warp == kVWarp) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: residual tile and key tiles; warp kVWarp: value tiles.  A stage is
    // refilled once the MMA that read it has completed; the key tiles run ahead of
    // the value tiles, whose stages free up only after the second contraction.
    const bool keys = warp == 0;
    // (test hook: the value tiles are never loaded, so the waits for them run out)
    const bool withhold = !keys && (test_hooks(status) & MUSE_TEST_WITHHOLD_VALUES);
    if (lane == 0 && !withhold) {
      if (keys) {
        mbar_expect_tx(&sm.qbar, (uint32_t)(D / 64) * BM * 128);
        for (int kb = 0; kb < D / 64; ++kb) tma_load_2d(sm.q[kb], &map_q, kb * 64, (int)(q.lab + r0), &sm.qbar);
      }
      uint64_t *full = keys ? sm.fullk : sm.fullv;
      uint64_t *empty = keys ? sm.emptyk : sm.emptyv;
      TileIter<BN> it;
      it.begin(koff, k.C, kend, klo, khi);
      int t = 0;
      for (; !it.done(); it.next(), ++t) {
        const KTile kt = it.get();
        const int st = t % NST;
        const int nbox = kt.npad > 64 ? 2 : 1;
        if (t >= NST && !mbar_wait<true>(&empty[st], ((t / NST) - 1) & 1, abort_flag, status)) break;
        if (keys) {
          mbar_expect_tx(&full[st], (uint32_t)nbox * (D / 64) * 64 * 128);
          for (int rb = 0; rb < nbox; ++rb)
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_2d(sm.k[st][kb] + rb * 64 * 64, &map_k, kb * 64, (int)(k.lab + kt.x0 + rb * 64),
                          &full[st]);
        } else {
          mbar_expect_tx(&full[st], (uint32_t)nbox * DV * 128);
          for (int rb = 0; rb < nbox; ++rb)
            tma_load_2d(sm.vt[st][rb], &map_vt, kcol0 + kt.x0 + rb * 64, p * DV, &full[st]);
        }
      }
      // copies still in flight land before the CTA may exit
      for (int u = max(0, t - NST); u < t; ++u) mbar_drain(&full[u % NST], (u / NST) & 1, status);
    }
  } else if (warp >= kEWarp && warp < kVWarp) {
    // ------------------------------------------------------------ epilogue-data producers
    // warp kEWarp + par stages the tiles of parity par (stages par, par + 2, ...)
    const int par = warp - kEWarp;
    TileIter<BN> it;
    it.begin(koff, k.C, kend, klo, khi);
    int t = 0;
    for (; !it.done(); it.next(), ++t) {
      if ((t & 1) != par) continue;
      const KTile kt = it.get();
      const int st = t % NST;
      int ok = 1;
      if (t >= NST && lane == 0) ok = mbar_wait<true>(&sm.emptye[st], ((t / NST) - 1) & 1, abort_flag, status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      // tilt weights of the staged query clusters over the tile's columns
      for (int e = lane; e < nslots * (BN / 4); e += 32) {
        const int sl = e / (BN / 4), v = e % (BN / 4);
        const int col = kt.x0 + 4 * v, i = i_first + sl;
        const bool in = i < q.C && col < wl && 4 * v < kt.npad;
        cp_async16(&sm.w[st][sl][4 * v], in ? (const void *)(Wi + (int64_t)i * wl + col) : (const void *)W,
                   in ? 16u : 0u);
      }
      // coefficients of the tile's key clusters for the CTA's rows
      for (int sg = 0; sg < kt.nseg; ++sg) {
        const int row = r0 + 4 * lane;
        const bool in = row < cl;
        const int64_t at = (int64_t)(kt.j + sg) * cl + row;
        cp_async16(&sm.c0[st][sg][4 * lane], in ? (const void *)(C0 + at) : (const void *)W, in ? 16u : 0u);
        cp_async16(&sm.c1[st][sg][4 * lane], in ? (const void *)(C1 + at) : (const void *)W, in ? 16u : 0u);
      }
      if constexpr (RET) {
        // the tile's key blocks (8 per copy) and their per-8 ranges (8-aligned tile start)
        const int64_t g0 = (k.lab + kt.x0) / 8;
        const int64_t gend = (k.lab + k.n + 7) / 8;  // the instance's groups end here
        for (int v = lane; v < BN / 8; v += 32) {
          const bool in = 8 * v < kt.npad && g0 + v < gend;
          cp_async16(&sm.kblk[st][8 * v], in ? (const void *)(ra.kblk + 8 * (g0 + v)) : (const void *)W,
                     in ? 16u : 0u);
          cp_async4(&sm.kgrp[st][v], in ? (const void *)(ra.kgrp + g0 + v) : (const void *)W, in ? 4u : 0u);
        }
      }
      cp_async_arrive(&sm.fulle[st]);
      // column -> key cluster of the tile (0xFF outside [c, c+n)), by comparison with
      // the tile's cluster boundaries held in registers
      int bnd[kTileSegs - 1];  // first key of the tile's clusters 1 .. nseg-1
#pragma unroll
      for (int b = 0; b < kTileSegs - 1; ++b) bnd[b] = b + 1 < kt.nseg ? koff[kt.j + b + 1] : 0x7FFFFFFF;
      for (int col = lane; col < BN; col += 32) {
        const int key = kt.x0 + col;
        int sg = 0xFF;
        if (col < kt.npad && key >= kt.c && key < kt.c + kt.n) {
          sg = 0;
#pragma unroll
          for (int b = 0; b < kTileSegs - 1; ++b) sg += key >= bnd[b] ? 1 : 0;
        }
        sm.seg[st][col] = (unsigned char)sg;
      }
      // per 16-column chunk: valid-column mask (a contiguous run) << 16, the key
      // clusters of its first and last valid columns (bits 0-3, 4-7) and the first
      // column of the second one (bits 8-12; 16 for one cluster), or kComplex when
      // more than two clusters share the chunk
      if (lane < BN / 16) {
        const int cx = kt.x0 + 16 * lane;
        const int k0 = max(kt.c, cx), k1 = min(kt.c + kt.n, cx + 16);
        int code = 16 << 8;  // no valid column: mask 0, P = 0
        if (16 * lane < kt.npad && k0 < k1) {
          int s0 = 0, s1 = 0, split = 16;
#pragma unroll
          for (int b = 0; b < kTileSegs - 1; ++b) {
            s0 += k0 >= bnd[b] ? 1 : 0;
            s1 += k1 - 1 >= bnd[b] ? 1 : 0;
          }
#pragma unroll
          for (int b = 0; b < kTileSegs - 1; ++b)
            if (b == s0 && s1 == s0 + 1) split = bnd[b] - cx;
          const uint32_t m16 = ((1u << (k1 - cx)) - 1u) & ~((1u << (k0 - cx)) - 1u);
          code = s1 > s0 + 1 ? kComplex : (s0 | (s1 << 4) | (split << 8));
          code |= (int)(m16 << 16);
        }
        sm.chunk[st][lane] = code;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.fulle[st]);  // releases the segment map with the stage
    }
    if (lane == 0)
      for (int u = max(0, t - NST); u < t; ++u)
        if ((u & 1) == par) mbar_drain(&sm.fulle[u % NST], (u / NST) & 1, status);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Two in-order streams: S(t) = Qt . K(t)^T (needs K(t), and the S buffer of tile
    // t-2 read by its group) and O += P(t) V(t) (needs P(t) and V(t)).  Whichever is
    // ready is issued, the first contraction first, so that neither epilogue group
    // waits behind the other.
    if (lane == 0) {
      bool ok = mbar_wait<true>(&sm.qbar, 0, abort_flag, status);
      tc_fence_after();
      TileIter<BN> it;
      it.begin(koff, k.C, kend, klo, khi);
      int g1 = 0, g2 = 0;  // next tile of each contraction
      int idle = 0;
      uint64_t t_idle = 0;
      const uint64_t idle_limit = wait_limit<true>(status);
      while (ok && (!it.done() || g2 < g1)) {
        bool progressed = false;
        if (!it.done()) {
          const int st = g1 % NST, buf = g1 % kSBuf;
          // the buffer's previous tile has gone through O += P V
          if ((g1 < kSBuf || mbar_test(&sm.spfree[buf], ((g1 / kSBuf) - 1) & 1)) &&
              mbar_test(&sm.fullk[st], (g1 / NST) & 1)) {
            tc_fence_after();
            const KTile kt = it.get();
            const uint32_t id = idesc(BM, kt.npad);
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t a = sdesc(sm.q[kk >> 2] + (kk & 3) * 16);
              const uint64_t b = sdesc(sm.k[st][kk >> 2] + (kk & 3) * 16);
              tc_mma(tmem + s_col(buf), a, b, id, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sm.sfull[buf]);
            tc_commit(&sm.emptyk[st]);  // the key tile is consumed
            sm.tnpad[g1 & 3] = kt.npad;
            ++g1;
            it.next();
            progressed = true;
          }
        }
        if (g2 < g1) {
          const int st = g2 % NST, pb = g2 % kSBuf;
          if (mbar_test(&sm.pready[pb], (g2 / kSBuf) & 1) && mbar_test(&sm.fullv[st], (g2 / NST) & 1)) {
            tc_fence_after();
            const uint32_t id = idesc(BM, DV);
            const int npad = sm.tnpad[g2 & 3];
            for (int kk = 0; kk < npad / 16; ++kk) {
              const uint64_t b = sdesc(sm.vt[st][kk >> 2] + (kk & 3) * 16);
              tc_mma_ts(tmem_o, tmem + s_col(pb) + kk * 8, b, id, (g2 > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&sm.spfree[pb]);
            tc_commit(&sm.emptyv[st]);
            ++g2;
            progressed = true;
          }
        }
        if (progressed) {
          idle = 0;
          continue;
        }
        // nothing ready: poll again, within the same time limit as every other wait
        if ((++idle & 255) == 0) {
          if (*abort_flag) {
            ok = false;
          } else {
            const uint64_t now = now_ns();
            if (idle == 256) {
              t_idle = now;
            } else if (now - t_idle > idle_limit) {
              *abort_flag = 1;
              report(status, MUSE_ERR_TIMEOUT);
              ok = false;
            }
          }
        }
      }
      tc_commit(&sm.obar);  // also tracks every MMA issued, on the abort path too
      mbar_drain(&sm.obar, 0, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;  // tiles of parity grp (and, at the end, half of O)
    const int r = quad * 32 + lane;
    const int n = r0 + r;
    const bool valid = n < q.n;
    const int i = valid ? q_cluster[q.lab + n] : i_first;
    const int slot = i - i_first;
    const bool staged = slot < nslots;
    const bool wfast = __all_sync(0xffffffffu, staged);  // every row of the warp has staged weights
    const float *wrow = Wi + (int64_t)i * wl;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    int brow = 0;                 // RET: the row's query block (0 masks every key)
    const int32_t *so = nullptr;  // RET: the row's selected (cluster, block) slots
    constexpr int kSelReg = 8;    // RET: selected clusters kept in registers
    int selc[kSelReg];
#pragma unroll
    for (int t1 = 0; t1 < kSelReg; ++t1) selc[t1] = -1;
    if constexpr (RET) {
      if (valid) {
        brow = q_perm[q.lab + n] / ra.S;
        so = ra.sel + (((int64_t)p * ra.Cq + i) * ra.nb + brow) * ra.K12 * 2;
        if (brow > 0) {
#pragma unroll
          for (int t1 = 0; t1 < kSelReg; ++t1)
            if (t1 < ra.k1) selc[t1] = so[2 * t1 * ra.k2];
          if (ra.k1 <= kSelReg && ra.K12 <= 16 && grp == 0)
            for (int e = 0; e < ra.K12; ++e) sm.xblk[r][e] = so[2 * e + 1];
        }
      }
    }
    // the table is read by both groups' threads of the same row
    if constexpr (RET) asm volatile("bar.sync 2, %0;" ::"r"(32 * kEpiWarps) : "memory");
    const bool xfast = ra.k1 <= kSelReg && ra.K12 <= 16;  // selection held in registers/table
    TileIter<BN> it;
    it.begin(koff, k.C, kend, klo, khi);
    int t = 0;
    bool ok = true;
    for (; !it.done(); it.next(), ++t) {
      if ((t & 1) != grp) continue;
      const KTile kt = it.get();
      const int buf = t % kSBuf, st = t % NST;
      // (a wait that gave up in one lane stops the whole warp: the TMEM accesses below
      // are warp-collective)
      if (!__all_sync(0xffffffffu, mbar_wait<true>(&sm.sfull[buf], (t / kSBuf) & 1, abort_flag, status) &&
                                       mbar_wait<true>(&sm.fulle[st], (t / NST) & 1, abort_flag, status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float *wsm = &sm.w[st][staged ? slot : 0][0];
      const int nch16 = kt.npad / 16;
      uint32_t xseg = 0;  // RET: tile segments holding a cluster the row selected
      uint32_t tmap = 0xFFFFFFFFu;  // RET: 4 bits per tile segment: its selected slot (15: none)
      if constexpr (RET) {
#pragma unroll
        for (int t1 = 0; t1 < kSelReg; ++t1) {
          const int d = selc[t1] - kt.j;
          if (selc[t1] >= 0 && d >= 0 && d < kt.nseg) {
            xseg |= 1u << d;
            tmap = (tmap & ~(15u << (4 * d))) | ((uint32_t)t1 << (4 * d));
          }
        }
        if (so && brow > 0)
          for (int t1 = kSelReg; t1 < ra.k1; ++t1) {
            const int d = so[2 * t1 * ra.k2] - kt.j;
            if (so[2 * t1 * ra.k2] >= 0 && d >= 0 && d < kt.nseg) xseg |= 1u << d;
          }
      }
      // P for 16 columns of S held in x, stored as 8 packed bf16 columns over the same
      // buffer: chunk cb's P lands in S columns 8 cb .. 8 cb + 7, which belong to S chunk
      // cb / 2, already read (and waited for) by this thread; the load in flight is of
      // chunk cb + 1, columns 16 cb + 16 on

      auto chunk = [&](int cb, const uint32_t(&x)[16]) {
        const int code = sm.chunk[st][cb];
        uint32_t keep = 0xFFFFu;  // RET: the row's causal and exclusion mask of the chunk
        if constexpr (RET) {
          // the chunk's block range, conservative: every key of its two 8-key groups
          const int ga = sm.kgrp[st][2 * cb], gb = sm.kgrp[st][2 * cb + 1];
          const int blo = min(ga & 0xFFFF, gb & 0xFFFF), bhi = max(ga >> 16, gb >> 16);
          const bool straddle = blo < brow && bhi >= brow;
          const bool xchunk = xseg != 0u && blo < brow;
          if (blo >= brow) keep = 0u;
          if (straddle || xchunk) {
            const uint4 ka = *reinterpret_cast<const uint4 *>(&sm.kblk[st][cb * 16]);
            const uint4 kb = *reinterpret_cast<const uint4 *>(&sm.kblk[st][cb * 16 + 8]);
            if (straddle) keep = lt_bits16(ka, kb, (uint32_t)brow * 0x10001u);
            if (xchunk) {
              if (xfast && !(code & kComplex))
                keep &= excl_fast(ka, kb, code, tmap, sm.xblk[r], ra.k2);
              else
                keep &= excl_bits<D, DV>(sm, st, cb, xseg, kt.j, so, ra.k1, ra.k2);
            }
          }
        }
        uint32_t pk[8];
        if (wfast && !(code & kComplex)) {
          // at most two key clusters over the chunk's valid columns
          const int glo = code & 15, ghi = (code >> 4) & 15, split = (code >> 8) & 31;
          const uint32_t msk = ((uint32_t)code >> 16) & keep;
          const float b0 = sm.c0[st][glo][r], b1 = sm.c1[st][glo][r];
          float w[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 v4 = *reinterpret_cast<const float4 *>(wsm + cb * 16 + 4 * u);
            w[4 * u] = v4.x; w[4 * u + 1] = v4.y; w[4 * u + 2] = v4.z; w[4 * u + 3] = v4.w;
          }
          float pv[16];
          if (glo == ghi) {
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              float t0, t1;
              fma2(t0, t1, b1, b1, __uint_as_float(x[e]), __uint_as_float(x[e + 1]), b0, b0);
              mul2(pv[e], pv[e + 1], w[e], w[e + 1], t0, t1);
            }
          } else {
            const float h0 = sm.c0[st][ghi][r], h1 = sm.c1[st][ghi][r];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const bool lo0 = e < split, lo1 = e + 1 < split;
              float t0, t1;
              fma2(t0, t1, lo0 ? b1 : h1, lo1 ? b1 : h1, __uint_as_float(x[e]), __uint_as_float(x[e + 1]),
                   lo0 ? b0 : h0, lo1 ? b0 : h0);
              mul2(pv[e], pv[e + 1], w[e], w[e + 1], t0, t1);
            }
          }
          if (msk != 0xFFFFu) {
            // columns outside the tile's keys: their S may come from unrelated rows
#pragma unroll
            for (int e = 0; e < 16; ++e) pv[e] = ((msk >> e) & 1u) ? pv[e] : 0.f;
          }
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            __nv_bfloat162 h = __floats2bfloat162_rn(pv[e], pv[e + 1]);
            pk[e >> 1] = *reinterpret_cast<uint32_t *>(&h);
          }
        } else {
          F16 xv;
#pragma unroll
          for (int e = 0; e < 16; ++e) xv.v[e] = __uint_as_float(x[e]);
          const P8 pr = mixed_chunk<D, DV>(sm, st, cb, r, staged ? wsm : wrow + kt.x0, xv);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t hm = (((keep >> (2 * e)) & 1u) ? 0x0000FFFFu : 0u) |
                                (((keep >> (2 * e + 1)) & 1u) ? 0xFFFF0000u : 0u);
            pk[e] = pr.v[e] & hm;
          }
        }
        tmem_st8(tmem + lane_base + s_col(buf) + cb * 8, pk);
      };
      // S chunks alternate between two register sets: the load of chunk cb+1 is in
      // flight while chunk cb is processed
      uint32_t xa[16], xb[16];
      int nl = 1;  // chunks whose load has been issued
      auto landed = [&]() { tmem_ld_wait(); };
      tmem_ld16_async(tmem + lane_base + s_col(buf), xa);
      landed();
      for (int cb = 0; cb < nch16; cb += 2) {
        if (nl < nch16) tmem_ld16_async(tmem + lane_base + s_col(buf) + (nl++) * 16, xb);
        chunk(cb, xa);
        landed();
        if (cb + 1 >= nch16) break;
        if (nl < nch16) tmem_ld16_async(tmem + lane_base + s_col(buf) + (nl++) * 16, xa);
        chunk(cb + 1, xb);
        landed();
      }
      if (!ok) break;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.pready[buf]);
        mbar_arrive(&sm.emptye[st]);  // the tile's epilogue data is consumed
      }
    }
    if (ok && t > 0 && __all_sync(0xffffffffu, mbar_wait<true>(&sm.obar, 0, abort_flag, status))) {
      tc_fence_after();
      const int row = valid ? q_perm[q.lab + n] : 0;
      for (int cb = grp; cb < DV / 16; cb += 2) {
        float o[16];
        tmem_ld16(tmem_o + lane_base + cb * 16, o);
        if (!valid) continue;
        if (half >= 0) {  // half the keys: a float32 partial, added by refine_halves
          float4 *dst = reinterpret_cast<float4 *>(sp.opart + ((int64_t)pslot * BM + r) * DV + cb * 16);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
        } else if (O) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            __nv_bfloat162 h = __floats2bfloat162_rn(o[e], o[e + 1]);
            pk[e >> 1] = *reinterpret_cast<uint32_t *>(&h);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(O + ((int64_t)p * N + row) * DV + cb * 16);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
          const int64_t rr = (int64_t)p * mt.in.out_stride + mt.in.out0[s] + row;
          float4 *dst = reinterpret_cast<float4 *>(part_o + rr * DV + cb * 16);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
        }
      }
      if (valid && !O && grp == 0) {
        const int64_t rr = (int64_t)p * mt.in.out_stride + mt.in.out0[s] + row;
        part_lse[rr] = lse[q.lab + n];
      }
    } else if (t == 0 && valid) {
      if constexpr (RET) {
        // every row of the CTA lies in block 0: no key precedes it, the partial is empty
        const int row = q_perm[q.lab + n];
        const int64_t rr = (int64_t)p * mt.in.out_stride + mt.in.out0[s] + row;
        float4 *dst = reinterpret_cast<float4 *>(part_o + rr * DV);
        for (int c = grp; c < DV / 4; c += 2) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (grp == 0) part_lse[rr] = lse[q.lab + n];
      } else if (half >= 0) {  // a half with no keys: a zero partial
        float4 *dst = reinterpret_cast<float4 *>(sp.opart + ((int64_t)pslot * BM + r) * DV);
        for (int c = grp; c < DV / 4; c += 2) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else if (grp == 0) {
        // an instance with no keys cannot occur (every key range is non-empty)
        report(status, MUSE_ERR_DEVICE);
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

// The refinement and its retrieval mode: one CTA per SM, 416 threads.
template <int D, int DV, bool RET>
__global__ void __launch_bounds__(kThreads, 1)
refine_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_vt, MuseTables mt, int N,
                 const int32_t *__restrict__ q_perm, const int32_t *__restrict__ q_cluster,
                 const int32_t *__restrict__ k_offsets, const float *__restrict__ W,
                 const float *__restrict__ c0g, const float *__restrict__ c1g,
                 const float *__restrict__ lse, __nv_bfloat16 *__restrict__ O,
                 float *__restrict__ part_o, float *__restrict__ part_lse, int *status,
                 const __grid_constant__ BlockMap bm, const RetArgs ra, const SplitArgs sp) {
  refine_tc_body<D, DV, RET>(map_q, map_k, map_vt, mt, N, q_perm, q_cluster, k_offsets, W, c0g,
                             c1g, lse, O, part_o, part_lse, status, bm, ra, sp);
}

// O rows of the split units: the two halves' float32 partials added, bf16, natural order.
// One CTA per split unit, a thread per row.
template <int DV>
__global__ void __launch_bounds__(BM)
refine_halves(MuseTables mt, int N, const int32_t *__restrict__ q_perm, const float *__restrict__ opart,
              __nv_bfloat16 *__restrict__ O, SplitArgs sp) {
  const int unit = sp.full + (int)blockIdx.x, p = unit / sp.tpp, r0 = (unit % sp.tpp) * BM;
  const Task q = make_task(mt.q, p * mt.q.nseg);
  const int n = r0 + (int)threadIdx.x;
  if (n >= q.n) return;
  const int row = q_perm[q.lab + n];
  const float4 *a = reinterpret_cast<const float4 *>(opart + ((int64_t)(2 * blockIdx.x) * BM + threadIdx.x) * DV);
  const float4 *b = reinterpret_cast<const float4 *>(opart + ((int64_t)(2 * blockIdx.x + 1) * BM + threadIdx.x) * DV);
  uint2 *dst = reinterpret_cast<uint2 *>(O + ((int64_t)p * N + row) * DV);
#pragma unroll 4
  for (int u = 0; u < DV / 4; ++u) {
    const float4 x = a[u], y = b[u];
    __nv_bfloat162 h0 = __floats2bfloat162_rn(x.x + y.x, x.y + y.y);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(x.z + y.z, x.w + y.w);
    dst[u] = make_uint2(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1));
  }
}

// ------------------------------------------------------------------ host side
template <int D, int DV, bool RET>
static cudaError_t launch(const MuseTables &mt, int N, int P, SortedSide qs, const int32_t *q_perm,
                          SortedSide ks, const int32_t *k_offsets, const void *vt, StageBufs b,
                          void *O, float *part_o, float *part_lse, int *status, cudaStream_t st,
                          const RetArgs &ra) {
  CUtensorMap mq, mk, mv;
  const int ldv = vt_ld(mt.k.row_stride);
  if (!make_map(&mq, qs.rows, D, (uint64_t)P * mt.q.row_stride, D, BM) ||
      !make_map(&mk, ks.rows, D, (uint64_t)P * mt.k.row_stride, D, 64) ||
      !make_map(&mv, vt, ldv, (uint64_t)P * DV, ldv, DV))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem<D, DV>) + 1024;
  auto kern = refine_tc_kernel<D, DV, RET>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
  if (fa.maxThreadsPerBlock < kThreads) return cudaErrorLaunchOutOfResources;
  const BlockMap bm = make_block_map(mt.q, BM);
  // One CTA per SM: with T units (problem, 128-row tile) the last wave holds T % SMs of them.
  // In the single-instance output mode, when at most half an SM count is left over, those
  // units are split into key halves so that the last wave is about full and half as long.
  SplitArgs sp{0, 0, b.opart};
  int dev = 0, sms = 0;
  if (!RET && O && mt.in.ninst == 1 && b.opart && cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0) {
    const int T = bm.total * P, R = T % sms;
    if (R > 0 && 2 * R <= sms && 2 * R <= kSplitSlots && mt.k.nrow[0] >= 16) {
      sp.tpp = bm.total;
      sp.full = T - R;
    }
  }
  cudaGetLastError();  // (attribute queries leave no error behind)
  if (sp.tpp > 0) {
    const int R = bm.total * P - sp.full;
    kern<<<dim3(sp.full + 2 * R), kThreads, smem, st>>>(mq, mk, mv, mt, N, q_perm, qs.cluster, k_offsets,
                                                         b.W, b.c0, b.c1, b.lse, (__nv_bfloat16 *)O,
                                                         part_o, part_lse, status, bm, ra, sp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    refine_halves<DV><<<R, BM, 0, st>>>(mt, N, q_perm, sp.opart, (__nv_bfloat16 *)O, sp);
    count_launches(2);
    return cudaGetLastError();
  }
  dim3 grid(bm.total, P);
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, mt, N, q_perm, qs.cluster, k_offsets, b.W, b.c0,
                                     b.c1, b.lse, (__nv_bfloat16 *)O, part_o, part_lse, status, bm,
                                     ra, sp);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tcr

bool tc_supported(int dtype, int D, int Dv) {
  return dtype == MUSE_BF16 && (D == 64 || D == 128) && (Dv == 64 || Dv == 128);
}

cudaError_t run_refine_tc(const MuseTables &mt, int D, int Dv, int N, int P, SortedSide qs,
                          const int32_t *q_perm, SortedSide ks, const int32_t *k_offsets,
                          const void *vt, StageBufs b, void *O, float *part_o, float *part_lse,
                          int *status, cudaStream_t st) {
  const tcr::RetArgs ra{};
#define MUSE_REFINE_TC(DD, DDV)                                                              \
  if (D == DD && Dv == DDV)                                                                  \
    return tcr::launch<DD, DDV, false>(mt, N, P, qs, q_perm, ks, k_offsets, vt, b, O, part_o, \
                                       part_lse, status, st, ra);
  MUSE_REFINE_TC(64, 64)
  MUSE_REFINE_TC(64, 128)
  MUSE_REFINE_TC(128, 64)
  MUSE_REFINE_TC(128, 128)
#undef MUSE_REFINE_TC
  return cudaErrorInvalidValue;
}

cudaError_t run_refine_tc_ret(const MuseTables &mt, int D, int Dv, int N, int P, SortedSide qs,
                              const int32_t *q_perm, SortedSide ks, const int32_t *k_offsets,
                              const void *vt, StageBufs b, float *part_o, float *part_lse,
                              const unsigned short *kblk, const int *kgrp, const int32_t *pend,
                              const int32_t *sel, int S, int k1, int k2, int *status,
                              cudaStream_t st) {
  tcr::RetArgs ra;
  ra.kblk = kblk;
  ra.kgrp = kgrp;
  ra.pend = pend;
  ra.sel = sel;
  ra.S = S;
  ra.nb = N / S;
  ra.k1 = k1;
  ra.k2 = k2;
  ra.K12 = k1 * k2 > 1 ? k1 * k2 : 1;
  ra.Cq = mt.q.C[0];
#define MUSE_REFINE_TC(DD, DDV)                                                                 \
  if (D == DD && Dv == DDV)                                                                     \
    return tcr::launch<DD, DDV, true>(mt, N, P, qs, q_perm, ks, k_offsets, vt, b, nullptr, part_o, \
                                      part_lse, status, st, ra);
  MUSE_REFINE_TC(64, 64)
  MUSE_REFINE_TC(64, 128)
  MUSE_REFINE_TC(128, 64)
  MUSE_REFINE_TC(128, 128)
#undef MUSE_REFINE_TC
  return cudaErrorInvalidValue;
}

}  // namespace muse
