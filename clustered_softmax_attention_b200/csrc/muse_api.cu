// extern "C" entry points of libmuse: argument validation, segment tables,
// workspace layout and the launch sequence of every call.  Declarations and the
// meaning of every argument: include/muse.h.
#include <math.h>

#include <atomic>
#include <mutex>
#include <string.h>
#include <vector>

#include "internal.h"
#include "tc.h"

namespace muse {

// ---------------------------------------------------------------------------
// Device status block (common.cuh): one per device.  Its status word is read and
// cleared by muse_last_device_status, its test-hook words set by muse_set_test_hooks.
// ---------------------------------------------------------------------------
static __device__ __align__(16) int g_status_word[kStatusInts];

static std::atomic<uint64_t> g_launches{0};
static std::atomic<void *> g_prof_start{nullptr}, g_prof_stop{nullptr};

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static int *status_ptr() {
  static std::mutex mu;
  static int *ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int *>(p);
  }
  return ptrs[dev];
}

int *device_status_word() { return status_ptr(); }

static thread_local cudaError_t t_last_cuda = cudaSuccess;
muse_status cuda_fail(cudaError_t e) {
  t_last_cuda = e;
  return MUSE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Workspace: a bump allocator over the caller's buffer (or a size count when
// base == nullptr).  Every piece is 256-byte aligned.
// ---------------------------------------------------------------------------
struct Bump {
  char *base;
  size_t off = 0;
  explicit Bump(void *b) : base(static_cast<char *>(b)) {}
  template <typename T>
  T *take(size_t count) {
    const size_t o = off;
    off = align_up(off + count * sizeof(T));
    return base ? reinterpret_cast<T *>(base + o) : nullptr;
  }
};

static size_t elem_size(int dtype) { return dtype == MUSE_F32 ? 4 : 2; }
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static muse_status check_dims(const muse_dims &d, bool need_dv) {
  if (d.dtype != MUSE_F32 && d.dtype != MUSE_BF16) return MUSE_ERR_DTYPE;
  if (d.B <= 0 || d.H <= 0 || d.N <= 0) return MUSE_ERR_SHAPE;
  if (d.D != 64 && d.D != 128) return MUSE_ERR_SHAPE;
  if (need_dv && d.Dv != 64 && d.Dv != 128) return MUSE_ERR_SHAPE;
  if ((int64_t)d.B * d.H > 65535) return MUSE_ERR_SHAPE;
  if ((int64_t)d.N * 128 > (int64_t)1 << 31) return MUSE_ERR_SHAPE;
  if (!isfinite(d.scale)) return MUSE_ERR_INVALID_ARG;
  return MUSE_OK;
}

static bool valid_C(int C, int n) { return C >= 1 && C <= n && C <= kMaxClusters; }

// One segment covering the whole sequence.
static SegTable whole_side(int N, int C) {
  SegTable t;
  memset(&t, 0, sizeof(t));
  t.nseg = 1;
  t.row_stride = N;
  t.cen_stride = C;
  t.off_stride = C + 1;
  t.max_rows = N;
  t.max_C = C;
  t.row0[0] = 0;
  t.nrow[0] = N;
  t.C[0] = C;
  return t;
}

static InstTable whole_inst(int N, int Cq, int Ck) {
  InstTable in;
  memset(&in, 0, sizeof(in));
  in.ninst = 1;
  in.w_stride = Cq * w_ld(N);
  in.z_stride = Cq * Ck;
  in.c_stride = Ck * w_ld(N);
  in.out_stride = N;
  return in;
}

// Squares of the causal decomposition: level l (side s = block*2^(l-1)), odd r with
// r*s < N: queries [r s, min((r+1) s, N)), keys [(r-1) s, r s).
struct Square {
  int lev, q0, q1, k0, k1;
};
static std::vector<Square> causal_squares(int N, int block) {
  std::vector<Square> out;
  int lev = 1;
  for (int64_t s = block; s < N; s *= 2, ++lev)
    for (int64_t r = 1; r * s < N; r += 2)
      out.push_back({lev, (int)(r * s), (int)std::min<int64_t>((r + 1) * s, N), (int)((r - 1) * s),
                     (int)(r * s)});
  return out;
}

}  // namespace muse

using namespace muse;

extern "C" int muse_causal_levels(int N, int block) {
  if (N <= 0 || block <= 0) return 0;
  int L = 0;
  for (int64_t s = block; s < N; s *= 2) ++L;
  return L;
}

namespace muse {

static bool build_causal(int N, int block, int Cq, int Ck, MuseTables &mt, int &levels) {
  levels = muse_causal_levels(N, block);
  std::vector<Square> sq = causal_squares(N, block);
  if ((int)sq.size() > kMaxSeg || sq.empty()) return false;
  memset(&mt, 0, sizeof(mt));
  SegTable &q = mt.q, &k = mt.k;
  InstTable &in = mt.in;
  q.nseg = k.nseg = in.ninst = (int)sq.size();
  int cq_acc = 0, ck_acc = 0, oq = 0, ok = 0, w = 0, z = 0, c = 0;
  for (size_t s = 0; s < sq.size(); ++s) {
    const Square &x = sq[s];
    const int nq = x.q1 - x.q0, nk = x.k1 - x.k0;
    const int cq = std::min(Cq, nq), ck = std::min(Ck, nk);
    q.row0[s] = x.q0; q.nrow[s] = nq; q.C[s] = cq; q.lab0[s] = (x.lev - 1) * N + x.q0;
    q.cen0[s] = cq_acc; q.off0[s] = oq;
    k.row0[s] = x.k0; k.nrow[s] = nk; k.C[s] = ck; k.lab0[s] = (x.lev - 1) * N + x.k0;
    k.cen0[s] = ck_acc; k.off0[s] = ok;
    in.w0[s] = w; in.z0[s] = z; in.cc0[s] = c; in.out0[s] = (x.lev - 1) * N;
    cq_acc += cq; ck_acc += ck; oq += cq + 1; ok += ck + 1;
    w += cq * w_ld(nk); z += cq * ck; c += ck * w_ld(nq);
    q.max_rows = std::max(q.max_rows, nq); k.max_rows = std::max(k.max_rows, nk);
    q.max_C = std::max(q.max_C, cq); k.max_C = std::max(k.max_C, ck);
  }
  q.row_stride = k.row_stride = levels * N;
  q.cen_stride = cq_acc; k.cen_stride = ck_acc;
  q.off_stride = oq; k.off_stride = ok;
  in.w_stride = w; in.z_stride = z; in.c_stride = c; in.out_stride = levels * N;
  return true;
}

// Workspace of the refinement (sorted copies, tilt weights, coefficients).
struct RefineWs {
  SortedSide qs, ks;
  void *vs;
  int32_t *v_cluster;
  StageBufs sb;
};

static void plan_refine(Bump &bp, const MuseTables &mt, const muse_dims &d, int P, RefineWs &r,
                        bool need_logZ_mu) {
  const size_t es = elem_size(d.dtype);
  const size_t qrows = (size_t)P * mt.q.row_stride, krows = (size_t)P * mt.k.row_stride;
  r.qs.rows = bp.take<char>(qrows * d.D * es);
  r.qs.cluster = bp.take<int32_t>(qrows);
  r.ks.rows = bp.take<char>(krows * d.D * es);
  r.ks.cluster = bp.take<int32_t>(krows);
  r.vs = bp.take<char>((size_t)P * d.Dv * vt_ld(mt.k.row_stride) * es);
  r.v_cluster = bp.take<int32_t>(krows);
  memset(&r.sb, 0, sizeof(r.sb));
  r.sb.W = bp.take<float>((size_t)P * mt.in.w_stride);
  if (need_logZ_mu) {
    r.sb.logZ = bp.take<float>((size_t)P * mt.in.z_stride);
    r.sb.mu_k = bp.take<float>((size_t)P * mt.in.z_stride * d.D);
  }
  r.sb.c0 = bp.take<float>((size_t)P * mt.in.c_stride);
  r.sb.c1 = bp.take<float>((size_t)P * mt.in.c_stride);
  r.sb.lse = bp.take<float>(qrows);
  r.sb.opart = bp.take<float>((size_t)kSplitCtas * 128 * d.Dv);
}

struct KmWs {
  KmeansOut q, k;
  char *scratch;
};

static void plan_kmeans_pair(Bump &bp, const MuseTables &mt, const muse_dims &d, int P, KmWs &w) {
  auto side = [&](const SegTable &t, KmeansOut &o) {
    o.labels = bp.take<int32_t>((size_t)P * t.row_stride);
    o.centroids = bp.take<float>((size_t)P * t.cen_stride * d.D);
    o.perm = bp.take<int32_t>((size_t)P * t.row_stride);
    o.offsets = bp.take<int32_t>((size_t)P * t.off_stride);
  };
  side(mt.q, w.q);
  side(mt.k, w.k);
  w.scratch = bp.take<char>(kmeans_pair_ws_bytes(&mt.q, &mt.k, P, d.D));
}

#define MUSE_TRY(expr)                                  \
  do {                                                  \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_);        \
  } while (0)

// Inside a stream capture the event becomes an event-record node of the graph, so
// every replay records it; outside a capture it is an ordinary record.
static cudaError_t record_profile_event(void *ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  if (cs == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags((cudaEvent_t)ev, st, cudaEventRecordExternal);
  return cudaEventRecord((cudaEvent_t)ev, st);
}

cudaError_t profile_mark(bool start, cudaStream_t st) {
  void *ev0 = g_prof_start.load(), *ev1 = g_prof_stop.load();
  if (!ev0 || !ev1) return cudaSuccess;
  return record_profile_event(start ? ev0 : ev1, st);
}

// The refinement's two evaluations of the same sum: the pair form costs 2 N^2 (D + Dv)
// tensor flops per problem; the summary form 2 Dv D N per unit of up to 224 rows of one
// query cluster (about N / 224 + Cq / 2 units) plus 2 Dv (D + 16) Ck N.  The summary form
// is taken when it needs under three quarters of the pair form's flops.
static bool summary_form_cheaper(int N, int Cq, int Ck, int D, int Dv) {
  const double n = N, pair = 2.0 * n * n * (D + Dv);
  const double summ = 2.0 * Dv * D * n * (n / 224.0 + Cq / 2.0) + 2.0 * Dv * (D + 16) * (double)Ck * n;
  return summ < 0.75 * pair;
}

// Whether the full method's refinement runs in summary form.  form: 0 = by the flop rule,
// 1 = wherever supported, 2 = never; out: the call writes O (not the causal partials).
static bool use_summary_form(const muse_dims &d, const MuseTables &mt, bool monopole, int form,
                             bool out) {
  return out && !monopole && form != 2 && tc_supported(d.dtype, d.D, d.Dv) &&
         refine_sf_supported(d.dtype, d.D, d.Dv, mt) &&
         (form == 1 || summary_form_cheaper(d.N, mt.q.C[0], mt.k.C[0], d.D, d.Dv));
}

// The refinement launch sequence shared by every path.
static muse_status refine_path(const void *Q, const void *K, const void *V, const muse_dims &d,
                               int P, const MuseTables &mt, const float *q_centroids,
                               const int32_t *q_perm, const int32_t *q_offsets,
                               const int32_t *k_perm, const int32_t *k_offsets,
                               const float *logZ_in, const float *mu_k_in, RefineWs &r, void *O,
                               float *part_o, float *part_lse, cudaStream_t st,
                               bool monopole = false, int form = 0) {
  MUSE_TRY(run_sort_side(Q, d.dtype, d.D, d.N, mt.q, P, q_perm, q_offsets, q_centroids, r.qs, st));
  MUSE_TRY(run_sort_side(K, d.dtype, d.D, d.N, mt.k, P, k_perm, k_offsets, nullptr, r.ks, st));
  const bool use_tc = tc_supported(d.dtype, d.D, d.Dv);
  if (use_tc) {
    MUSE_TRY(run_sort_side_t(V, d.dtype, d.Dv, d.N, mt.k, P, k_perm, r.vs, st));
  } else {
    SortedSide vsd{r.vs, r.v_cluster};
    MUSE_TRY(run_sort_side(V, d.dtype, d.Dv, d.N, mt.k, P, k_perm, k_offsets, nullptr, vsd, st));
  }
  StageBufs sb = r.sb;
  if (logZ_in) {
    sb.logZ = const_cast<float *>(logZ_in);
    sb.mu_k = const_cast<float *>(mu_k_in);
    MUSE_TRY(run_tilt_weights(mt, d.dtype, d.D, P, d.scale, q_centroids, r.ks, logZ_in, sb.W, st));
  } else {
    MUSE_TRY(run_summaries(mt, d.dtype, d.D, d.Dv, P, d.scale, q_centroids, r.ks, nullptr,
                           k_offsets, sb, st));
  }
  // the dipole terms carry the logit scale; the monopole-only ablation drops them
  MUSE_TRY(run_coeffs(mt, d.dtype, d.D, P, d.scale, r.qs, q_offsets, sb, monopole ? 0.f : d.scale, st));
  MUSE_TRY(profile_mark(true, st));
  if (use_summary_form(d, mt, monopole, form, O != nullptr)) {
    MUSE_TRY(run_refine_sf(mt, d.N, P, r.qs.rows, q_perm, q_offsets, r.ks.rows, k_offsets, r.vs, sb,
                           O, status_ptr(), st));
  } else if (use_tc) {
    MUSE_TRY(run_refine_tc(mt, d.D, d.Dv, d.N, P, r.qs, q_perm, r.ks, k_offsets, r.vs, sb, O,
                           part_o, part_lse, status_ptr(), st));
  } else {
    MUSE_TRY(run_refine(mt, d.dtype, d.D, d.Dv, d.N, P, r.qs, q_perm, r.ks, r.vs, sb, O, part_o,
                        part_lse, st));
  }
  MUSE_TRY(profile_mark(false, st));
  return MUSE_OK;
}

}  // namespace muse

// ===========================================================================
// Entry points
// ===========================================================================

extern "C" const char *muse_status_string(muse_status s) {
  switch (s) {
    case MUSE_OK: return "MUSE_OK";
    case MUSE_ERR_INVALID_ARG: return "MUSE_ERR_INVALID_ARG";
    case MUSE_ERR_SHAPE: return "MUSE_ERR_SHAPE";
    case MUSE_ERR_DTYPE: return "MUSE_ERR_DTYPE";
    case MUSE_ERR_WORKSPACE: return "MUSE_ERR_WORKSPACE";
    case MUSE_ERR_CUDA: return "MUSE_ERR_CUDA";
    case MUSE_ERR_TIMEOUT: return "MUSE_ERR_TIMEOUT";
    case MUSE_ERR_DEVICE: return "MUSE_ERR_DEVICE";
  }
  return "MUSE_ERR_UNKNOWN";
}

extern "C" uint64_t muse_launch_counter(void) { return g_launches.load(); }

extern "C" void muse_set_profile_events(void *start, void *stop) {
  g_prof_start.store(start);
  g_prof_stop.store(stop);
}

extern "C" muse_status muse_last_device_status(muse_stream_t st) {
  if (cudaStreamSynchronize((cudaStream_t)st) != cudaSuccess) return MUSE_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int)) != cudaSuccess) return MUSE_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return MUSE_ERR_CUDA;
  return (muse_status)v;
}

extern "C" muse_status muse_set_test_hooks(unsigned hooks, uint64_t wait_limit_ns) {
  if (hooks & ~(unsigned)MUSE_TEST_WITHHOLD_VALUES) return MUSE_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MUSE_ERR_CUDA;
  int words[3];
  words[0] = (int)hooks;
  memcpy(&words[1], &wait_limit_ns, sizeof(uint64_t));
  if (cudaMemcpyToSymbol(g_status_word, words, sizeof(words), sizeof(int)) != cudaSuccess) {
    const cudaError_t e_ = cudaGetLastError();
    return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return MUSE_ERR_CUDA;
  return MUSE_OK;
}

// --------------------------------------------------------------------------- sizes

static size_t ws_kmeans(const muse_dims &d, int C) {
  SegTable t = whole_side(d.N, C);
  return kmeans_ws_bytes(t, d.B * d.H, d.D);
}

static size_t ws_summaries(const muse_dims &d, int Cq, int Ck, bool need_v, bool need_mu) {
  const int P = d.B * d.H;
  MuseTables mt;
  mt.q = whole_side(d.N, Cq);
  mt.k = whole_side(d.N, Ck);
  mt.in = whole_inst(d.N, Cq, Ck);
  Bump bp(nullptr);
  const size_t es = elem_size(d.dtype);
  bp.take<char>((size_t)P * d.N * d.D * es);
  bp.take<int32_t>((size_t)P * d.N);
  if (need_v) bp.take<char>((size_t)P * d.N * d.Dv * es);
  bp.take<float>((size_t)P * mt.in.w_stride);
  if (need_mu) {
    bp.take<float>((size_t)P * mt.in.z_stride * d.D);
    bp.take<float>((size_t)P * mt.in.z_stride * d.Dv);
  }
  return bp.off;
}

static size_t ws_refine(const muse_dims &d, int Cq, int Ck) {
  MuseTables mt;
  mt.q = whole_side(d.N, Cq);
  mt.k = whole_side(d.N, Ck);
  mt.in = whole_inst(d.N, Cq, Ck);
  Bump bp(nullptr);
  RefineWs r;
  plan_refine(bp, mt, d, d.B * d.H, r, false);
  return bp.off;
}

// the partially specialised dipole's covariances (after the forward pass's buffers)
static size_t ws_partial_dipole(const muse_dims &d, int Cq, int Ck) {
  return partial_dipole_ws_floats(d.B * d.H, Cq, Ck, d.D, d.Dv) * sizeof(float) + 256;
}

// the tilted value means of the summary-form ablations (after the forward pass's buffers)
static size_t ws_value_means(const muse_dims &d, int Cq, int Ck) {
  return (size_t)d.B * d.H * Cq * Ck * d.Dv * sizeof(float) + 256;
}

static size_t ws_forward(const muse_dims &d, int Cq, int Ck) {
  MuseTables mt;
  mt.q = whole_side(d.N, Cq);
  mt.k = whole_side(d.N, Ck);
  mt.in = whole_inst(d.N, Cq, Ck);
  Bump bp(nullptr);
  KmWs kw;
  plan_kmeans_pair(bp, mt, d, d.B * d.H, kw);
  RefineWs r;
  plan_refine(bp, mt, d, d.B * d.H, r, true);
  return bp.off;
}

static size_t ws_causal(const muse_dims &d, int block, int Cq, int Ck) {
  MuseTables mt;
  int L = 0;
  if (!build_causal(d.N, block, Cq, Ck, mt, L)) return 0;
  const int P = d.B * d.H;
  Bump bp(nullptr);
  KmWs kw;
  plan_kmeans_pair(bp, mt, d, P, kw);
  RefineWs r;
  plan_refine(bp, mt, d, P, r, true);
  bp.take<float>((size_t)P * L * d.N * d.Dv);
  bp.take<float>((size_t)P * L * d.N);
  return bp.off;
}

extern "C" size_t muse_workspace_size(const char *entry, muse_dims d, int Cq, int Ck, int block,
                                      int k1, int k2) {
  if (!entry) return 0;
  const bool dv_needed = strcmp(entry, "muse_kmeans") != 0;
  if (check_dims(d, dv_needed) != MUSE_OK) return 0;
  if (!strcmp(entry, "muse_kmeans")) return valid_C(Cq, d.N) ? ws_kmeans(d, Cq) : 0;
  if (!valid_C(Cq, d.N) && strcmp(entry, "muse_causal_blocks") != 0) return 0;
  if (!strcmp(entry, "muse_tilted_summaries"))
    return valid_C(Ck, d.N) ? ws_summaries(d, Cq, Ck, true, true) : 0;
  if (!strcmp(entry, "muse_dipole_refine")) return valid_C(Ck, d.N) ? ws_refine(d, Cq, Ck) : 0;
  if (!strcmp(entry, "muse_forward")) return valid_C(Ck, d.N) ? ws_forward(d, Cq, Ck) : 0;
  if (!strcmp(entry, "muse_forward_ex"))
    return valid_C(Ck, d.N)
               ? ws_forward(d, Cq, Ck) + ws_partial_dipole(d, Cq, Ck) + ws_value_means(d, Cq, Ck)
               : 0;
  if (!strcmp(entry, "muse_causal_blocks")) {
    if (block <= 0 || block % 64 || d.N % block || Cq < 1 || Ck < 1 || Cq > kMaxClusters ||
        Ck > kMaxClusters)
      return 0;
    return ws_causal(d, block, Cq, Ck);
  }
  if (!strcmp(entry, "muse_retrieve_exact")) return muse_retrieval_ws(d, block, Cq, Ck, k1, k2);
  if (!strcmp(entry, "muse_backward")) return valid_C(Ck, d.N) ? muse_backward_ws(d, Cq, Ck) : 0;
  return 0;
}

// --------------------------------------------------------------------------- muse_kmeans

extern "C" muse_status muse_kmeans(const void *X, muse_dims d, int C, int iters, int32_t *labels,
                                   float *centroids, int32_t *perm, int32_t *offsets, void *ws,
                                   size_t ws_bytes, muse_stream_t st) {
  muse_status s = check_dims(d, false);
  if (s != MUSE_OK) return s;
  if (!X || !labels || !centroids || !perm || !offsets) return MUSE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(labels) || !aligned16(centroids) || !aligned16(perm) ||
      !aligned16(offsets))
    return MUSE_ERR_INVALID_ARG;
  if (!valid_C(C, d.N) || iters < 1 || iters > 1000) return MUSE_ERR_INVALID_ARG;
  const size_t need = ws_kmeans(d, C);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MUSE_ERR_WORKSPACE;
  SegTable t = whole_side(d.N, C);
  KmeansOut o{labels, centroids, perm, offsets};
  if (run_kmeans(X, d.dtype, d.D, d.N, t, d.B * d.H, iters, o, (char *)ws, status_ptr(),
                 (cudaStream_t)st) != cudaSuccess) {
    const cudaError_t e_ = cudaGetLastError();
    return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
  }
  return MUSE_OK;
}

// --------------------------------------------------------------------------- summaries

extern "C" muse_status muse_tilted_summaries(const float *q_centroids, const void *K,
                                             const void *V, const int32_t *k_perm,
                                             const int32_t *k_offsets, muse_dims d, int Cq, int Ck,
                                             float *logZ, float *mu_k, float *mu_v, float *cov,
                                             void *ws, size_t ws_bytes, muse_stream_t st) {
  const bool need_v = mu_v || cov;
  muse_status s = check_dims(d, need_v);
  if (s != MUSE_OK) return s;
  if (!q_centroids || !K || !k_perm || !k_offsets || !logZ || (need_v && !V))
    return MUSE_ERR_INVALID_ARG;
  for (const void *p : {(const void *)q_centroids, K, V, (const void *)k_perm,
                        (const void *)k_offsets, (const void *)logZ, (const void *)mu_k,
                        (const void *)mu_v, (const void *)cov})
    if (p && !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  if (!valid_C(Cq, d.N) || !valid_C(Ck, d.N)) return MUSE_ERR_INVALID_ARG;
  const size_t need = ws_summaries(d, Cq, Ck, true, true);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MUSE_ERR_WORKSPACE;
  const int P = d.B * d.H;
  MuseTables mt;
  mt.q = whole_side(d.N, Cq);
  mt.k = whole_side(d.N, Ck);
  mt.in = whole_inst(d.N, Cq, Ck);
  Bump bp(ws);
  const size_t es = elem_size(d.dtype);
  SortedSide ks{bp.take<char>((size_t)P * d.N * d.D * es), bp.take<int32_t>((size_t)P * d.N)};
  void *vs = bp.take<char>((size_t)P * d.N * d.Dv * es);
  StageBufs sb;
  memset(&sb, 0, sizeof(sb));
  sb.W = bp.take<float>((size_t)P * mt.in.w_stride);
  float *mk_int = bp.take<float>((size_t)P * mt.in.z_stride * d.D);
  float *mv_int = bp.take<float>((size_t)P * mt.in.z_stride * d.Dv);
  sb.logZ = logZ;
  sb.mu_k = mu_k ? mu_k : (cov ? mk_int : nullptr);
  sb.mu_v = mu_v ? mu_v : (cov ? mv_int : nullptr);
  sb.cov = cov;
  cudaStream_t cs = (cudaStream_t)st;
  if (run_sort_side(K, d.dtype, d.D, d.N, mt.k, P, k_perm, k_offsets, nullptr, ks, cs) !=
      cudaSuccess)
    return MUSE_ERR_CUDA;
  if (need_v) {
    SortedSide vsd{vs, ks.cluster};
    if (run_sort_side(V, d.dtype, d.Dv, d.N, mt.k, P, k_perm, k_offsets, nullptr, vsd, cs) !=
        cudaSuccess)
      return MUSE_ERR_CUDA;
  }
  if (run_summaries(mt, d.dtype, d.D, d.Dv, P, d.scale, q_centroids, ks, vs, k_offsets, sb, cs) !=
      cudaSuccess)
    return MUSE_ERR_CUDA;
  return MUSE_OK;
}

// --------------------------------------------------------------------------- refine

extern "C" muse_status muse_dipole_refine(const void *Q, const void *K, const void *V,
                                          const int32_t *q_labels, const float *q_centroids,
                                          const int32_t *q_perm, const int32_t *q_offsets,
                                          const int32_t *k_perm, const int32_t *k_offsets,
                                          const float *logZ, const float *mu_k,
                                          const float *mu_v, const float *cov, muse_dims d,
                                          int Cq, int Ck, void *O, void *ws, size_t ws_bytes,
                                          muse_stream_t st) {
  muse_status s = check_dims(d, true);
  if (s != MUSE_OK) return s;
  const void *ptrs[] = {Q, K, V, q_centroids, q_perm, q_offsets, k_perm, k_offsets, logZ, mu_k, O};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  for (const void *p : {(const void *)q_labels, (const void *)mu_v, (const void *)cov})
    if (p && !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  if (!mu_v != !cov) return MUSE_ERR_INVALID_ARG;  // both materialised, or neither
  if (!valid_C(Cq, d.N) || !valid_C(Ck, d.N)) return MUSE_ERR_INVALID_ARG;
  const size_t need = ws_refine(d, Cq, Ck);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MUSE_ERR_WORKSPACE;
  const int P = d.B * d.H;
  if (cov) {
    // the summaries are given: the refinement reads them as they are
    if (run_refine_summaries(d.dtype, d.D, d.Dv, d.N, P, Cq, Ck, d.scale, Q, q_centroids, q_perm,
                             q_offsets, q_labels, logZ, mu_k, mu_v, cov, O, status_ptr(),
                             (cudaStream_t)st) != cudaSuccess) {
      const cudaError_t e_ = cudaGetLastError();
      return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
    }
    return MUSE_OK;
  }
  MuseTables mt;
  mt.q = whole_side(d.N, Cq);
  mt.k = whole_side(d.N, Ck);
  mt.in = whole_inst(d.N, Cq, Ck);
  Bump bp(ws);
  RefineWs r;
  plan_refine(bp, mt, d, P, r, false);
  return refine_path(Q, K, V, d, P, mt, q_centroids, q_perm, q_offsets, k_perm, k_offsets, logZ,
                     mu_k, r, O, nullptr, nullptr, (cudaStream_t)st);
}

// --------------------------------------------------------------------------- forward

extern "C" muse_status muse_forward_ex(const void *Q, const void *K, const void *V, muse_dims d,
                                       int Cq, int Ck, int iters, unsigned flags, void *O, void *ws,
                                       size_t ws_bytes, muse_stream_t st) {
  muse_status s = check_dims(d, true);
  if (s != MUSE_OK) return s;
  const unsigned abl = MUSE_FLAG_MONOPOLE | MUSE_FLAG_PARTIAL_DIPOLE;
  const unsigned frm = MUSE_FLAG_REFINE_SUMMARY | MUSE_FLAG_REFINE_PAIR;
  if ((flags & ~(abl | frm)) || (flags & abl) == abl || (flags & frm) == frm ||
      ((flags & abl) && (flags & frm)))
    return MUSE_ERR_INVALID_ARG;
  const bool partial = (flags & MUSE_FLAG_PARTIAL_DIPOLE) != 0;
  const int form = (flags & MUSE_FLAG_REFINE_SUMMARY) ? 1 : (flags & MUSE_FLAG_REFINE_PAIR) ? 2 : 0;
  const void *ptrs[] = {Q, K, V, O};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  if (!valid_C(Cq, d.N) || !valid_C(Ck, d.N) || iters < 1 || iters > 1000)
    return MUSE_ERR_INVALID_ARG;
  // the ablations in summary form (no O(N^2) contraction) where the output kernel fits
  const bool summary = (flags & abl) != 0 && coef_out_supported(d.dtype, d.D, d.Dv, Ck);
  const size_t need = ws_forward(d, Cq, Ck) + (partial ? ws_partial_dipole(d, Cq, Ck) : 0) +
                      (summary ? ws_value_means(d, Cq, Ck) : 0);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MUSE_ERR_WORKSPACE;
  const int P = d.B * d.H;
  MuseTables mt;
  mt.q = whole_side(d.N, Cq);
  mt.k = whole_side(d.N, Ck);
  mt.in = whole_inst(d.N, Cq, Ck);
  Bump bp(ws);
  KmWs kw;
  plan_kmeans_pair(bp, mt, d, P, kw);
  RefineWs r;
  plan_refine(bp, mt, d, P, r, true);
  float *pd_ws = partial ? bp.take<float>(partial_dipole_ws_floats(P, Cq, Ck, d.D, d.Dv)) : nullptr;
  float *mu_v = summary ? bp.take<float>((size_t)P * mt.in.z_stride * d.Dv) : nullptr;
  cudaStream_t cs = (cudaStream_t)st;
  int *stat = status_ptr();
  if (run_kmeans_pair(Q, mt.q, kw.q, K, mt.k, kw.k, d.dtype, d.D, d.N, P, iters, kw.scratch, stat,
                      cs) != cudaSuccess) {
    const cudaError_t e_ = cudaGetLastError();
    return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
  }
  if (summary) {
    // O_n = sum_j p_j mu_v,ij (+ s Cbar_i qt_n) from the summaries: sorted copies (values
    // row-major), tilt weights / logZ / mu_k, the tilted value means, the aggregated
    // covariances for the partial dipole, then one output kernel
    MUSE_TRY(run_sort_side(Q, d.dtype, d.D, d.N, mt.q, P, kw.q.perm, kw.q.offsets, kw.q.centroids,
                           r.qs, cs));
    MUSE_TRY(run_sort_side(K, d.dtype, d.D, d.N, mt.k, P, kw.k.perm, kw.k.offsets, nullptr, r.ks, cs));
    SortedSide vsd{r.vs, r.v_cluster};
    MUSE_TRY(run_sort_side(V, d.dtype, d.Dv, d.N, mt.k, P, kw.k.perm, kw.k.offsets, nullptr, vsd, cs));
    StageBufs sb = r.sb;
    MUSE_TRY(run_summaries(mt, d.dtype, d.D, d.Dv, P, d.scale, kw.q.centroids, r.ks, nullptr,
                           kw.k.offsets, sb, cs));
    MUSE_TRY(run_tilt_values(mt, d.dtype, d.Dv, P, kw.k.offsets, sb.W, r.vs, mu_v, cs));
    sb.mu_v = mu_v;
    const float *cbar = nullptr;
    if (partial) {
      MUSE_TRY(run_partial_dipole(mt, d.dtype, d.D, d.Dv, d.N, P, d.scale, r.qs, kw.q.perm, r.ks, V,
                                  kw.k.perm, kw.k.offsets, sb.logZ, pd_ws, nullptr, cs));
      cbar = partial_dipole_cbar(pd_ws, P, mt.k.max_C, d.D, d.Dv);
    }
    MUSE_TRY(profile_mark(true, cs));
    MUSE_TRY(run_coef_out(mt, d.D, d.N, P, d.scale, r.qs.rows, kw.q.perm, kw.q.offsets, sb, cbar, O,
                          stat, cs));
    MUSE_TRY(profile_mark(false, cs));
    return MUSE_OK;
  }
  // the partially specialised dipole adds s Cbar_i qt to the monopole-only result
  muse_status s2 = refine_path(Q, K, V, d, P, mt, kw.q.centroids, kw.q.perm, kw.q.offsets,
                               kw.k.perm, kw.k.offsets, nullptr, nullptr, r, O, nullptr, nullptr,
                               cs, (flags & abl) != 0, form);
  if (s2 != MUSE_OK || !partial) return s2;
  MUSE_TRY(run_partial_dipole(mt, d.dtype, d.D, d.Dv, d.N, P, d.scale, r.qs, kw.q.perm, r.ks, V,
                              kw.k.perm, kw.k.offsets, r.sb.logZ, pd_ws, O, cs));
  return MUSE_OK;
}

extern "C" int muse_refine_form(muse_dims d, int Cq, int Ck, unsigned flags) {
  if (check_dims(d, true) != MUSE_OK || !valid_C(Cq, d.N) || !valid_C(Ck, d.N)) return -1;
  const unsigned frm = MUSE_FLAG_REFINE_SUMMARY | MUSE_FLAG_REFINE_PAIR;
  if ((flags & ~frm) || (flags & frm) == frm) return -1;
  MuseTables mt;
  mt.q = whole_side(d.N, Cq);
  mt.k = whole_side(d.N, Ck);
  mt.in = whole_inst(d.N, Cq, Ck);
  const int form = (flags & MUSE_FLAG_REFINE_SUMMARY) ? 1 : (flags & MUSE_FLAG_REFINE_PAIR) ? 2 : 0;
  return use_summary_form(d, mt, false, form, true) ? 1 : 0;
}

extern "C" muse_status muse_forward(const void *Q, const void *K, const void *V, muse_dims d,
                                    int Cq, int Ck, int iters, void *O, void *ws, size_t ws_bytes,
                                    muse_stream_t st) {
  return muse_forward_ex(Q, K, V, d, Cq, Ck, iters, 0u, O, ws, ws_bytes, st);
}

// --------------------------------------------------------------------------- causal

extern "C" muse_status muse_causal_blocks(const void *Q, const void *K, const void *V,
                                          muse_dims d, int block, int Cq, int Ck, int iters,
                                          void *O, int32_t *q_labels_out, int32_t *k_labels_out,
                                          void *ws, size_t ws_bytes, muse_stream_t st) {
  muse_status s = check_dims(d, true);
  if (s != MUSE_OK) return s;
  const void *ptrs[] = {Q, K, V, O};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  if ((q_labels_out && !aligned16(q_labels_out)) || (k_labels_out && !aligned16(k_labels_out)))
    return MUSE_ERR_INVALID_ARG;
  if (block <= 0 || block % 64 || d.N % block) return MUSE_ERR_SHAPE;
  if (Cq < 1 || Ck < 1 || Cq > kMaxClusters || Ck > kMaxClusters || iters < 1 || iters > 1000)
    return MUSE_ERR_INVALID_ARG;
  if (causal_squares(d.N, block).size() > (size_t)kMaxSeg) return MUSE_ERR_SHAPE;
  const int P = d.B * d.H;
  const int levels = muse_causal_levels(d.N, block);
  cudaStream_t cs = (cudaStream_t)st;
  if (levels == 0) {
    // one block: the diagonal is the whole causal attention
    if (run_diag_merge(Q, K, V, d.dtype, d.D, d.Dv, d.N, P, block, 0, d.scale, nullptr, nullptr,
                       O, cs) != cudaSuccess) {
      const cudaError_t e_ = cudaGetLastError();
      return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
    }
    return MUSE_OK;
  }
  MuseTables mt;
  int L = 0;
  build_causal(d.N, block, Cq, Ck, mt, L);
  if ((int64_t)P * mt.q.nseg > 65535) return MUSE_ERR_SHAPE;
  const size_t need = ws_causal(d, block, Cq, Ck);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MUSE_ERR_WORKSPACE;
  Bump bp(ws);
  KmWs kw;
  plan_kmeans_pair(bp, mt, d, P, kw);
  RefineWs r;
  plan_refine(bp, mt, d, P, r, true);
  float *part_o = bp.take<float>((size_t)P * L * d.N * d.Dv);
  float *part_lse = bp.take<float>((size_t)P * L * d.N);
  if (q_labels_out) kw.q.labels = q_labels_out;
  if (k_labels_out) kw.k.labels = k_labels_out;
  // rows outside every square of a level keep label -1
  if (cudaMemsetAsync(kw.q.labels, 0xff, (size_t)P * L * d.N * sizeof(int32_t), cs) != cudaSuccess ||
      cudaMemsetAsync(kw.k.labels, 0xff, (size_t)P * L * d.N * sizeof(int32_t), cs) != cudaSuccess) {
    const cudaError_t e_ = cudaGetLastError();
    return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
  }
  int *stat = status_ptr();
  if (run_kmeans_pair(Q, mt.q, kw.q, K, mt.k, kw.k, d.dtype, d.D, d.N, P, iters, kw.scratch, stat,
                      cs) != cudaSuccess) {
    const cudaError_t e_ = cudaGetLastError();
    return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
  }
  s = refine_path(Q, K, V, d, P, mt, kw.q.centroids, kw.q.perm, kw.q.offsets, kw.k.perm,
                  kw.k.offsets, nullptr, nullptr, r, nullptr, part_o, part_lse, cs);
  if (s != MUSE_OK) return s;
  if (run_diag_merge(Q, K, V, d.dtype, d.D, d.Dv, d.N, P, block, L, d.scale, part_o, part_lse, O,
                     cs) != cudaSuccess) {
    const cudaError_t e_ = cudaGetLastError();
    return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
  }
  return MUSE_OK;
}

// --------------------------------------------------------------------------- backward

extern "C" muse_status muse_backward(const void *Q, const void *K, const void *V, const void *dO,
                                     const int32_t *q_perm, const int32_t *q_offsets,
                                     const int32_t *k_perm, const int32_t *k_offsets, muse_dims d,
                                     int Cq, int Ck, void *dQ, void *dK, void *dV, void *ws,
                                     size_t ws_bytes, muse_stream_t st) {
  muse_status s = check_dims(d, true);
  if (s != MUSE_OK) return s;
  const void *ptrs[] = {Q, K, V, dO, q_perm, q_offsets, k_perm, k_offsets, dQ, dK, dV};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return MUSE_ERR_INVALID_ARG;
  if (!valid_C(Cq, d.N) || !valid_C(Ck, d.N)) return MUSE_ERR_INVALID_ARG;
  const size_t need = muse_backward_ws(d, Cq, Ck);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MUSE_ERR_WORKSPACE;
  if (run_backward(Q, K, V, dO, q_perm, q_offsets, k_perm, k_offsets, d, Cq, Ck, dQ, dK, dV, ws,
                   (cudaStream_t)st) != cudaSuccess) {
    const cudaError_t e_ = cudaGetLastError();
    return cuda_fail(e_ != cudaSuccess ? e_ : cudaErrorUnknown);
  }
  return MUSE_OK;
}

extern "C" const char *muse_last_error_detail(void) {
  return t_last_cuda == cudaSuccess ? "" : cudaGetErrorString(t_last_cuda);
}
