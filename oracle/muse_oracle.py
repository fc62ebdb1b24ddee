"""Float64 CPU oracle for the Multipole Semantic Attention (MuSe) forward pass.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously correct
statement of what the CUDA library computes.  Only the test-suite, the package's
``smoke()`` check and the CPU-baseline leg of ``bench.py`` may import it; the
product path never does, and it shares no code with the CUDA sources.

Sources (page title, then section):
  [review]   pith.science review of arXiv 2509.10406, "Multipole Semantic Attention:
             A Fast Approximation of Softmax Attention for Pretraining"
  [summary]  gist.science, "Technische Samenvatting: Multipole Semantic Attention (MuSe)"
  [abstract] fugumt.com listing of arXiv 2509.10406v2, abstract

Notation: per (batch, head) Q, K in R^{N x D}, V in R^{N x Dv}; s is the logit scale in
exp(s q.k).  Query clusters i (centroid qbar_i), key clusters j (member set S_j).
q = qbar_i + qt (the residual), k = k_j + kt ([summary] "Kernmechanismen", item 1,
"Decompositie").

Every routine is float64.  Inputs are the already-rounded values the GPU sees.

Readings taken where the pages leave a step open:
  * K-means starts from the first C rows, runs T rounds of (assign, update); the
    labels are those of round T and the centroids are the update after it.  An
    empty cluster keeps its previous centroid.  Ties go to the lowest cluster index.
  * log Z_ij is the SUM form logsumexp_{k in S_j} s qbar_i.k (it carries log|S_j|), so
    clusters are weighted by their total mass.
  * The dipole carries the logit scale: the residual enters exp(s qt.k), so its
    first-order term is s C_ij qt.
  * Causal: binary hierarchical decomposition (exact diagonal blocks plus one
    MuSe square per level), every square with its own K-means.
  * Retrieval: global clusters; block scores log Z_{i,j,b'}; top-k1 clusters by the
    prefix logsumexp, then top-k2 blocks per chosen cluster, ties to the lower index.

Parity pins for every function live in tests/test_oracle_pins.py.  Parity unpinned:
the absolute RSE values on synthetic data (the pages' RSE figures come from trained
activations) and the constant in front of the Tr(Cov(qt)Cov(kt)) error order.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Tuple

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------------------
# K-means (Lloyd), separately on queries and on keys.
# [review] "What carries the argument" and "Core claim": queries and keys are
# partitioned separately; [summary] "Kernmechanismen", item 1 (separate clustering
# of queries and keys, because attention is translation-invariant in the keys but not
# in the queries).
# ----------------------------------------------------------------------------

def kmeans_distances(X: np.ndarray, C: np.ndarray, chunk: int = 0) -> np.ndarray:
    """Squared Euclidean distances ||x_n - c_c||^2 by direct differences, [n, C].

    Rows go through in chunks (default: about 4M differences at a time) only to bound the
    temporary array; every distance is the same sum of squared differences either way."""
    X = np.asarray(X, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    if chunk <= 0:
        chunk = max(1, (1 << 22) // max(1, C.shape[0] * C.shape[1]))
    out = np.empty((X.shape[0], C.shape[0]))
    for a in range(0, X.shape[0], chunk):
        diff = X[a:a + chunk, None, :] - C[None, :, :]
        out[a:a + chunk] = np.einsum("ncd,ncd->nc", diff, diff)
    return out


def kmeans_assign(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """Nearest centroid per row; ties go to the lowest index (argmin keeps the first)."""
    return np.argmin(kmeans_distances(X, C), axis=1).astype(np.int64)


def kmeans_assign_gap(X: np.ndarray, C: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Labels plus the normalised top-2 gap (d2 - d1) / (||x||^2 + ||c_a||^2).

    The gap decides whether a label disagreement with another implementation is a
    legal near-tie: the rounding error of any expanded-form distance scales with
    ||x||^2 + ||c||^2, not with d1 (which can be ~0).
    """
    d = kmeans_distances(X, C)
    lab = np.argmin(d, axis=1)
    if C.shape[0] == 1:
        return lab.astype(np.int64), np.full(X.shape[0], np.inf)
    part = np.partition(d, 1, axis=1)
    norm = (np.asarray(X, np.float64) ** 2).sum(1) + (np.asarray(C, np.float64)[lab] ** 2).sum(1)
    gap = (part[:, 1] - part[:, 0]) / np.maximum(norm, 1e-300)
    return lab.astype(np.int64), gap


def kmeans_update(X: np.ndarray, labels: np.ndarray, C_prev: np.ndarray) -> np.ndarray:
    """Each centroid becomes the mean of its members; an empty cluster keeps C_prev."""
    X = np.asarray(X, dtype=np.float64)
    C = np.array(C_prev, dtype=np.float64, copy=True)
    for c in range(C.shape[0]):
        members = X[labels == c]
        if members.shape[0] > 0:
            C[c] = members.sum(axis=0) / members.shape[0]
    return C


def kmeans_init(X: np.ndarray, n_clusters: int) -> np.ndarray:
    """Initial centroids: the first C rows."""
    return np.array(X[:n_clusters], dtype=np.float64, copy=True)


def kmeans(X: np.ndarray, n_clusters: int, iters: int,
           history: bool = False):
    """Lloyd K-means: T rounds of (assign, update) from the first-C-rows start.

    Returns (labels of round T, centroids after round T's update) and, when
    ``history`` is set, the list of centroids before each round.
    """
    C = kmeans_init(X, n_clusters)
    hist = []
    labels = None
    for _ in range(iters):
        hist.append(C.copy())
        labels = kmeans_assign(X, C)
        C = kmeans_update(X, labels, C)
    if history:
        return labels, C, hist
    return labels, C


def kmeans_objective(X: np.ndarray, labels: np.ndarray, C: np.ndarray) -> float:
    """Within-cluster sum of squared distances."""
    diff = np.asarray(X, np.float64) - np.asarray(C, np.float64)[labels]
    return float((diff * diff).sum())


def cluster_means(X: np.ndarray, labels: np.ndarray, n_clusters: int) -> np.ndarray:
    """Mean of the members of each cluster (zero for an empty cluster)."""
    X = np.asarray(X, dtype=np.float64)
    out = np.zeros((n_clusters, X.shape[1]))
    for c in range(n_clusters):
        m = X[labels == c]
        if m.shape[0]:
            out[c] = m.sum(0) / m.shape[0]
    return out


# ----------------------------------------------------------------------------
# Stage 1: exponentially tilted monopole summaries and the tilted dipole.
# [review] "What carries the argument": each key/value cluster is a distribution; the
# log-normaliser and the value output are derivatives of its cumulant generating
# function; truncating after the first cumulants gives the monopole (tilted centroids)
# and the dipole (key-value covariance contracted with the residual query).
# [review] "Assumptions & free parameters": M_j(q) = E exp(q.k) over cluster j.
# [review] referee minor comment on Algorithm 3: the dipole of Eq. (6) is the
# exponentially tilted Cov_ij(v, k).
# [summary] "Kernmechanismen", item 2: coarse query centroids attend to key clusters
# with exponentially tilted centroids, specialised to each query cluster.
# ----------------------------------------------------------------------------

def tilted_summaries(qbar: np.ndarray, K: np.ndarray, V: np.ndarray,
                     k_labels: np.ndarray, n_kclusters: int, scale: float,
                     want_cov: bool = True):
    """For every query centroid i and key cluster j:

      l_k      = s * qbar_i . k                      (k in S_j)
      logZ_ij  = log sum_{k in S_j} exp(l_k)          (max-shifted)
      w_k      = exp(l_k - logZ_ij)                   (tilted weights, sum to 1)
      mu_k,ij  = sum_k w_k k,      mu_v,ij = sum_k w_k v
      C_ij     = sum_k w_k (v - mu_v,ij)(k - mu_k,ij)^T     [Dv x D], centred (two-pass)

    Empty key clusters get logZ = -inf and zero moments.
    Returns logZ [Cq,Ck], mu_k [Cq,Ck,D], mu_v [Cq,Ck,Dv], cov [Cq,Ck,Dv,D] (or None).
    """
    qbar = np.asarray(qbar, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    Cq, D = qbar.shape
    Dv = V.shape[1]
    Ck = n_kclusters
    logZ = np.full((Cq, Ck), NEG_INF)
    mu_k = np.zeros((Cq, Ck, D))
    mu_v = np.zeros((Cq, Ck, Dv))
    cov = np.zeros((Cq, Ck, Dv, D)) if want_cov else None
    for j in range(Ck):
        idx = np.nonzero(k_labels == j)[0]
        if idx.size == 0:
            continue
        Kj, Vj = K[idx], V[idx]
        ell = scale * (qbar @ Kj.T)                      # [Cq, n_j]
        m = ell.max(axis=1)
        lz = m + np.log(np.exp(ell - m[:, None]).sum(axis=1))
        w = np.exp(ell - lz[:, None])
        logZ[:, j] = lz
        mu_k[:, j] = w @ Kj
        mu_v[:, j] = w @ Vj
        if want_cov:
            step = max(1, 2_000_000 // max(1, idx.size * max(D, Dv)))
            for a in range(0, Cq, step):
                b = min(Cq, a + step)
                Vc = Vj[None, :, :] - mu_v[a:b, j][:, None, :]    # [c, n_j, Dv]
                Kc = Kj[None, :, :] - mu_k[a:b, j][:, None, :]    # [c, n_j, D]
                cov[a:b, j] = np.matmul((w[a:b, :, None] * Vc).transpose(0, 2, 1), Kc)
    return logZ, mu_k, mu_v, cov


# ----------------------------------------------------------------------------
# Stage 2: per-query refinement.
# [review] "What carries the argument": the two-stage scheme drops only the
# residual-residual term qt.kt.  [summary] "Kernmechanismen", items 1-2: the expansion
# of exp((q_i + qt).(k_j + kt)) keeps three of its four terms; fine queries refine the
# cluster summaries with their residuals.
# ----------------------------------------------------------------------------

def refine(Q: np.ndarray, q_labels: np.ndarray, qbar: np.ndarray, logZ: np.ndarray,
           mu_k: np.ndarray, mu_v: np.ndarray, cov: np.ndarray, scale: float,
           zero_residual: bool = False, rows: Optional[np.ndarray] = None,
           return_lse: bool = False, dipole: bool = True):
    """For query n in cluster i, qt = q_n - qbar_i:

      a_j  = logZ_ij + s * qt . mu_k,ij
      p    = softmax_j(a)
      O_n  = sum_j p_j (mu_v,ij + s * C_ij qt)

    ``zero_residual`` forces qt = 0 (the monopole-only result at the centroid).
    ``dipole=False`` drops the s C_ij qt term: the monopole-only ablation ([review]
    "invented entities": the dipole correction, whose removal the paper's Table 3
    measures), O_n = sum_j p_j mu_v,ij with the same weights p.
    ``rows`` restricts the output to those query rows (others are left zero).
    With ``return_lse`` also returns logsumexp_j a_j per row (for merging partial sums).
    """
    Q = np.asarray(Q, np.float64)
    N = Q.shape[0]
    Dv = mu_v.shape[2]
    O = np.zeros((N, Dv))
    lse = np.full(N, NEG_INF)
    sel = np.zeros(N, bool)
    if rows is None:
        sel[:] = True
    else:
        sel[np.asarray(rows)] = True
    for i in np.unique(q_labels[sel]):
        idx = np.nonzero((q_labels == i) & sel)[0]
        Qt = Q[idx] - qbar[i][None, :]
        if zero_residual:
            Qt = np.zeros_like(Qt)
        a = logZ[i][None, :] + scale * (Qt @ mu_k[i].T)           # [n_i, Ck]
        m = a.max(axis=1)
        e = np.exp(a - m[:, None])
        l = e.sum(axis=1)
        p = e / l[:, None]
        Ck, Dv_, D = cov[i].shape
        dip = (cov[i].reshape(Ck * Dv_, D) @ Qt.T).reshape(Ck, Dv_, idx.size)  # C_ij qt
        term = mu_v[i][:, :, None] + (scale * dip if dipole else 0.0)  # [Ck, Dv, n_i]
        O[idx] = np.einsum("nj,jvn->nv", p, term)
        lse[idx] = m + np.log(l)
    if return_lse:
        return O, lse
    return O


def muse_from_labels(Q, K, V, q_labels, k_labels, Cq: int, Ck: int, scale: float,
                     qbar: Optional[np.ndarray] = None, rows: Optional[np.ndarray] = None,
                     return_lse: bool = False, zero_residual: bool = False,
                     dipole: bool = True):
    """MuSe output from given clusterings.  qbar defaults to the member means.

    With ``rows`` the summaries are built only for the query clusters those rows use.
    """
    Q = np.asarray(Q, np.float64)
    q_labels = np.asarray(q_labels)
    k_labels = np.asarray(k_labels)
    if qbar is None:
        qbar = cluster_means(Q, q_labels, Cq)
    if rows is not None:
        used = np.unique(q_labels[np.asarray(rows)])
        remap = -np.ones(Cq, np.int64)
        remap[used] = np.arange(used.size)
        logZ, mu_k, mu_v, cov = tilted_summaries(qbar[used], K, V, k_labels, Ck, scale)
        lab = np.where(q_labels >= 0, remap[np.clip(q_labels, 0, Cq - 1)], -1)
        return refine(Q, lab, qbar[used], logZ, mu_k, mu_v, cov, scale,
                      zero_residual=zero_residual, rows=rows, return_lse=return_lse,
                      dipole=dipole)
    logZ, mu_k, mu_v, cov = tilted_summaries(qbar, K, V, k_labels, Ck, scale)
    return refine(Q, q_labels, qbar, logZ, mu_k, mu_v, cov, scale,
                  zero_residual=zero_residual, return_lse=return_lse, dipole=dipole)


# ----------------------------------------------------------------------------
# The partially specialised dipole ([review] "Axioms" / "ad hoc to paper": the
# covariance of each key cluster is taken without the exponential tilt by the query
# centroid, Cov_j(v,k) over the cluster's members, "aggregated per query cluster";
# referee comment on Algorithm 3: it is Cov_j(v,k), not the tilted Cov_ij(v,k)).
# The aggregation weights are not printed; the reading taken here weights cluster j
# by the monopole softmax at the centroid, pi_ij = softmax_j(logZ_ij).
# ----------------------------------------------------------------------------

def key_cluster_covariances(K: np.ndarray, V: np.ndarray, k_labels: np.ndarray,
                            n_kclusters: int) -> np.ndarray:
    """Cov_j = (1/|S_j|) sum_{k in S_j} (v - vbar_j)(k - kbar_j)^T  [Ck, Dv, D]
    (two-pass: means first; zero for an empty cluster)."""
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    out = np.zeros((n_kclusters, V.shape[1], K.shape[1]))
    for j in range(n_kclusters):
        idx = np.nonzero(k_labels == j)[0]
        if idx.size == 0:
            continue
        kc = K[idx] - K[idx].mean(axis=0)
        vc = V[idx] - V[idx].mean(axis=0)
        out[j] = vc.T @ kc / idx.size
    return out


def muse_partial_dipole_from_labels(Q, K, V, q_labels, k_labels, Cq: int, Ck: int,
                                    scale: float, qbar: Optional[np.ndarray] = None):
    """O_n = sum_j p_j mu_v,ij + s Cbar_i qt_n, with p_j = softmax_j(logZ_ij + s qt.mu_k,ij)
    (the monopole part of the full method) and Cbar_i = sum_j pi_ij Cov_j,
    pi_ij = softmax_j(logZ_ij)."""
    Q = np.asarray(Q, np.float64)
    q_labels = np.asarray(q_labels)
    if qbar is None:
        qbar = cluster_means(Q, q_labels, Cq)
    logZ, mu_k, mu_v, cov = tilted_summaries(qbar, K, V, k_labels, Ck, scale, want_cov=False)
    O = refine(Q, q_labels, qbar, logZ, mu_k, mu_v, np.zeros((Cq, Ck, mu_v.shape[2], Q.shape[1])),
               scale, dipole=False)
    covs = key_cluster_covariances(K, V, k_labels, Ck)
    for i in np.unique(q_labels):
        m = logZ[i].max()
        pi = np.exp(logZ[i] - m)          # exp(-inf) = 0 for empty clusters
        pi /= pi.sum()
        cbar = np.einsum("j,jvd->vd", pi, covs)
        idx = np.nonzero(q_labels == i)[0]
        O[idx] += scale * (Q[idx] - qbar[i][None, :]) @ cbar.T
    return O


# ----------------------------------------------------------------------------
# Backward pass: the gradient of the same approximation.
# [review] referee report and "What carries the argument": MuSe is used for pretraining,
# so the approximation itself is differentiated (the pages never measure it).  Reading
# taken: the clustering is held fixed (K-means assignments are discrete), the query
# centroid qbar_i is the mean of its members (as K-means leaves it), so gradients flow
# into Q through both qbar_i and the residuals; the key clustering enters only through
# the member sets S_j.
# ----------------------------------------------------------------------------

def muse_backward_from_labels(Q, K, V, q_labels, k_labels, Cq: int, Ck: int, scale: float, dO):
    """(dQ, dK, dV) = gradients of sum(O * dO) for O = muse_from_labels(Q, K, V, ...), labels
    fixed, qbar the member means.  Chain rule through the definitions, in reverse order:

      refinement   O_n = sum_j p_nj y_nj,  y_nj = mu_v,ij + s C_ij qt_n,
                   p_n = softmax_j(a_nj),  a_nj = logZ_ij + s qt_n . mu_k,ij
      summaries    w_ik = exp(s qbar_i.k - logZ_ij), mu_k = sum w k, mu_v = sum w v,
                   C_ij = sum w v k^T - mu_v mu_k^T   (equal to the centred form)
      centroids    qt_n = q_n - qbar_i,  qbar_i = mean of the members of cluster i
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    dO = np.asarray(dO, np.float64)
    q_labels = np.asarray(q_labels)
    k_labels = np.asarray(k_labels)
    s = scale
    N, D = Q.shape
    Dv = V.shape[1]
    qbar = cluster_means(Q, q_labels, Cq)
    logZ, mu_k, mu_v, cov = tilted_summaries(qbar, K, V, k_labels, Ck, s)
    dQt = np.zeros((N, D))
    dlogZ = np.zeros((Cq, Ck))
    dmuk = np.zeros((Cq, Ck, D))
    dmuv = np.zeros((Cq, Ck, Dv))
    dC = np.zeros((Cq, Ck, Dv, D))
    live = np.isfinite(logZ)
    # --- refinement, per query cluster
    for i in np.unique(q_labels):
        idx = np.nonzero(q_labels == i)[0]
        Qt = Q[idx] - qbar[i][None, :]
        a = np.where(live[i][None, :], logZ[i][None, :] + s * (Qt @ mu_k[i].T), NEG_INF)
        m = a.max(axis=1)
        p = np.exp(a - m[:, None])
        p /= p.sum(axis=1)[:, None]
        y = mu_v[i][None, :, :] + s * np.einsum("jvd,nd->njv", cov[i], Qt)   # [n, Ck, Dv]
        dy = p[:, :, None] * dO[idx][:, None, :]                               # dO/dy
        dp = np.einsum("nv,njv->nj", dO[idx], y)
        da = p * (dp - (p * dp).sum(axis=1)[:, None])                         # softmax
        dlogZ[i] += da.sum(axis=0)
        dQt[idx] += s * (da @ mu_k[i]) + s * np.einsum("jvd,njv->nd", cov[i], dy)
        dmuk[i] += s * (da.T @ Qt)
        dmuv[i] += dy.sum(axis=0)
        dC[i] += s * np.einsum("njv,nd->jvd", dy, Qt)
    # --- summaries, per key cluster (all query centroids at once)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dqbar = np.zeros((Cq, D))
    for j in range(Ck):
        kidx = np.nonzero(k_labels == j)[0]
        if kidx.size == 0:
            continue
        Kj, Vj = K[kidx], V[kidx]
        ell = s * (qbar @ Kj.T)                                  # [Cq, nj]
        w = np.exp(ell - logZ[:, j][:, None])
        G = dC[:, j]                                             # [Cq, Dv, D]
        Gk = np.einsum("ivd,nd->inv", G, Kj)                     # G k_k
        Gv = np.einsum("ivd,nv->ind", G, Vj)                     # G^T v_k
        dmuv_t = dmuv[:, j] - np.einsum("ivd,id->iv", G, mu_k[:, j])   # through -mu_v mu_k^T
        dmuk_t = dmuk[:, j] - np.einsum("ivd,iv->id", G, mu_v[:, j])
        dw = (np.einsum("nv,inv->in", Vj, Gk)                    # v^T G k
              + dmuk_t @ Kj.T + dmuv_t @ Vj.T)
        dVj = np.einsum("in,inv->nv", w, Gk) + w.T @ dmuv_t
        dKj = np.einsum("in,ind->nd", w, Gv) + w.T @ dmuk_t
        dell = w * (dw - (w * dw).sum(axis=1)[:, None]) + w * dlogZ[:, j][:, None]
        dqbar += s * (dell @ Kj)
        dKj += s * (dell.T @ qbar)
        dK[kidx] += dKj
        dV[kidx] += dVj
    # --- residuals and centroids
    dQ = dQt.copy()
    for i in np.unique(q_labels):
        idx = np.nonzero(q_labels == i)[0]
        dQ[idx] += (dqbar[i] - dQt[idx].sum(axis=0))[None, :] / idx.size
    return dQ, dK, dV


def muse_acausal(Q, K, V, Cq: int, Ck: int, iters: int, scale: float,
                 return_labels: bool = False, dipole: bool = True):
    """Full acausal MuSe: K-means on Q and on K, summaries, refinement."""
    ql, qc = kmeans(Q, Cq, iters)
    kl, _ = kmeans(K, Ck, iters)
    O = muse_from_labels(Q, K, V, ql, kl, Cq, Ck, scale, qbar=qc, dipole=dipole)
    if return_labels:
        return O, ql, kl
    return O


# ----------------------------------------------------------------------------
# Exact softmax attention (the quantity MuSe approximates).
# ----------------------------------------------------------------------------

def exact_attention(Q, K, V, scale: float, causal: bool = False,
                    rows: Optional[np.ndarray] = None, return_lse: bool = False,
                    chunk: int = 256):
    """E_n = sum_k softmax_k(s q_n . k) v_k; causal keeps k <= n."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    N = Q.shape[0]
    rws = np.arange(N) if rows is None else np.asarray(rows)
    O = np.zeros((N, V.shape[1]))
    lse = np.full(N, NEG_INF)
    for a in range(0, rws.size, chunk):
        r = rws[a:a + chunk]
        L = scale * (Q[r] @ K.T)
        if causal:
            L = np.where(np.arange(K.shape[0])[None, :] <= r[:, None], L, NEG_INF)
        m = L.max(axis=1)
        e = np.exp(L - m[:, None])
        l = e.sum(axis=1)
        O[r] = (e @ V) / l[:, None]
        lse[r] = m + np.log(l)
    if return_lse:
        return O, lse
    return O


def merge_partials(parts: List[Tuple[np.ndarray, np.ndarray]]) -> np.ndarray:
    """Combine normalised partial outputs (lse, o) of disjoint key sets into one softmax."""
    lses = np.stack([p[0] for p in parts])            # [P, N]
    M = lses.max(axis=0)
    M = np.where(np.isfinite(M), M, 0.0)
    wts = np.exp(lses - M[None, :])                   # exp(-inf) = 0
    num = sum(wts[k][:, None] * parts[k][1] for k in range(len(parts)))
    den = wts.sum(axis=0)
    return num / den[:, None]


def rse(O: np.ndarray, E: np.ndarray) -> float:
    """Relative squared error ||O - E||_F^2 / ||E||_F^2."""
    O = np.asarray(O, np.float64)
    E = np.asarray(E, np.float64)
    return float(((O - E) ** 2).sum() / (E ** 2).sum())


def max_rel_err(O: np.ndarray, ref: np.ndarray) -> float:
    """max |O - ref| / max |ref| (normwise infinity-relative error)."""
    O = np.asarray(O, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(O - ref).max() / max(np.abs(ref).max(), 1e-300))


# ----------------------------------------------------------------------------
# Causal attention: hierarchical block decomposition.
# [review] Figure 2 caption and "Assumptions & free parameters" (invented entity
# "Hierarchical block decomposition for causal attention"): the lower-triangular
# attention matrix is split into blocks; the diagonal blocks are exact ("Flash"),
# the below-diagonal blocks use MuSe; O(NCD log N) ([abstract]).
# ----------------------------------------------------------------------------

def causal_squares(N: int, S: int) -> List[Tuple[int, int, int, int, int, int]]:
    """Below-diagonal squares of the binary decomposition.

    Level l = 1, 2, ... has side s_l = S * 2^(l-1); for odd r with r*s_l < N the
    square's queries are [r s_l, min((r+1) s_l, N)) and its keys [(r-1) s_l, r s_l).
    Returns (level, r, q0, q1, k0, k1).  For a query in block b the levels whose bit
    (l-1) of b is set cover the keys [0, b*S) exactly once.
    """
    out = []
    lev, s = 1, S
    while s < N:
        r = 1
        while r * s < N:
            out.append((lev, r, r * s, min((r + 1) * s, N), (r - 1) * s, r * s))
            r += 2
        lev += 1
        s *= 2
    return out


def diagonal_exact(Q, K, V, S: int, scale: float):
    """Exact causal attention inside each S-row diagonal block: (lse, o) per row."""
    Q = np.asarray(Q, np.float64)
    N = Q.shape[0]
    O = np.zeros((N, np.asarray(V).shape[1]))
    lse = np.full(N, NEG_INF)
    for b0 in range(0, N, S):
        b1 = min(N, b0 + S)
        o, l = exact_attention(Q[b0:b1], K[b0:b1], V[b0:b1], scale, causal=True,
                               return_lse=True)
        O[b0:b1] = o
        lse[b0:b1] = l
    return lse, O


def muse_causal(Q, K, V, S: int, Cq: int, Ck: int, iters: int, scale: float,
                labels: Optional[Dict[Tuple[int, int], Tuple[np.ndarray, np.ndarray]]] = None,
                return_labels: bool = False, rows: Optional[np.ndarray] = None):
    """Causal MuSe: exact diagonal blocks + one acausal MuSe instance per square.

    Each square clusters its own query range and key range with
    C_eff = min(C, range length).  ``labels`` maps (level, r) to the (query, key)
    labels of that square (teacher forcing); otherwise K-means runs here.
    ``rows`` restricts the work to the squares and outputs of those query rows
    (the other rows of the result are not meaningful).
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    N = Q.shape[0]
    rws = None if rows is None else np.asarray(rows)
    parts = [diagonal_exact(Q, K, V, S, scale)]
    used = {}
    for (lev, r, q0, q1, k0, k1) in causal_squares(N, S):
        if rws is not None and not ((rws >= q0) & (rws < q1)).any():
            continue
        cq = min(Cq, q1 - q0)
        ck = min(Ck, k1 - k0)
        if labels is not None and (lev, r) in labels:
            ql, kl = labels[(lev, r)]
            qbar = None
        else:
            ql, qbar = kmeans(Q[q0:q1], cq, iters)
            kl, _ = kmeans(K[k0:k1], ck, iters)
        used[(lev, r)] = (ql, kl)
        sub = None if rws is None else rws[(rws >= q0) & (rws < q1)] - q0
        o, l = muse_from_labels(Q[q0:q1], K[k0:k1], V[k0:k1], ql, kl, cq, ck, scale,
                                qbar=qbar, return_lse=True, rows=sub)
        lse = np.full(N, NEG_INF)
        oo = np.zeros((N, V.shape[1]))
        lse[q0:q1] = l
        oo[q0:q1] = o
        parts.append((lse, oo))
    O = merge_partials(parts)
    if return_labels:
        return O, used
    return O


# ----------------------------------------------------------------------------
# Causal accumulation + retrieval (paper v4).
# [summary] "Kernmechanismen", item 3 (causal accumulation: the context is cut into
# spatial blocks; a block sees the summaries of all preceding blocks) and item 4
# (retrieval: top-k1 key clusters by tilted summary score, then top-k2 spatial blocks
# inside them; exact attention on the retrieved (cluster, block) pairs and the local
# block diagonal; the rest through the approximate summaries).
# ----------------------------------------------------------------------------

def block_logZ(qbar, K, k_labels, n_kclusters: int, S: int, scale: float) -> np.ndarray:
    """logZ_{i,j,b'} = log sum over keys of cluster j in block b' of exp(s qbar_i.k)."""
    qbar = np.asarray(qbar, np.float64)
    K = np.asarray(K, np.float64)
    N = K.shape[0]
    nb = (N + S - 1) // S
    out = np.full((qbar.shape[0], n_kclusters, nb), NEG_INF)
    blk = np.arange(N) // S
    for j in range(n_kclusters):
        for b in range(nb):
            idx = np.nonzero((k_labels == j) & (blk == b))[0]
            if idx.size:
                ell = scale * (qbar @ K[idx].T)
                m = ell.max(axis=1)
                out[:, j, b] = m + np.log(np.exp(ell - m[:, None]).sum(axis=1))
    return out


def _lse(x: np.ndarray) -> float:
    x = np.asarray(x, np.float64)
    if x.size == 0 or not np.isfinite(x.max()):
        return NEG_INF
    m = x.max()
    return float(m + math.log(np.exp(x - m).sum()))


def retrieval_select(logZb: np.ndarray, k1: int, k2: int) -> np.ndarray:
    """Selected (cluster, block) pairs per (query cluster i, query block b).

    sigma_ij = logsumexp over b' < b of logZ_{i,j,b'}; the k1 largest finite sigma_ij
    (ties to the lower j) give the clusters; inside each, the k2 largest finite
    logZ_{i,j,b'} with b' < b (ties to the lower b').  Slot t*k2 + u holds the u-th block
    of the t-th cluster; unused slots hold (-1, -1).  Block 0 selects nothing.
    Returns int64 [Cq, nb, k1*k2, 2].
    """
    Cq, Ck, nb = logZb.shape
    sel = -np.ones((Cq, nb, max(1, k1 * k2), 2), np.int64)
    for i in range(Cq):
        for b in range(1, nb):
            sig = np.array([_lse(logZb[i, j, :b]) for j in range(Ck)])
            cand = [j for j in range(Ck) if np.isfinite(sig[j])]
            cand.sort(key=lambda j: (-sig[j], j))
            for t, j in enumerate(cand[:k1]):
                blocks = [bb for bb in range(b) if np.isfinite(logZb[i, j, bb])]
                blocks.sort(key=lambda bb: (-logZb[i, j, bb], bb))
                for u, bb in enumerate(blocks[:k2]):
                    sel[i, b, t * k2 + u] = (j, bb)
    return sel


def muse_retrieval(Q, K, V, S: int, Cq: int, Ck: int, iters: int, k1: int, k2: int,
                   scale: float, q_labels=None, k_labels=None, selection=None,
                   rows: Optional[np.ndarray] = None, return_all: bool = False):
    """Causal MuSe with retrieval.

    Query n in block b, cluster i: exact terms over the diagonal keys [bS, n] and over
    the keys of every selected pair (j, b'); for every key cluster j a tilted
    monopole+dipole summary (tilt qbar_i) of its remaining keys in blocks < b, used as
    in the acausal refinement; all terms share one softmax normaliser.
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    N = Q.shape[0]
    if q_labels is None:
        q_labels, qbar = kmeans(Q, Cq, iters)
    else:
        qbar = cluster_means(Q, q_labels, Cq)
    if k_labels is None:
        k_labels, _ = kmeans(K, Ck, iters)
    q_labels = np.asarray(q_labels)
    k_labels = np.asarray(k_labels)
    blk = np.arange(N) // S
    need_sel = selection is None
    rws = np.arange(N) if rows is None else np.asarray(rows)
    groups = sorted(set((int(q_labels[n]), int(blk[n])) for n in rws))
    if need_sel:
        logZb = block_logZ(qbar, K, k_labels, Ck, S, scale)
        selection = retrieval_select(logZb, k1, k2)
    O = np.zeros((N, V.shape[1]))
    for (i, b) in groups:
        idx = np.array([n for n in rws if q_labels[n] == i and blk[n] == b])
        picked = set()
        for (j, bb) in selection[i, b]:
            if j >= 0:
                picked.add((int(j), int(bb)))
        retrieved = np.array([k for k in range(b * S)
                              if (int(k_labels[k]), int(blk[k])) in picked], dtype=np.int64)
        # remainder summaries per key cluster, tilt qbar_i
        rest_mask = np.zeros(N, bool)
        rest_mask[:b * S] = True
        rest_mask[retrieved] = False
        logZ_r, mu_k_r, mu_v_r, cov_r = tilted_summaries(
            qbar[i:i + 1], K[rest_mask], V[rest_mask], k_labels[rest_mask], Ck, scale)
        for n in idx:
            qt = Q[n] - qbar[i]
            logits = []
            values = []
            diag = np.arange(b * S, n + 1)
            keys = np.concatenate([diag, retrieved])
            if keys.size:
                logits.append(scale * (K[keys] @ Q[n]))
                values.append(V[keys])
            a = logZ_r[0] + scale * (mu_k_r[0] @ qt)
            ok = np.isfinite(a)
            if ok.any():
                logits.append(a[ok])
                values.append(mu_v_r[0][ok] + scale * (cov_r[0][ok] @ qt))
            L = np.concatenate(logits)
            Vs = np.concatenate(values, axis=0)
            m = L.max()
            e = np.exp(L - m)
            O[n] = (e @ Vs) / e.sum()
    if return_all:
        return O, q_labels, k_labels, selection
    return O
