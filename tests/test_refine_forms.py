"""The two evaluations of the refinement that the CUDA path implements, checked in float64
against the oracle's direct transcription of the formula (CPU only).

The formula (pith.science review of arXiv 2509.10406, "What carries the argument"): for
query n in cluster i with residual qt = q_n - qbar_i,
    p = softmax_j(logZ_ij + s qt.mu_k,ij),   O_n = sum_j p_j (mu_v,ij + s C_ij qt),
C_ij the tilted covariance of values and keys in key cluster j.  With u_j = qt.mu_k,ij,
c0 = p_j (1 - s u_j), c1 = s p_j and the tilted weights w_ik = exp(s qbar_i.k - logZ_ij):
  pair form     O_n = sum_k w_ik (c0_nj(k) + c1_nj(k) qt.k) v_k          (refine_tc.cu)
  summary form  O_n = sum_j c0_nj mu_v,ij + sum_j c1_nj C'_ij qt,
                C'_ij = sum_{k in S_j} w_ik v_k k^T (uncentred)           (refine_sf.cu)
Both rest on sum_{k in S_j} w_ik = 1 and C_ij = C'_ij - mu_v,ij mu_k,ij^T.  A dropped
term or a misplaced scale in either reading fails these comparisons.
"""
import numpy as np
import pytest

from clustered_softmax_attention_b200.inputs import small_problem
from oracle import muse_oracle as mo


def _both_forms(Q, K, V, ql, kl, Cq, Ck, s):
    qbar = mo.cluster_means(Q, ql, Cq)
    logZ, mu_k, mu_v, cov = mo.tilted_summaries(qbar, K, V, kl, Ck, s)
    N, Dv = Q.shape[0], V.shape[1]
    pair = np.zeros((N, Dv))
    summ = np.zeros((N, Dv))
    checks = []
    for i in range(Cq):
        rows = np.nonzero(ql == i)[0]
        if rows.size == 0:
            continue
        qt = Q[rows] - qbar[i]
        u = qt @ mu_k[i].T                                   # [n, Ck]
        a = logZ[i][None, :] + s * u
        e = np.exp(a - a.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)
        c0, c1 = p * (1.0 - s * u), s * p
        for j in range(Ck):
            idx = np.nonzero(kl == j)[0]
            if idx.size == 0:
                continue
            w = np.exp(s * (K[idx] @ qbar[i]) - logZ[i, j])  # tilted weights, sum to 1
            checks.append(abs(w.sum() - 1.0))
            S = qt @ K[idx].T                                # qt.k per (row, key)
            pair[rows] += ((c0[:, j:j + 1] + c1[:, j:j + 1] * S) * w[None, :]) @ V[idx]
            Cu = (w[:, None] * V[idx]).T @ K[idx]            # C'_ij, [Dv, D]
            np.testing.assert_allclose(Cu - np.outer(mu_v[i, j], mu_k[i, j]), cov[i, j],
                                       rtol=1e-9, atol=1e-12)
            summ[rows] += c0[:, j:j + 1] * mu_v[i, j][None, :] + c1[:, j:j + 1] * (qt @ Cu.T)
    ref = mo.refine(Q, ql, qbar, logZ, mu_k, mu_v, cov, s)
    return pair, summ, ref, max(checks)


@pytest.mark.parametrize("seed,N,D,Dv,Cq,Ck,s", [(1, 300, 8, 6, 5, 7, 0.7),
                                                  (2, 257, 16, 16, 9, 3, 1.0),
                                                  (3, 120, 4, 10, 1, 12, 1.9)])
def test_pair_and_summary_forms_equal_the_formula(seed, N, D, Dv, Cq, Ck, s):
    Q, K, V = small_problem(seed, N, D, Dv, 6, 0.4)
    ql = mo.kmeans(Q, Cq, 4)[0]
    kl = mo.kmeans(K, Ck, 4)[0]
    pair, summ, ref, wsum = _both_forms(Q, K, V, ql, kl, Cq, Ck, s)
    assert wsum < 1e-12
    scale = np.abs(ref).max()
    assert np.abs(pair - ref).max() <= 1e-11 * scale
    assert np.abs(summ - ref).max() <= 1e-11 * scale


def test_summary_form_needs_the_centring_in_c0():
    """c0 = p (without - s u) would miss the -mu_v (mu_k . qt) part of C_ij qt."""
    Q, K, V = small_problem(4, 200, 8, 8, 5, 0.5)
    ql = mo.kmeans(Q, 4, 4)[0]
    kl = mo.kmeans(K, 6, 4)[0]
    qbar = mo.cluster_means(Q, ql, 4)
    logZ, mu_k, mu_v, cov = mo.tilted_summaries(qbar, K, V, kl, 6, 1.0)
    ref = mo.refine(Q, ql, qbar, logZ, mu_k, mu_v, cov, 1.0)
    wrong = np.zeros_like(ref)
    for i in range(4):
        rows = np.nonzero(ql == i)[0]
        qt = Q[rows] - qbar[i]
        a = logZ[i][None, :] + qt @ mu_k[i].T
        p = np.exp(a - a.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        for j in range(6):
            idx = np.nonzero(kl == j)[0]
            if idx.size == 0:
                continue
            w = np.exp(K[idx] @ qbar[i] - logZ[i, j])
            Cu = (w[:, None] * V[idx]).T @ K[idx]
            wrong[rows] += p[:, j:j + 1] * mu_v[i, j][None, :] + p[:, j:j + 1] * (qt @ Cu.T)
    assert np.abs(wrong - ref).max() > 1e-6 * np.abs(ref).max()
