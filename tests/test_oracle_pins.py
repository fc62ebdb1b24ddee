"""Pins for the float64 oracle: each check ties it to something other than itself.

Hand-derived closed forms (tests/golden), library routines (torch SDPA, sklearn
K-means), limits where MuSe is exact, calculus identities (the dipole is the
Jacobian of softmax attention), invariances, and the truncation-error order.
No GPU is used here.
"""
import glob
import json
import math
import os

import numpy as np
import pytest

from oracle import muse_oracle as mo
from clustered_softmax_attention_b200.inputs import small_problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _closed(expr_tree):
    """Evaluate nested lists of closed-form expression strings with math only."""
    env = {"exp": math.exp, "log": math.log, "inf": math.inf, "__builtins__": {}}
    if isinstance(expr_tree, str):
        return eval(expr_tree, env)  # noqa: S307 - fixture expressions are ours
    return [_closed(e) for e in expr_tree]


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------- goldens

def _goldens(kind):
    names = sorted(os.path.basename(p) for p in glob.glob(os.path.join(GOLDEN, "*.json")))
    return [n for n in names if _load(n).get("kind", "muse") == kind]


@pytest.mark.parametrize("name", _goldens("muse"))
def test_golden_closed_forms(name):
    g = _load(name)
    Q, K, V = (np.array(g[k], float) for k in ("Q", "K", "V"))
    s = g["scale"]
    ql, kl = np.array(g["q_labels"]), np.array(g["k_labels"])
    exp = g["expected"]
    qbar = mo.cluster_means(Q, ql, g["Cq"])
    logZ, mu_k, mu_v, cov = mo.tilted_summaries(qbar, K, V, kl, g["Ck"], s)
    np.testing.assert_allclose(logZ, np.array(_closed(exp["logZ"])), rtol=1e-13, atol=1e-14)
    for key, val in (("mu_k", mu_k), ("mu_v", mu_v), ("cov", cov)):
        if key in exp:
            np.testing.assert_allclose(val, np.array(_closed(exp[key])), rtol=1e-13, atol=1e-14)
    O = mo.refine(Q, ql, qbar, logZ, mu_k, mu_v, cov, s)
    np.testing.assert_allclose(O, np.array(_closed(exp["O"])), rtol=1e-12, atol=1e-14)
    if "E" in exp:
        E = mo.exact_attention(Q, K, V, s)
        np.testing.assert_allclose(E, np.array(_closed(exp["E"])), rtol=1e-13)
    if "kmeans_rounds" in g:
        for t, want in g["kmeans_rounds"].items():
            lab, cen = mo.kmeans(K, g["Ck"], int(t))
            assert lab.tolist() == want["labels"]
            np.testing.assert_allclose(cen, np.array(_closed(want["centroids"])), rtol=0, atol=1e-15)


@pytest.mark.parametrize("name", _goldens("kmeans_gap"))
def test_golden_kmeans_gap_normaliser(name):
    """The label-parity gap (d2 - d1) / (||x||^2 + ||c_a||^2) on hand-derived rows where d1 is
    0, where the runner-up's norm differs from the assigned centroid's, and an exact tie."""
    g = _load(name)
    X, C = np.array(_closed(g["X"])), np.array(_closed(g["C"]))
    lab, gap = mo.kmeans_assign_gap(X, C)
    assert lab.tolist() == g["labels"]
    assert mo.kmeans_assign(X, C).tolist() == g["labels"]
    np.testing.assert_allclose(gap, np.array(_closed(g["gap"])), rtol=1e-13, atol=0)


@pytest.mark.parametrize("name", _goldens("retrieval_select"))
def test_golden_retrieval_selection(name):
    """Cluster ranking by the prefix logsumexp, block ranking inside each chosen cluster,
    ties to the lower index, -inf excluded, slot order, fewer candidates than k1 or k2."""
    g = _load(name)
    lzb = np.array(_closed(g["logZb"]), dtype=np.float64)
    for case in g["cases"]:
        sel = mo.retrieval_select(lzb, case["k1"], case["k2"])
        assert sel.tolist() == case["slots"], (case["k1"], case["k2"])


# --------------------------------------------------------------------------- exact attention

def test_exact_attention_matches_torch_sdpa():
    import torch
    Q, K, V = small_problem(1, 50, 8, 5, 4, 0.3)
    for causal in (False, True):
        for s in (1.0, 0.7):
            E = mo.exact_attention(Q, K, V, s, causal=causal)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.tensor(Q)[None], torch.tensor(K)[None], torch.tensor(V)[None],
                is_causal=causal, scale=s)[0].numpy()
            np.testing.assert_allclose(E, ref, rtol=1e-12, atol=1e-14)


def test_merge_partials_is_joint_softmax():
    Q, K, V = small_problem(2, 40, 6, 3, 4, 0.4)
    parts = []
    for lo, hi in ((0, 7), (7, 30), (30, 40)):
        o, l = mo.exact_attention(Q, K[lo:hi], V[lo:hi], 1.3, return_lse=True)
        parts.append((l, o))
    np.testing.assert_allclose(mo.merge_partials(parts), mo.exact_attention(Q, K, V, 1.3),
                               rtol=1e-12, atol=1e-14)


def test_rse_and_max_rel_err_definitions():
    E = np.array([[3.0, 4.0], [0.0, 0.0]])
    O = E + np.array([[0.0, 0.0], [1.0, 0.0]])
    assert mo.rse(O, E) == pytest.approx(1.0 / 25.0)
    assert mo.max_rel_err(O, E) == pytest.approx(1.0 / 4.0)


# --------------------------------------------------------------------------- K-means

def test_kmeans_matches_sklearn_lloyd_per_round():
    from sklearn.cluster import KMeans
    X, _, _ = small_problem(3, 300, 5, 1, 6, 0.25)
    C = 6
    for T in (1, 2, 3):
        lab, cen = mo.kmeans(X, C, T)
        assert np.bincount(lab, minlength=C).min() > 0
        km = KMeans(n_clusters=C, init=X[:C].copy(), n_init=1, max_iter=T, tol=0.0,
                    algorithm="lloyd").fit(X)
        if km.n_iter_ == T:
            np.testing.assert_allclose(cen, km.cluster_centers_, rtol=1e-12, atol=1e-13)
            # sklearn's labels are the assignment to its final centroids
            assert (mo.kmeans_assign(X, cen) == km.labels_).all()


def test_kmeans_converged_matches_sklearn():
    from sklearn.cluster import KMeans
    X, _, _ = small_problem(4, 400, 6, 1, 5, 0.2)
    lab, cen = mo.kmeans(X, 5, 60)
    km = KMeans(n_clusters=5, init=X[:5].copy(), n_init=1, max_iter=60, tol=0.0,
                algorithm="lloyd").fit(X)
    assert (lab == km.labels_).all()
    np.testing.assert_allclose(cen, km.cluster_centers_, rtol=1e-12, atol=1e-13)


def test_kmeans_recovers_separated_mixture():
    rng = np.random.default_rng(7)
    comps, D = 8, 6
    means = rng.standard_normal((comps, D)) * 10.0
    idx = np.concatenate([np.arange(comps), rng.integers(0, comps, 500)])
    X = means[idx] + 0.01 * rng.standard_normal((idx.size, D))
    lab, cen = mo.kmeans(X, comps, 5)
    # the first C rows are one point per component, so cluster c is component c
    assert (lab == idx).all()
    np.testing.assert_allclose(cen, means, atol=0.01)


def test_kmeans_objective_nonincreasing():
    X, _, _ = small_problem(5, 500, 8, 1, 20, 0.5)
    _, _, hist = mo.kmeans(X, 16, 12, history=True)
    objs = []
    for C in hist:
        lab = mo.kmeans_assign(X, C)
        objs.append(mo.kmeans_objective(X, lab, C))
    assert all(b <= a + 1e-12 for a, b in zip(objs, objs[1:]))


def test_kmeans_empty_cluster_keeps_centroid_and_gap():
    X = np.array([[0.0], [0.1], [10.0]])
    C0 = np.array([[0.0], [5.0], [100.0]])
    lab = mo.kmeans_assign(X, C0)
    assert lab.tolist() == [0, 0, 1]
    C1 = mo.kmeans_update(X, lab, C0)
    assert C1[2, 0] == 100.0 and C1[0, 0] == pytest.approx(0.05) and C1[1, 0] == 10.0
    lab2, gap = mo.kmeans_assign_gap(np.array([[1.0]]), np.array([[0.0], [2.0]]))
    assert lab2[0] == 0 and gap[0] == 0.0


# --------------------------------------------------------------------------- limits where MuSe is exact

def test_singleton_key_clusters_are_exact_for_any_query_clustering():
    """Ck = N: every key is its own cluster, kt = 0, C = 0 -> exact attention."""
    Q, K, V = small_problem(8, 48, 6, 4, 5, 0.3)
    rng = np.random.default_rng(0)
    for s in (1.0, 2.5):
        ql = rng.integers(0, 5, size=48)
        O = mo.muse_from_labels(Q, K, V, ql, np.arange(48), 5, 48, s)
        np.testing.assert_allclose(O, mo.exact_attention(Q, K, V, s), rtol=1e-10, atol=1e-12)


def test_singleton_query_clusters_are_exact_for_any_key_clustering():
    """Cq = N: qt = 0 -> exact attention, whatever the key clusters."""
    Q, K, V = small_problem(9, 40, 5, 3, 4, 0.3)
    rng = np.random.default_rng(1)
    for s in (1.0, 3.0):
        kl = rng.integers(0, 3, size=40)
        O = mo.muse_from_labels(Q, K, V, np.arange(40), kl, 40, 3, s)
        np.testing.assert_allclose(O, mo.exact_attention(Q, K, V, s), rtol=1e-10, atol=1e-12)
    # the full pipeline with Cq = N: the first-N start makes every query its own centroid
    O = mo.muse_acausal(Q, K, V, 40, 3, 4, 1.0)
    np.testing.assert_allclose(O, mo.exact_attention(Q, K, V, 1.0), rtol=1e-10, atol=1e-12)


def test_zero_residual_is_exact_attention_at_the_centroid():
    """qt := 0 gives sum_j softmax(logZ_ij) mu_v,ij = exact attention evaluated at qbar_i."""
    Q, K, V = small_problem(10, 60, 6, 4, 6, 0.4)
    ql, qc = mo.kmeans(Q, 5, 3)
    kl, _ = mo.kmeans(K, 7, 3)
    O = mo.muse_from_labels(Q, K, V, ql, kl, 5, 7, 1.7, qbar=qc, zero_residual=True)
    E = mo.exact_attention(qc[ql], K, V, 1.7)
    np.testing.assert_allclose(O, E, rtol=1e-10, atol=1e-12)


def test_single_key_cluster_is_first_order_taylor_of_attention():
    """Ck = 1: O(q) = E(qbar) + J(qbar) qt with J the Jacobian of softmax attention.

    The dipole s*C must equal dE/dq at the centroid (central differences, float64),
    which fixes its sign, its transpose (Dv x D with D != Dv) and the factor s.
    """
    Q, K, V = small_problem(11, 30, 4, 3, 3, 0.5)
    s = 1.6
    qbar = Q.mean(0, keepdims=True)
    logZ, mu_k, mu_v, cov = mo.tilted_summaries(qbar, K, V, np.zeros(30, int), 1, s)
    h = 1e-5
    J = np.zeros((3, 4))
    for d in range(4):
        e = np.zeros((1, 4))
        e[0, d] = h
        J[:, d] = (mo.exact_attention(qbar + e, K, V, s) - mo.exact_attention(qbar - e, K, V, s))[0] / (2 * h)
    np.testing.assert_allclose(s * cov[0, 0], J, rtol=1e-7, atol=1e-10)
    np.testing.assert_allclose(mu_v[0, 0], mo.exact_attention(qbar, K, V, s)[0], rtol=1e-12)
    O = mo.refine(Q, np.zeros(30, int), qbar, logZ, mu_k, mu_v, cov, s)
    np.testing.assert_allclose(O, mu_v[0, 0][None] + (Q - qbar) @ (s * cov[0, 0]).T, rtol=1e-12)


# --------------------------------------------------------------------------- invariances

def test_key_translation_invariance_and_query_translation_dependence():
    Q, K, V = small_problem(12, 80, 6, 4, 4, 0.15)
    O = mo.muse_acausal(Q, K, V, 6, 5, 6, 1.0)
    rng = np.random.default_rng(3)
    for norm in (0.5, 10.0):
        t = rng.standard_normal(6)
        t *= norm / np.linalg.norm(t)
        Ot = mo.muse_acausal(Q, K + t, V, 6, 5, 6, 1.0)
        np.testing.assert_allclose(Ot, O, rtol=1e-9, atol=1e-11)
    t = rng.standard_normal(6)
    Oq = mo.muse_acausal(Q + t, K, V, 6, 5, 6, 1.0)
    assert np.abs(Oq - O).max() > 1e-3


# --------------------------------------------------------------------------- truncation-error order

def _order_problem(eq, ek, seed=0, N=64, D=4, Dv=3, cq=4, ck=4):
    rng = np.random.default_rng(seed)
    qc = rng.standard_normal((cq, D))
    kc = rng.standard_normal((ck, D))
    ql = np.arange(N) % cq
    kl = np.arange(N) % ck
    nq = rng.standard_normal((N, D))
    nk = rng.standard_normal((N, D))
    V = rng.standard_normal((N, Dv))
    return qc[ql] + eq * nq, kc[kl] + ek * nk, V, ql, kl


def _err(eq, ek, cq=4, ck=4):
    Q, K, V, ql, kl = _order_problem(eq, ek, cq=cq, ck=ck)
    O = mo.muse_from_labels(Q, K, V, ql, kl, cq, ck, 1.0)
    return np.abs(O - mo.exact_attention(Q, K, V, 1.0)).max()


def test_truncation_error_is_second_order_in_each_residual():
    """Dropping only qt.kt leaves an error of order Tr(Cov(qt)Cov(kt)) ~ eq^2 ek^2."""
    eps = np.array([1e-3, 3e-3, 1e-2, 3e-2, 1e-1])
    fixed = 0.05
    eq_err = np.array([_err(e, fixed) for e in eps])
    ek_err = np.array([_err(fixed, e) for e in eps])
    slope_q = np.polyfit(np.log(eps), np.log(eq_err), 1)[0]
    slope_k = np.polyfit(np.log(eps), np.log(ek_err), 1)[0]
    assert 1.8 <= slope_q <= 2.2, slope_q
    assert 1.8 <= slope_k <= 2.2, slope_k
    # error / (Tr Cov qt * Tr Cov kt) stays bounded as both shrink
    ratios = [_err(e, e) / (e * e * e * e) for e in (1e-2, 3e-3, 1e-3)]
    assert max(ratios) / min(ratios) < 2.0


def test_monopole_only_would_be_first_order():
    """Without the dipole the error would fall only linearly: guards the dipole's presence."""
    def err_no_dip(eq):
        Q, K, V, ql, kl = _order_problem(eq, 0.05)
        qbar = mo.cluster_means(Q, ql, 4)
        logZ, mu_k, mu_v, cov = mo.tilted_summaries(qbar, K, V, kl, 4, 1.0)
        O = mo.refine(Q, ql, qbar, logZ, mu_k, mu_v, cov, 1.0, dipole=False)
        return np.abs(O - mo.exact_attention(Q, K, V, 1.0)).max()
    eps = np.array([1e-3, 1e-2, 1e-1])
    slope = np.polyfit(np.log(eps), np.log([err_no_dip(e) for e in eps]), 1)[0]
    assert 0.8 <= slope <= 1.2


def test_monopole_only_single_key_cluster_is_attention_at_the_centroid():
    """Monopole only, Ck = 1: every query of cluster i gets sum_k softmax(s qbar_i.k) v_k,
    exact attention evaluated at its centroid, whatever its residual."""
    rng = np.random.default_rng(21)
    N, D, Dv, Cq, s = 48, 5, 3, 4, 0.7
    Q = rng.standard_normal((N, D))
    K = rng.standard_normal((N, D))
    V = rng.standard_normal((N, Dv))
    ql = rng.integers(0, Cq, N)
    ql[:Cq] = np.arange(Cq)
    O = mo.muse_from_labels(Q, K, V, ql, np.zeros(N, np.int64), Cq, 1, s, dipole=False)
    qbar = mo.cluster_means(Q, ql, Cq)
    at_centroid = mo.exact_attention(qbar, K, V, s)
    np.testing.assert_allclose(O, at_centroid[ql], rtol=1e-12, atol=1e-12)
    # the dipole term is what moves the output off the centroid's value
    O_dip = mo.muse_from_labels(Q, K, V, ql, np.zeros(N, np.int64), Cq, 1, s)
    assert np.abs(O_dip - O).max() > 1e-3


def test_monopole_only_singleton_queries_is_exact():
    """Monopole only with Cq = N: qt = 0, so the dropped term vanishes and the result is
    exact attention for any key clustering."""
    rng = np.random.default_rng(22)
    N, D, Dv = 40, 4, 3
    Q, K, V = rng.standard_normal((N, D)), rng.standard_normal((N, D)), rng.standard_normal((N, Dv))
    kl = rng.integers(0, 5, N)
    O = mo.muse_from_labels(Q, K, V, np.arange(N), kl, N, 5, 1.0, dipole=False)
    np.testing.assert_allclose(O, mo.exact_attention(Q, K, V, 1.0), rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------- tiny brute force

def _bruteforce_muse(Q, K, V, ql, kl, Cq, Ck, s):
    """Same definitions, written as scalar loops (N <= 16)."""
    N, D = len(Q), len(Q[0])
    Dv = len(V[0])
    qbar = []
    for i in range(Cq):
        mem = [Q[n] for n in range(N) if ql[n] == i]
        qbar.append([sum(m[d] for m in mem) / len(mem) if mem else 0.0 for d in range(D)])
    out = []
    for n in range(N):
        i = ql[n]
        qt = [Q[n][d] - qbar[i][d] for d in range(D)]
        a, terms = [], []
        for j in range(Ck):
            mem = [k for k in range(N) if kl[k] == j]
            if not mem:
                continue
            ell = [s * sum(qbar[i][d] * K[k][d] for d in range(D)) for k in mem]
            mx = max(ell)
            lz = mx + math.log(sum(math.exp(x - mx) for x in ell))
            w = [math.exp(x - lz) for x in ell]
            muk = [sum(w[t] * K[k][d] for t, k in enumerate(mem)) for d in range(D)]
            muv = [sum(w[t] * V[k][e] for t, k in enumerate(mem)) for e in range(Dv)]
            cq_ = [sum(w[t] * (V[k][e] - muv[e]) * sum((K[k][d] - muk[d]) * qt[d] for d in range(D))
                       for t, k in enumerate(mem)) for e in range(Dv)]
            a.append(lz + s * sum(qt[d] * muk[d] for d in range(D)))
            terms.append([muv[e] + s * cq_[e] for e in range(Dv)])
        mx = max(a)
        p = [math.exp(x - mx) for x in a]
        tot = sum(p)
        out.append([sum(p[t] * terms[t][e] for t in range(len(a))) / tot for e in range(Dv)])
    return np.array(out)


def test_tiny_bruteforce_agrees():
    Q, K, V = small_problem(13, 14, 3, 2, 3, 0.6)
    ql = np.array([0, 1, 2, 0, 1, 2, 0, 0, 1, 1, 2, 2, 0, 1])
    kl = np.array([0, 0, 1, 1, 2, 2, 3, 3, 0, 1, 2, 3, 0, 1])
    for s in (1.0, 0.4):
        O = mo.muse_from_labels(Q, K, V, ql, kl, 3, 5, s)   # key cluster 4 is empty
        ref = _bruteforce_muse(Q.tolist(), K.tolist(), V.tolist(), ql.tolist(), kl.tolist(), 3, 5, s)
        np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-14)


def test_row_subset_matches_full():
    Q, K, V = small_problem(14, 90, 5, 4, 5, 0.3)
    ql, qc = mo.kmeans(Q, 6, 3)
    kl, _ = mo.kmeans(K, 6, 3)
    full = mo.muse_from_labels(Q, K, V, ql, kl, 6, 6, 1.0)
    rows = np.array([0, 17, 44, 89])
    sub = mo.muse_from_labels(Q, K, V, ql, kl, 6, 6, 1.0, rows=rows)
    np.testing.assert_allclose(sub[rows], full[rows], rtol=1e-13)


# --------------------------------------------------------------------------- causal decomposition

def test_causal_squares_cover_each_prefix_once():
    for N, S in ((64, 8), (72, 8), (40, 8), (16, 16)):
        cover = np.zeros((N, N), int)
        for n in range(N):
            b = n // S
            cover[n, b * S:n + 1] += 1
        for (lev, r, q0, q1, k0, k1) in mo.causal_squares(N, S):
            cover[q0:q1, k0:k1] += 1
        assert (cover == np.tril(np.ones((N, N), int))).all(), (N, S)


def test_causal_limits_are_exact():
    Q, K, V = small_problem(15, 64, 5, 3, 4, 0.3)
    E = mo.exact_attention(Q, K, V, 1.0, causal=True)
    # one block: the diagonal is the whole causal attention
    np.testing.assert_allclose(mo.muse_causal(Q, K, V, 64, 4, 4, 3, 1.0), E, rtol=1e-12)
    # C >= range length in every square: singleton clusters everywhere -> exact
    np.testing.assert_allclose(mo.muse_causal(Q, K, V, 8, 64, 64, 3, 1.0), E, rtol=1e-10, atol=1e-12)
    # ragged N (not a power-of-two multiple of S)
    Q2, K2, V2 = Q[:44], K[:44], V[:44]
    E2 = mo.exact_attention(Q2, K2, V2, 1.0, causal=True)
    np.testing.assert_allclose(mo.muse_causal(Q2, K2, V2, 8, 64, 64, 3, 1.0), E2, rtol=1e-10, atol=1e-12)


def test_causal_is_close_to_exact_on_clustered_data():
    Q, K, V = small_problem(16, 128, 6, 4, 4, 0.05)
    O = mo.muse_causal(Q, K, V, 16, 4, 4, 5, 1.0)
    assert mo.rse(O, mo.exact_attention(Q, K, V, 1.0, causal=True)) < 1e-4


# --------------------------------------------------------------------------- retrieval

def test_block_logz_merges_to_cluster_logz():
    Q, K, V = small_problem(17, 64, 5, 3, 4, 0.3)
    ql, qc = mo.kmeans(Q, 4, 3)
    kl, _ = mo.kmeans(K, 5, 3)
    lzb = mo.block_logZ(qc, K, kl, 5, 16, 1.3)
    lz, _, _, _ = mo.tilted_summaries(qc, K, V, kl, 5, 1.3, want_cov=False)
    np.testing.assert_allclose(np.logaddexp.reduce(lzb, axis=2), lz, rtol=1e-12)


def test_retrieval_select_against_bruteforce_ranking():
    rng = np.random.default_rng(5)
    lzb = rng.standard_normal((3, 6, 5))
    lzb[rng.random(lzb.shape) < 0.3] = -np.inf
    lzb[1, 2, :] = lzb[1, 3, :]          # exact ties between clusters 2 and 3
    sel = mo.retrieval_select(lzb, 2, 2)
    for i in range(3):
        assert (sel[i, 0] == -1).all()
        for b in range(1, 5):
            sig = {j: np.logaddexp.reduce(lzb[i, j, :b]) for j in range(6)}
            ranked = [j for j, v in sorted(sig.items(), key=lambda kv: (-kv[1], kv[0])) if v > -np.inf][:2]
            want = []
            for j in ranked:
                bl = [bb for bb, v in sorted(enumerate(lzb[i, j, :b]), key=lambda kv: (-kv[1], kv[0]))
                      if v > -np.inf][:2]
                want += [(j, bb) for bb in bl] + [(-1, -1)] * (2 - len(bl))
            want += [(-1, -1)] * (4 - len(want))
            assert [tuple(x) for x in sel[i, b]] == want


def test_retrieval_limits_are_exact():
    Q, K, V = small_problem(18, 64, 5, 3, 4, 0.3)
    S = 16
    E = mo.exact_attention(Q, K, V, 1.0, causal=True)
    # everything retrieved: exact
    O = mo.muse_retrieval(Q, K, V, S, 4, 5, 3, k1=5, k2=4, scale=1.0)
    np.testing.assert_allclose(O, E, rtol=1e-10, atol=1e-12)
    # singleton queries (qt = 0): exact whatever is retrieved
    for k1, k2 in ((0, 0), (2, 1), (1, 3)):
        O = mo.muse_retrieval(Q, K, V, S, 64, 5, 3, k1=k1, k2=k2, scale=1.0)
        np.testing.assert_allclose(O, E, rtol=1e-10, atol=1e-12)
    # singleton keys, nothing retrieved: the remainder summaries are exact
    O = mo.muse_retrieval(Q, K, V, S, 4, 64, 3, k1=0, k2=0, scale=1.0)
    np.testing.assert_allclose(O, E, rtol=1e-10, atol=1e-12)


def test_retrieval_block_zero_uses_only_the_diagonal():
    Q, K, V = small_problem(19, 48, 4, 3, 3, 0.3)
    O = mo.muse_retrieval(Q, K, V, 16, 3, 3, 2, k1=1, k2=1, scale=1.0)
    E0 = mo.exact_attention(Q[:16], K[:16], V[:16], 1.0, causal=True)
    np.testing.assert_allclose(O[:16], E0, rtol=1e-12)


# --------------------------------------------------------------------------- partial dipole

def test_partial_dipole_equals_full_when_the_centroid_is_zero():
    """One query cluster whose centroid is 0 and one key cluster: the tilt by qbar = 0 is
    uniform, so the tilted C_ij is the plain Cov_j and pi = 1; the partially specialised
    dipole must then equal the full method (two different code paths)."""
    rng = np.random.default_rng(31)
    N, D, Dv, s = 40, 5, 3, 0.8
    Q = 0.3 * rng.standard_normal((N, D))
    Q -= Q.mean(axis=0)
    K, V = rng.standard_normal((N, D)), rng.standard_normal((N, Dv))
    ql, kl = np.zeros(N, np.int64), np.zeros(N, np.int64)
    Op = mo.muse_partial_dipole_from_labels(Q, K, V, ql, kl, 1, 1, s)
    Of = mo.muse_from_labels(Q, K, V, ql, kl, 1, 1, s)
    np.testing.assert_allclose(Op, Of, rtol=1e-12, atol=1e-12)


def test_key_cluster_covariance_is_numpy_cov():
    """Cov_j against numpy's biased covariance of the stacked (v, k) members."""
    rng = np.random.default_rng(32)
    N, D, Dv = 50, 4, 3
    K, V = rng.standard_normal((N, D)), rng.standard_normal((N, Dv))
    kl = rng.integers(0, 3, N)
    covs = mo.key_cluster_covariances(K, V, kl, 4)
    for j in range(3):
        idx = kl == j
        full = np.cov(np.hstack([V[idx], K[idx]]).T, bias=True)
        np.testing.assert_allclose(covs[j], full[:Dv, Dv:], rtol=1e-12, atol=1e-14)
    assert (covs[3] == 0).all()


def test_partial_dipole_is_first_order_in_the_centroid():
    """The untilted covariance leaves an error linear in the query centroid (the pages'
    O(qbar qt kt^2) bound): with one key cluster (so both weightings are 1), qt fixed and
    qbar scaled, the partial dipole departs from the full one in proportion to qbar."""
    rng = np.random.default_rng(33)
    N, D, Dv = 60, 4, 3
    base = rng.standard_normal(D)
    noise = 0.05 * rng.standard_normal((N, D))
    K, V = rng.standard_normal((N, D)), rng.standard_normal((N, Dv))
    ql, kl = np.zeros(N, np.int64), np.zeros(N, np.int64)
    diffs = []
    for a in (1e-3, 1e-2, 1e-1):
        Q = a * base[None, :] + noise - noise.mean(axis=0)
        Op = mo.muse_partial_dipole_from_labels(Q, K, V, ql, kl, 1, 1, 1.0)
        Of = mo.muse_from_labels(Q, K, V, ql, kl, 1, 1, 1.0)
        diffs.append(np.abs(Op - Of).max())
    slope = np.polyfit(np.log([1e-3, 1e-2, 1e-1]), np.log(diffs), 1)[0]
    assert 0.8 <= slope <= 1.2, slope


# --------------------------------------------------------------------------- the pages' trends

def _trend_problem(seed):
    from clustered_softmax_attention_b200.inputs import small_problem
    return small_problem(seed, 512, 16, 8, 24, 0.25)


def test_more_clusters_lower_error_and_the_dipole_helps():
    """The pages' qualitative claims (review "free parameters": error falls from C = 32 to
    C = 128; "invented entities": removing the dipole raises the error), on synthetic
    mixtures: the RSE against exact attention falls as C grows, and the monopole-only
    result is worse than the full method at every C."""
    for seed in (1, 2):
        Q, K, V = _trend_problem(seed)
        E = mo.exact_attention(Q, K, V, 1.0)
        errs, mono = [], []
        for C in (4, 16, 64):
            ql, qc = mo.kmeans(Q, C, 5)
            kl, _ = mo.kmeans(K, C, 5)
            errs.append(mo.rse(mo.muse_from_labels(Q, K, V, ql, kl, C, C, 1.0, qbar=qc), E))
            mono.append(mo.rse(mo.muse_from_labels(Q, K, V, ql, kl, C, C, 1.0, qbar=qc,
                                                   dipole=False), E))
        assert errs[0] > errs[1] > errs[2], errs
        assert all(m > e for m, e in zip(mono, errs)), (mono, errs)


def test_more_kmeans_rounds_do_not_raise_the_error():
    """Review "free parameters": the error drops from 1 to 5 K-means iterations."""
    tot1 = tot5 = 0.0
    for seed in (3, 4, 5):
        Q, K, V = _trend_problem(seed)
        E = mo.exact_attention(Q, K, V, 1.0)
        for T in (1, 5):
            ql, qc = mo.kmeans(Q, 16, T)
            kl, _ = mo.kmeans(K, 16, T)
            r = mo.rse(mo.muse_from_labels(Q, K, V, ql, kl, 16, 16, 1.0, qbar=qc), E)
            if T == 1:
                tot1 += r
            else:
                tot5 += r
    assert tot5 < tot1, (tot1, tot5)


def test_retrieval_error_does_not_rise_with_k1_and_k2():
    """gist.science "Kernmechanismen" item 4: retrieval is the accuracy upgrade of the causal
    accumulation -- exact attention on the retrieved (cluster, block) pairs replaces their
    summaries.  On seeded mixtures with 5 % outlier keys (x4 norm), the RSE against exact
    causal attention must not rise as k1 and k2 grow, and retrieving every pair is exact."""
    from clustered_softmax_attention_b200.inputs import draw_problem
    steps = ((0, 0), (1, 1), (2, 2), (4, 4), (8, 4), (16, 8))
    for seed in (1, 2, 3):
        rng = np.random.Generator(np.random.PCG64(seed))
        Q, K, V = draw_problem(rng, 1024, 16, 16, 24, 0.3 / 4, 0.05, 4.0)
        E = mo.exact_attention(Q, K, V, 1.0, causal=True)
        ql, _ = mo.kmeans(Q, 16, 5)
        kl, _ = mo.kmeans(K, 16, 5)
        errs = [mo.rse(mo.muse_retrieval(Q, K, V, 128, 16, 16, 5, k1, k2, 1.0,
                                         q_labels=ql, k_labels=kl), E) for k1, k2 in steps]
        assert all(b <= a * (1 + 1e-9) for a, b in zip(errs, errs[1:])), (seed, errs)
        assert errs[0] > 10 * errs[4], (seed, errs)   # retrieval makes a real difference
        assert errs[-1] < 1e-20, (seed, errs)          # k1 = Ck, k2 = nb: everything exact


# --------------------------------------------------------------------------- backward pass

def _fd_grad(f, X, h=1e-6):
    g = np.zeros_like(X)
    for idx in np.ndindex(X.shape):
        Xp, Xm = X.copy(), X.copy()
        Xp[idx] += h
        Xm[idx] -= h
        g[idx] = (f(Xp) - f(Xm)) / (2 * h)
    return g


@pytest.mark.parametrize("seed,D,Dv,s", [(0, 3, 2, 0.9), (1, 2, 4, 1.7), (2, 4, 4, 0.4)])
def test_backward_matches_central_differences(seed, D, Dv, s):
    """The backward pass against central finite differences of the forward oracle (labels
    fixed, qbar the member means), with an empty key cluster and a singleton query cluster."""
    rng = np.random.default_rng(seed)
    N, Cq, Ck = 14, 3, 4
    Q, K, V = rng.standard_normal((N, D)), rng.standard_normal((N, D)), rng.standard_normal((N, Dv))
    ql = np.concatenate([[0, 1, 2], rng.integers(0, 2, N - 3)])   # cluster 2: one member
    kl = np.concatenate([[0, 1, 2], rng.integers(0, 3, N - 3)])   # cluster 3: empty
    dO = rng.standard_normal((N, Dv))
    dQ, dK, dV = mo.muse_backward_from_labels(Q, K, V, ql, kl, Cq, Ck, s, dO)
    loss = lambda Q_, K_, V_: float((mo.muse_from_labels(Q_, K_, V_, ql, kl, Cq, Ck, s) * dO).sum())
    for got, fd in ((dQ, _fd_grad(lambda X: loss(X, K, V), Q)),
                    (dK, _fd_grad(lambda X: loss(Q, X, V), K)),
                    (dV, _fd_grad(lambda X: loss(Q, K, X), V))):
        np.testing.assert_allclose(got, fd, rtol=0, atol=1e-7 * np.abs(fd).max())


@pytest.mark.parametrize("case", ["singleton_keys", "singleton_queries"])
def test_backward_is_exact_attention_gradient_in_the_exact_limits(case):
    """Ck = N or Cq = N makes the approximation equal to exact attention as a function of
    (Q, K, V), so its gradient must equal exact attention's, taken by torch autograd."""
    import torch
    Q, K, V = small_problem(41, 24, 5, 3, 4, 0.3)
    rng = np.random.default_rng(9)
    dO = rng.standard_normal((24, 3))
    if case == "singleton_keys":
        ql, kl, Cq, Ck = rng.integers(0, 4, 24), np.arange(24), 4, 24
    else:
        ql, kl, Cq, Ck = np.arange(24), rng.integers(0, 5, 24), 24, 5
    dQ, dK, dV = mo.muse_backward_from_labels(Q, K, V, ql, kl, Cq, Ck, 1.3, dO)
    t = [torch.tensor(x, requires_grad=True) for x in (Q, K, V)]
    O = torch.nn.functional.scaled_dot_product_attention(t[0][None], t[1][None], t[2][None],
                                                         scale=1.3)[0]
    (O * torch.tensor(dO)).sum().backward()
    for got, ref in zip((dQ, dK, dV), t):
        np.testing.assert_allclose(got, ref.grad.numpy(), rtol=1e-10, atol=1e-12)
