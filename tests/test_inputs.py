"""The seeded synthetic inputs (CPU): the recipe the workloads are measured on.

Per (b,h): component means N(0, I/D); queries and keys independent draws of
mean[uniform component] + sigma N(0, I); values N(0, 1); for the retrieval workload
exactly round(0.05 N) key rows scaled x4; float32, or bfloat16 by round-to-nearest-even.
"""
import math

import numpy as np
import pytest

from clustered_softmax_attention_b200.inputs import (WORKLOAD_ORDER, WORKLOADS, draw_problem,
                                                     make_inputs, round_to_bf16)


def test_round_to_bf16_is_round_to_nearest_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1);
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: ties go up (even)
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e-3])
    r = round_to_bf16(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2 ** -6 and r[3] == 1.0
    assert r[4] == -2.5
    # every result is a bfloat16 (the low 16 bits of the float32 are zero) within half an ulp
    bits = r.astype(np.float32).view(np.uint32)
    assert (bits & 0xFFFF == 0).all()
    assert abs(float(r[5]) - 3.0e-3) <= 2.0 ** (math.floor(math.log2(3.0e-3)) - 8)


def test_draw_problem_statistics_and_outliers():
    rng = np.random.Generator(np.random.PCG64(5))
    N, D, Dv = 4000, 64, 32
    Q, K, V = draw_problem(rng, N, D, Dv, components=8, sigma=0.1)
    assert Q.shape == (N, D) and K.shape == (N, D) and V.shape == (N, Dv)
    assert abs(V.mean()) < 0.02 and abs(V.std() - 1.0) < 0.02
    # the same seed with outliers: exactly round(0.05 N) key rows, scaled by 4
    rng2 = np.random.Generator(np.random.PCG64(6))
    _, K0, _ = draw_problem(rng2, 1000, 16, 4, 4, 0.2)
    rng3 = np.random.Generator(np.random.PCG64(6))
    _, K1, _ = draw_problem(rng3, 1000, 16, 4, 4, 0.2, outlier_frac=0.05, outlier_scale=4.0)
    scaled = np.nonzero(~np.isclose(K0, K1).all(axis=1))[0]
    assert scaled.size == round(0.05 * 1000)
    np.testing.assert_allclose(K1[scaled], 4.0 * K0[scaled])


@pytest.mark.parametrize("name", WORKLOAD_ORDER)
def test_workloads_are_seeded_and_shaped(name):
    w = WORKLOADS[name]
    # one problem, drawn as the full draw would draw it
    Q, K, V = make_inputs(w, heads=[0])
    assert Q.shape == (1, 1, w.N, w.D) and V.shape == (1, 1, w.N, w.Dv)
    assert Q.dtype == np.float32
    Q2, _, _ = make_inputs(w, heads=[0])
    np.testing.assert_array_equal(Q, Q2)
    if w.dtype == "bf16":
        assert (Q.view(np.uint32) & 0xFFFF == 0).all()


def test_head_subset_matches_full_draw():
    w = WORKLOADS["acausal_n1k_f32"]
    full = make_inputs(w)
    sub = make_inputs(w, heads=[0])
    for a, b in zip(full, sub):
        np.testing.assert_array_equal(a.reshape(-1, *a.shape[2:])[0], b[0, 0])
