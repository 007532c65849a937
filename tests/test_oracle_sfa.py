"""Pins of the oracle's sparse feature attention ("Scaling Attention via
Feature Sparsity", §2): the codes against a brute-force sort with the tie
rule, the score as the sum over the intersection of the supports (explicit
loops), k = d as dense softmax attention, and k = 1 scores that vanish
unless the two largest coordinates coincide."""

import numpy as np
import torch

import oracle

S = 0.25


def test_codes_brute_force_with_ties():
    x = np.array([[0.5, -2.0, 2.0, 0.1, -0.5, 1.0]])
    vals, idx = oracle.sfa_codes(x, 3)
    # |x| = .5 2 2 .1 .5 1: the two 2s, then 1 (index 5)
    assert idx.tolist() == [[1, 2, 5]]
    assert vals.tolist() == [[-2.0, 2.0, 1.0]]
    vals, idx = oracle.sfa_codes(x, 4)      # 0.5 ties at indices 0 and 4: 0 wins
    assert idx.tolist() == [[0, 1, 2, 5]]
    rng = np.random.default_rng(1)
    X = np.round(rng.standard_normal((20, 9)) * 2) / 2    # many ties
    for kf in (1, 3, 9):
        v, i = oracle.sfa_codes(X, kf)
        for r in range(20):
            order = sorted(range(9), key=lambda c: (-abs(X[r, c]), c))[:kf]
            assert list(i[r]) == sorted(order)
            assert np.array_equal(v[r], X[r, sorted(order)])


def test_overlap_score_by_loops():
    rng = np.random.default_rng(2)
    d, kf, n = 12, 4, 6
    Q = rng.standard_normal((1, 1, n, d))
    K = rng.standard_normal((1, 1, n, d))
    V = rng.standard_normal((1, 1, n, d))
    qv, qi = oracle.sfa_codes(Q, kf)
    kv, ki = oracle.sfa_codes(K, kf)
    o = oracle.sfa_attention(Q, K, V, kf, S)
    for t in range(n):
        a = []
        for j in range(n):
            common = set(qi[0, 0, t]) & set(ki[0, 0, j])
            sc = 0.0
            for c in common:
                sc += qv[0, 0, t, list(qi[0, 0, t]).index(c)] * kv[0, 0, j, list(ki[0, 0, j]).index(c)]
            a.append(S * sc)
        w = np.exp(np.array(a) - max(a))
        np.testing.assert_allclose(o[0, 0, t], (w @ V[0, 0]) / w.sum(), rtol=1e-12, atol=1e-12)


def test_full_support_is_dense_attention():
    rng = np.random.default_rng(3)
    Q, K, V = (rng.standard_normal((2, 3, 10, 8)) for _ in range(3))
    o = oracle.sfa_attention(Q, K, V, 8, S)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.tensor(Q), torch.tensor(K), torch.tensor(V),
                                                           scale=S).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)


def test_single_feature_scores_need_the_same_top_coordinate():
    rng = np.random.default_rng(4)
    d = 6
    Q = rng.standard_normal((1, 1, 8, d))
    K = rng.standard_normal((1, 1, 8, d))
    Qs = oracle.sfa_densify(*oracle.sfa_codes(Q, 1), d)
    Ks = oracle.sfa_densify(*oracle.sfa_codes(K, 1), d)
    sc = Qs[0, 0] @ Ks[0, 0].T
    qa = np.abs(Q[0, 0]).argmax(axis=1)
    ka = np.abs(K[0, 0]).argmax(axis=1)
    for t in range(8):
        for j in range(8):
            if qa[t] != ka[j]:
                assert sc[t, j] == 0.0
            else:
                assert sc[t, j] == Q[0, 0, t, qa[t]] * K[0, 0, j, ka[j]]
