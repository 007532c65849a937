"""Pins of the oracle's covariance-aware routing (PISA "Roteamento Consciente
de Covariância": a block's score takes in both its attention score and the
norm M_j = ‖H_j − H̄‖₂ of its first-order deviation from the head's mean).

The pins fix M_j by things other than the oracle's SVD call: a rank-one
construction whose spectral norm is a product of vector norms, identical
blocks (every H_j equal, so M_j = 0), and the largest eigenvalue of AᵀA from
a symmetric eigen-solver; the "cov" score is checked by explicit loops and
against the "dot" order when M_j = 0."""

import numpy as np

import oracle

S = 0.3


def _rank_one_blocks(rng, nb, blk, d):
    """Keys k̄_j + a_n u and values b_n w + c_j with per-block coefficients:
    H_j = (Σ_n a_n b_n) u wᵀ = γ_j u wᵀ, so H_j − H̄ = (γ_j − γ̄) u wᵀ."""
    u = rng.standard_normal(d)
    w = rng.standard_normal(d)
    kbar = rng.standard_normal((nb, d))
    a = rng.standard_normal((nb, blk))
    a -= a.mean(axis=1, keepdims=True)           # zero-mean deviations per block
    b = rng.standard_normal((nb, blk))
    c = rng.standard_normal((nb, d))
    K = kbar[:, None, :] + a[:, :, None] * u[None, None, :]
    V = b[:, :, None] * w[None, None, :] + c[:, None, :]
    gamma = (a * b).sum(axis=1)
    return K.reshape(nb * blk, d), V.reshape(nb * blk, d), gamma, u, w


def test_covnorm_rank_one_closed_form():
    rng = np.random.default_rng(3)
    nb, blk, d = 9, 16, 7
    K, V, gamma, u, w = _rank_one_blocks(rng, nb, blk, d)
    st = oracle.block_pool(None, K[None, None], V[None, None], blk, covariance=True)
    expect = np.abs(gamma - gamma.mean()) * np.linalg.norm(u) * np.linalg.norm(w)
    np.testing.assert_allclose(st["covnorm"][0, 0], expect, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(st["hbar"][0, 0], gamma.mean() * np.outer(u, w), atol=1e-12)


def test_covnorm_identical_blocks_is_zero_and_cov_orders_like_dot():
    rng = np.random.default_rng(4)
    nb, blk, d = 6, 8, 5
    Kb = rng.standard_normal((blk, d))
    Vb = rng.standard_normal((blk, d))
    shift = rng.standard_normal((nb, d))         # distinct centroids, same deviations
    K = (Kb[None] + shift[:, None]).reshape(nb * blk, d)
    V = np.tile(Vb, (nb, 1))
    Q = rng.standard_normal((nb * blk, d))
    st = oracle.block_pool(Q[None, None], K[None, None], V[None, None], blk, covariance=True)
    np.testing.assert_allclose(st["covnorm"], 0.0, atol=1e-12)
    cov = oracle.route_scores(st["qmean"], st["kmean"], "cov", covnorm=st["covnorm"], scale=S, block=blk)
    dot = oracle.route_scores(st["qmean"], st["kmean"], "dot")
    np.testing.assert_allclose(cov, S * dot, atol=1e-12)


def test_covnorm_equals_largest_eigenvalue_of_gram():
    rng = np.random.default_rng(5)
    nb, blk, d = 5, 12, 6
    K = rng.standard_normal((nb * blk, d))
    V = rng.standard_normal((nb * blk, d))
    st = oracle.block_pool(None, K[None, None], V[None, None], blk, covariance=True)
    # H_j by explicit loops, then sqrt(λ_max(AᵀA)) with a symmetric solver
    Hs = []
    for j in range(nb):
        H = np.zeros((d, d))
        kb = K[j * blk:(j + 1) * blk].mean(axis=0)
        for n in range(blk):
            H += np.outer(K[j * blk + n] - kb, V[j * blk + n])
        Hs.append(H)
    Hbar = sum(Hs) / nb
    for j in range(nb):
        A = Hs[j] - Hbar
        lam = np.linalg.eigvalsh(A.T @ A).max()
        assert abs(st["covnorm"][0, 0, j] - np.sqrt(lam)) <= 1e-10 * max(1.0, np.sqrt(lam))


def test_cov_score_brute_force():
    rng = np.random.default_rng(6)
    B, H, nqb, nb, d, blk = 1, 2, 3, 4, 5, 8
    qm = rng.standard_normal((B, H, nqb, d))
    km = rng.standard_normal((B, H, nb, d))
    M = rng.random((B, H, nb)) * 10.0
    got = oracle.route_scores(qm, km, "cov", covnorm=M, scale=S, block=blk)
    for h in range(H):
        for i in range(nqb):
            qn = np.sqrt(sum(x * x for x in qm[0, h, i]))
            for j in range(nb):
                dot = sum(qm[0, h, i, c] * km[0, h, j, c] for c in range(d))
                ref = S * dot + np.log(1.0 + S * qn * M[0, h, j] / blk)
                assert abs(got[0, h, i, j] - ref) <= 1e-12


def test_cov_score_prefers_heterogeneous_blocks_at_equal_attention():
    # two blocks with the same centroid: the one with the larger deviation
    # norm scores higher, so it is the one computed exactly
    qm = np.array([[[[1.0, 0.0]]]])
    km = np.array([[[[0.5, 0.5], [0.5, 0.5]]]])
    M = np.array([[[1.0, 5.0]]])
    sc = oracle.route_scores(qm, km, "cov", covnorm=M, scale=S, block=4)
    assert sc[0, 0, 0, 1] > sc[0, 0, 0, 0]
    assert list(oracle.topk_from_scores(sc, 1)[0, 0, 0]) == [1]
