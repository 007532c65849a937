"""Pins of the oracle's backward pass of the sparse prefill (drop and
zero_order tails): central finite differences of the forward oracle, torch
autograd of dense float64 attention when every block is selected, and zero
gradients when nothing is attended."""

import numpy as np
import pytest
import torch

import oracle

S = 0.4


def _case(rng, nb=4, blk=3, d=4, H=2):
    N = nb * blk
    Q, K, V = (rng.standard_normal((1, H, N, d)) for _ in range(3))
    idx = np.array([[[sorted(rng.choice(nb, 2, replace=False)) for _ in range(nb)] for _ in range(H)]])
    dO = rng.standard_normal((1, H, N, d))
    return Q, K, V, idx, dO, blk


@pytest.mark.parametrize("tail", ["zero_order", "drop"])
def test_finite_differences(tail):
    rng = np.random.default_rng(11)
    Q, K, V, idx, dO, blk = _case(rng)
    dQ, dK, dV = oracle.sparse_attention_backward(Q, K, V, idx, blk, tail, S, dO)

    def f(Qx, Kx, Vx):
        return float((oracle.sparse_attention(Qx, Kx, Vx, idx, blk, tail, S) * dO).sum())

    h = 1e-6
    for arr, grad, which in ((Q, dQ, 0), (K, dK, 1), (V, dV, 2)):
        for pos in [(0, 0, 0, 0), (0, 1, 5, 2), (0, 0, 11, 3), (0, 1, 7, 1)]:
            plus = [Q.copy(), K.copy(), V.copy()]
            minus = [Q.copy(), K.copy(), V.copy()]
            plus[which][pos] += h
            minus[which][pos] -= h
            num = (f(*plus) - f(*minus)) / (2 * h)
            assert abs(num - grad[pos]) <= 1e-6 * max(1.0, abs(num)), (tail, which, pos, num, grad[pos])


def test_all_selected_matches_autograd():
    rng = np.random.default_rng(12)
    nb, blk, d = 3, 4, 5
    N = nb * blk
    Q, K, V, dO = (rng.standard_normal((1, 2, N, d)) for _ in range(4))
    idx = np.tile(np.arange(nb), (1, 2, nb, 1))
    dQ, dK, dV = oracle.sparse_attention_backward(Q, K, V, idx, blk, "zero_order", S, dO)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=S)
    o.backward(torch.tensor(dO))
    np.testing.assert_allclose(dQ, tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.numpy(), atol=1e-12)


def test_drop_without_selection_has_no_gradient():
    rng = np.random.default_rng(13)
    Q, K, V, _, dO, blk = _case(rng)
    idx = np.zeros((1, 2, 4, 0), dtype=np.int64)
    for g in oracle.sparse_attention_backward(Q, K, V, idx, blk, "drop", S, dO):
        assert not g.any()


# ---- the rows' log-sum-exp (what sa_sparse_attn_fwd_lse writes) -------------

@pytest.mark.parametrize("tail", ["zero_order", "drop"])
def test_lse_every_block_selected_is_dense_logsumexp(tail):
    # with every block selected there are no pseudo-keys: torch's logsumexp of
    # the dense logits, in log2 units
    rng = np.random.default_rng(21)
    nb, blk, d = 4, 3, 4
    Q, K = (rng.standard_normal((1, 2, nb * blk, d)) for _ in range(2))
    idx = np.tile(np.arange(nb), (1, 2, nb, 1))
    got = oracle.sparse_attention_lse(Q, K, idx, blk, tail, S)
    ref = torch.logsumexp(S * torch.from_numpy(Q) @ torch.from_numpy(K).transpose(-1, -2), dim=-1) / np.log(2.0)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_lse_centroids_only():
    # zero_order with nothing selected: log2 Σ_j B e^{s q·k̄_j} = log2 B +
    # logsumexp_j(s q·k̄_j) / ln 2, the centroids taken with torch's mean
    rng = np.random.default_rng(22)
    nb, blk, d = 5, 4, 3
    Q, K = (rng.standard_normal((1, 1, nb * blk, d)) for _ in range(2))
    idx = np.zeros((1, 1, nb, 0), dtype=np.int64)
    got = oracle.sparse_attention_lse(Q, K, idx, blk, "zero_order", S)
    kbar = torch.from_numpy(K).reshape(1, 1, nb, blk, d).mean(dim=3)
    ref = np.log2(blk) + torch.logsumexp(S * torch.from_numpy(Q) @ kbar.transpose(-1, -2), dim=-1) / np.log(2.0)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_lse_without_keys_is_infinite():
    rng = np.random.default_rng(23)
    Q, K = (rng.standard_normal((1, 1, 6, 2)) for _ in range(2))
    got = oracle.sparse_attention_lse(Q, K, np.zeros((1, 1, 2, 0), dtype=np.int64), 3, "drop", S)
    assert np.all(np.isinf(got)) and np.all(got > 0)
