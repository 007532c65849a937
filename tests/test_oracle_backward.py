"""Pins of the oracle's backward pass of the sparse prefill (every tail of
the prefill): central finite differences of the forward oracle, torch
autograd of dense float64 attention when every block is selected, torch
autograd of float64 re-statements of PISA's hybrid order and of SLA2's
mixture written with dense masks, the limits where the first-order and
mixed tails reduce to the zero-order and drop ones, and zero gradients when
nothing is attended."""

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


ALPHA = np.array([[0.3, 0.8, 0.5, 0.6], [0.9, 0.2, 0.4, 0.7]])   # [H, d] of _case


@pytest.mark.parametrize("tail", ["zero_order", "drop", "first_order", "linear_mix"])
def test_finite_differences(tail):
    rng = np.random.default_rng(11)
    Q, K, V, idx, dO, blk = _case(rng)
    alpha = ALPHA if tail == "linear_mix" else None
    dQ, dK, dV = oracle.sparse_attention_backward(Q, K, V, idx, blk, tail, S, dO, alpha=alpha)

    def f(Qx, Kx, Vx):
        return float((oracle.sparse_attention(Qx, Kx, Vx, idx, blk, tail, S, alpha=alpha) * dO).sum())

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


# ---- PISA's hybrid order (first_order) ----------------------------------

def _first_order_torch(Q, K, V, idx, blk, scale):
    """PISA's hybrid order restated with dense masks over all tokens and all
    block centroids (float64 torch, differentiable)."""
    Bsz, H, N, d = Q.shape
    nb = N // blk
    Kb, Vb = K.reshape(Bsz, H, nb, blk, d), V.reshape(Bsz, H, nb, blk, d)
    kbar, vsum = Kb.mean(dim=3), Vb.sum(dim=3)
    hbar = torch.einsum("bhjnc,bhjne->bhce", Kb - kbar.unsqueeze(3), Vb) / nb
    sel = torch.zeros(Bsz, H, nb, nb, dtype=torch.bool)             # [.., query block, key block]
    for b in range(Bsz):
        for h in range(H):
            for i in range(nb):
                sel[b, h, i, list(idx[b, h, i])] = True
    sel_tok = sel.repeat_interleave(blk, dim=2).repeat_interleave(blk, dim=3)   # [.., N, N]
    uns_row = (~sel).repeat_interleave(blk, dim=2)                               # [.., N, nb]
    a = scale * Q @ K.transpose(-1, -2)
    c = scale * Q @ kbar.transpose(-1, -2)
    m = torch.maximum(a.masked_fill(~sel_tok, -1e300).amax(-1), c.masked_fill(~uns_row, -1e300).amax(-1))
    wa = torch.exp(a - m[..., None]) * sel_tok
    wc = torch.exp(c - m[..., None]) * uns_row
    num = wa @ V + wc @ vsum + (scale * Q @ hbar) * wc.sum(-1, keepdim=True)
    den = wa.sum(-1) + blk * wc.sum(-1)
    return num / den[..., None]


def test_first_order_matches_autograd_of_a_masked_restatement():
    rng = np.random.default_rng(14)
    Q, K, V, idx, dO, blk = _case(rng, nb=5, blk=3, d=4)
    dQ, dK, dV = oracle.sparse_attention_backward(Q, K, V, idx, blk, "first_order", S, dO)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    o = _first_order_torch(tq, tk, tv, idx, blk, S)
    np.testing.assert_allclose(o.detach().numpy(), oracle.sparse_attention(Q, K, V, idx, blk, "first_order", S),
                               rtol=1e-12, atol=1e-12)
    o.backward(torch.tensor(dO))
    for got, t in ((dQ, tq), (dK, tk), (dV, tv)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_first_order_with_block_constant_keys():
    # constant keys inside every block give H̄ = 0: the output, dQ and dV are
    # the zero-order ones; dK still differs, through H̄'s dependence on K
    rng = np.random.default_rng(15)
    Q, K, V, idx, dO, blk = _case(rng)
    K = np.repeat(K[:, :, ::blk], blk, axis=2)
    fo = oracle.sparse_attention_backward(Q, K, V, idx, blk, "first_order", S, dO)
    zo = oracle.sparse_attention_backward(Q, K, V, idx, blk, "zero_order", S, dO)
    np.testing.assert_allclose(fo[0], zo[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fo[2], zo[2], rtol=1e-12, atol=1e-13)
    assert np.abs(fo[1] - zo[1]).max() > 1e-3


# ---- SLA2's mixture (linear_mix) ------------------------------------------

def _linear_mix_torch(Q, K, V, idx, blk, scale, alpha, eps=1e-6):
    """SLA2's α⊙O_s + (1−α)⊙O_l restated with dense token masks."""
    Bsz, H, N, d = Q.shape
    nb = N // blk
    sel = torch.zeros(Bsz, H, nb, nb, dtype=torch.bool)
    for b in range(Bsz):
        for h in range(H):
            for i in range(nb):
                sel[b, h, i, list(idx[b, h, i])] = True
    sel_tok = sel.repeat_interleave(blk, dim=2).repeat_interleave(blk, dim=3)
    a = (scale * Q @ K.transpose(-1, -2)).masked_fill(~sel_tok, float("-inf"))
    has = sel_tok.any(-1, keepdim=True)
    p = torch.softmax(torch.where(has, a, torch.zeros_like(a)), dim=-1) * has
    o_s = p @ V
    lin = torch.relu(Q) @ torch.relu(K).transpose(-1, -2) * (~sel_tok)
    o_l = (lin @ V) / (lin.sum(-1, keepdim=True) + eps)
    al = alpha[None, :, None, :]
    return al * o_s + (1 - al) * o_l


def test_linear_mix_matches_autograd_of_a_masked_restatement():
    rng = np.random.default_rng(16)
    Q, K, V, idx, dO, blk = _case(rng, nb=5, blk=3, d=4)
    dQ, dK, dV = oracle.sparse_attention_backward(Q, K, V, idx, blk, "linear_mix", S, dO, alpha=ALPHA)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    o = _linear_mix_torch(tq, tk, tv, idx, blk, S, torch.tensor(ALPHA))
    np.testing.assert_allclose(o.detach().numpy(),
                               oracle.sparse_attention(Q, K, V, idx, blk, "linear_mix", S, alpha=ALPHA),
                               rtol=1e-12, atol=1e-12)
    o.backward(torch.tensor(dO))
    for got, t in ((dQ, tq), (dK, tk), (dV, tv)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_linear_mix_limits():
    rng = np.random.default_rng(17)
    Q, K, V, idx, dO, blk = _case(rng)
    # α = 1: the drop backward
    ones = np.ones_like(ALPHA)
    lm = oracle.sparse_attention_backward(Q, K, V, idx, blk, "linear_mix", S, dO, alpha=ones)
    dr = oracle.sparse_attention_backward(Q, K, V, idx, blk, "drop", S, dO)
    for x, y in zip(lm, dr):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-13)
    # every block selected: no linear branch; the drop backward of α⊙dO
    nb = idx.shape[2]
    full = np.tile(np.arange(nb), (1, 2, nb, 1))
    lm = oracle.sparse_attention_backward(Q, K, V, full, blk, "linear_mix", S, dO, alpha=ALPHA)
    dr = oracle.sparse_attention_backward(Q, K, V, full, blk, "drop", S, dO * ALPHA[None, :, None, :])
    for x, y in zip(lm, dr):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-13)
    # α = 0 and nothing selected: ReLU linear attention over all tokens (torch autograd)
    empty = np.zeros((1, 2, nb, 0), dtype=np.int64)
    lm = oracle.sparse_attention_backward(Q, K, V, empty, blk, "linear_mix", S, dO, alpha=np.zeros_like(ALPHA))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    fq, fk = torch.relu(tq), torch.relu(tk)
    o = (fq @ (fk.transpose(-1, -2) @ tv)) / (fq @ fk.sum(-2, keepdim=True).transpose(-1, -2) + 1e-6)
    o.backward(torch.tensor(dO))
    for got, t in zip(lm, (tq, tk, tv)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=1e-10, atol=1e-12)


# ---- the straight-through backward of a quantised forward (o_forward) ------

@pytest.mark.parametrize("tail", ["zero_order", "drop"])
def test_backward_with_the_forwards_own_output_is_unchanged(tail):
    rng = np.random.default_rng(18)
    Q, K, V, idx, dO, blk = _case(rng)
    O = oracle.sparse_attention(Q, K, V, idx, blk, tail, S)
    a = oracle.sparse_attention_backward(Q, K, V, idx, blk, tail, S, dO)
    b = oracle.sparse_attention_backward(Q, K, V, idx, blk, tail, S, dO, o_forward=O)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-14)


def test_backward_shift_of_delta_closed_form():
    # o_forward = O + E shifts δ by Δ_t = dO_t·E_t; dS = P (dP − δ) moves by
    # −P Δ, so dQ moves by −s Δ_t Σ_k P_tk k_k = −s Δ_t · (attention of Q to K
    # with the keys as values), and dV does not move
    rng = np.random.default_rng(19)
    Q, K, V, idx, dO, blk = _case(rng)
    O = oracle.sparse_attention(Q, K, V, idx, blk, "zero_order", S)
    E = 0.05 * rng.standard_normal(O.shape)
    a = oracle.sparse_attention_backward(Q, K, V, idx, blk, "zero_order", S, dO)
    b = oracle.sparse_attention_backward(Q, K, V, idx, blk, "zero_order", S, dO, o_forward=O + E)
    shift = (dO * E).sum(axis=-1, keepdims=True)
    pk = oracle.sparse_attention(Q, K, K, idx, blk, "zero_order", S)
    np.testing.assert_allclose(b[0] - a[0], -S * shift * pk, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(b[2], a[2], rtol=1e-12, atol=1e-14)
