"""Pins of the oracle's first_order tail (PISA "Algoritmo Central": the
zero-order block terms plus the global first-order correction
(s q_t) H̄ Σ_{j∈U} e^{s q_t.k̄_j} of the numerator).

Each pin fixes the result by something other than the oracle's own formula:
block-constant keys make the correction vanish; blocks that share their
deviations from the centroid make H̄ equal every block's H_j, so the hybrid
order is the per-block first-order Taylor sum, written out token by token
here; and the approximation error must shrink as the square of the in-block
deviations, against linearly for the zero-order tail."""

import numpy as np
import pytest

import oracle

S = 0.35


def _dense(q, K, V, scale):
    a = scale * q @ K.T
    w = np.exp(a - a.max(axis=1, keepdims=True))
    return (w @ V) / w.sum(axis=1, keepdims=True)


def _shared_deviation_inputs(rng, nb, blk, d, eps):
    """Keys k̄_j + eps Δ_n with the same zero-mean Δ in every block; values
    v_n + c_j (one pattern, a per-block offset), so H_j = eps Σ_n Δ_n v_nᵀ for
    every block j."""
    kbar = rng.standard_normal((nb, d))
    delta = rng.standard_normal((blk, d))
    delta -= delta.mean(axis=0)
    vpat = rng.standard_normal((blk, d))
    voff = rng.standard_normal((nb, d))
    K = (kbar[:, None, :] + eps * delta[None, :, :]).reshape(nb * blk, d)
    V = (vpat[None, :, :] + voff[:, None, :]).reshape(nb * blk, d)
    return K, V, kbar, delta, vpat, voff


def test_hbar_closed_form_and_block_constant_keys():
    rng = np.random.default_rng(1)
    nb, blk, d = 6, 8, 5
    K, V, kbar, delta, vpat, voff = _shared_deviation_inputs(rng, nb, blk, d, 0.3)
    st = oracle.block_pool(None, K[None, None], V[None, None], blk, first_order=True)
    # every block has H_j = 0.3 Σ_n Δ_n v_nᵀ (the offsets drop out: ΣΔ = 0)
    np.testing.assert_allclose(st["hbar"][0, 0], 0.3 * delta.T @ vpat, atol=1e-12)
    # block-constant keys: H̄ = 0 and first_order == zero_order == dense
    Kc = np.repeat(kbar, blk, axis=0)
    q = rng.standard_normal((blk, d))
    Q = np.concatenate([q] * nb)[None, None]
    idx = np.tile(np.array([1, 4]), (1, 1, nb, 1))
    o1 = oracle.sparse_attention(Q, Kc[None, None], V[None, None], idx, blk, "first_order", S)
    o0 = oracle.sparse_attention(Q, Kc[None, None], V[None, None], idx, blk, "zero_order", S)
    np.testing.assert_allclose(o1, o0, atol=1e-13)
    np.testing.assert_allclose(o1[0, 0, :blk], _dense(q, Kc, V, S), atol=1e-12)


def test_equals_per_block_first_order_taylor():
    rng = np.random.default_rng(2)
    nb, blk, d = 7, 8, 6
    K, V, kbar, delta, vpat, voff = _shared_deviation_inputs(rng, nb, blk, d, 0.2)
    q = rng.standard_normal((blk, d))
    sel = [0, 3]
    uns = [j for j in range(nb) if j not in sel]
    # brute force: exact over S, e^{s q.k̄_j} (1 + s q.(k_n − k̄_j)) per token over U
    num = np.zeros((blk, d))
    den = np.zeros(blk)
    for t in range(blk):
        for j in range(nb):
            for n in range(blk):
                k = K[j * blk + n]
                v = V[j * blk + n]
                if j in sel:
                    w = np.exp(S * q[t] @ k)
                else:
                    w = np.exp(S * q[t] @ kbar[j]) * (1.0 + S * q[t] @ (k - kbar[j]))
                num[t] += w * v
                den[t] += w
    ref = num / den[:, None]
    Q = np.zeros((1, 1, nb * blk, d))
    Q[0, 0, :blk] = q
    idx = np.tile(np.array(sel), (1, 1, nb, 1))
    got = oracle.sparse_attention(Q, K[None, None], V[None, None], idx, blk, "first_order", S)[0, 0, :blk]
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_error_is_second_order_in_the_deviations():
    rng = np.random.default_rng(3)
    nb, blk, d = 8, 16, 8
    q = rng.standard_normal((blk, d))
    errs = {"zero_order": [], "first_order": []}
    for eps in (0.08, 0.04, 0.02):
        r2 = np.random.default_rng(7)            # same pattern, smaller deviations
        K, V, *_ = _shared_deviation_inputs(r2, nb, blk, d, eps)
        Q = np.zeros((1, 1, nb * blk, d))
        Q[0, 0, :blk] = q
        idx = np.zeros((1, 1, nb, 0), dtype=np.int64)          # every block in the tail
        ref = _dense(q, K, V, S)
        for tail in errs:
            o = oracle.sparse_attention(Q, K[None, None], V[None, None], idx, blk, tail, S)[0, 0, :blk]
            errs[tail].append(np.abs(o - ref).max())
    for tail, order in (("zero_order", 1), ("first_order", 2)):
        e = errs[tail]
        ratios = [e[i + 1] / e[i] for i in range(len(e) - 1)]
        for r in ratios:
            assert abs(np.log2(r) + order) < 0.35, (tail, e)
    assert errs["first_order"][-1] < 0.1 * errs["zero_order"][-1]


@pytest.mark.parametrize("k", [0, 3])
def test_all_blocks_selected_or_none_consistent(k):
    # with every block selected the tail is empty: first_order == drop == dense
    rng = np.random.default_rng(4 + k)
    nb, blk, d = 4, 8, 4
    Q = rng.standard_normal((1, 2, nb * blk, d))
    K = rng.standard_normal((1, 2, nb * blk, d))
    V = rng.standard_normal((1, 2, nb * blk, d))
    idx = np.tile(np.arange(nb), (1, 2, nb, 1))
    o1 = oracle.sparse_attention(Q, K, V, idx, blk, "first_order", S)
    o2 = oracle.sparse_attention(Q, K, V, idx, blk, "drop", S)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
