"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test fixes a part of the oracle against a closed form, a hand-derived
worked example (tests/golden), a library routine it must reduce to, or brute
force written independently here with Python loops.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sdpa(q, k, v, scale, mask=None):
    """Library softmax attention in float64 (torch SDPA on CPU)."""
    t = lambda a: torch.as_tensor(np.asarray(a, dtype=np.float64))
    m = None if mask is None else torch.as_tensor(mask)
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=m, scale=scale).numpy()


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --------------------------------------------------------------------------
# block statistics
# --------------------------------------------------------------------------

def test_block_pool_closed_form_ramp():
    # keys k[n, c] = a_c + b_c * n inside every block: mean a + b (B-1)/2,
    # population variance b^2 (B^2 - 1) / 12
    Bk, nb, d = 8, 3, 5
    rng = np.random.default_rng(0)
    a = rng.standard_normal((nb, d))
    b = rng.standard_normal((nb, d))
    n = np.arange(Bk)
    K = (a[:, None, :] + b[:, None, :] * n[None, :, None]).reshape(1, 1, nb * Bk, d)
    V = np.ones_like(K) * 3.0
    st = oracle.block_pool(None, K, V, Bk, variance=True)
    np.testing.assert_allclose(st["kmean"][0, 0], a + b * (Bk - 1) / 2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st["kvar"][0, 0], b * b * (Bk * Bk - 1) / 12, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(st["vsum"][0, 0], 3.0 * Bk)


def test_block_pool_brute_force_and_linear_stats():
    Bsz, H, N, d, blk = 1, 2, 12, 3, 4
    Q, K, V = _rand((Bsz, H, N, d), 1), _rand((Bsz, H, N, d), 2), _rand((Bsz, H, N, d), 3)
    st = oracle.block_pool(Q, K, V, blk, variance=True, linear=True)
    for h in range(H):
        for j in range(N // blk):
            toks = range(j * blk, (j + 1) * blk)
            for c in range(d):
                qm = sum(Q[0, h, n, c] for n in toks) / blk
                km = sum(K[0, h, n, c] for n in toks) / blk
                kv = sum((K[0, h, n, c] - km) ** 2 for n in toks) / blk
                vs = sum(V[0, h, n, c] for n in toks)
                zr = sum(max(K[0, h, n, c], 0.0) for n in toks)
                assert math.isclose(st["qmean"][0, h, j, c], qm, abs_tol=1e-12)
                assert math.isclose(st["kmean"][0, h, j, c], km, abs_tol=1e-12)
                assert math.isclose(st["kvar"][0, h, j, c], kv, abs_tol=1e-12)
                assert math.isclose(st["vsum"][0, h, j, c], vs, abs_tol=1e-12)
                assert math.isclose(st["zrelu"][0, h, j, c], zr, abs_tol=1e-12)
        for c in range(d):
            for e in range(d):
                ht = sum(max(K[0, h, n, c], 0.0) * V[0, h, n, e] for n in range(N))
                assert math.isclose(st["htot"][0, h, c, e], ht, abs_tol=1e-11)
            assert math.isclose(st["ztot"][0, h, c],
                                sum(max(K[0, h, n, c], 0.0) for n in range(N)), abs_tol=1e-11)


def test_block_pool_constant_block_has_zero_variance():
    K = np.repeat(_rand((1, 1, 4, 1, 6), 4), 16, axis=3).reshape(1, 1, 64, 6)
    st = oracle.block_pool(None, K, K, 16, variance=True)
    assert np.abs(st["kvar"]).max() < 1e-25


# --------------------------------------------------------------------------
# router
# --------------------------------------------------------------------------

def test_route_scores_brute_force():
    d, nq, nb = 4, 3, 5
    qm, km = _rand((1, 1, nq, d), 5), _rand((1, 1, nb, d), 6)
    pq, pk = _rand((d, d), 7), _rand((d, d), 8)
    kv = np.abs(_rand((1, 1, nb, d), 9))
    s = 0.7
    dot = oracle.route_scores(qm, km, "dot")
    proj = oracle.route_scores(qm, km, "proj", proj_q=pq, proj_k=pk)
    t2 = oracle.route_scores(qm, km, "taylor2", kvar=kv, scale=s)
    for i in range(nq):
        for j in range(nb):
            q, k = qm[0, 0, i], km[0, 0, j]
            assert math.isclose(dot[0, 0, i, j], sum(q[c] * k[c] for c in range(d)), abs_tol=1e-12)
            a = [sum(q[r] * pq[r, c] for r in range(d)) for c in range(d)]
            b = [sum(k[r] * pk[r, c] for r in range(d)) for c in range(d)]
            assert math.isclose(proj[0, 0, i, j], sum(x * y for x, y in zip(a, b)), abs_tol=1e-11)
            # the SPLA score itself, exp(q'.kbar)(1 + 1/2 q'^T diag(var) q'), q' = s q
            raw = math.exp(s * sum(q[c] * k[c] for c in range(d))) * (
                1 + 0.5 * sum((s * q[c]) ** 2 * kv[0, 0, j, c] for c in range(d)))
            assert math.isclose(t2[0, 0, i, j], math.log(raw), abs_tol=1e-12)


def test_taylor2_equals_dot_order_without_variance():
    qm, km = _rand((1, 2, 8, 6), 10), _rand((1, 2, 32, 6), 11)
    t2 = oracle.route_scores(qm, km, "taylor2", kvar=np.zeros_like(km), scale=0.3)
    dot = oracle.route_scores(qm, km, "dot")
    np.testing.assert_array_equal(oracle.topk_from_scores(t2, 7), oracle.topk_from_scores(dot, 7))


def test_golden_taylor2_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "spla_taylor2_worked.json")))
    K = np.array(g["K"])[None, None]
    st = oracle.block_pool(None, K, K, g["block"], variance=True)
    np.testing.assert_allclose(st["kmean"][0, 0], g["expected_kmean"], atol=1e-15)
    np.testing.assert_allclose(st["kvar"][0, 0], g["expected_kvar"], atol=1e-15)
    q = np.array(g["qmean"])[None, None, None]
    t2 = oracle.route_scores(q, st["kmean"], "taylor2", kvar=st["kvar"], scale=g["scale"])
    np.testing.assert_allclose(t2[0, 0, 0], g["expected_log_scores"], rtol=1e-14)
    dot = oracle.route_scores(q, st["kmean"], "dot")
    np.testing.assert_allclose(dot[0, 0, 0], g["expected_dot"], rtol=1e-14)


def test_decode_route_scores_group_sum_brute_force():
    Bsz, Hq, Hkv, nb, d = 1, 4, 2, 5, 3
    q, km = _rand((Bsz, Hq, d), 12), _rand((Bsz, Hkv, nb, d), 13)
    kv = np.abs(_rand((Bsz, Hkv, nb, d), 14))
    s = 0.5
    sc = oracle.decode_route_scores(q, km, kv, s)
    g = Hq // Hkv
    for kh in range(Hkv):
        for j in range(nb):
            tot = 0.0
            for h in range(kh * g, (kh + 1) * g):
                qq = q[0, h]
                tot += math.exp(s * sum(qq[c] * km[0, kh, j, c] for c in range(d))) * (
                    1 + 0.5 * sum((s * qq[c]) ** 2 * kv[0, kh, j, c] for c in range(d)))
            assert math.isclose(sc[0, kh, j], math.log(tot), abs_tol=1e-12)


def test_topk_brute_force_definition():
    rng = np.random.default_rng(15)
    for trial in range(40):
        nb = int(rng.integers(1, 8))
        k = int(rng.integers(0, nb + 1))
        sc = rng.integers(-2, 3, size=nb).astype(float)   # many ties on purpose
        got = list(oracle.topk_from_scores(sc, k))
        valid = []
        for sub in itertools.combinations(range(nb), k):
            rest = [u for u in range(nb) if u not in sub]
            if all(sc[j] > sc[u] or (sc[j] == sc[u] and j < u) for j in sub for u in rest):
                valid.append(list(sub))
        assert valid == [got]


def test_topk_hand_ties_and_keep_count():
    assert list(oracle.topk_from_scores(np.array([1.0, 3.0, 3.0, 2.0, 3.0]), 2)) == [1, 2]
    assert list(oracle.topk_from_scores(np.array([0.0, 0.0, 0.0]), 2)) == [0, 1]
    assert oracle.k_from_percent(10, 256) == 26
    assert oracle.k_from_percent(5, 512) == 26
    assert oracle.k_from_percent(50, 4) == 2


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _all_idx(Bsz, H, nqb, nb):
    return np.broadcast_to(np.arange(nb), (Bsz, H, nqb, nb)).copy()


def _rand_idx(rng, Bsz, H, nqb, nb, k):
    return np.stack([np.stack([np.stack([np.sort(rng.choice(nb, k, replace=False))
                                         for _ in range(nqb)]) for _ in range(H)])
                     for _ in range(Bsz)])


@pytest.mark.parametrize("tail", ["zero_order", "drop", "linear_mix"])
def test_all_blocks_selected_is_dense_attention(tail):
    Bsz, H, N, d, blk = 1, 2, 64, 8, 16
    Q, K, V = _rand((Bsz, H, N, d), 20), _rand((Bsz, H, N, d), 21), _rand((Bsz, H, N, d), 22)
    s = 1 / math.sqrt(d)
    idx = _all_idx(Bsz, H, N // blk, N // blk)
    alpha = np.full((H, d), 1.0) if tail == "linear_mix" else None
    alpha_any = np.random.default_rng(0).uniform(0.2, 0.9, (H, d))
    O = oracle.sparse_attention(Q, K, V, idx, blk, tail, s, alpha=alpha)
    np.testing.assert_allclose(O, _sdpa(Q, K, V, s), rtol=1e-11, atol=1e-12)
    if tail == "linear_mix":
        # U empty: the linear branch is 0, so O = alpha * dense
        O2 = oracle.sparse_attention(Q, K, V, idx, blk, tail, s, alpha=alpha_any)
        np.testing.assert_allclose(O2, alpha_any[None, :, None, :] * _sdpa(Q, K, V, s),
                                   rtol=1e-11, atol=1e-12)


def test_zero_order_is_exact_for_block_size_one():
    Bsz, H, N, d = 1, 1, 24, 5
    Q, K, V = _rand((Bsz, H, N, d), 23), _rand((Bsz, H, N, d), 24), _rand((Bsz, H, N, d), 25)
    idx = _rand_idx(np.random.default_rng(1), Bsz, H, N, N, 5)
    O = oracle.sparse_attention(Q, K, V, idx, 1, "zero_order", 0.4)
    np.testing.assert_allclose(O, _sdpa(Q, K, V, 0.4), rtol=1e-11, atol=1e-12)


def test_zero_order_is_exact_for_block_constant_keys():
    Bsz, H, N, d, blk = 1, 2, 96, 6, 8
    K = np.repeat(_rand((Bsz, H, N // blk, 1, d), 26), blk, axis=3).reshape(Bsz, H, N, d)
    Q, V = _rand((Bsz, H, N, d), 27), _rand((Bsz, H, N, d), 28)
    for k in (0, 3, 12):
        idx = _rand_idx(np.random.default_rng(k), Bsz, H, N // blk, N // blk, k)
        O = oracle.sparse_attention(Q, K, V, idx, blk, "zero_order", 0.5)
        np.testing.assert_allclose(O, _sdpa(Q, K, V, 0.5), rtol=1e-10, atol=1e-12)


def test_zero_order_without_selection_is_attention_over_block_pseudo_tokens():
    # all blocks unselected: softmax over nb pseudo-tokens with key kbar_j,
    # value vsum_j / B and logit bias ln B (B e^{x} = e^{x + ln B})
    Bsz, H, N, d, blk = 1, 1, 64, 4, 8
    Q, K, V = _rand((Bsz, H, N, d), 29), _rand((Bsz, H, N, d), 30), _rand((Bsz, H, N, d), 31)
    idx = np.zeros((Bsz, H, N // blk, 0), dtype=np.int64)
    O = oracle.sparse_attention(Q, K, V, idx, blk, "zero_order", 0.6)
    kb = K.reshape(Bsz, H, N // blk, blk, d).mean(axis=3)
    vb = V.reshape(Bsz, H, N // blk, blk, d).mean(axis=3)
    bias = np.full((N, N // blk), math.log(blk))
    np.testing.assert_allclose(O, _sdpa(Q, kb, vb, 0.6, mask=bias), rtol=1e-11, atol=1e-12)


def test_drop_is_masked_softmax_attention():
    Bsz, H, N, d, blk = 1, 2, 64, 4, 8
    Q, K, V = _rand((Bsz, H, N, d), 32), _rand((Bsz, H, N, d), 33), _rand((Bsz, H, N, d), 34)
    idx = _rand_idx(np.random.default_rng(2), Bsz, H, N // blk, N // blk, 3)
    O = oracle.sparse_attention(Q, K, V, idx, blk, "drop", 0.5)
    for h in range(H):
        mask = np.zeros((N, N), dtype=bool)
        for i in range(N // blk):
            for j in idx[0, h, i]:
                mask[i * blk:(i + 1) * blk, j * blk:(j + 1) * blk] = True
        ref = _sdpa(Q[0, h], K[0, h], V[0, h], 0.5, mask=mask)
        np.testing.assert_allclose(O[0, h], ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("tail", ["zero_order", "drop", "linear_mix"])
def test_value_shift_shifts_output(tail):
    # row normalisation: V -> V + c shifts every output row by exactly c
    # (the linear branch needs eps = 0 for this to be exact)
    Bsz, H, N, d, blk = 1, 2, 48, 4, 8
    Q, K, V = _rand((Bsz, H, N, d), 35), _rand((Bsz, H, N, d), 36), _rand((Bsz, H, N, d), 37)
    Q = np.abs(Q)  # keeps relu(q).z > 0 so the eps-free linear branch is defined
    idx = _rand_idx(np.random.default_rng(3), Bsz, H, N // blk, N // blk, 2)
    alpha = np.random.default_rng(4).uniform(0.2, 0.9, (H, d))
    c = np.array([0.5, -1.25, 2.0, 0.0])
    O1 = oracle.sparse_attention(Q, K, V, idx, blk, tail, 0.5, alpha=alpha, eps=0.0)
    O2 = oracle.sparse_attention(Q, K, V + c, idx, blk, tail, 0.5, alpha=alpha, eps=0.0)
    np.testing.assert_allclose(O2, O1 + c, rtol=1e-10, atol=1e-11)


def test_permuting_tokens_inside_blocks_leaves_output_unchanged():
    Bsz, H, N, d, blk = 1, 1, 64, 4, 16
    Q, K, V = _rand((Bsz, H, N, d), 38), _rand((Bsz, H, N, d), 39), _rand((Bsz, H, N, d), 40)
    idx = _rand_idx(np.random.default_rng(5), Bsz, H, N // blk, N // blk, 1)
    perm = np.concatenate([j * blk + np.random.default_rng(j).permutation(blk)
                           for j in range(N // blk)])
    alpha = np.full((H, d), 0.5)
    for tail in ("zero_order", "drop", "linear_mix"):
        O1 = oracle.sparse_attention(Q, K, V, idx, blk, tail, 0.5, alpha=alpha)
        O2 = oracle.sparse_attention(Q, K[:, :, perm], V[:, :, perm], idx, blk, tail, 0.5, alpha=alpha)
        np.testing.assert_allclose(O1, O2, rtol=1e-11, atol=1e-12)


def _brute(Q, K, V, sel, blk, tail, s, alpha, eps):
    """Token-by-token evaluation of the three tails with Python floats."""
    N, d = len(K), len(K[0])
    nb = N // blk
    out = []
    for q in Q:
        def lg(k):
            return s * sum(q[c] * k[c] for c in range(d))
        S = [n for j in sel for n in range(j * blk, (j + 1) * blk)]
        U = [j for j in range(nb) if j not in sel]
        if tail == "zero_order":
            terms = [(lg(K[n]), 1.0, V[n]) for n in S]
            for j in U:
                kb = [sum(K[n][c] for n in range(j * blk, (j + 1) * blk)) / blk for c in range(d)]
                vs = [sum(V[n][c] for n in range(j * blk, (j + 1) * blk)) for c in range(d)]
                terms.append((lg(kb), float(blk), [x / blk for x in vs]))
            m = max(t[0] for t in terms)
            den = sum(w * math.exp(a - m) for a, w, _ in terms)
            out.append([sum(w * math.exp(a - m) * v[c] for a, w, v in terms) / den for c in range(d)])
            continue
        if S:
            m = max(lg(K[n]) for n in S)
            den = sum(math.exp(lg(K[n]) - m) for n in S)
            os_ = [sum(math.exp(lg(K[n]) - m) * V[n][c] for n in S) / den for c in range(d)]
        else:
            os_ = [0.0] * d
        if tail == "drop":
            out.append(os_)
            continue
        Ut = [n for j in U for n in range(j * blk, (j + 1) * blk)]
        fq = [max(x, 0.0) for x in q]
        den = sum(fq[c] * max(K[n][c], 0.0) for n in Ut for c in range(d)) + eps
        ol = [sum(sum(fq[c] * max(K[n][c], 0.0) for c in range(d)) * V[n][e] for n in Ut) / den
              for e in range(d)]
        out.append([alpha[e] * os_[e] + (1 - alpha[e]) * ol[e] for e in range(d)])
    return out


@pytest.mark.parametrize("tail", ["zero_order", "drop", "linear_mix"])
@pytest.mark.parametrize("k", [0, 1, 3])
def test_attention_brute_force(tail, k):
    Bsz, H, N, d, blk = 1, 1, 16, 3, 4
    Q, K, V = _rand((Bsz, H, N, d), 41 + k), _rand((Bsz, H, N, d), 42), _rand((Bsz, H, N, d), 43)
    idx = _rand_idx(np.random.default_rng(6 + k), Bsz, H, N // blk, N // blk, k)
    alpha = np.random.default_rng(7).uniform(0.2, 0.9, (H, d))
    O = oracle.sparse_attention(Q, K, V, idx, blk, tail, 0.7, alpha=alpha)
    for i in range(N // blk):
        rows = Q[0, 0, i * blk:(i + 1) * blk].tolist()
        ref = _brute(rows, K[0, 0].tolist(), V[0, 0].tolist(), list(idx[0, 0, i]), blk, tail,
                     0.7, alpha[0].tolist(), 1e-6)
        np.testing.assert_allclose(O[0, 0, i * blk:(i + 1) * blk], ref, rtol=1e-10, atol=1e-12)


def test_golden_zero_order_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "pisa_zero_order_worked.json")))
    Q, K, V = (np.array(g[n])[None, None] for n in ("Q", "K", "V"))
    idx = np.array(g["block_idx"])[None, None]
    alpha = np.array(g["alpha"])[None]
    for tail, want in g["expected_rows_0_1"].items():
        O = oracle.sparse_attention(Q, K, V, idx, g["block"], tail, g["scale"],
                                    alpha=alpha, eps=g["eps"])
        np.testing.assert_allclose(O[0, 0, :2, 0], want, rtol=1e-13)


def test_linear_mix_limits():
    Bsz, H, N, d, blk = 1, 2, 32, 4, 8
    Q, K, V = _rand((Bsz, H, N, d), 44), _rand((Bsz, H, N, d), 45), _rand((Bsz, H, N, d), 46)
    idx = _rand_idx(np.random.default_rng(8), Bsz, H, N // blk, N // blk, 2)
    one = np.ones((H, d))
    np.testing.assert_allclose(oracle.sparse_attention(Q, K, V, idx, blk, "linear_mix", 0.5, alpha=one),
                               oracle.sparse_attention(Q, K, V, idx, blk, "drop", 0.5),
                               rtol=1e-12, atol=1e-13)
    # alpha = 0 and nothing selected: ReLU linear attention over all tokens,
    # evaluated here with torch on the feature-mapped matrices
    idx0 = np.zeros((Bsz, H, N // blk, 0), dtype=np.int64)
    O = oracle.sparse_attention(Q, K, V, idx0, blk, "linear_mix", 0.5, alpha=np.zeros((H, d)))
    fq = torch.relu(torch.as_tensor(Q))
    fk = torch.relu(torch.as_tensor(K))
    A = fq @ fk.transpose(-1, -2)
    ref = (A @ torch.as_tensor(V)) / (A.sum(-1, keepdim=True) + 1e-6)
    np.testing.assert_allclose(O, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_sampled_query_blocks_match_full_output():
    Bsz, H, N, d, blk = 2, 2, 32, 4, 8
    Q, K, V = _rand((Bsz, H, N, d), 47), _rand((Bsz, H, N, d), 48), _rand((Bsz, H, N, d), 49)
    idx = _rand_idx(np.random.default_rng(9), Bsz, H, N // blk, N // blk, 2)
    O = oracle.sparse_attention(Q, K, V, idx, blk, "zero_order", 0.5)
    picks = [(1, 0, 2), (0, 1, 3), (1, 1, 0)]
    S = oracle.sparse_attention(Q, K, V, idx, blk, "zero_order", 0.5, qblocks=picks)
    for r, (b, h, i) in enumerate(picks):
        np.testing.assert_array_equal(S[r], O[b, h, i * blk:(i + 1) * blk])


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------

def test_decode_all_blocks_is_dense_gqa_attention():
    Bsz, Hq, Hkv, N, d, blk = 2, 4, 2, 64, 8, 8
    q, Kc, Vc = _rand((Bsz, Hq, d), 50), _rand((Bsz, Hkv, N, d), 51), _rand((Bsz, Hkv, N, d), 52)
    s = 1 / math.sqrt(d)
    o, idx, sc = oracle.decode_attention(q, Kc, Vc, blk, N // blk, s)
    g = Hq // Hkv
    kx = np.repeat(Kc, g, axis=1)
    vx = np.repeat(Vc, g, axis=1)
    ref = _sdpa(q[:, :, None, :], kx, vx, s)[:, :, 0, :]
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_decode_matches_prefill_oracle_row():
    Bsz, Hq, Hkv, N, d, blk, k = 1, 4, 2, 64, 8, 8, 3
    q, Kc, Vc = _rand((Bsz, Hq, d), 53), _rand((Bsz, Hkv, N, d), 54), _rand((Bsz, Hkv, N, d), 55)
    s = 0.4
    o, idx, sc = oracle.decode_attention(q, Kc, Vc, blk, k, s)
    st = oracle.block_pool(None, Kc, Vc, blk, variance=True)
    np.testing.assert_allclose(sc, oracle.decode_route_scores(q, st["kmean"], st["kvar"], s))
    np.testing.assert_array_equal(idx, oracle.topk_from_scores(sc, k))
    g = Hq // Hkv
    for h in range(Hq):
        kh = h // g
        Qrow = np.zeros((1, 1, blk, d))
        Qrow[0, 0, 0] = q[0, h]
        pre = oracle.sparse_attention(Qrow, Kc[:, kh:kh + 1], Vc[:, kh:kh + 1],
                                      idx[0, kh][None, None, None], blk, "zero_order", s,
                                      qblocks=[(0, 0, 0)])
        np.testing.assert_allclose(o[0, h], pre[0, 0], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# FP8 e4m3
# --------------------------------------------------------------------------

def test_e4m3_codes_are_fixed_points_and_match_torch():
    vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    fin = vals[np.isfinite(vals)]
    assert len(fin) == 254 and np.abs(fin).max() == 448.0
    np.testing.assert_array_equal(oracle.e4m3_round(fin), fin)
    # midpoints of consecutive codes (ties) and random values in range
    pos = np.unique(fin[fin >= 0])
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(60)
    rnd = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000) * 0.01,
                          mids, -mids])
    ref = torch.as_tensor(rnd).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.e4m3_round(rnd), ref)


def test_e4m3_saturates():
    np.testing.assert_array_equal(oracle.e4m3_round(np.array([500.0, -1e9, 449.0, 464.1])),
                                  [448.0, -448.0, 448.0, 448.0])


def test_quantise_blocks_error_bound():
    X = _rand((1, 2, 256, 16), 61) * 3
    deq, codes, sigma = oracle.quantise_blocks_e4m3(X, 128)
    assert sigma.shape == (1, 2, 2)
    xs = (X.reshape(1, 2, 2, 128, 16) / sigma[..., None, None].astype(np.float64)).reshape(X.shape)
    assert np.abs(codes).max() <= 448.0
    # half an ulp of e4m3 at the value's binade (2^-9 spacing below 2^-6)
    e = np.maximum(np.floor(np.log2(np.maximum(np.abs(xs), 1e-30))), -6)
    ulp = 2.0 ** (e - 3)
    assert np.all(np.abs(codes - xs) <= ulp / 2 + 1e-6 * ulp)
    assert np.all(np.abs(deq - X) <= (ulp / 2 + 1e-6 * ulp) * sigma.max())


def test_fp8_attention_is_exact_on_e4m3_representable_blocks():
    # build per-block inputs whose absmax is 448 * sigma and whose values are
    # e4m3 values times sigma: quantisation is then lossless, so the quantised
    # forward equals the float64 attention (drop tail has no centroids)
    rng = np.random.default_rng(70)
    Bsz, H, N, d, blk = 1, 2, 256, 16, 128
    vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 64)]
    def make():
        X = rng.choice(vals, size=(Bsz, H, N, d))
        X[:, :, ::blk, 0] = 448.0          # pins each block's absmax to 448
        return X * 2.0 ** -10              # a power-of-two scale keeps x / sigma exact
    Q, K, V = make(), make(), make()
    idx = _rand_idx(np.random.default_rng(71), Bsz, H, N // blk, N // blk, 1)
    np.testing.assert_array_equal(oracle.quantise_blocks_e4m3(Q, blk)[0], Q)
    a = oracle.fp8_attention(Q, K, V, idx, blk, "drop", 0.3)
    b = oracle.sparse_attention(Q, K, V, idx, blk, "drop", 0.3)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_quantise_blocks_ragged_last_block():
    X = _rand((1, 1, 300, 8), 72)
    deq, codes, sigma = oracle.quantise_blocks_e4m3(X, 128)
    assert deq.shape == X.shape and sigma.shape == (1, 1, 3)
    np.testing.assert_allclose(sigma[0, 0, 2], np.float32(np.abs(X[0, 0, 256:]).max()) / np.float32(448.0))
