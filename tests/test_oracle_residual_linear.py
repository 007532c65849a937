"""Pins of the oracle's residual_linear tail (SPLA §2.2-2.3: the exact sparse
attention plus the RMS-normalised residual linear attention over the
unselected blocks, with the exponential feature map).

The pins fix it by: the dense case (every block selected leaves no residual,
so the output is textbook softmax attention), explicit token loops, the
subtraction form the GPU uses (all-block state minus the selected blocks'),
and the scale invariance of the RMS norm."""

import math

import numpy as np
import torch

import oracle

S = 0.3


def _dense(q, K, V, scale):
    a = scale * q @ K.T
    w = np.exp(a - a.max(axis=1, keepdims=True))
    return (w @ V) / w.sum(axis=1, keepdims=True)


def test_all_selected_is_dense_attention():
    rng = np.random.default_rng(1)
    B, Hq, Hkv, N, d, blk = 1, 4, 2, 64, 8, 8
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    o, _, _ = oracle.decode_attention(q, K, V, blk, N // blk, S, tail="residual_linear")
    g = Hq // Hkv
    for h in range(Hq):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q[0, h][None, None, None]), torch.tensor(K[0, h // g][None, None]),
            torch.tensor(V[0, h // g][None, None]), scale=S)[0, 0, 0].numpy()
        np.testing.assert_allclose(o[0, h], ref, atol=1e-12)


def test_brute_force_token_loops():
    rng = np.random.default_rng(2)
    nb, blk, d = 5, 4, 3
    K = rng.standard_normal((nb * blk, d))
    V = rng.standard_normal((nb * blk, d))
    q = rng.standard_normal((2, d))
    sel = [1, 3]
    got = oracle.sparse_attention(np.concatenate([q, np.zeros((nb * blk - 2, d))])[None, None],
                                  K[None, None], V[None, None],
                                  np.tile(np.array(sel), (1, 1, nb, 1)), blk, "residual_linear", S)[0, 0, :2]
    for t in range(2):
        num = [0.0] * d
        den = 0.0
        lin = [0.0] * d
        for j in range(nb):
            for n in range(blk):
                k = K[j * blk + n]
                v = V[j * blk + n]
                if j in sel:
                    w = math.exp(S * sum(q[t, c] * k[c] for c in range(d)))
                    den += w
                    for c in range(d):
                        num[c] += w * v[c]
                else:
                    f = sum(math.exp(q[t, c]) * math.exp(k[c]) for c in range(d))
                    for c in range(d):
                        lin[c] += f * v[c]
        rms = math.sqrt(sum(x * x for x in lin) / d + 1e-6)
        ref = [num[c] / den + lin[c] / rms for c in range(d)]
        np.testing.assert_allclose(got[t], ref, rtol=1e-12, atol=1e-12)


def test_subtraction_form_equals_direct_sum():
    # φ(q)ᵀ(S_all − S_sel) with S = Σ φ(k) vᵀ: the IO-saving form of SPLA §2.2
    rng = np.random.default_rng(3)
    nb, blk, d = 6, 8, 5
    K = rng.standard_normal((nb * blk, d))
    V = rng.standard_normal((nb * blk, d))
    q = rng.standard_normal((blk, d))
    sel = [0, 4]
    S_all = np.exp(K).T @ V
    tok = np.concatenate([np.arange(j * blk, (j + 1) * blk) for j in sel])
    S_sel = np.exp(K[tok]).T @ V[tok]
    o_rla = np.exp(q) @ (S_all - S_sel)
    rms = np.sqrt((o_rla * o_rla).mean(axis=1) + 1e-6)
    ref = _dense(q, K[tok], V[tok], S) + o_rla / rms[:, None]
    Q = np.zeros((nb * blk, d))
    Q[:blk] = q
    got = oracle.sparse_attention(Q[None, None], K[None, None], V[None, None],
                                  np.tile(np.array(sel), (1, 1, nb, 1)), blk, "residual_linear", S)[0, 0, :blk]
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)


def test_rms_norm_scale_invariance():
    # scaling V by c scales the exact part by c and leaves the normalised
    # residual unchanged (its RMS is far above eps here)
    rng = np.random.default_rng(4)
    B, Hq, Hkv, N, d, blk = 1, 2, 1, 64, 8, 8
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    idx = np.array([[[1, 5]]])
    o1, _, _ = oracle.decode_attention(q, K, V, blk, 2, S, tail="residual_linear", block_idx=idx)
    o3, _, _ = oracle.decode_attention(q, K, 3.0 * V, blk, 2, S, tail="residual_linear", block_idx=idx)
    d1, _, _ = oracle.decode_attention(q, K, V, blk, 2, S, tail="drop", block_idx=idx)
    np.testing.assert_allclose(o3 - 3.0 * d1, o1 - d1, rtol=1e-9, atol=1e-9)
