"""Plain float64 CPU oracle of the backward pass of the sparse prefill.

TEST INFRASTRUCTURE: only the tests and ``bench.py``'s CPU legs use this
module.  It shares no code with the CUDA library.

The forward is ``sparse_attention`` of the tails "drop" and "zero_order"
(PISA "Algoritmo Central": exact terms over the selected blocks S_i, and for
every unselected block j one pseudo-key k̄_j = mean of the block's keys with
value v̄_j = vsum_j / B and weight B e^{s q·k̄_j}).  Written as attention of
query block i to the key list [k_n, n ∈ S_i] + [k̄_j, j ∈ U_i] with logit
biases [0 ...] + [ln B ...], the gradients are those of softmax attention
(the chain rule through o = P V, P = softmax(s Q Kᵀ + bias)):

    dV_keys = Pᵀ dO,  dP = dO V_keysᵀ,  δ_t = dO_t · o_t,
    dS = P ⊙ (dP − δ),  dQ = s dS K_keys,  dK_keys = s dSᵀ Q,

and a pseudo-key's gradients reach the tokens of its block through
k̄_j = (1/B) Σ_n k_n and v̄_j = (1/B) Σ_n v_n: every token n of block j gets
dk̄_j / B and dv̄_j / B (added to what it gets as an exact key of the query
blocks that selected block j).

The rows' log-sum-exp of that key list (``sparse_attention_lse``, log2
units) is what the GPU forward can hand to its backward.

Pins (``tests/test_oracle_backward.py``): central finite differences of the
forward oracle on tiny inputs (both tails); with every block selected the
gradients equal torch autograd of float64 softmax attention; drop with no
selected block has zero gradients.  The log-sum-exp equals torch's
``logsumexp`` of the dense logits when every block is selected, log2 B plus
``logsumexp`` of the centroid logits when none is, and +inf without keys.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def sparse_attention_lse(Q, K, block_idx, block: int, tail: str, scale: float) -> np.ndarray:
    """[B,H,N] float64: each query row's log-sum-exp of its logits in log2
    units, log2 Σ exp(s q·k + bias) over the row's key list of
    ``sparse_attention_backward`` (exact keys bias 0, pseudo-keys ln B); +inf
    for a row without keys."""
    if tail not in ("drop", "zero_order"):
        raise ValueError("the log-sum-exp is defined for the drop and zero_order tails")
    Q, K = _f64(Q), _f64(K)
    Bsz, H, N, d = K.shape
    nb = N // block
    idx = np.asarray(block_idx)
    out = np.full((Bsz, H, N), np.inf)
    for b in range(Bsz):
        for h in range(H):
            Kh = K[b, h]
            kbar = Kh.reshape(nb, block, d).mean(axis=1)
            for i in range(N // block):
                rows = slice(i * block, (i + 1) * block)
                sel = sorted(int(j) for j in idx[b, h, i])
                uns = [j for j in range(nb) if j not in set(sel)] if tail == "zero_order" else []
                tok = [n for j in sel for n in range(j * block, (j + 1) * block)]
                keys = np.concatenate([Kh[tok], kbar[uns]]) if tok or uns else np.zeros((0, d))
                if keys.shape[0] == 0:
                    continue
                bias = np.concatenate([np.zeros(len(tok)), np.full(len(uns), np.log(block))])
                a = scale * Q[b, h, rows] @ keys.T + bias
                mx = a.max(axis=1, keepdims=True)
                out[b, h, rows] = (mx[:, 0] + np.log(np.exp(a - mx).sum(axis=1))) / np.log(2.0)
    return out


def sparse_attention_backward(Q, K, V, block_idx, block: int, tail: str, scale: float, dO):
    """(dQ, dK, dV) [B,H,N,d] float64 of sparse_attention(tail) at (Q, K, V)
    for the output cotangent dO [B,H,N,d]; tail "drop" or "zero_order"."""
    if tail not in ("drop", "zero_order"):
        raise ValueError("backward is defined for the drop and zero_order tails")
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    Bsz, H, N, d = K.shape
    nb = N // block
    idx = np.asarray(block_idx)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for b in range(Bsz):
        for h in range(H):
            Kh, Vh = K[b, h], V[b, h]
            kbar = Kh.reshape(nb, block, d).mean(axis=1)
            vbar = Vh.reshape(nb, block, d).mean(axis=1)
            for i in range(N // block):
                rows = slice(i * block, (i + 1) * block)
                q, g = Q[b, h, rows], dO[b, h, rows]
                sel = sorted(int(j) for j in idx[b, h, i])
                uns = [j for j in range(nb) if j not in set(sel)] if tail == "zero_order" else []
                tok = np.concatenate([np.arange(j * block, (j + 1) * block) for j in sel]) if sel else \
                    np.zeros(0, dtype=np.int64)
                keys = np.concatenate([Kh[tok], kbar[uns]])
                vals = np.concatenate([Vh[tok], vbar[uns]])
                bias = np.concatenate([np.zeros(len(tok)), np.full(len(uns), np.log(block))])
                if keys.shape[0] == 0:
                    continue                       # output 0: no gradient
                a = scale * q @ keys.T + bias
                p = np.exp(a - a.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                o = p @ vals
                dvals = p.T @ g
                dp = g @ vals.T
                delta = (g * o).sum(axis=1, keepdims=True)
                ds = p * (dp - delta)
                dQ[b, h, rows] += scale * ds @ keys
                dkeys = scale * ds.T @ q
                ne = len(tok)
                dK[b, h, tok] += dkeys[:ne]
                dV[b, h, tok] += dvals[:ne]
                for r, j in enumerate(uns):
                    dK[b, h, j * block:(j + 1) * block] += dkeys[ne + r] / block
                    dV[b, h, j * block:(j + 1) * block] += dvals[ne + r] / block
    return dQ, dK, dV
