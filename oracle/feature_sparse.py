"""Plain float64 CPU oracle of sparse feature attention (SFA).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use this module.  It shares no code with the
CUDA library.

Source: "Scaling Attention via Feature Sparsity", §2 "Metodologia Proposta:
Sparse Feature Attention": every query and key keeps only its k coordinates
of largest magnitude (a top-k operator on the Q and K projections), and the
attention score of a (query, key) pair is taken over the overlap of their
supports, Σ_{c ∈ supp(q) ∩ supp(k)} q_c k_c, followed by the usual softmax
over the keys and the weighted sum of the (dense) values.  FlashSFA computes
exactly this with an online softmax over tiles.

Readings taken where the page leaves a step open:

* the top-k is over |x_c| per token and head; a tie in magnitude goes to the
  smaller channel index; the kept coordinates keep their signed values;
* the softmax scale s multiplies the support-overlap score as it multiplies
  q·k in dense attention (s = 1/sqrt(d) of the full head dimension);
* attention is non-causal, as everywhere else in this repository (the
  page's language models are causal; the causal mask is a separate axis);
* V stays dense.

Pins (``tests/test_oracle_sfa.py``): k = d is dense softmax attention (torch
SDPA); the overlap score equals the dot product of the zero-filled sparse
vectors and, by explicit loops, the sum over the intersection of the
supports; k = 1 scores are non-zero only for pairs whose largest coordinate
is the same; the codes equal a brute-force sort with the tie rule.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def sfa_codes(X, kf: int):
    """Top-kf coordinates by magnitude of every vector of X [..., d].

    Returns (values [..., kf] float64, indices [..., kf] int64), the indices
    ascending within each vector; ties in |x| go to the smaller index.
    """
    X = _f64(X)
    d = X.shape[-1]
    if not 1 <= kf <= d:
        raise ValueError("kf must be in [1, d]")
    flat = X.reshape(-1, d)
    vals = np.empty((flat.shape[0], kf))
    idx = np.empty((flat.shape[0], kf), dtype=np.int64)
    # stable sort of -|x| keeps the smaller index first among equal magnitudes
    order = np.argsort(-np.abs(flat), axis=1, kind="stable")[:, :kf]
    order.sort(axis=1)
    for r in range(flat.shape[0]):
        idx[r] = order[r]
        vals[r] = flat[r, order[r]]
    return vals.reshape(X.shape[:-1] + (kf,)), idx.reshape(X.shape[:-1] + (kf,))


def sfa_densify(vals, idx, d: int) -> np.ndarray:
    """Zero-filled dense vectors [..., d] from codes (values, indices)."""
    vals = _f64(vals)
    idx = np.asarray(idx, dtype=np.int64)
    out = np.zeros(vals.shape[:-1] + (d,))
    np.put_along_axis(out, idx, vals, axis=-1)
    return out


def sfa_attention(Q, K, V, kf: int, scale: float, rows=None) -> np.ndarray:
    """SFA forward, [B,H,N,d] inputs, non-causal: softmax(s Q̃ K̃ᵀ) V with Q̃,
    K̃ the top-kf sparsified queries and keys (the support-overlap score is the
    dot product of the zero-filled sparse vectors).  ``rows``: optional query
    row indices (then only those rows are returned, [B,H,len(rows),d])."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    d = Q.shape[-1]
    if rows is not None:
        Q = Q[:, :, np.asarray(rows, dtype=np.int64)]
    Qs = sfa_densify(*sfa_codes(Q, kf), d)
    Ks = sfa_densify(*sfa_codes(K, kf), d)
    a = scale * np.einsum("bhic,bhjc->bhij", Qs, Ks)
    a -= a.max(axis=-1, keepdims=True)
    w = np.exp(a)
    return np.einsum("bhij,bhjc->bhic", w, V) / w.sum(axis=-1)[..., None]
