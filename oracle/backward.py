"""Plain float64 CPU oracle of the backward pass of the sparse prefill.

TEST INFRASTRUCTURE: only the tests and ``bench.py``'s CPU legs use this
module.  It shares no code with the CUDA library.

The forward is ``sparse_attention``.  For the tails "drop" and "zero_order"
(PISA "Algoritmo Central": exact terms over the selected blocks S_i, and for
every unselected block j one pseudo-key k̄_j = mean of the block's keys with
value v̄_j = vsum_j / B and weight B e^{s q·k̄_j}), written as attention of
query block i to the key list [k_n, n ∈ S_i] + [k̄_j, j ∈ U_i] with logit
biases [0 ...] + [ln B ...], the gradients are those of softmax attention
(the chain rule through o = P V, P = softmax(s Q Kᵀ + bias)):

    dV_keys = Pᵀ dO,  dP = dO V_keysᵀ,  δ_t = dO_t · o_t,
    dS = P ⊙ (dP − δ),  dQ = s dS K_keys,  dK_keys = s dSᵀ Q,

and a pseudo-key's gradients reach the tokens of its block through
k̄_j = (1/B) Σ_n k_n and v̄_j = (1/B) Σ_n v_n: every token n of block j gets
dk̄_j / B and dv̄_j / B (added to what it gets as an exact key of the query
blocks that selected block j).

"first_order" (PISA's hybrid order) adds λ_t f_t to the zero-order output,
with f_t = s H̄ᵀ q_t and λ_t = Σ_{j∈U} P_tj / B (the pseudo-keys' share of
the row's softmax, without the factor B).  So a pseudo-key's value seen by
row t is v̄_j + f_t / B; the softmax backward above then holds with
dP_tj = dO_t·(v̄_j + f_t / B), plus two more terms: dq_t += s λ_t H̄ dO_t,
and G = dL/dH̄ = s Σ_t λ_t q_t dO_tᵀ, which reaches every token m of block
j through H̄ = (1/nb) Σ_j Σ_{m∈j} (k_m − k̄_j) v_mᵀ as

    dk_m += G (v_m − v̄_j) / nb,   dv_m += Gᵀ (k_m − k̄_j) / nb.

"linear_mix" (SLA2 §2A) is o = α⊙O_s + (1−α)⊙O_l: O_s is the drop output,
whose backward above takes the cotangent α⊙dO; O_l = φ(q)ᵀ h_U / (φ(q)·z_U
+ ε) with φ = ReLU, h_U = Σ_{n∈U} φ(k_n) v_nᵀ, z_U = Σ_{n∈U} φ(k_n) over the
unselected tokens (O_l = 0 when U is empty).  With g = (1−α)⊙dO_t,
num = φ(q)ᵀ h_U and den = φ(q)·z_U + ε:

    dnum = g / den,  dden = −(g·O_l) / den,
    dφ(q) = h_U dnum + z_U dden,          dq = 1[q > 0] ⊙ dφ(q),
    dh_U = φ(q) dnumᵀ,  dz_U = φ(q) dden,
    for n ∈ U:  dk_n = 1[k_n > 0] ⊙ (dh_U v_n + dz_U),  dv_n = dh_Uᵀ φ(k_n).

The rows' log-sum-exp of the drop / zero-order key list
(``sparse_attention_lse``, log2 units) is what the GPU forward can hand to
its backward.

Pins (``tests/test_oracle_backward.py``): central finite differences of the
forward oracle on tiny inputs (every tail); with every block selected the
gradients equal torch autograd of float64 softmax attention; drop with no
selected block has zero gradients; first_order against torch autograd of a
float64 re-statement of PISA's hybrid order, and equal to zero_order when
the keys are constant inside each block (H̄ = 0); linear_mix against torch
autograd of a masked float64 re-statement, equal to drop (cotangent α⊙dO)
when no block is unselected, and to torch autograd of plain ReLU linear
attention when α = 0 and nothing is selected.  The log-sum-exp equals
torch's ``logsumexp`` of the dense logits when every block is selected,
log2 B plus ``logsumexp`` of the centroid logits when none is, and +inf
without keys.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def sparse_attention_lse(Q, K, block_idx, block: int, tail: str, scale: float) -> np.ndarray:
    """[B,H,N] float64: each query row's log-sum-exp of its logits in log2
    units, log2 Σ exp(s q·k + bias) over the row's key list of
    ``sparse_attention_backward`` (exact keys bias 0, pseudo-keys ln B); +inf
    for a row without keys.  "first_order" has the zero-order denominator
    (PISA's first-order term changes the numerator only), so its log-sum-exp
    is the zero-order one."""
    if tail not in ("drop", "zero_order", "first_order"):
        raise ValueError("the log-sum-exp is defined for the drop, zero_order and first_order tails")
    if tail == "first_order":
        tail = "zero_order"
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


def sparse_attention_backward(Q, K, V, block_idx, block: int, tail: str, scale: float, dO, *, alpha=None,
                              eps: float = 1e-6, o_forward=None):
    """(dQ, dK, dV) [B,H,N,d] float64 of sparse_attention(tail) at (Q, K, V)
    for the output cotangent dO [B,H,N,d]; tail "drop", "zero_order",
    "first_order" or "linear_mix" (with alpha [H,d] and the linear branch's
    eps).

    ``o_forward`` [B,H,N,d] (drop and zero_order): the output a quantised
    forward produced.  SLA2 §2C runs the forward of its low-precision sparse
    branch quantised and keeps the backward in 16 bits; read as a
    straight-through estimator, the gradients are those above at the
    unquantised operands, with δ_t = dO_t·o_t taken from the forward that
    ran (the only quantity of the backward that comes from the forward's
    output)."""
    if tail == "first_order":
        return _first_order_backward(Q, K, V, block_idx, block, scale, dO)
    if tail == "linear_mix":
        if alpha is None:
            raise ValueError("linear_mix needs alpha [H, d]")
        return _linear_mix_backward(Q, K, V, block_idx, block, scale, dO, alpha, eps)
    if tail not in ("drop", "zero_order"):
        raise ValueError(f"no backward for tail {tail!r}")
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    Of = None if o_forward is None else _f64(o_forward)
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
                o = p @ vals if Of is None else Of[b, h, rows]
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


def _first_order_backward(Q, K, V, block_idx, block: int, scale: float, dO):
    """Backward of PISA's hybrid order (the zero-order terms plus λ_t f_t)."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    Bsz, H, N, d = K.shape
    nb = N // block
    idx = np.asarray(block_idx)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for b in range(Bsz):
        for h in range(H):
            Kh, Vh = K[b, h], V[b, h]
            Kb, Vb = Kh.reshape(nb, block, d), Vh.reshape(nb, block, d)
            kbar, vbar = Kb.mean(axis=1), Vb.mean(axis=1)
            hbar = np.einsum("jnc,jne->ce", Kb - kbar[:, None], Vb) / nb      # H̄ [c, e]
            G = np.zeros((d, d))                                               # dL/dH̄
            for i in range(N // block):
                rows = slice(i * block, (i + 1) * block)
                q, g = Q[b, h, rows], dO[b, h, rows]
                sel = sorted(int(j) for j in idx[b, h, i])
                uns = [j for j in range(nb) if j not in set(sel)]
                tok = np.concatenate([np.arange(j * block, (j + 1) * block) for j in sel]) if sel else \
                    np.zeros(0, dtype=np.int64)
                ne, nu = len(tok), len(uns)
                keys = np.concatenate([Kh[tok], kbar[uns]])
                vals = np.concatenate([Vh[tok], vbar[uns]])
                if keys.shape[0] == 0:
                    continue
                bias = np.concatenate([np.zeros(ne), np.full(nu, np.log(block))])
                a = scale * q @ keys.T + bias
                p = np.exp(a - a.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                lam = p[:, ne:].sum(axis=1) / block                      # λ_t
                f = scale * q @ hbar                                     # f_t = s H̄ᵀ q_t
                o = p @ vals + lam[:, None] * f
                dp = g @ vals.T
                dp[:, ne:] += ((g * f).sum(axis=1) / block)[:, None]     # pseudo-key values v̄_j + f_t / B
                delta = (g * o).sum(axis=1, keepdims=True)
                ds = p * (dp - delta)
                dQ[b, h, rows] += scale * ds @ keys + scale * lam[:, None] * (g @ hbar.T)
                G += scale * (q * lam[:, None]).T @ g
                dkeys = scale * ds.T @ q
                dvals = p.T @ g
                dK[b, h, tok] += dkeys[:ne]
                dV[b, h, tok] += dvals[:ne]
                for r, j in enumerate(uns):
                    dK[b, h, j * block:(j + 1) * block] += dkeys[ne + r] / block
                    dV[b, h, j * block:(j + 1) * block] += dvals[ne + r] / block
            # H̄ = (1/nb) Σ_j Σ_{m∈j} (k_m − k̄_j) v_mᵀ
            dK[b, h] += ((Vb - vbar[:, None]).reshape(N, d) @ G.T) / nb
            dV[b, h] += ((Kb - kbar[:, None]).reshape(N, d) @ G) / nb
    return dQ, dK, dV


def _linear_mix_backward(Q, K, V, block_idx, block: int, scale: float, dO, alpha, eps: float):
    """Backward of SLA2's mixture α⊙O_s + (1−α)⊙O_l (ReLU linear branch over U)."""
    Q, K, V, dO, alpha = _f64(Q), _f64(K), _f64(V), _f64(dO), _f64(alpha)
    Bsz, H, N, d = K.shape
    nb = N // block
    idx = np.asarray(block_idx)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for b in range(Bsz):
        for h in range(H):
            Kh, Vh = K[b, h], V[b, h]
            al = alpha[h][None, :]
            for i in range(N // block):
                rows = slice(i * block, (i + 1) * block)
                q, g = Q[b, h, rows], dO[b, h, rows]
                sel = sorted(int(j) for j in idx[b, h, i])
                uns = [j for j in range(nb) if j not in set(sel)]
                tok = np.concatenate([np.arange(j * block, (j + 1) * block) for j in sel]) if sel else \
                    np.zeros(0, dtype=np.int64)
                utok = np.concatenate([np.arange(j * block, (j + 1) * block) for j in uns]) if uns else \
                    np.zeros(0, dtype=np.int64)
                if len(tok):
                    # O_s: softmax attention over the selected tokens, cotangent α⊙dO
                    gs = al * g
                    a = scale * q @ Kh[tok].T
                    p = np.exp(a - a.max(axis=1, keepdims=True))
                    p /= p.sum(axis=1, keepdims=True)
                    o_s = p @ Vh[tok]
                    dp = gs @ Vh[tok].T
                    ds = p * (dp - (gs * o_s).sum(axis=1, keepdims=True))
                    dQ[b, h, rows] += scale * ds @ Kh[tok]
                    dK[b, h, tok] += scale * ds.T @ q
                    dV[b, h, tok] += p.T @ gs
                if len(utok):
                    # O_l: ReLU linear attention over the unselected tokens, cotangent (1−α)⊙dO
                    gl = (1.0 - al) * g
                    phq, phk = np.maximum(q, 0.0), np.maximum(Kh[utok], 0.0)
                    h_u, z_u = phk.T @ Vh[utok], phk.sum(axis=0)
                    den = phq @ z_u + eps
                    o_l = (phq @ h_u) / den[:, None]
                    dnum = gl / den[:, None]
                    dden = -(gl * o_l).sum(axis=1) / den
                    dphq = dnum @ h_u.T + dden[:, None] * z_u[None, :]
                    dQ[b, h, rows] += (q > 0) * dphq
                    dh = phq.T @ dnum
                    dz = phq.T @ dden
                    dK[b, h, utok] += (Kh[utok] > 0) * (Vh[utok] @ dh.T + dz[None, :])
                    dV[b, h, utok] += phk @ dh
    return dQ, dK, dV
