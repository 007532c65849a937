"""Plain float64 CPU oracle of the block-sparse attention hot path.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use this module.  It shares no code with the
CUDA library.

Notation (PISA, "Algoritmo Central"): a query block i owns the rows t of
block i; its KV blocks are split into the selected set S_i (computed exactly)
and the unselected set U_i (approximated or dropped).  ``B`` in the formulas is
the block size (tokens per block), ``s`` the softmax scale.

Readings taken where the pages leave a step open (each is restated in the
design notes of the repository):

* the softmax scale multiplies every logit, including the centroid logit of
  PISA's zero-order term:  alpha_{t,j} = exp(s * q_t . kbar_j);
* the denominator's zero-order term for an unselected block is
  B * exp(s * q_t . kbar_j)  (the zero-order Taylor term of sum_n e^{s q k_n};
  the first-order term of the denominator vanishes because the keys' deviations
  from their centroid sum to zero);
* "Cov(k)" of the SPLA score is the per-channel population variance (divide
  by B) of the block's keys, and the score is compared in log form
  s q.kbar + log1p(0.5 s^2 sum_c q_c^2 var_c), which orders blocks the same way;
* top-k keeps the k largest scores, a tie goes to the smaller block index, and
  the kept indices are returned in ascending order;
* the SLA2 linear branch uses the ReLU feature map (SALAD), runs over the
  unselected blocks only, and adds eps = 1e-6 to its denominator;
* PISA's covariance-aware routing: M_j = ‖H_j − H̄‖₂ is the spectral norm,
  and the score adds the first-order error bound to the zero-order mass of the
  block, s q̄.k̄_j + log1p(s ‖q̄_i‖ M_j / B) (the page says the score
  "incorporates" both without a formula; this is the plainest combination the
  error argument gives);
* SPLA's residual linear attention (decode tail "residual_linear"): the
  feature map is φ(x) = exp(x) on the unscaled q and k, o_rla = ō − õ is the
  difference of the UNNORMALISED linear attentions over all blocks and over
  the selected ones (φ(q)ᵀ Σ_{n∈U} φ(k_n) v_nᵀ, the state that "accumulates
  only the unselected blocks"), and the gated sum is o = o_sparse +
  RMSNorm(o_rla) with unit gain (the RMS norm's scale is the only parameter
  the page names; no trained value exists here) and eps = 1e-6; o_sparse is
  the drop output;
* GQA decode shares one selection per (batch, KV head); the group's score for
  a block is the log of the sum over the group's query heads of each head's
  SPLA block mass (a logsumexp of the log-form scores).

Pins (the tests under ``tests/test_oracle_*.py``):
  block_pool          closed forms on ramps / constant blocks; brute force
  route_scores        brute-force loops; taylor2 == dot order when var == 0
  topk_from_scores    brute-force sort on tiny inputs, hand-made ties
  first_order tail    H̄ = 0 (block-constant keys) -> zero_order; identical
                      per-block deviations -> PISA's per-block first-order
                      Taylor sum by brute force; error O(ε²) vs zero_order's
                      O(ε) as the in-block deviations shrink
  residual_linear     all blocks selected -> drop (= dense); brute-force
                      token loops; the subtraction form φ(q)ᵀ(S_all − S_sel)
                      equals the direct sum; RMS-norm scale invariance
  covnorm / "cov"     rank-one deviations H_j − H̄ = (γ_j − γ̄) u wᵀ -> closed
                      form |γ_j − γ̄|·|u|·|w|; identical blocks -> M_j = 0 and
                      "cov" = s·"dot"; the square root of the largest
                      eigenvalue of AᵀA (a symmetric eigen-solver, not the
                      SVD); brute-force score loops
  sparse_attention    k = nb -> dense softmax attention (torch SDPA, fp64);
                      block size 1 / block-constant keys -> dense; V+c -> O+c;
                      hand-derived worked example (tests/golden); brute force
  decode_attention    k = nb -> dense single-query attention; equals the
                      prefill oracle on one row with the same selection
  e4m3_round          every one of the 256 e4m3 codes and random values
                      against torch.float8_e4m3fn
  quantise_blocks_e4m3  bounds of the format (|error| <= half an ulp)
  fp8_attention       on inputs already e4m3-exact per block the quantised
                      forward equals sparse_attention (drop tail; zero-order
                      tail with e4m3-exact block means over three centroid
                      groups); a hand-quantised two-group worked example of
                      the centroid path (bf16 then e4m3 ties, one scale per
                      128 blocks, value means vsum/B)
"""

from __future__ import annotations

from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

EPS_LINEAR = 1e-6
E4M3_MAX = 448.0


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Block statistics
# ---------------------------------------------------------------------------

def block_pool(Q, K, V, block: int, *, variance: bool = False,
               linear: bool = False, first_order: bool = False,
               covariance: bool = False) -> dict:
    """Per-block statistics of Q, K and V, all float64.

    Follows PISA "Implementação de Hardware", step "Pré-computação"
    (centroids kbar_j and value sums), SLA2 §2B (mean pooling of adjacent
    token blocks for the router) and SPLA §2.1 (block mean and diagonal block
    covariance of the keys).

    Q, K, V: arrays [B, H, N, d]; Q may be None.  N must be a multiple of
    ``block``.  Returns a dict with
      qmean [B,H,nqb,d]  mean of the queries of each block (if Q is given)
      kmean [B,H,nb,d]   mean of the keys of each block (kbar_j)
      vsum  [B,H,nb,d]   sum of the values of each block
      kvar  [B,H,nb,d]   per-channel population variance of the keys
                         (only with ``variance``)
      zrelu [B,H,nb,d]   sum over the block of relu(k)   (only with ``linear``)
      ztot  [B,H,d]      sum over all tokens of relu(k)  (only with ``linear``)
      htot  [B,H,d,d]    sum over all tokens of relu(k_n) v_n^T
                         (only with ``linear``)
      hbar  [B,H,d,d]    PISA's global first-order statistic H̄: the mean over
                         the head's blocks of H_j = Σ_{n∈j} (k_n − k̄_j) v_nᵀ
                         (only with ``first_order`` or ``covariance``)
      covnorm [B,H,nb]   M_j = ‖H_j − H̄‖₂, the spectral norm (largest singular
                         value) of each block's first-order deviation from the
                         mean, PISA "Roteamento Consciente de Covariância"
                         (only with ``covariance``)
    """
    K = _f64(K)
    V = _f64(V)
    Bsz, H, N, d = K.shape
    if N % block:
        raise ValueError("N must be a multiple of the block size")
    nb = N // block
    Kb = K.reshape(Bsz, H, nb, block, d)
    Vb = V.reshape(Bsz, H, nb, block, d)
    out = {}
    if Q is not None:
        Q = _f64(Q)
        if Q.shape[2] % block:
            raise ValueError("query length must be a multiple of the block size")
        out["qmean"] = Q.reshape(Bsz, H, Q.shape[2] // block, block, d).mean(axis=3)
    kmean = Kb.mean(axis=3)
    out["kmean"] = kmean
    out["vsum"] = Vb.sum(axis=3)
    if variance:
        dev = Kb - kmean[:, :, :, None, :]
        out["kvar"] = (dev * dev).mean(axis=3)
    if linear:
        R = np.maximum(Kb, 0.0)
        out["zrelu"] = R.sum(axis=3)
        out["ztot"] = out["zrelu"].sum(axis=2)
        Rt = np.maximum(K, 0.0)
        out["htot"] = np.einsum("bhnc,bhne->bhce", Rt, V)
    if first_order or covariance:
        # H_j = Σ_n (k_n − k̄_j) v_nᵀ for every block, then their mean
        dev = Kb - kmean[:, :, :, None, :]
        Hj = np.einsum("bhjnc,bhjne->bhjce", dev, Vb)
        out["hbar"] = Hj.mean(axis=2)
        if covariance:
            # largest singular value of each d×d deviation matrix (LAPACK SVD)
            out["covnorm"] = np.linalg.norm(Hj - out["hbar"][:, :, None], ord=2, axis=(-2, -1))
    return out


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------

def route_scores(qmean, kmean, mode: str, *, proj_q=None, proj_k=None,
                 kvar=None, scale: Optional[float] = None, covnorm=None,
                 block: Optional[int] = None) -> np.ndarray:
    """Block scores [B,H,nqb,nb] of the router.

    mode "dot":     q̄_i . k̄_j on mean-pooled blocks (SLA2 §2B, pooling of
                    adjacent blocks; the original SLA router's static top-k).
    mode "proj":    (q̄_i P_q) . (k̄_j P_k), the inference form of SLA2's
                    learnable router (SLA2 §2B, projections proj_q, proj_k).
    mode "taylor2": SPLA §2.1 score exp(q.k̄)(1 + ½ qᵀ diag(Var k) q) with the
                    scale folded into q (q' = s q̄_i), in log form
                    s q̄.k̄ + log1p(½ s² Σ_c q̄_c² var_c).
    mode "cov":     PISA's covariance-aware score (§2 "Roteamento Consciente
                    de Covariância"): the block's zero-order mass B e^{s q̄.k̄_j}
                    plus the bound e^{s q̄.k̄_j} s‖q̄‖ M_j on the norm of the
                    first-order term the hybrid order leaves out for it
                    (‖α s qᵀ(H_j − H̄)‖ ≤ α s ‖q‖ M_j), in log form without
                    the constant log B:
                    s q̄.k̄_j + log1p(s ‖q̄_i‖ M_j / B).
                    Needs covnorm (M_j), block (B) and scale.
    """
    qm = _f64(qmean)
    km = _f64(kmean)
    if mode == "dot":
        return np.einsum("bhic,bhjc->bhij", qm, km)
    if mode == "proj":
        pq = qm @ _f64(proj_q)
        pk = km @ _f64(proj_k)
        return np.einsum("bhic,bhjc->bhij", pq, pk)
    if mode == "taylor2":
        if kvar is None or scale is None:
            raise ValueError("taylor2 needs kvar and scale")
        s = float(scale)
        lin = s * np.einsum("bhic,bhjc->bhij", qm, km)
        quad = 0.5 * s * s * np.einsum("bhic,bhjc->bhij", qm * qm, _f64(kvar))
        return lin + np.log1p(quad)
    if mode == "cov":
        if covnorm is None or scale is None or block is None:
            raise ValueError("cov needs covnorm, scale and block")
        s = float(scale)
        lin = s * np.einsum("bhic,bhjc->bhij", qm, km)
        qn = np.sqrt((qm * qm).sum(axis=-1))                       # [B,H,nqb]
        bound = s * qn[..., :, None] * _f64(covnorm)[..., None, :] / float(block)
        return lin + np.log1p(bound)
    raise ValueError(f"unknown route mode {mode!r}")


def decode_route_scores(q, kmean, kvar, scale: float) -> np.ndarray:
    """Group-shared SPLA scores for GQA decode, [B, Hkv, nb].

    q [B,Hq,d]; kmean, kvar [B,Hkv,nb,d].  Query head h reads KV head
    h // (Hq/Hkv).  Each head's log score is SPLA §2.1's
    s q.k̄_j + log1p(½ s² Σ_c q_c² var_jc); the group's score is the log of the
    sum over its heads of exp(that), computed as a logsumexp.
    """
    q = _f64(q)
    km = _f64(kmean)
    kv = _f64(kvar)
    Bsz, Hq, d = q.shape
    Hkv = km.shape[1]
    g = Hq // Hkv
    s = float(scale)
    qg = q.reshape(Bsz, Hkv, g, d)
    lin = s * np.einsum("bkgc,bkjc->bkgj", qg, km)
    quad = 0.5 * s * s * np.einsum("bkgc,bkjc->bkgj", qg * qg, kv)
    per_head = lin + np.log1p(quad)            # [B, Hkv, g, nb]
    mx = per_head.max(axis=2, keepdims=True)
    return (mx + np.log(np.exp(per_head - mx).sum(axis=2, keepdims=True)))[:, :, 0, :]


def k_from_percent(pct: int, nb: int) -> int:
    """Number of kept blocks for "keep pct% of the KV blocks": ceil(pct*nb/100)."""
    return -((-int(pct) * int(nb)) // 100)


def topk_from_scores(scores, k: int) -> np.ndarray:
    """Indices of the k largest scores along the last axis, ascending.

    A tie is broken in favour of the smaller block index.  The selected set
    S_i of PISA "Algoritmo Central" (critical blocks) / SLA2 §2B top-k.
    """
    sc = np.asarray(scores)
    nb = sc.shape[-1]
    if not 0 <= k <= nb:
        raise ValueError("k out of range")
    flat = sc.reshape(-1, nb)
    out = np.empty((flat.shape[0], k), dtype=np.int64)
    for r in range(flat.shape[0]):
        order = sorted(range(nb), key=lambda j: (-float(flat[r, j]), j))
        out[r] = sorted(order[:k])
    return out.reshape(sc.shape[:-1] + (k,))


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _block_tokens(blocks: Sequence[int], block: int) -> np.ndarray:
    if len(blocks) == 0:
        return np.zeros(0, dtype=np.int64)
    b = np.asarray(blocks, dtype=np.int64)
    return (b[:, None] * block + np.arange(block)[None, :]).reshape(-1)


def _attend_rows(q, K, V, sel: Sequence[int], nb: int, block: int, tail: str,
                 scale: float, alpha_h=None, eps: float = EPS_LINEAR,
                 centroids=None, hbar=None) -> np.ndarray:
    """Output rows o_t for query rows q [R, d] against one head's K, V [N, d].

    PISA "Algoritmo Central":  o_t = N_t / D_t with
      N_t = Σ_{j∈S} Σ_n e^{s q_t.k_{j,n}} v_{j,n} + Σ_{j∈U} e^{s q_t.k̄_j} Σ_n v_{j,n}
      D_t = Σ_{j∈S} Σ_n e^{s q_t.k_{j,n}}         + Σ_{j∈U} B e^{s q_t.k̄_j}
    (zero_order).  "first_order" is PISA's hybrid order: the zero_order terms
    plus the global first-order correction of the numerator,
      N_t += (s q_t) H̄ Σ_{j∈U} e^{s q_t.k̄_j},
    with H̄ the mean over all blocks of H_j = Σ_{n∈j} (k_n − k̄_j) v_nᵀ (the
    first-order term of the denominator is zero: the deviations sum to zero).
    "drop" keeps only the S terms (the keep-or-drop baseline PISA and SPLA
    contrast with).  "linear_mix" is SLA2 §2A O = α⊙O_s + (1−α)⊙O_l with O_s
    the drop output and O_l the ReLU linear attention (SALAD §2) over U:
      O_l = φ(q)ᵀ Σ_{n∈U} φ(k_n) v_nᵀ / (φ(q)·Σ_{n∈U} φ(k_n) + eps).
    "residual_linear" is SPLA's sparse plus residual linear attention
    (§2.2-2.3): o = O_s + RMSNorm(o_rla) with o_rla = φ(q)ᵀ Σ_{n∈U} φ(k_n) v_nᵀ,
    φ = exp elementwise, RMSNorm(x) = x / sqrt(mean(x²) + eps) (unit gain).
    """
    sel = sorted(int(j) for j in sel)
    uns = [j for j in range(nb) if j not in set(sel)]
    tok = _block_tokens(sel, block)
    Ks, Vs = K[tok], V[tok]
    R, d = q.shape
    a = scale * (q @ Ks.T)                      # exact logits [R, |S|B]
    if tail in ("zero_order", "first_order"):
        if centroids is None:
            kbar = K.reshape(nb, block, d).mean(axis=1)[uns]      # [|U|, d]
            vsum = V.reshape(nb, block, d).sum(axis=1)[uns]       # [|U|, d]
        else:   # given block centroids k̄_j and value means v̄_j = vsum_j / B
            kbar = centroids[0][uns]
            vsum = block * centroids[1][uns]
        c = scale * (q @ kbar.T)                               # [R, |U|]
        m = np.full(R, -np.inf)
        if a.shape[1]:
            m = np.maximum(m, a.max(axis=1))
        if c.shape[1]:
            m = np.maximum(m, c.max(axis=1))
        wa = np.exp(a - m[:, None])
        wc = np.exp(c - m[:, None])
        num = wa @ Vs + wc @ vsum
        den = wa.sum(axis=1) + block * wc.sum(axis=1)
        if tail == "first_order":
            if hbar is None:
                Kb = K.reshape(nb, block, d)
                dev = Kb - Kb.mean(axis=1, keepdims=True)
                hbar = np.einsum("jnc,jne->ce", dev, V.reshape(nb, block, d)) / nb
            num = num + ((scale * q) @ _f64(hbar)) * wc.sum(axis=1)[:, None]
        return num / den[:, None]
    if tail in ("drop", "linear_mix", "residual_linear"):
        if a.shape[1]:
            m = a.max(axis=1)
            wa = np.exp(a - m[:, None])
            o_s = (wa @ Vs) / wa.sum(axis=1)[:, None]
        else:
            o_s = np.zeros((R, d))
        if tail == "drop":
            return o_s
        if tail == "residual_linear":
            # SPLA §2.2-2.3: the residual linear attention over the unselected
            # tokens with the exponential feature map, φ(q)ᵀ Σ_{n∈U} φ(k_n) v_nᵀ
            # (unnormalised: the RMS norm scales it), added to the exact part
            # after an RMS norm of unit gain
            tokU = _block_tokens(uns, block)
            o_l = (np.exp(q) @ np.exp(K[tokU]).T) @ V[tokU]
            rms = np.sqrt((o_l * o_l).mean(axis=1) + eps)
            return o_s + o_l / rms[:, None]
        utok = _block_tokens(uns, block)
        phi_k = np.maximum(K[utok], 0.0)
        phi_q = np.maximum(q, 0.0)
        h_u = phi_k.T @ V[utok]                  # Σ_{n∈U} φ(k_n) v_nᵀ   [d, d]
        z_u = phi_k.sum(axis=0)                  # Σ_{n∈U} φ(k_n)        [d]
        o_l = (phi_q @ h_u) / (phi_q @ z_u + eps)[:, None]
        al = _f64(alpha_h)[None, :]
        return al * o_s + (1.0 - al) * o_l
    raise ValueError(f"unknown tail mode {tail!r}")


def sparse_attention(Q, K, V, block_idx, block: int, tail: str, scale: float,
                     *, alpha=None, eps: float = EPS_LINEAR,
                     qblocks: Optional[Iterable[Tuple[int, int, int]]] = None):
    """Prefill output of the method, float64.

    Q, K, V [B,H,N,d]; block_idx [B,H,nqb,k] (the selected KV blocks S_i of
    every query block i, as integers); alpha [H,d] for ``linear_mix``.
    The query block size equals the KV block size.

    Without ``qblocks`` returns O [B,H,N,d].  With ``qblocks`` (an iterable of
    (b, h, i)) returns an array [len, block, d] holding only those query blocks,
    in the same order, for sampled checks at large sizes.
    """
    Q = np.asarray(Q)
    K = np.asarray(K)
    V = np.asarray(V)
    Bsz, H, N, d = K.shape
    nb = N // block
    idx = np.asarray(block_idx)
    if alpha is not None:
        alpha = _f64(alpha)
    if tail == "linear_mix" and alpha is None:
        raise ValueError("linear_mix needs alpha [H, d]")

    def hbar_of(Kh, Vh):
        if tail != "first_order":
            return None
        Kb = Kh.reshape(nb, block, d)
        dev = Kb - Kb.mean(axis=1, keepdims=True)
        return np.einsum("jnc,jne->ce", dev, Vh.reshape(nb, block, d)) / nb

    if qblocks is not None:
        qb = list(qblocks)
        out = np.empty((len(qb), block, d))
        cache = {}
        for r, (b, h, i) in enumerate(qb):
            key = (b, h)
            if key not in cache:
                Kh, Vh = _f64(K[b, h]), _f64(V[b, h])
                cache = {key: (Kh, Vh, hbar_of(Kh, Vh))}
            Kh, Vh, Hb = cache[key]
            q = _f64(Q[b, h, i * block:(i + 1) * block])
            out[r] = _attend_rows(q, Kh, Vh, idx[b, h, i], nb, block, tail, scale,
                                  None if alpha is None else alpha[h], eps, hbar=Hb)
        return out

    O = np.empty((Bsz, H, Q.shape[2], d))
    for b in range(Bsz):
        for h in range(H):
            Kh, Vh = _f64(K[b, h]), _f64(V[b, h])
            Hb = hbar_of(Kh, Vh)
            for i in range(Q.shape[2] // block):
                q = _f64(Q[b, h, i * block:(i + 1) * block])
                O[b, h, i * block:(i + 1) * block] = _attend_rows(
                    q, Kh, Vh, idx[b, h, i], nb, block, tail, scale,
                    None if alpha is None else alpha[h], eps, hbar=Hb)
    return O


def decode_attention(q, Kcache, Vcache, block: int, topk: int, scale: float, *,
                     tail: str = "zero_order", block_idx=None,
                     pairs: Optional[Iterable[Tuple[int, int]]] = None):
    """GQA decode of one query token per sequence, float64.

    q [B,Hq,d]; Kcache, Vcache [B,Hkv,N,d].  For every (batch, KV head) the
    block statistics of SPLA §2.1 (mean, diagonal variance) and PISA's value
    sums are computed from the cache, the group-shared taylor2 route picks
    ``topk`` blocks (unless ``block_idx`` [B,Hkv,topk] is given), and each of
    the group's query heads attends exactly to the selected blocks plus
    PISA's zero-order term for the rest (or drops them, or adds SPLA's
    residual linear attention over them: tail "residual_linear").

    Returns (o [B,Hq,d], block_idx [B,Hkv,topk], scores [B,Hkv,nb]).  With
    ``pairs`` (an iterable of (b, kv_head)) only those pairs are computed; the
    other entries are NaN / -1.
    """
    q = _f64(q)
    Bsz, Hq, d = q.shape
    Hkv, N = Kcache.shape[1], Kcache.shape[2]
    g = Hq // Hkv
    nb = N // block
    todo = list(pairs) if pairs is not None else [(b, k) for b in range(Bsz) for k in range(Hkv)]
    o = np.full((Bsz, Hq, d), np.nan)
    idx_out = np.full((Bsz, Hkv, topk), -1, dtype=np.int64)
    sc_out = np.full((Bsz, Hkv, nb), np.nan)
    for b, kh in todo:
        Kh = _f64(Kcache[b, kh])
        Vh = _f64(Vcache[b, kh])
        st = block_pool(None, Kh[None, None], Vh[None, None], block, variance=True)
        qg = q[b, kh * g:(kh + 1) * g]
        sc = decode_route_scores(qg[None], st["kmean"][0][None], st["kvar"][0][None], scale)[0, 0]
        sc_out[b, kh] = sc
        if block_idx is None:
            sel = topk_from_scores(sc, topk)
        else:
            sel = np.sort(np.asarray(block_idx[b, kh], dtype=np.int64))
        idx_out[b, kh] = sel
        o[b, kh * g:(kh + 1) * g] = _attend_rows(qg, Kh, Vh, sel, nb, block, tail, scale)
    return o, idx_out, sc_out


# ---------------------------------------------------------------------------
# FP8 e4m3 (SLA2 §2C: low-precision sparse branch)
# ---------------------------------------------------------------------------

def e4m3_round(x) -> np.ndarray:
    """Round to the nearest value of the e4m3fn format, ties to even, saturating.

    e4m3fn: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; normal
    values (1 + m/8) 2^(e-7) for e in 1..15 except the all-ones pattern
    S.1111.111 (NaN); subnormals m/8 * 2^-6; largest finite 448; no infinity.
    Out-of-range magnitudes saturate to ±448 (the "satfinite" convention).
    """
    x = _f64(x)
    out = np.empty_like(x)
    ax = np.abs(x)
    nan = np.isnan(x)
    with np.errstate(divide="ignore", invalid="ignore"):
        mant, ex = np.frexp(ax)            # ax = mant * 2^ex, mant in [0.5, 1)
        e = ex - 1                         # ax in [2^e, 2^(e+1))
        e = np.maximum(e, -6)              # below 2^-6 the spacing is 2^-9 (subnormal)
        ulp = np.ldexp(1.0, e - 3)
        q = np.rint(ax / ulp) * ulp        # np.rint rounds half to even
    q = np.minimum(q, E4M3_MAX)
    out[:] = np.copysign(q, x)
    out[ax == 0] = x[ax == 0]
    out[nan] = np.nan
    return out


def quantise_blocks_e4m3(X, block: int = 128):
    """Per-(batch, head, token block) absmax-scaled e4m3 quantisation.

    SLA2 §2C quantises the sparse branch to 8 bits; the scale layout is a
    reading: one float32 scale per block of ``block`` tokens (a ragged last
    block has its own scale), σ = absmax / 448 (σ = 1 for an all-zero block),
    codes = e4m3(x / σ) with the division done in float32.  Returns (dequantised float64 X̂, codes as float64,
    σ [B,H,N/block] float32).
    """
    X32 = np.asarray(X, dtype=np.float32)
    Bsz, H, N, d = X32.shape
    nb = -(-N // block)
    if nb * block != N:   # a ragged last block: zero rows do not change its absmax
        X32 = np.concatenate([X32, np.zeros((Bsz, H, nb * block - N, d), np.float32)], axis=2)
    Xb = X32.reshape(Bsz, H, nb, block, d)
    amax = np.abs(Xb).max(axis=(3, 4))
    sigma = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    scaled = (Xb / sigma[:, :, :, None, None]).astype(np.float32)
    codes = e4m3_round(scaled)
    deq = codes * sigma[:, :, :, None, None].astype(np.float64)
    return (deq.reshape(Bsz, H, nb * block, d)[:, :, :N], codes.reshape(Bsz, H, nb * block, d)[:, :, :N],
            sigma)


def _bf16(x) -> np.ndarray:
    """Round to bfloat16 (nearest, ties to even) and back to float64."""
    import torch
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def fp8_attention(Q, K, V, block_idx, block: int, tail: str, scale: float, *,
                  qblocks: Optional[Iterable[Tuple[int, int, int]]] = None,
                  absolute_values: bool = False):
    """The e4m3 quantised forward of the sparse branch, float64 (P unquantised).

    SLA2 §2C runs the sparse branch in 8 bits; reading: Q, K, V are replaced by
    their per-(batch, head, block) e4m3 values (``quantise_blocks_e4m3``), and
    the zero-order tail uses the block centroids k̄_j and value means vsum_j/B
    of the unquantised inputs, stored in bfloat16 and quantised to e4m3 with one
    scale per group of 128 blocks.  The attention itself is PISA's N_t / D_t in
    float64.  Same return convention as ``sparse_attention``.

    With ``absolute_values`` the values (and value means) are replaced by their
    absolute values, which gives Σ_n p_n |v_n| / l per output element: the
    scale of the error that rounding each p_n to e4m3 can cause.
    """
    Qd = quantise_blocks_e4m3(Q, block)[0]
    Kd = quantise_blocks_e4m3(K, block)[0]
    Vd = quantise_blocks_e4m3(V, block)[0]
    if absolute_values:
        Vd = np.abs(Vd)
    Bsz, H, N, d = np.asarray(K).shape
    nb = N // block
    idx = np.asarray(block_idx)
    cent = None
    if tail == "zero_order":
        K64, V64 = _f64(K), _f64(V)
        kb = _bf16(K64.reshape(Bsz, H, nb, block, d).mean(axis=3))
        vb = _bf16(V64.reshape(Bsz, H, nb, block, d).sum(axis=3) / block)
        cent = (quantise_blocks_e4m3(kb, 128)[0], quantise_blocks_e4m3(vb, 128)[0])
        if absolute_values:
            cent = (cent[0], np.abs(cent[1]))
    todo = list(qblocks) if qblocks is not None else [
        (b, h, i) for b in range(Bsz) for h in range(H) for i in range(N // block)]
    out = np.empty((len(todo), block, d))
    for r, (b, h, i) in enumerate(todo):
        c = None if cent is None else (cent[0][b, h], cent[1][b, h])
        out[r] = _attend_rows(Qd[b, h, i * block:(i + 1) * block], Kd[b, h], Vd[b, h], idx[b, h, i], nb,
                              block, tail, scale, centroids=c)
    if qblocks is not None:
        return out
    return out.reshape(Bsz, H, N // block, block, d).reshape(Bsz, H, N, d)


def dense_equivalent_flops(Bsz: int, H: int, N: int, d: int) -> float:
    """4·B·H·N²·d: the FLOPs of dense attention of the same shape."""
    return 4.0 * Bsz * H * float(N) * N * d


__all__ = [
    "block_pool", "route_scores", "decode_route_scores", "k_from_percent",
    "topk_from_scores", "sparse_attention", "decode_attention", "e4m3_round",
    "quantise_blocks_e4m3", "fp8_attention", "dense_equivalent_flops", "EPS_LINEAR", "E4M3_MAX",
]

