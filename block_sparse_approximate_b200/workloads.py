"""Seeded synthetic inputs for the tests, the benchmark and the smoke check.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, and both the CUDA path and the CPU oracle consume what it
returns.  Everything is generated with ``torch.Generator`` on the requested
device (values for one seed therefore differ between a CPU and a CUDA
generator; a test always feeds one generated tensor to both sides).

Workloads (the pages' own workloads are video diffusion transformers and
long-context LLM decoding; these synthetic inputs stand in for them):

* ``tiny``      B=1, H=2, N=1024, d=64, fp32, Q,K,V ~ N(0,1); block 64;
                dot router, top-4 KV blocks per query block; zero-order tail.
* ``video_dit`` B=1, H=12, N=32768 tokens on an 8x64x64 latent grid, d=128,
                bf16; Q and K are smooth fields (sum of 8 random sinusoids per
                head and channel) plus N(0, 0.5) noise, V ~ N(0,1); block 128;
                dot router, keep 10% of KV blocks; zero-order tail.
* ``sla2_mix``  B=1, H=40, N=65536 on a 16x64x64 grid, generated as
                ``video_dit``; block 128; projected router with proj_q, proj_k
                ~ N(0, 1/d); keep 5%; linear_mix with alpha ~ U(0.2, 0.9).
* ``video_dit_pisa``  ``video_dit`` (same seed, same inputs) with PISA's
                covariance-aware router and hybrid-order (first-order) tail.
* ``fp8``       ``video_dit`` shapes, e4m3 sparse branch; zero-order tail.
* ``decode``    16 sequences, 32 query heads, 8 KV heads, d=128, bf16 cache of
                131072 tokens: K, V ~ N(0,1) plus an N(0, 0.5) offset per
                (64-token block, channel); q ~ N(0,1); block 64; taylor2 router,
                top-64 blocks; zero-order tail.
* ``sfa``       sparse feature attention ("Scaling Attention via Feature
                Sparsity"): B=1, H=12, N=16384, d=128, bf16, Q,K,V ~ N(0,1),
                seed 6; the top-16 of 128 features of every query and key
                (the page's example k = 16, d = 128); every 128-token tile of
                keys attends (non-causal).
* ``decode_rla``  ``decode`` (same seed, same caches) with SPLA's residual
                linear attention over the unselected blocks instead of the
                zero-order tail.

N(m, v) above names the variance v.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch

__all__ = ["Workload", "WORKLOADS", "prefill_inputs", "decode_inputs",
           "video_field", "keep_count"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str                 # "fp32" | "bf16"
    block: int
    route: str                 # "dot" | "proj" | "taylor2" | "cov"
    tail: str                  # "drop" | "zero_order" | "first_order" | "linear_mix"
    seed: int
    topk: Optional[int] = None
    keep_pct: Optional[int] = None
    grid: Optional[Tuple[int, int, int]] = None
    fp8: bool = False
    decode: bool = False
    Hkv: Optional[int] = None
    extra: dict = field(default_factory=dict)

    @property
    def nb(self) -> int:
        return self.N // self.block

    @property
    def k(self) -> int:
        return self.topk if self.topk is not None else keep_count(self.keep_pct, self.nb)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


def keep_count(pct: int, nb: int) -> int:
    """Blocks kept for "keep pct% of the KV blocks": ceil(pct * nb / 100)."""
    return -((-int(pct) * int(nb)) // 100)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, N=1024, d=64, dtype="fp32", block=64,
                     route="dot", tail="zero_order", seed=0, topk=4),
    "video_dit": Workload("video_dit", B=1, H=12, N=8 * 64 * 64, d=128, dtype="bf16",
                          block=128, route="dot", tail="zero_order", seed=1,
                          keep_pct=10, grid=(8, 64, 64)),
    "sla2_mix": Workload("sla2_mix", B=1, H=40, N=16 * 64 * 64, d=128, dtype="bf16",
                         block=128, route="proj", tail="linear_mix", seed=2,
                         keep_pct=5, grid=(16, 64, 64)),
    "video_dit_pisa": Workload("video_dit_pisa", B=1, H=12, N=8 * 64 * 64, d=128, dtype="bf16",
                               block=128, route="cov", tail="first_order", seed=1,
                               keep_pct=10, grid=(8, 64, 64)),
    "fp8": Workload("fp8", B=1, H=12, N=8 * 64 * 64, d=128, dtype="bf16",
                    block=128, route="dot", tail="zero_order", seed=3,
                    keep_pct=10, grid=(8, 64, 64), fp8=True),
    "decode": Workload("decode", B=16, H=32, N=131072, d=128, dtype="bf16",
                       block=64, route="taylor2", tail="zero_order", seed=4,
                       topk=64, decode=True, Hkv=8),
    "sfa": Workload("sfa", B=1, H=12, N=16384, d=128, dtype="bf16", block=128, route="dot",
                    tail="drop", seed=6, topk=128, extra={"kf": 16}),
    "decode_rla": Workload("decode_rla", B=16, H=32, N=131072, d=128, dtype="bf16",
                           block=64, route="taylor2", tail="residual_linear", seed=4,
                           topk=64, decode=True, Hkv=8),
}

_DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def video_field(B: int, H: int, grid: Tuple[int, int, int], d: int,
                gen: torch.Generator, device, n_waves: int = 8,
                noise_var: float = 0.5) -> torch.Tensor:
    """Smooth field over a (T, Y, X) latent grid plus Gaussian noise, [B,H,T*Y*X,d] fp32.

    Per (batch, head, channel): the sum of ``n_waves`` sinusoids
    sin(2π(f_t t/T + f_y y/Y + f_x x/X) + φ) of amplitude 1, the integer
    frequency triples drawn without replacement from {0,1,2}^3 minus the zero
    triple, φ ~ U(0, 2π); then noise of variance ``noise_var``.  Tokens are in
    raster order (t, y, x).
    """
    T, Y, X = grid
    dev = torch.device(device)
    freqs = torch.tensor([(a, b, c) for a in range(3) for b in range(3) for c in range(3)
                          if (a, b, c) != (0, 0, 0)], dtype=torch.float32, device=dev)
    nf = freqs.shape[0]
    t = torch.arange(T, device=dev, dtype=torch.float32) / T
    y = torch.arange(Y, device=dev, dtype=torch.float32) / Y
    x = torch.arange(X, device=dev, dtype=torch.float32) / X
    out = torch.empty(B, H, T * Y * X, d, dtype=torch.float32, device=dev)
    two_pi = 2.0 * math.pi
    for b in range(B):
        for h in range(H):
            # frequency choice and phases for the d channels of this head
            keys = torch.rand(d, nf, generator=gen, device=dev)
            pick = keys.argsort(dim=1)[:, :n_waves]                      # [d, w]
            f = freqs[pick]                                              # [d, w, 3]
            phi = torch.rand(d, n_waves, generator=gen, device=dev) * two_pi
            at = two_pi * f[..., 0, None] * t                            # [d, w, T]
            ay = two_pi * f[..., 1, None] * y                            # [d, w, Y]
            ax = two_pi * f[..., 2, None] * x                            # [d, w, X]
            ang = (at[..., :, None, None] + ay[..., None, :, None] + ax[..., None, None, :]
                   + phi[..., None, None, None])                         # [d, w, T, Y, X]
            val = torch.sin(ang).sum(dim=1).reshape(d, T * Y * X)
            out[b, h] = val.t()
    out += torch.randn(out.shape, generator=gen, device=dev) * math.sqrt(noise_var)
    return out


def prefill_inputs(w: Workload, device="cpu", *, H: Optional[int] = None,
                   N: Optional[int] = None) -> dict:
    """Q, K, V [B,H,N,d] (workload dtype) plus the router / mix parameters.

    ``H`` and ``N`` shrink the workload for tests (for a grid workload ``N``
    shrinks the time axis and must be a multiple of Y*X).
    """
    dev = torch.device(device)
    gen = _gen(w.seed, dev)
    Hh = H if H is not None else w.H
    dt = _DT[w.dtype]
    if w.grid is None:
        Nn = N if N is not None else w.N
        Q = torch.randn(w.B, Hh, Nn, w.d, generator=gen, device=dev)
        K = torch.randn(w.B, Hh, Nn, w.d, generator=gen, device=dev)
        V = torch.randn(w.B, Hh, Nn, w.d, generator=gen, device=dev)
    else:
        T, Y, X = w.grid
        if N is not None:
            if N % (Y * X):
                raise ValueError("N must be a multiple of Y*X for a grid workload")
            T = N // (Y * X)
        Q = video_field(w.B, Hh, (T, Y, X), w.d, gen, dev)
        K = video_field(w.B, Hh, (T, Y, X), w.d, gen, dev)
        V = torch.randn(Q.shape, generator=gen, device=dev)
    out = {"Q": Q.to(dt).contiguous(), "K": K.to(dt).contiguous(), "V": V.to(dt).contiguous()}
    if w.route == "proj":
        sd = 1.0 / math.sqrt(w.d)
        out["proj_q"] = (torch.randn(w.d, w.d, generator=gen, device=dev) * sd).contiguous()
        out["proj_k"] = (torch.randn(w.d, w.d, generator=gen, device=dev) * sd).contiguous()
    if w.tail == "linear_mix":
        out["alpha"] = (0.2 + 0.7 * torch.rand(Hh, w.d, generator=gen, device=dev)).contiguous()
    return out


def block_linear_inputs(B: int, H: int, nb: int, block: int, d: int, dtype, seed: int, device="cpu",
                        dev_std: float = 0.5, mix: float = 4.0, noise: float = 0.1) -> dict:
    """Q, K, V [B,H,nb*block,d] whose values follow the keys' in-block deviations.

    Every key block j has a centroid c_j ~ N(0, I) and deviations
    e_n ~ N(0, dev_std² I) shifted to zero mean over the block: k_n = c_j + e_n.
    Values are v_n = e_n M + noise·N(0, I) with one M ~ N(0, mix²/d) per head,
    so the blocks share a first-order statistic Σ_n e_n v_nᵀ of order
    block·dev_std²·M; queries are N(0, I).
    """
    dev = torch.device(device)
    gen = _gen(seed, dev)
    N = nb * block
    c = torch.randn(B, H, nb, 1, d, generator=gen, device=dev)
    e = torch.randn(B, H, nb, block, d, generator=gen, device=dev) * dev_std
    e = e - e.mean(dim=3, keepdim=True)
    K = (c + e).reshape(B, H, N, d)
    M = torch.randn(B, H, d, d, generator=gen, device=dev) * (mix / math.sqrt(d))
    V = e.reshape(B, H, N, d) @ M + noise * torch.randn(B, H, N, d, generator=gen, device=dev)
    Q = torch.randn(B, H, N, d, generator=gen, device=dev)
    return {n: x.to(dtype).contiguous() for n, x in (("Q", Q), ("K", K), ("V", V))}


def decode_inputs(w: Workload, device="cpu", *, B: Optional[int] = None,
                  N: Optional[int] = None, Hkv: Optional[int] = None,
                  offset_var: float = 0.5) -> dict:
    """q [B,Hq,d] and bf16 caches Kcache, Vcache [B,Hkv,N,d].

    K and V are N(0,1) plus, for every (64-token block, channel), an offset of
    variance ``offset_var`` added to all tokens of that block (independent
    offsets for K and V).  Generated one sequence at a time to bound memory.
    """
    dev = torch.device(device)
    gen = _gen(w.seed, dev)
    Bn = B if B is not None else w.B
    Nn = N if N is not None else w.N
    hkv = Hkv if Hkv is not None else w.Hkv
    g = w.H // w.Hkv
    Hq = hkv * g
    blk = w.block
    if Nn % blk:
        raise ValueError("cache length must be a multiple of the block size")
    dt = _DT[w.dtype]
    q = torch.randn(Bn, Hq, w.d, generator=gen, device=dev).to(dt).contiguous()
    Kc = torch.empty(Bn, hkv, Nn, w.d, dtype=dt, device=dev)
    Vc = torch.empty(Bn, hkv, Nn, w.d, dtype=dt, device=dev)
    sd = math.sqrt(offset_var)
    for b in range(Bn):
        for dst in (Kc, Vc):
            base = torch.randn(hkv, Nn // blk, blk, w.d, generator=gen, device=dev)
            off = torch.randn(hkv, Nn // blk, 1, w.d, generator=gen, device=dev) * sd
            dst[b] = (base + off).reshape(hkv, Nn, w.d).to(dt)
    return {"q": q, "Kcache": Kc, "Vcache": Vc}
