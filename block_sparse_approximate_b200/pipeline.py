"""The hot path as a sequence of C-ABI calls with preallocated buffers.

A prefill step is block_pool -> route -> sparse_attn_fwd; a decode step is
decode_fwd over precomputed cache statistics.  The buffers are allocated once
(torch device memory) and every call goes through ``binding``; nothing here
computes.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import binding as bd
from .workloads import Workload


@dataclass
class PrefillBuffers:
    stats: dict
    block_idx: torch.Tensor
    scores: Optional[torch.Tensor]
    out: torch.Tensor


def alloc_prefill(w: Workload, Q: torch.Tensor, want_scores: bool = False) -> PrefillBuffers:
    B, H, N, d = Q.shape
    nb = N // w.block
    dev = Q.device
    f = dict(device=dev, dtype=torch.float32)
    st = {"qmean": torch.empty(B, H, nb, d, **f), "kmean": torch.empty(B, H, nb, d, **f),
          "vsum": torch.empty(B, H, nb, d, **f)}
    if w.route == "taylor2":
        st["kvar"] = torch.empty(B, H, nb, d, **f)
    if w.tail == "linear_mix":
        st["zrelu"] = torch.empty(B, H, nb, d, **f)
        st["htot"] = torch.empty(B, H, d, d, **f)
        st["ztot"] = torch.empty(B, H, d, **f)
    if Q.dtype == torch.bfloat16 and w.tail in ("zero_order", "first_order"):
        st["kmean_bf16"] = torch.empty(B, H, nb, d, device=dev, dtype=torch.bfloat16)
        st["vmean_bf16"] = torch.empty(B, H, nb, d, device=dev, dtype=torch.bfloat16)
    if w.tail == "first_order" or w.route == "cov":
        st["hbar"] = torch.empty(B, H, d, d, **f)
    if w.tail == "first_order" and Q.dtype == torch.bfloat16:
        st["hbarT_bf16"] = torch.empty(B, H, d, d, device=dev, dtype=torch.bfloat16)
    if w.route == "cov":
        st["covnorm"] = torch.empty(B, H, nb, **f)
    idx = torch.empty(B, H, nb, w.k, device=dev, dtype=torch.int32)
    sc = torch.empty(B, H, nb, nb, **f) if want_scores else None
    return PrefillBuffers(st, idx, sc, torch.empty_like(Q))


class PrefillStep:
    """Callable running one prefill step of workload ``w`` on fixed buffers."""

    def __init__(self, w: Workload, inputs: dict, want_scores: bool = False):
        self.w = w
        self.inp = inputs
        Q = inputs["Q"]
        self.buf = alloc_prefill(w, Q, want_scores)
        B, H, N, d = Q.shape
        self.shape = bd.Shape(B, H, N, d, w.block)
        self.dtype = bd._dtype_code(Q)
        self.cst = bd._stats_struct(self.buf.stats)
        self.lib = bd.load()

    def __call__(self, stream=None):
        lib, w, inp, buf = self.lib, self.w, self.inp, self.buf
        s = bd._stream(stream)
        bd._check("sa_block_pool", lib.sa_block_pool(inp["Q"].data_ptr(), inp["K"].data_ptr(),
                                                     inp["V"].data_ptr(), self.dtype, self.shape,
                                                     ctypes.byref(self.cst), s))
        bd._check("sa_route", lib.sa_route(ctypes.byref(self.cst), self.shape, bd.ROUTE[w.route],
                                           bd._ptr(inp.get("proj_q")), bd._ptr(inp.get("proj_k")),
                                           float(w.scale), int(w.k), buf.block_idx.data_ptr(),
                                           bd._ptr(buf.scores), s))
        bd._check("sa_sparse_attn_fwd",
                  lib.sa_sparse_attn_fwd(inp["Q"].data_ptr(), inp["K"].data_ptr(), inp["V"].data_ptr(),
                                         self.dtype, self.shape, buf.block_idx.data_ptr(), int(w.k),
                                         bd.TAIL[w.tail], bd._ptr(inp.get("alpha")),
                                         ctypes.byref(self.cst), float(w.scale), buf.out.data_ptr(), s))
        return buf.out

    # kernels this step launches (block_pool [+ linear totals], route, attention)
    def launches(self) -> int:
        return 3 + (1 if self.w.tail == "linear_mix" else 0)


class DecodeStep:
    """Callable running one decode step (route + split attention + combine)."""

    def __init__(self, w: Workload, inputs: dict, stats: dict):
        self.w = w
        self.inp = inputs
        self.stats = stats
        q, Kc = inputs["q"], inputs["Kcache"]
        B, Hq, d = q.shape
        Hkv, N = Kc.shape[1], Kc.shape[2]
        self.shape = bd.DecodeShape(B, Hq, Hkv, N, d, w.block)
        self.lib = bd.load()
        ws = int(self.lib.sa_decode_workspace_size(self.shape, int(w.k)))
        self.ws = torch.empty(max(ws, 256), device=q.device, dtype=torch.uint8)
        self.out = torch.empty_like(q)
        self.idx = torch.empty(B, Hkv, w.k, device=q.device, dtype=torch.int32)
        self.scores = torch.empty(B, Hkv, N // w.block, device=q.device, dtype=torch.float32)
        self.cst = bd._stats_struct(stats)

    def __call__(self, stream=None):
        inp = self.inp
        bd._check("sa_decode_fwd",
                  self.lib.sa_decode_fwd(inp["q"].data_ptr(), inp["Kcache"].data_ptr(),
                                         inp["Vcache"].data_ptr(), bd.SA_BF16, self.shape,
                                         ctypes.byref(self.cst), int(self.w.k), float(self.w.scale),
                                         bd.TAIL[self.w.tail], self.idx.data_ptr(),
                                         self.scores.data_ptr(), self.out.data_ptr(),
                                         self.ws.data_ptr(), self.ws.numel(), bd._stream(stream)))
        return self.out

    def launches(self) -> int:
        return 4


class Fp8PrefillStep:
    """One step of the e4m3 sparse branch: block statistics (bf16 inputs) ->
    router -> per-block e4m3 quantisation of Q, K, V and of the centroid tiles
    -> e4m3 sparse attention."""

    def __init__(self, w: Workload, inputs: dict):
        self.w = w
        self.inp = inputs
        Q = inputs["Q"]
        self.buf = alloc_prefill(w, Q)
        B, H, N, d = Q.shape
        self.shape = (B, H, N, d, w.block)
        self.ops = None

    def __call__(self, stream=None):
        w, inp, buf = self.w, self.inp, self.buf
        bd._check("sa_block_pool", bd.load().sa_block_pool(
            inp["Q"].data_ptr(), inp["K"].data_ptr(), inp["V"].data_ptr(), bd.SA_BF16, bd.Shape(*self.shape),
            ctypes.byref(bd._stats_struct(buf.stats)), bd._stream(stream)))
        bd._check("sa_route", bd.load().sa_route(
            ctypes.byref(bd._stats_struct(buf.stats)), bd.Shape(*self.shape), bd.ROUTE[w.route], None, None,
            float(w.scale), int(w.k), buf.block_idx.data_ptr(), None, bd._stream(stream)))
        self.ops = bd.fp8_operands(inp["Q"], inp["K"], inp["V"], buf.stats, stream=stream)
        return bd.sparse_attn_fwd_fp8(self.ops, self.shape, buf.block_idx, w.tail, w.scale, out=buf.out,
                                      stream=stream)

    def launches(self) -> int:
        return 2 + 5 + 1
