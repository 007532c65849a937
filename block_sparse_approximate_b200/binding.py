"""ctypes binding of libsparseattn (argument marshalling only).

Every function here validates tensor placement, allocates the outputs with
torch on the inputs' device, passes raw device pointers and the current CUDA
stream to the C entry point of the same name, and raises ``SparseAttnError``
on a non-OK status.  All computation happens in the library's CUDA kernels;
there is no fallback: if ``libsparseattn.so`` has not been built, ``load()``
raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparseattn.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_ALIGNMENT, SA_ERR_CUDA, SA_ERR_WORKSPACE = range(6)
SA_FP32, SA_BF16 = 0, 1
ROUTE = {"dot": 0, "proj": 1, "taylor2": 2, "cov": 3}
TAIL = {"drop": 0, "zero_order": 1, "linear_mix": 2, "first_order": 3, "residual_linear": 4}

# every entry point declared in include/sparseattn.h
EXPORTS = ("sa_block_pool", "sa_route", "sa_sparse_attn_fwd", "sa_decode_workspace_size",
           "sa_decode_fwd", "sa_decode_fwd_static", "sa_quantize_e4m3", "sa_sparse_attn_fwd_fp8",
           "sa_sfa_encode", "sa_sfa_densify", "sa_sfa_workspace_size", "sa_sfa_attn_fwd",
           "sa_sparse_attn_bwd_workspace_size", "sa_sparse_attn_bwd", "sa_sparse_attn_fwd_lse",
           "sa_sparse_attn_bwd_lse", "sa_sparse_attn_bwd_linear_mix_workspace_size", "sa_sparse_attn_bwd_linear_mix",
           "sa_device_error", "sa_last_error", "sa_version")


class SparseAttnError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("block", ctypes.c_int32)]


class DecodeShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("block", ctypes.c_int32)]


_STAT_FIELDS = ("qmean", "kmean", "vsum", "kvar", "zrelu", "htot", "ztot", "kmean_bf16", "vmean_bf16",
                "hbar", "hbarT_bf16", "covnorm", "sexp", "kvar_bf16")


class BlockStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _STAT_FIELDS]


_FP8_FIELDS = ("q", "k", "v", "q_scale", "k_scale", "v_scale", "v_scale_max", "kbar", "vbar",
               "kbar_scale", "vbar_scale")


class Fp8Operands(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _FP8_FIELDS]


_lib = None


def load():
    """Loads libsparseattn.so (built in-tree) and declares its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m block_sparse_approximate_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    lib.sa_block_pool.argtypes = [vp, vp, vp, ctypes.c_int, Shape, ctypes.POINTER(BlockStats), vp]
    lib.sa_route.argtypes = [ctypes.POINTER(BlockStats), Shape, ctypes.c_int, vp, vp, f32, i32, vp, vp, vp]
    lib.sa_sparse_attn_fwd.argtypes = [vp, vp, vp, ctypes.c_int, Shape, vp, i32, ctypes.c_int, vp,
                                       ctypes.POINTER(BlockStats), f32, vp, vp]
    lib.sa_decode_workspace_size.argtypes = [DecodeShape, i32]
    lib.sa_decode_workspace_size.restype = sz
    lib.sa_decode_fwd.argtypes = [vp, vp, vp, ctypes.c_int, DecodeShape, ctypes.POINTER(BlockStats),
                                  i32, f32, ctypes.c_int, vp, vp, vp, vp, sz, vp]
    lib.sa_decode_fwd_static.argtypes = [vp, vp, vp, ctypes.c_int, DecodeShape, ctypes.POINTER(BlockStats),
                                         i32, f32, ctypes.c_int, vp, vp, vp, vp]
    lib.sa_quantize_e4m3.argtypes = [vp, ctypes.c_int64, i32, i32, i32, vp, vp, vp, vp]
    lib.sa_sparse_attn_fwd_fp8.argtypes = [ctypes.POINTER(Fp8Operands), Shape, vp, i32, ctypes.c_int, f32, vp, vp]
    i64 = ctypes.c_int64
    lib.sa_sfa_encode.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp]
    lib.sa_sfa_densify.argtypes = [vp, vp, i64, i32, i32, vp, vp]
    lib.sa_sfa_workspace_size.argtypes = [Shape]
    lib.sa_sfa_workspace_size.restype = sz
    lib.sa_sfa_attn_fwd.argtypes = [vp, vp, vp, ctypes.c_int, Shape, f32, vp, vp, sz, vp]
    lib.sa_sparse_attn_bwd_workspace_size.argtypes = [Shape, i32]
    lib.sa_sparse_attn_bwd_workspace_size.restype = sz
    lib.sa_sparse_attn_bwd.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, Shape, vp, i32, ctypes.c_int,
                                       ctypes.POINTER(BlockStats), f32, vp, vp, vp, vp, sz, vp]
    lib.sa_sparse_attn_fwd_lse.argtypes = [vp, vp, vp, ctypes.c_int, Shape, vp, i32, ctypes.c_int,
                                           ctypes.POINTER(BlockStats), f32, vp, vp, vp]
    lib.sa_sparse_attn_bwd_lse.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int, Shape, vp, i32, ctypes.c_int,
                                           ctypes.POINTER(BlockStats), f32, vp, vp, vp, vp, sz, vp]
    lib.sa_sparse_attn_bwd_linear_mix_workspace_size.argtypes = [Shape, i32]
    lib.sa_sparse_attn_bwd_linear_mix_workspace_size.restype = sz
    lib.sa_sparse_attn_bwd_linear_mix.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, Shape, vp, i32, vp,
                                                  ctypes.POINTER(BlockStats), f32, vp, vp, vp, vp, sz, vp]
    for fn in ("sa_block_pool", "sa_route", "sa_sparse_attn_fwd", "sa_decode_fwd", "sa_decode_fwd_static",
               "sa_quantize_e4m3", "sa_sparse_attn_fwd_fp8", "sa_sfa_encode", "sa_sfa_densify", "sa_sfa_attn_fwd",
               "sa_sparse_attn_bwd", "sa_sparse_attn_fwd_lse", "sa_sparse_attn_bwd_lse",
               "sa_sparse_attn_bwd_linear_mix"):
        getattr(lib, fn).restype = ctypes.c_int
    lib.sa_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    lib.sa_device_error.restype = ctypes.c_int
    lib.sa_last_error.restype = ctypes.c_char_p
    lib.sa_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != SA_OK:
        raise SparseAttnError(fn, status, load().sa_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SA_FP32
    if t.dtype == torch.bfloat16:
        return SA_BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def _stats_struct(stats: dict) -> BlockStats:
    return BlockStats(*[_ptr(stats.get(n)) for n in _STAT_FIELDS])


def device_error() -> int:
    """Reads and clears the device-side error word (0 = no kernel gave up)."""
    v = ctypes.c_uint32(0)
    _check("sa_device_error", load().sa_device_error(ctypes.byref(v)))
    return int(v.value)


def version() -> str:
    return load().sa_version().decode()


def block_pool(Q: Optional[torch.Tensor], K: torch.Tensor, V: torch.Tensor, block: int, *,
               variance: bool = False, linear: bool = False, centroids_bf16: bool = False,
               first_order: bool = False, covariance: bool = False, residual: bool = False,
               stream=None) -> dict:
    """Block statistics of (Q,) K, V [B,H,N,d]; returns a dict of float32 tensors."""
    lib = load()
    Bsz, H, N, d = K.shape
    nb = N // block
    dev = K.device
    f = dict(device=dev, dtype=torch.float32)
    st = {"kmean": torch.empty(Bsz, H, nb, d, **f), "vsum": torch.empty(Bsz, H, nb, d, **f)}
    if Q is not None:
        st["qmean"] = torch.empty(Bsz, H, nb, d, **f)
    if variance:
        st["kvar"] = torch.empty(Bsz, H, nb, d, **f)
    if linear:
        st["zrelu"] = torch.empty(Bsz, H, nb, d, **f)
        st["htot"] = torch.empty(Bsz, H, d, d, **f)
        st["ztot"] = torch.empty(Bsz, H, d, **f)
    if centroids_bf16:
        st["kmean_bf16"] = torch.empty(Bsz, H, nb, d, device=dev, dtype=torch.bfloat16)
        st["vmean_bf16"] = torch.empty(Bsz, H, nb, d, device=dev, dtype=torch.bfloat16)
        if variance:
            st["kvar_bf16"] = torch.empty(Bsz, H, nb, d, device=dev, dtype=torch.bfloat16)
    if first_order or covariance:
        st["hbar"] = torch.empty(Bsz, H, d, d, **f)
        if centroids_bf16 and first_order:
            st["hbarT_bf16"] = torch.empty(Bsz, H, d, d, device=dev, dtype=torch.bfloat16)
    if covariance:
        st["covnorm"] = torch.empty(Bsz, H, nb, **f)
    if residual:
        st["sexp"] = torch.empty(Bsz, H, d, d, **f)
    cst = _stats_struct(st)
    _check("sa_block_pool", lib.sa_block_pool(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K),
                                              Shape(Bsz, H, N, d, block), ctypes.byref(cst),
                                              _stream(stream)))
    return st


def route(stats: dict, shape, mode: str, topk: int, *, proj_q=None, proj_k=None,
          scale: float = 1.0, want_scores: bool = False, stream=None):
    """Top-k KV blocks per query block: returns (block_idx int32 [B,H,nqb,topk], scores or None)."""
    lib = load()
    Bsz, H, N, d, block = shape
    nb = N // block
    dev = stats["kmean"].device
    idx = torch.empty(Bsz, H, nb, topk, device=dev, dtype=torch.int32)
    sc = torch.empty(Bsz, H, nb, nb, device=dev, dtype=torch.float32) if want_scores else None
    cst = _stats_struct(stats)
    _check("sa_route", lib.sa_route(ctypes.byref(cst), Shape(Bsz, H, N, d, block), ROUTE[mode],
                                    _ptr(proj_q), _ptr(proj_k), float(scale), int(topk),
                                    _ptr(idx), _ptr(sc), _stream(stream)))
    return idx, sc


def sparse_attn_fwd(Q, K, V, block_idx, block: int, tail: str, stats: dict, scale: float, *,
                    alpha=None, out=None, lse=None, stream=None) -> torch.Tensor:
    """Sparse prefill forward; returns O with the shape and dtype of Q.  With
    ``lse`` (float32 [B,H,N]) the rows' log2 log-sum-exp is written there
    (sa_sparse_attn_fwd_lse)."""
    lib = load()
    Bsz, H, N, d = Q.shape
    O = out if out is not None else torch.empty_like(Q)
    topk = block_idx.shape[-1] if block_idx is not None else 0
    cst = _stats_struct(stats or {})
    if lse is not None:
        _check("sa_sparse_attn_fwd_lse",
               lib.sa_sparse_attn_fwd_lse(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), Shape(Bsz, H, N, d, block),
                                          _ptr(block_idx) if topk > 0 else None, int(topk), TAIL[tail],
                                          ctypes.byref(cst), float(scale), _ptr(O), _ptr(lse), _stream(stream)))
        return O
    _check("sa_sparse_attn_fwd",
           lib.sa_sparse_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q),
                                  Shape(Bsz, H, N, d, block),
                                  _ptr(block_idx) if topk > 0 else None, int(topk), TAIL[tail],
                                  _ptr(alpha), ctypes.byref(cst), float(scale), _ptr(O),
                                  _stream(stream)))
    return O


def decode_stats_bf16(stats: dict) -> dict:
    """The view of block statistics that makes sa_decode_fwd read the bf16
    copies (kmean_bf16, kvar_bf16, vmean_bf16; kmean left NULL), plus sexp."""
    return {n: stats[n] for n in ("kmean_bf16", "kvar_bf16", "vmean_bf16", "sexp") if n in stats}


def decode_workspace_size(B: int, Hq: int, Hkv: int, N: int, d: int, block: int, topk: int) -> int:
    return int(load().sa_decode_workspace_size(DecodeShape(B, Hq, Hkv, N, d, block), int(topk)))


def decode_fwd(q, Kcache, Vcache, stats: dict, block: int, topk: int, scale: float, *,
               tail: str = "zero_order", workspace=None, want_route: bool = True, out=None,
               stream=None):
    """GQA decode; returns (o [B,Hq,d], block_idx [B,Hkv,topk] or None, scores [B,Hkv,nb] or None)."""
    lib = load()
    Bsz, Hq, d = q.shape
    Hkv, N = Kcache.shape[1], Kcache.shape[2]
    nb = N // block
    dev = q.device
    ws_bytes = decode_workspace_size(Bsz, Hq, Hkv, N, d, block, topk)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), device=dev, dtype=torch.uint8)
    o = out if out is not None else torch.empty_like(q)
    idx = torch.empty(Bsz, Hkv, topk, device=dev, dtype=torch.int32) if want_route else None
    sc = torch.empty(Bsz, Hkv, nb, device=dev, dtype=torch.float32) if want_route else None
    cst = _stats_struct(stats)
    _check("sa_decode_fwd",
           lib.sa_decode_fwd(_ptr(q), _ptr(Kcache), _ptr(Vcache), _dtype_code(q),
                             DecodeShape(Bsz, Hq, Hkv, N, d, block), ctypes.byref(cst), int(topk),
                             float(scale), TAIL[tail], _ptr(idx), _ptr(sc), _ptr(o),
                             _ptr(workspace), workspace.numel(), _stream(stream)))
    return o, idx, sc


def decode_fwd_static(q, Kcache, Vcache, stats: dict, block: int, topk: int, scale: float, *,
                      tail: str = "zero_order", out=None, stream=None):
    """decode_fwd with the library's static scratch instead of a workspace
    (see sa_decode_fwd_static); returns (o, block_idx, scores)."""
    lib = load()
    Bsz, Hq, d = q.shape
    Hkv, N = Kcache.shape[1], Kcache.shape[2]
    nb = N // block
    dev = q.device
    o = out if out is not None else torch.empty_like(q)
    idx = torch.empty(Bsz, Hkv, topk, device=dev, dtype=torch.int32)
    sc = torch.empty(Bsz, Hkv, nb, device=dev, dtype=torch.float32)
    cst = _stats_struct(stats)
    _check("sa_decode_fwd_static",
           lib.sa_decode_fwd_static(_ptr(q), _ptr(Kcache), _ptr(Vcache), _dtype_code(q),
                                    DecodeShape(Bsz, Hq, Hkv, N, d, block), ctypes.byref(cst), int(topk),
                                    float(scale), TAIL[tail], _ptr(idx), _ptr(sc), _ptr(o),
                                    _stream(stream)))
    return o, idx, sc


def quantize_e4m3(X: torch.Tensor, block: int = 128, *, want_max: bool = False, stream=None):
    """Per-block e4m3 codes of a bf16 tensor [B,H,N,d]: returns (codes uint8
    [B,H,N,d], scales float32 [B,H,ceil(N/block)], scale_max [B,H] or None)."""
    lib = load()
    Bsz, H, N, d = X.shape
    nblk = (N + block - 1) // block
    codes = torch.empty(X.shape, device=X.device, dtype=torch.uint8)
    scales = torch.empty(Bsz, H, nblk, device=X.device, dtype=torch.float32)
    smax = torch.empty(Bsz, H, device=X.device, dtype=torch.float32) if want_max else None
    _check("sa_quantize_e4m3", lib.sa_quantize_e4m3(_ptr(X), Bsz * H, N, d, block, _ptr(codes), _ptr(scales),
                                                    _ptr(smax), _stream(stream)))
    return codes, scales, smax


def fp8_operands(Q, K, V, stats: dict, block: int = 128, stream=None) -> dict:
    """Quantises Q, K, V and (if present) the bf16 centroid tiles of ``stats``."""
    q, qs, _ = quantize_e4m3(Q, block, stream=stream)
    k, ks, _ = quantize_e4m3(K, block, stream=stream)
    v, vs, vmax = quantize_e4m3(V, block, want_max=True, stream=stream)
    ops = {"q": q, "k": k, "v": v, "q_scale": qs, "k_scale": ks, "v_scale": vs, "v_scale_max": vmax}
    if stats.get("kmean_bf16") is not None:
        ops["kbar"], ops["kbar_scale"], _ = quantize_e4m3(stats["kmean_bf16"].view(torch.bfloat16), 128,
                                                          stream=stream)
        ops["vbar"], ops["vbar_scale"], _ = quantize_e4m3(stats["vmean_bf16"].view(torch.bfloat16), 128,
                                                          stream=stream)
    return ops


def sparse_attn_fwd_fp8(ops: dict, shape, block_idx, tail: str, scale: float, *, out=None, stream=None):
    """e4m3 sparse prefill; ``ops`` from fp8_operands; returns bf16 O [B,H,N,d]."""
    lib = load()
    Bsz, H, N, d, block = shape
    O = out if out is not None else torch.empty(Bsz, H, N, d, device=ops["q"].device, dtype=torch.bfloat16)
    topk = block_idx.shape[-1] if block_idx is not None else 0
    cops = Fp8Operands(*[_ptr(ops.get(n)) for n in _FP8_FIELDS])
    _check("sa_sparse_attn_fwd_fp8",
           lib.sa_sparse_attn_fwd_fp8(ctypes.byref(cops), Shape(Bsz, H, N, d, block),
                                      _ptr(block_idx) if topk > 0 else None, int(topk), TAIL[tail],
                                      float(scale), _ptr(O), _stream(stream)))
    return O


def sfa_encode(X: torch.Tensor, kf: int, *, want_dense: bool = True, stream=None):
    """Sparse feature codes of a bf16 tensor [..., d]: returns (vals bf16 [..., kf],
    idx uint8 [..., kf], dense bf16 [..., d] zero-filled rows or None)."""
    lib = load()
    d = X.shape[-1]
    rows = X.numel() // d
    vals = torch.empty(X.shape[:-1] + (kf,), device=X.device, dtype=torch.bfloat16)
    idx = torch.empty(X.shape[:-1] + (kf,), device=X.device, dtype=torch.uint8)
    dense = torch.empty_like(X) if want_dense else None
    _check("sa_sfa_encode", lib.sa_sfa_encode(_ptr(X), rows, d, int(kf), _ptr(vals), _ptr(idx), _ptr(dense),
                                              _stream(stream)))
    return vals, idx, dense


def sfa_densify(vals: torch.Tensor, idx: torch.Tensor, d: int, *, stream=None) -> torch.Tensor:
    """Zero-filled rows [..., d] bf16 from sparse feature codes."""
    lib = load()
    kf = vals.shape[-1]
    rows = vals.numel() // kf
    dense = torch.empty(vals.shape[:-1] + (d,), device=vals.device, dtype=torch.bfloat16)
    _check("sa_sfa_densify", lib.sa_sfa_densify(_ptr(vals), _ptr(idx), rows, int(d), int(kf), _ptr(dense),
                                                _stream(stream)))
    return dense


def sfa_attn_fwd(Qs, Ks, V, block: int, scale: float, *, workspace=None, out=None, stream=None) -> torch.Tensor:
    """Sparse feature attention on zero-filled sparse Q, K [B,H,N,d] and dense V."""
    lib = load()
    Bsz, H, N, d = Qs.shape
    shape = Shape(Bsz, H, N, d, block)
    ws = int(lib.sa_sfa_workspace_size(shape))
    if workspace is None:
        workspace = torch.empty(max(ws, 256), device=Qs.device, dtype=torch.uint8)
    O = out if out is not None else torch.empty_like(Qs)
    _check("sa_sfa_attn_fwd", lib.sa_sfa_attn_fwd(_ptr(Qs), _ptr(Ks), _ptr(V), _dtype_code(Qs), shape, float(scale),
                                                  _ptr(O), _ptr(workspace), workspace.numel(), _stream(stream)))
    return O


def sparse_attn_bwd(Q, K, V, O, dO, block_idx, block: int, tail: str, stats: dict, scale: float, *,
                    lse=None, workspace=None, stream=None):
    """Backward of sparse_attn_fwd (drop, zero_order): returns float32 (dQ, dK, dV).
    ``lse``: the forward's log-sum-exp (sparse_attn_fwd(..., lse=...)), which
    sa_sparse_attn_bwd_lse uses instead of recomputing it."""
    lib = load()
    Bsz, H, N, d = Q.shape
    topk = block_idx.shape[-1] if block_idx is not None else 0
    shape = Shape(Bsz, H, N, d, block)
    ws = int(lib.sa_sparse_attn_bwd_workspace_size(shape, int(topk)))
    if workspace is None:
        workspace = torch.empty(max(ws, 256), device=Q.device, dtype=torch.uint8)
    f = dict(device=Q.device, dtype=torch.float32)
    dQ, dK, dV = torch.empty(Q.shape, **f), torch.empty(K.shape, **f), torch.empty(V.shape, **f)
    cst = _stats_struct(stats or {})
    if lse is not None:
        _check("sa_sparse_attn_bwd_lse",
               lib.sa_sparse_attn_bwd_lse(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(lse), _dtype_code(Q),
                                          shape, _ptr(block_idx) if topk > 0 else None, int(topk), TAIL[tail],
                                          ctypes.byref(cst), float(scale), _ptr(dQ), _ptr(dK), _ptr(dV),
                                          _ptr(workspace), workspace.numel(), _stream(stream)))
        return dQ, dK, dV
    _check("sa_sparse_attn_bwd",
           lib.sa_sparse_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _dtype_code(Q), shape,
                                  _ptr(block_idx) if topk > 0 else None, int(topk), TAIL[tail], ctypes.byref(cst),
                                  float(scale), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(workspace), workspace.numel(),
                                  _stream(stream)))
    return dQ, dK, dV


def sparse_attn_bwd_linear_mix(Q, K, V, O, dO, block_idx, block: int, alpha, stats: dict, scale: float, *,
                               workspace=None, stream=None):
    """Backward of sparse_attn_fwd(..., "linear_mix", alpha=alpha): returns float32 (dQ, dK, dV)."""
    lib = load()
    Bsz, H, N, d = Q.shape
    topk = block_idx.shape[-1] if block_idx is not None else 0
    shape = Shape(Bsz, H, N, d, block)
    ws = int(lib.sa_sparse_attn_bwd_linear_mix_workspace_size(shape, int(topk)))
    if workspace is None:
        workspace = torch.empty(max(ws, 256), device=Q.device, dtype=torch.uint8)
    f = dict(device=Q.device, dtype=torch.float32)
    dQ, dK, dV = torch.empty(Q.shape, **f), torch.empty(K.shape, **f), torch.empty(V.shape, **f)
    cst = _stats_struct(stats or {})
    _check("sa_sparse_attn_bwd_linear_mix",
           lib.sa_sparse_attn_bwd_linear_mix(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _dtype_code(Q), shape,
                                             _ptr(block_idx) if topk > 0 else None, int(topk), _ptr(alpha),
                                             ctypes.byref(cst), float(scale), _ptr(dQ), _ptr(dK), _ptr(dV),
                                             _ptr(workspace), workspace.numel(), _stream(stream)))
    return dQ, dK, dV
