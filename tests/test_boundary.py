"""The C-ABI library: it loads, exports every declared entry point, and its
host-side argument validation returns the documented status codes (these
checks run before any CUDA call, so no GPU is needed)."""
import ctypes
import os
import re

import pytest

from block_sparse_approximate_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^\S.*?\b(sa_\w+)\s*\(", txt, flags=re.M))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert {"sa_block_pool", "sa_route", "sa_sparse_attn_fwd", "sa_decode_fwd"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(bd.EXPORTS) <= declared


def _header():
    return open(os.path.join(ROOT, "include", "sparseattn.h")).read()


def test_binding_mirrors_header_layouts():
    # the ctypes structs and enum maps follow the header's declarations
    txt = _header()
    body = re.search(r"typedef struct \{(.*?)\} sa_block_stats;", txt, flags=re.S).group(1)
    fields = re.findall(r"^\s*(?:float|uint16_t)\*\s*(\w+);", body, flags=re.M)
    assert tuple(fields) == bd._STAT_FIELDS
    tails = dict((n.lower(), int(v)) for n, v in re.findall(r"SA_TAIL_(\w+)\s*=\s*(\d+)", txt))
    assert tails == bd.TAIL
    routes = dict((n.lower(), int(v)) for n, v in re.findall(r"SA_ROUTE_(\w+)\s*=\s*(\d+)", txt))
    assert routes == bd.ROUTE


def test_version(lib):
    assert "sm_100a" in bd.version()


def _stats(**kw):
    return bd.BlockStats(*[kw.get(n) for n in bd._STAT_FIELDS])


FAKE = 0x10000  # never dereferenced: validation fails (or returns) before any launch


def test_block_pool_validation(lib):
    st = _stats(kmean=FAKE, vsum=FAKE)
    assert lib.sa_block_pool(None, None, FAKE, 1, bd.Shape(1, 1, 256, 128, 128), ctypes.byref(st), None) \
        == bd.SA_ERR_INVALID_ARG
    assert lib.sa_block_pool(None, FAKE, FAKE, 1, bd.Shape(1, 1, 256, 96, 128), ctypes.byref(st), None) \
        == bd.SA_ERR_UNSUPPORTED
    assert lib.sa_block_pool(None, FAKE, FAKE, 1, bd.Shape(1, 1, 250, 128, 128), ctypes.byref(st), None) \
        == bd.SA_ERR_INVALID_ARG
    assert lib.sa_block_pool(None, FAKE + 4, FAKE, 1, bd.Shape(1, 1, 256, 128, 128), ctypes.byref(st), None) \
        == bd.SA_ERR_ALIGNMENT
    assert "16-byte" in lib.sa_last_error().decode()
    # empty problem: nothing to launch
    assert lib.sa_block_pool(None, FAKE, FAKE, 1, bd.Shape(1, 1, 0, 128, 128), ctypes.byref(st), None) == bd.SA_OK
    st2 = _stats(kmean=FAKE, vsum=FAKE, hbarT_bf16=FAKE)     # hbarT_bf16 without hbar
    assert lib.sa_block_pool(None, FAKE, FAKE, 1, bd.Shape(1, 1, 256, 128, 128), ctypes.byref(st2), None) \
        == bd.SA_ERR_INVALID_ARG
    st3 = _stats(kmean=FAKE, vsum=FAKE, covnorm=FAKE)        # covnorm without hbar
    assert lib.sa_block_pool(None, FAKE, FAKE, 1, bd.Shape(1, 1, 256, 128, 128), ctypes.byref(st3), None) \
        == bd.SA_ERR_INVALID_ARG


def test_route_validation(lib):
    st = _stats(qmean=FAKE, kmean=FAKE)
    sh = bd.Shape(1, 1, 1024, 128, 128)
    assert lib.sa_route(ctypes.byref(st), sh, 0, None, None, 1.0, 9, FAKE, None, None) == bd.SA_ERR_INVALID_ARG
    assert lib.sa_route(ctypes.byref(st), sh, 1, None, None, 1.0, 2, FAKE, None, None) == bd.SA_ERR_INVALID_ARG
    assert lib.sa_route(ctypes.byref(st), sh, 2, None, None, 1.0, 2, FAKE, None, None) == bd.SA_ERR_INVALID_ARG
    assert lib.sa_route(ctypes.byref(st), sh, 7, None, None, 1.0, 2, FAKE, None, None) == bd.SA_ERR_INVALID_ARG
    assert lib.sa_route(ctypes.byref(st), sh, 3, None, None, 1.0, 2, FAKE, None, None) \
        == bd.SA_ERR_INVALID_ARG            # cov without covnorm
    big = bd.Shape(1, 1, 8192 * 64, 128, 64)
    assert lib.sa_route(ctypes.byref(st), big, 0, None, None, 1.0, 2, FAKE, None, None) == bd.SA_ERR_UNSUPPORTED


def test_sparse_attn_validation(lib):
    sh = bd.Shape(1, 1, 1024, 128, 128)
    none = _stats()
    f = lib.sa_sparse_attn_fwd
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 1, None, ctypes.byref(none), 0.1, FAKE, None) \
        == bd.SA_ERR_INVALID_ARG            # zero_order without kmean / vsum
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 2, None, ctypes.byref(none), 0.1, FAKE, None) \
        == bd.SA_ERR_INVALID_ARG            # linear_mix without alpha and totals
    assert f(FAKE, FAKE, FAKE, 1, sh, None, 2, 0, None, ctypes.byref(none), 0.1, FAKE, None) \
        == bd.SA_ERR_INVALID_ARG            # topk > 0 without block_idx
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 9, 0, None, ctypes.byref(none), 0.1, FAKE, None) \
        == bd.SA_ERR_INVALID_ARG            # topk > nb
    assert f(FAKE, FAKE, FAKE, 5, sh, FAKE, 2, 0, None, ctypes.byref(none), 0.1, FAKE, None) \
        == bd.SA_ERR_UNSUPPORTED            # unknown dtype
    assert f(FAKE, FAKE + 8, FAKE, 1, sh, FAKE, 2, 0, None, ctypes.byref(none), 0.1, FAKE, None) \
        == bd.SA_ERR_ALIGNMENT
    zo = _stats(kmean=FAKE, vsum=FAKE)
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 3, None, ctypes.byref(zo), 0.1, FAKE, None) \
        == bd.SA_ERR_INVALID_ARG            # first_order without hbar
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 4, None, ctypes.byref(zo), 0.1, FAKE, None) \
        == bd.SA_ERR_UNSUPPORTED            # residual_linear is a decode tail
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 5, None, ctypes.byref(zo), 0.1, FAKE, None) \
        == bd.SA_ERR_INVALID_ARG            # unknown tail mode


def test_lse_entry_validation(lib):
    # the log-sum-exp entries: lse2 required, only the bf16 tensor-core forward produces it
    sh = bd.Shape(1, 1, 1024, 128, 128)
    none = _stats()
    f = lib.sa_sparse_attn_fwd_lse
    # every case returns before a launch (the pointers are never dereferenced)
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 0, ctypes.byref(none), 0.1, FAKE, None, None) \
        == bd.SA_ERR_INVALID_ARG            # no lse2
    assert f(FAKE, FAKE, FAKE, 0, sh, FAKE, 2, 0, ctypes.byref(none), 0.1, FAKE, FAKE, None) \
        == bd.SA_ERR_UNSUPPORTED            # fp32 runs on the CUDA-core kernel
    assert f(FAKE, FAKE, FAKE, 1, bd.Shape(1, 1, 1024, 64, 128), FAKE, 2, 0, ctypes.byref(none), 0.1, FAKE,
             FAKE, None) == bd.SA_ERR_UNSUPPORTED   # d = 64
    lin = _stats(zrelu=FAKE, htot=FAKE, ztot=FAKE)
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 2, ctypes.byref(lin), 0.1, FAKE, FAKE, None) \
        == bd.SA_ERR_INVALID_ARG            # the linear mix (no alpha through this entry)
    fo_cuda = _stats(kmean=FAKE, vsum=FAKE, hbar=FAKE)
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 3, ctypes.byref(fo_cuda), 0.1, FAKE, FAKE, None) \
        == bd.SA_ERR_UNSUPPORTED            # first-order tail without the bf16 tiles: CUDA-core kernel
    assert f(FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 0, ctypes.byref(none), 0.1, FAKE, FAKE + 4, None) \
        == bd.SA_ERR_ALIGNMENT
    g = lib.sa_sparse_attn_bwd_lse
    big = 1 << 40
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, sh, FAKE, 2, 0, ctypes.byref(none), 0.1, FAKE, FAKE, FAKE,
             FAKE, big, None) == bd.SA_ERR_INVALID_ARG   # no lse2
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, 1, sh, FAKE, 2, 0, ctypes.byref(none), 0.1, FAKE, FAKE, FAKE,
             FAKE, big, None) == bd.SA_ERR_ALIGNMENT
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, sh, FAKE, 2, 2, ctypes.byref(none), 0.1, FAKE, FAKE, FAKE,
             FAKE, big, None) == bd.SA_ERR_UNSUPPORTED   # linear_mix has no backward


def test_decode_validation_and_workspace(lib):
    sh = bd.DecodeShape(16, 32, 8, 131072, 128, 64)
    ws = lib.sa_decode_workspace_size(sh, 64)
    assert ws > 16 * 32 * 128 * 4
    assert lib.sa_decode_workspace_size(bd.DecodeShape(1, 6, 4, 1024, 128, 64), 4) == 0   # Hq % Hkv
    st = _stats(kmean=FAKE, kvar=FAKE, vsum=FAKE)
    f = lib.sa_decode_fwd
    assert f(FAKE, FAKE, FAKE, 1, sh, ctypes.byref(st), 64, 0.1, 1, None, None, FAKE, FAKE, ws - 1, None) \
        == bd.SA_ERR_WORKSPACE
    assert f(FAKE, FAKE, FAKE, 0, sh, ctypes.byref(st), 64, 0.1, 1, None, None, FAKE, FAKE, ws, None) \
        == bd.SA_ERR_UNSUPPORTED            # fp32 caches
    assert f(FAKE, FAKE, FAKE, 1, sh, ctypes.byref(st), 64, 0.1, 2, None, None, FAKE, FAKE, ws, None) \
        == bd.SA_ERR_UNSUPPORTED            # linear_mix decode
    assert f(FAKE, FAKE, FAKE, 1, sh, ctypes.byref(st), 64, 0.1, 4, None, None, FAKE, FAKE, ws, None) \
        == bd.SA_ERR_INVALID_ARG            # residual_linear without stats->sexp
    # the residual partial sums fit over the statistics pass's partial states
    # here, so the workspace (and the static scratch bound) does not grow
    assert ws < 8 * 2 ** 20
    assert f(FAKE, FAKE, FAKE, 1, sh, ctypes.byref(st), 5000, 0.1, 1, None, None, FAKE, FAKE, ws, None) \
        == bd.SA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, sh, ctypes.byref(st), 64, 0.1, 1, None, None, FAKE, FAKE + 16, ws, None) \
        == bd.SA_ERR_ALIGNMENT              # workspace must be 256-byte aligned
