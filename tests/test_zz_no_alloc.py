"""sa_decode_fwd_static: decode for callers that cannot allocate device memory.

Such callers (a plugin or foreign-function host that only passes tensors it
was given, a serving loop that must not call cudaMalloc) use this entry
point, whose scratch is a static device array inside the library.  The test
calls it through the C ABI twice in a row on fresh inputs, so the second call
runs on the scratch the first one left behind, and compares each result with
the workspace entry point sa_decode_fwd.  It is collected last so that a run
stopping at the first failure has already run every other test.
"""
import ctypes
import math

import pytest
import torch

from block_sparse_approximate_b200 import binding as bd
from tests._parity import BF16_TOL, assert_no_device_error, assert_tol, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(seed, B=4, Hq=16, Hkv=4, N=16384, d=128, block=64):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=g, device=DEV).to(torch.bfloat16)
    Kc = (torch.randn(B, Hkv, N // block, block, d, generator=g, device=DEV)
          + 0.7 * torch.randn(B, Hkv, N // block, 1, d, generator=g, device=DEV)).reshape(B, Hkv, N, d)
    Vc = torch.randn(B, Hkv, N, d, generator=g, device=DEV)
    return q, Kc.to(torch.bfloat16).contiguous(), Vc.to(torch.bfloat16).contiguous()


def test_static_scratch_decode_matches_workspace_decode(lib):
    block, topk = 64, 24
    for call, seed in enumerate((31, 32)):
        q, Kc, Vc = _inputs(seed)
        st = bd.block_pool(None, Kc, Vc, block, variance=True)
        s = 1 / math.sqrt(q.shape[-1])
        o_ref, idx_ref, sc_ref = bd.decode_fwd(q, Kc, Vc, st, block, topk, s)
        B, Hq, d = q.shape
        Hkv, N = Kc.shape[1], Kc.shape[2]
        o = torch.empty_like(q)
        idx = torch.empty(B, Hkv, topk, device=DEV, dtype=torch.int32)
        sc = torch.empty(B, Hkv, N // block, device=DEV, dtype=torch.float32)
        cst = bd._stats_struct(st)
        status = lib.sa_decode_fwd_static(q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), bd.SA_BF16,
                                          bd.DecodeShape(B, Hq, Hkv, N, d, block), ctypes.byref(cst),
                                          topk, s, bd.TAIL["zero_order"], idx.data_ptr(), sc.data_ptr(),
                                          o.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert status == bd.SA_OK, lib.sa_last_error().decode()
        torch.cuda.synchronize()
        assert_no_device_error()
        assert torch.equal(idx, idx_ref), f"call {call}: selected blocks differ"
        assert_tol(np64(sc), np64(sc_ref), (1e-5, 1e-6), f"call {call}: route scores")
        assert_tol(np64(o), np64(o_ref), BF16_TOL, f"call {call}: output")


def test_static_scratch_rejects_problems_larger_than_the_array(lib):
    # 64 sequences x 64 query heads x 131072 tokens needs far more than 8 MiB
    sh = bd.DecodeShape(64, 64, 8, 131072, 128, 64)
    assert lib.sa_decode_workspace_size(sh, 64) > 8 * 2 ** 20
    fake = 0x10000   # rejected on the host before anything launches
    st = bd.BlockStats(*[fake if n in ("kmean", "kvar", "vsum") else None for n in bd._STAT_FIELDS])
    status = lib.sa_decode_fwd_static(fake, fake, fake, bd.SA_BF16, sh, ctypes.byref(st), 64, 0.1,
                                      bd.TAIL["zero_order"], None, None, fake, None)
    assert status == bd.SA_ERR_WORKSPACE
    assert "static scratch" in lib.sa_last_error().decode()
