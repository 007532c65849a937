"""sa_decode_fwd_static: decode for callers that cannot allocate device memory.

Such callers (a plugin or foreign-function host that only passes the tensors
it was given, a serving loop that must not call cudaMalloc because it can
synchronise the device) use this entry point, whose scratch is a static
device array inside the library.  The test calls it through the C ABI twice
in a row: first a larger zero-order problem, then a smaller one with the
residual linear tail, whose per-segment sums overlay the partial states the
first call left in the array, so the second call runs on a scratch laid out
differently from its own.  Both entry points run the same kernels, so each
result must equal the workspace entry point sa_decode_fwd's bit for bit.
The file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes
import math

import pytest
import torch

from block_sparse_approximate_b200 import binding as bd
from tests._parity import assert_no_device_error

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(seed, B, Hq, Hkv, N, d=128, block=64):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=g, device=DEV).to(torch.bfloat16)
    Kc = (torch.randn(B, Hkv, N // block, block, d, generator=g, device=DEV)
          + 0.7 * torch.randn(B, Hkv, N // block, 1, d, generator=g, device=DEV)).reshape(B, Hkv, N, d)
    Vc = torch.randn(B, Hkv, N, d, generator=g, device=DEV)
    return q, Kc.to(torch.bfloat16).contiguous(), Vc.to(torch.bfloat16).contiguous()


def _call_static(lib, q, Kc, Vc, st, block, topk, s, tail):
    B, Hq, d = q.shape
    Hkv, N = Kc.shape[1], Kc.shape[2]
    o = torch.empty_like(q)
    idx = torch.empty(B, Hkv, topk, device=DEV, dtype=torch.int32)
    sc = torch.empty(B, Hkv, N // block, device=DEV, dtype=torch.float32)
    cst = bd._stats_struct(st)
    status = lib.sa_decode_fwd_static(q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), bd.SA_BF16,
                                      bd.DecodeShape(B, Hq, Hkv, N, d, block), ctypes.byref(cst),
                                      topk, s, bd.TAIL[tail], idx.data_ptr(), sc.data_ptr(),
                                      o.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert status == bd.SA_OK, lib.sa_last_error().decode()
    return o, idx, sc


def test_static_scratch_decode_matches_workspace_decode(lib):
    block = 64
    calls = (  # (seed, B, Hq, Hkv, N, topk, tail): the second is smaller and lays its scratch out differently
        (31, 4, 16, 4, 16384, 24, "zero_order"),
        (32, 2, 16, 4, 8192, 12, "residual_linear"),
    )
    for call, (seed, B, Hq, Hkv, N, topk, tail) in enumerate(calls):
        q, Kc, Vc = _inputs(seed, B, Hq, Hkv, N)
        st = bd.block_pool(None, Kc, Vc, block, variance=True, residual=(tail == "residual_linear"))
        s = 1 / math.sqrt(q.shape[-1])
        o, idx, sc = _call_static(lib, q, Kc, Vc, st, block, topk, s, tail)
        torch.cuda.synchronize()
        o_ref, idx_ref, sc_ref = bd.decode_fwd(q, Kc, Vc, st, block, topk, s, tail=tail)
        torch.cuda.synchronize()
        assert_no_device_error()
        assert torch.equal(idx, idx_ref), f"call {call}: selected blocks differ"
        assert torch.equal(sc, sc_ref), f"call {call}: route scores differ"
        assert torch.equal(o, o_ref), f"call {call}: outputs differ"


def test_static_scratch_rejects_problems_larger_than_the_array(lib):
    # 64 sequences x 64 query heads x 131072 tokens needs far more than 8 MiB.
    # Every pointer is a real (small) device buffer, so the call could not
    # touch unmapped memory even if the size check came after a launch.
    sh = bd.DecodeShape(64, 64, 8, 131072, 128, 64)
    assert lib.sa_decode_workspace_size(sh, 64) > 8 * 2 ** 20
    buf = torch.zeros(1 << 16, device=DEV, dtype=torch.float32)
    p = buf.data_ptr()
    st = bd.BlockStats(*[p if n in ("kmean", "kvar", "vsum") else None for n in bd._STAT_FIELDS])
    status = lib.sa_decode_fwd_static(p, p, p, bd.SA_BF16, sh, ctypes.byref(st), 64, 0.1,
                                      bd.TAIL["zero_order"], None, None, p, None)
    torch.cuda.synchronize()
    assert status == bd.SA_ERR_WORKSPACE
    assert "static scratch" in lib.sa_last_error().decode()
    assert_no_device_error()
