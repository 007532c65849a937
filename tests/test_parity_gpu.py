"""GPU parity: every step of the path through the C-ABI against the CPU oracle
on the same seeded inputs (small sizes spanning several tiles and ragged
tails, plus edge cases).  Full-size workloads are in test_parity_full_gpu.py."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_approximate_b200 import binding as bd
from block_sparse_approximate_b200 import workloads as wl
from tests._parity import (BF16_TOL, FP32_TOL, assert_fp8_bound, assert_no_device_error, assert_stats_close,
                           assert_tol, check_topk_exact, np64, selection_agreement)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gauss(B, H, N, d, dtype, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return [torch.randn(B, H, N, d, generator=g, device=DEV).to(dtype).contiguous() for _ in range(3)]


# --------------------------------------------------------------------------
# block statistics
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,d,block,N", [(torch.float32, 64, 64, 1024), (torch.bfloat16, 128, 128, 4736),
                                             (torch.bfloat16, 128, 64, 2048), (torch.bfloat16, 64, 128, 1024)])
def test_block_pool(lib, dtype, d, block, N):
    Q, K, V = _gauss(2, 3, N, d, dtype, 1)
    st = bd.block_pool(Q, K, V, block, variance=True, linear=True, centroids_bf16=True)
    ref = oracle.block_pool(np64(Q), np64(K), np64(V), block, variance=True, linear=True)
    for n in ("qmean", "kmean", "vsum", "kvar", "zrelu", "ztot"):
        assert_stats_close(st[n], ref[n], n)
    assert_stats_close(st["htot"], ref["htot"], "htot", rtol=1e-4)
    assert_stats_close(st["kmean_bf16"].float(), ref["kmean"], "kmean_bf16", rtol=1e-2)
    assert_stats_close(st["vmean_bf16"].float(), ref["vsum"] / block, "vmean_bf16", rtol=1e-2)


@pytest.mark.parametrize("dtype,d,block,N", [(torch.float32, 64, 64, 1024), (torch.bfloat16, 128, 128, 4736),
                                             (torch.bfloat16, 128, 64, 2048), (torch.bfloat16, 64, 128, 1024)])
def test_block_pool_hbar(lib, dtype, d, block, N):
    # PISA's H̄ (bf16 with d = block = 128 takes the tensor-core path) and the
    # covariance norms M_j = ‖H_j − H̄‖₂ (power iteration to 1e-6 on λ)
    Q, K, V = _gauss(2, 3, N, d, dtype, 11)
    st = bd.block_pool(Q, K, V, block, centroids_bf16=True, first_order=True, covariance=True)
    ref = oracle.block_pool(np64(Q), np64(K), np64(V), block, first_order=True, covariance=True)
    assert_stats_close(st["hbar"], ref["hbar"], "hbar", rtol=1e-4)
    hT = np.swapaxes(ref["hbar"], -1, -2)
    assert_stats_close(st["hbarT_bf16"].float(), hT, "hbarT_bf16", rtol=2 ** -8)
    got = np64(st["covnorm"])
    np.testing.assert_allclose(got, ref["covnorm"], rtol=1e-3, atol=1e-4)


@pytest.mark.parametrize("dtype,d,block", [(torch.bfloat16, 128, 128), (torch.float32, 64, 64)])
def test_covnorm_rank_one(lib, dtype, d, block):
    # keys k̄_j + a_n u, values b_n w + c_j: H_j − H̄ = (γ_j − γ̄) u wᵀ, so
    # M_j = |γ_j − γ̄| |u| |w| (u, w, a, b chosen exactly representable in bf16)
    g = torch.Generator(device="cpu")
    g.manual_seed(13)
    nb = 12
    u = torch.randint(-4, 5, (d,), generator=g).double()
    w = torch.randint(-4, 5, (d,), generator=g).double()
    kbar = torch.randint(-8, 9, (nb, d), generator=g).double()
    r = torch.randint(-3, 4, (nb, block // 2), generator=g).double()
    a = torch.cat([r, -r], dim=1)                 # zero-mean deviations, small integers
    bcoef = torch.randint(-3, 4, (nb, block), generator=g).double() / 4
    cval = torch.randint(-8, 9, (nb, d), generator=g).double() / 8
    K = (kbar[:, None, :] + a[:, :, None] * u[None, None, :]).reshape(1, 1, nb * block, d)
    V = (bcoef[:, :, None] * w[None, None, :] + cval[:, None, :]).reshape(1, 1, nb * block, d)
    gam = (a * bcoef).sum(dim=1)
    expect = ((gam - gam.mean()).abs() * u.norm() * w.norm()).numpy()
    Kd, Vd = K.to(dtype).to(DEV), V.to(dtype).to(DEV)
    assert torch.equal(Kd.double().cpu(), K) and torch.equal(Vd.double().cpu(), V)
    st = bd.block_pool(None, Kd, Vd, block, covariance=True)
    np.testing.assert_allclose(np64(st["covnorm"])[0, 0], expect, rtol=1e-4, atol=1e-3)


def test_block_pool_hbar_large_offset(lib):
    # the deviation form: a large common key offset leaves H̄ unchanged
    Q, K, V = _gauss(1, 2, 2048, 128, torch.float32, 12)
    st0 = bd.block_pool(None, K, V, 128, first_order=True)
    st1 = bd.block_pool(None, (K + 1000.0).contiguous(), V, 128, first_order=True)
    ref = oracle.block_pool(None, np64(K), np64(V), 128, first_order=True)
    assert_stats_close(st0["hbar"], ref["hbar"], "hbar", rtol=1e-4)
    assert_stats_close(st1["hbar"], ref["hbar"], "hbar with offset", rtol=2e-3)


def test_block_pool_large_offset_variance(lib):
    # two-pass variance: a large common offset must not destroy the variance
    Q, K, V = _gauss(1, 2, 2048, 128, torch.float32, 2)
    K = (K + 1000.0).contiguous()
    st = bd.block_pool(None, K, V, 128, variance=True)
    ref = oracle.block_pool(None, np64(K), np64(V), 128, variance=True)
    np.testing.assert_allclose(np64(st["kvar"]), ref["kvar"], rtol=2e-3, atol=2e-3)


# --------------------------------------------------------------------------
# router
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["dot", "proj", "taylor2", "cov"])
@pytest.mark.parametrize("nb,k", [(37, 5), (256, 26), (16, 0), (16, 16), (97, 64), (97, 65), (300, 100),
                                  (600, 40), (1100, 64)])
def test_route(lib, mode, nb, k):
    d, block = 128, 128
    w = wl.WORKLOADS["video_dit"]
    if nb == 256:
        inp = wl.prefill_inputs(w, DEV, H=2, N=nb * block)
        Q, K, V = inp["Q"], inp["K"], inp["V"]
    else:
        Q, K, V = _gauss(1, 2, nb * block, d, torch.bfloat16, 3)
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    Pq = (torch.randn(d, d, generator=g, device=DEV) / math.sqrt(d)).contiguous()
    Pk = (torch.randn(d, d, generator=g, device=DEV) / math.sqrt(d)).contiguous()
    st = bd.block_pool(Q, K, V, block, variance=True, covariance=(mode == "cov"))
    s = 1 / math.sqrt(d)
    shape = (1, 2, nb * block, d, block)
    idx, sc = bd.route(st, shape, mode, k, proj_q=Pq, proj_k=Pk, scale=s, want_scores=True)
    ref = oracle.route_scores(np64(st["qmean"]), np64(st["kmean"]), mode, proj_q=np64(Pq),
                              proj_k=np64(Pk), kvar=np64(st["kvar"]), scale=s,
                              covnorm=np64(st["covnorm"]) if mode == "cov" else None, block=block)
    assert_stats_close(sc, ref, f"{mode} scores", rtol=2e-5)
    check_topk_exact(idx, sc, k)
    frac = selection_agreement(np64(sc), ref, k)
    assert frac >= 0.95


def test_route_tie_groups_cut_by_k(lib):
    # 24 distinct key blocks, each repeated 4 times: every dot score comes in
    # a group of 4 equal ones, and k = 10 keeps two groups and the two
    # smallest indices of the third (the selection is the same for every
    # score mode)
    d, block, nb = 128, 128, 96
    Q, K, V = _gauss(1, 1, nb * block, d, torch.float32, 7)
    K = K.reshape(1, 1, nb, block, d)[:, :, ::4].repeat_interleave(4, dim=2).reshape(1, 1, nb * block, d)
    st = bd.block_pool(Q, K.contiguous(), V, block)
    idx, sc = bd.route(st, (1, 1, nb * block, d, block), "dot", 10, want_scores=True)
    check_topk_exact(idx, sc, 10)
    s = np64(sc)[0, 0]
    assert (s.reshape(nb, 24, 4) == s.reshape(nb, 24, 4)[..., :1]).all()   # the groups do tie
    assert (np.diff(idx.cpu().numpy(), axis=-1) > 0).all()


def test_route_ties_pick_smaller_index(lib):
    # identical key blocks: every score ties, the smallest indices win
    d, block, nb = 128, 128, 12
    Q, K, V = _gauss(1, 1, nb * block, d, torch.float32, 6)
    K = K[:, :, :block].repeat(1, 1, nb, 1).contiguous()
    st = bd.block_pool(Q, K, V, block)
    idx, sc = bd.route(st, (1, 1, nb * block, d, block), "dot", 5, want_scores=True)
    assert (idx.cpu().numpy() == np.arange(5)).all()


# --------------------------------------------------------------------------
# sparse prefill
# --------------------------------------------------------------------------

def _prefill_case(Q, K, V, block, k, tail, mode="dot", alpha=None, seed=0, tol=BF16_TOL):
    B, H, N, d = Q.shape
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, block, linear=(tail == "linear_mix"),
                       centroids_bf16=(Q.dtype == torch.bfloat16), first_order=(tail == "first_order"))
    idx, sc = bd.route(st, (B, H, N, d, block), mode, k, want_scores=True)
    check_topk_exact(idx, sc, k)
    O = bd.sparse_attn_fwd(Q, K, V, idx, block, tail, st, s, alpha=alpha)
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle.sparse_attention(np64(Q), np64(K), np64(V), idx.cpu().numpy(), block, tail, s,
                                  alpha=None if alpha is None else np64(alpha))
    return assert_tol(np64(O), ref, tol, f"{tail} k={k}")


@pytest.mark.parametrize("tail", ["zero_order", "drop", "linear_mix", "first_order"])
def test_tiny_fp32(lib, tail):
    w = wl.WORKLOADS["tiny"]
    inp = wl.prefill_inputs(w, DEV)
    alpha = torch.rand(w.H, w.d, device=DEV) * 0.7 + 0.2 if tail == "linear_mix" else None
    _prefill_case(inp["Q"], inp["K"], inp["V"], w.block, w.k, tail, alpha=alpha, tol=FP32_TOL)


@pytest.mark.parametrize("tail", ["zero_order", "drop", "linear_mix", "first_order"])
@pytest.mark.parametrize("k", [0, 1, 4, 32])
def test_video_small_bf16(lib, tail, k):
    w = wl.WORKLOADS["video_dit"]
    inp = wl.prefill_inputs(w, DEV, H=2, N=4096)        # 1x64x64 grid, 32 blocks
    alpha = torch.rand(2, w.d, device=DEV) * 0.7 + 0.2 if tail == "linear_mix" else None
    _prefill_case(inp["Q"], inp["K"], inp["V"], w.block, k, tail, alpha=alpha)


@pytest.mark.parametrize("tail", ["zero_order", "drop", "linear_mix", "first_order"])
@pytest.mark.parametrize("dtype,d,block,nb,k", [
    (torch.bfloat16, 128, 128, 37, 5),     # ragged centroid tiles
    (torch.bfloat16, 128, 128, 133, 13),   # more than one 128-centroid tile, ragged
    (torch.bfloat16, 128, 64, 40, 6),
    (torch.bfloat16, 64, 128, 20, 3),
    (torch.float32, 128, 128, 9, 2),
    (torch.float32, 64, 64, 1, 1),         # a single block
])
def test_shapes(lib, tail, dtype, d, block, nb, k):
    Q, K, V = _gauss(2, 2, nb * block, d, dtype, 7 + nb)
    alpha = torch.rand(2, d, device=DEV) * 0.7 + 0.2 if tail == "linear_mix" else None
    tol = FP32_TOL if dtype == torch.float32 else BF16_TOL
    _prefill_case(Q, K, V, block, k, tail, alpha=alpha, tol=tol)


@pytest.mark.parametrize("dtype,nb,k", [(torch.bfloat16, 37, 5), (torch.bfloat16, 133, 13),
                                        (torch.float32, 37, 5), (torch.bfloat16, 9, 0)])
def test_first_order_tail_matters(lib, dtype, nb, k):
    # values tied to the keys' in-block deviations: the first-order term moves
    # the output far beyond the tolerance, and the GPU's first-order minus
    # zero-order difference matches the oracle's
    block, d = 128, 128
    inp = wl.block_linear_inputs(1, 2, nb, block, d, dtype, 21 + nb, DEV)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    tol = FP32_TOL if dtype == torch.float32 else BF16_TOL
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, block, centroids_bf16=(dtype == torch.bfloat16), first_order=True)
    idx, _ = bd.route(st, (1, 2, nb * block, d, block), "dot", k)
    o_fo = bd.sparse_attn_fwd(Q, K, V, idx, block, "first_order", st, s)
    o_zo = bd.sparse_attn_fwd(Q, K, V, idx, block, "zero_order", st, s)
    torch.cuda.synchronize()
    assert_no_device_error()
    args = (np64(Q), np64(K), np64(V), idx.cpu().numpy(), block)
    ref_fo = oracle.sparse_attention(*args, "first_order", s)
    ref_zo = oracle.sparse_attention(*args, "zero_order", s)
    assert np.abs(ref_fo - ref_zo).mean() > 10 * tol[1]
    assert_tol(np64(o_fo), ref_fo, tol, "first_order")
    assert_tol(np64(o_fo) - np64(o_zo), ref_fo - ref_zo, (2 * tol[0], 2 * tol[1]), "first_order - zero_order")


@pytest.mark.parametrize("k", [1, 4, 26])
def test_pisa_small(lib, k):
    # PISA end to end: covariance-aware routing on the GPU's statistics (scores
    # against the oracle's score of the same statistics, selection bit-exact
    # against the oracle's top-k of the GPU scores, selection agreement with
    # the oracle's statistics) and the hybrid-order tail on that selection
    w = wl.WORKLOADS["video_dit_pisa"]
    inp = wl.prefill_inputs(w, DEV, H=2, N=4096)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    B, H, N, d = Q.shape
    s = w.scale
    st = bd.block_pool(Q, K, V, w.block, centroids_bf16=True, first_order=True, covariance=True)
    idx, sc = bd.route(st, (B, H, N, d, w.block), "cov", k, scale=s, want_scores=True)
    check_topk_exact(idx, sc, k)
    ref_st = oracle.block_pool(np64(Q), np64(K), np64(V), w.block, covariance=True)
    ref_sc = oracle.route_scores(ref_st["qmean"], ref_st["kmean"], "cov", covnorm=ref_st["covnorm"],
                                 scale=s, block=w.block)
    # M_j comes from a power iteration stopped at 1e-6 on λ: scores within 2e-3
    np.testing.assert_allclose(np64(sc), ref_sc, rtol=1e-4, atol=2e-3)
    assert selection_agreement(np64(sc), ref_sc, k, gap_rel=5e-3) >= 0.9
    O = bd.sparse_attn_fwd(Q, K, V, idx, w.block, "first_order", st, s)
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle.sparse_attention(np64(Q), np64(K), np64(V), idx.cpu().numpy(), w.block, "first_order", s)
    assert_tol(np64(O), ref, BF16_TOL, f"pisa k={k}")


def test_empty_problem_is_a_no_op(lib):
    Q = torch.empty(1, 2, 0, 128, device=DEV, dtype=torch.bfloat16)
    st = {"kmean": torch.empty(1, 2, 0, 128, device=DEV), "vsum": torch.empty(1, 2, 0, 128, device=DEV)}
    idx = torch.empty(1, 2, 0, 0, device=DEV, dtype=torch.int32)
    O = bd.sparse_attn_fwd(Q, Q, Q, idx, 128, "zero_order", st, 0.1)
    assert O.shape == Q.shape


def test_value_shift_on_gpu(lib):
    # V + c shifts every output row by c (row normalisation, PISA §2)
    Q, K, V = _gauss(1, 2, 4096, 128, torch.float32, 11)
    c = torch.linspace(-1, 1, 128, device=DEV)
    for tail in ("zero_order", "drop"):
        st1 = bd.block_pool(Q, K, V, 128)
        idx, _ = bd.route(st1, (1, 2, 4096, 128, 128), "dot", 4)
        O1 = bd.sparse_attn_fwd(Q, K, V, idx, 128, tail, st1, 0.088)
        V2 = (V + c).contiguous()
        st2 = bd.block_pool(Q, K, V2, 128)
        O2 = bd.sparse_attn_fwd(Q, K, V2, idx, 128, tail, st2, 0.088)
        assert (O2 - O1 - c).abs().max().item() < 1e-4


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------

@pytest.mark.parametrize("tail", ["zero_order", "drop", "residual_linear"])
@pytest.mark.parametrize("B,Hq,Hkv,N,d,block,k", [
    (2, 8, 2, 8192, 128, 64, 16),
    (1, 4, 4, 4096, 128, 128, 5),
    (2, 8, 1, 2048, 64, 64, 0),
    (1, 4, 2, 2048, 128, 64, 32),           # every block selected
    (3, 6, 3, 64 * 77, 128, 64, 7),         # ragged split ranges
    # 8 heads per KV head, 2304 blocks, top-160: the merge takes 18 statistics
    # states and 20 exact states per head in chunks of 16, and the selected
    # blocks' zero-order terms in chunks of 64
    (1, 8, 1, 64 * 2304, 128, 64, 160),
])
def test_decode(lib, tail, B, Hq, Hkv, N, d, block, k):
    w = wl.WORKLOADS["decode"]
    g = torch.Generator(device=DEV)
    g.manual_seed(100 + N + k)
    q = torch.randn(B, Hq, d, generator=g, device=DEV).to(torch.bfloat16)
    Kc = (torch.randn(B, Hkv, N // block, block, d, generator=g, device=DEV)
          + 0.7 * torch.randn(B, Hkv, N // block, 1, d, generator=g, device=DEV)).reshape(B, Hkv, N, d).to(torch.bfloat16)
    Vc = torch.randn(B, Hkv, N, d, generator=g, device=DEV).to(torch.bfloat16)
    st = bd.block_pool(None, Kc, Vc, block, variance=True, residual=(tail == "residual_linear"))
    s = 1 / math.sqrt(d)
    o, idx, sc = bd.decode_fwd(q, Kc, Vc, st, block, k, s, tail=tail)
    torch.cuda.synchronize()
    check_topk_exact(idx, sc, k)
    ref_sc = oracle.decode_route_scores(np64(q), np64(st["kmean"]), np64(st["kvar"]), s)
    assert_stats_close(sc, ref_sc, "decode scores", rtol=2e-5)
    ref_o, _, _ = oracle.decode_attention(np64(q), np64(Kc), np64(Vc), block, k, s, tail=tail,
                                          block_idx=idx.cpu().numpy())
    assert_tol(np64(o), ref_o, BF16_TOL, f"decode {tail}")
    assert_no_device_error()
    del w


@pytest.mark.parametrize("case", ["tie_groups", "all_equal", "long_row"])
def test_decode_topk_edge_rows(lib, case):
    # tie_groups: 12 distinct key blocks repeated 4 times, so the scores come
    # in groups of 4 equal ones and k = 10 cuts the third group (the smallest
    # indices win); all_equal: one key block everywhere; long_row: 4000 blocks
    # per row (16 keys per thread of the top-k)
    d, block = 128, 64
    nb, k = {"tie_groups": (48, 10), "all_equal": (40, 5), "long_row": (4000, 64)}[case]
    g = torch.Generator(device=DEV)
    g.manual_seed(300 + nb)
    q = torch.randn(1, 4, d, generator=g, device=DEV).to(torch.bfloat16)
    Kb = torch.randn(1, 1, nb, block, d, generator=g, device=DEV)
    if case == "tie_groups":
        Kb = Kb[:, :, ::4].repeat_interleave(4, dim=2)
    elif case == "all_equal":
        Kb = Kb[:, :, :1].expand(1, 1, nb, block, d)
    Kc = Kb.reshape(1, 1, nb * block, d).to(torch.bfloat16).contiguous()
    Vc = torch.randn(1, 1, nb * block, d, generator=g, device=DEV).to(torch.bfloat16)
    st = bd.block_pool(None, Kc, Vc, block, variance=True)
    o, idx, sc = bd.decode_fwd(q, Kc, Vc, st, block, k, 1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert_no_device_error()
    check_topk_exact(idx, sc, k)
    if case == "all_equal":
        assert (idx.cpu().numpy().ravel() == np.arange(k)).all()
    if case == "tie_groups":
        s = np64(sc).ravel()
        assert (s.reshape(12, 4) == s.reshape(12, 4)[:, :1]).all()   # the groups do tie


def _bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.as_tensor(x).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("tail", ["zero_order", "drop", "residual_linear"])
@pytest.mark.parametrize("B,Hq,Hkv,N,d,block,k", [
    (2, 8, 2, 8192, 128, 64, 16),
    (1, 4, 4, 4096, 128, 128, 5),
    (2, 8, 1, 2048, 64, 64, 3),
    (3, 6, 3, 64 * 77, 128, 64, 7),         # ragged split ranges
    (4, 32, 4, 8192, 128, 64, 16),          # 8 heads per KV head; whole rows per CTA (fused top-k)
    (1, 8, 2, 64 * 300, 128, 64, 20),       # rows of three 128-block tiles, the last ragged
    (40, 8, 2, 64 * 300, 128, 64, 20),      # the same rows held whole by one CTA each (fused top-k)
    (1, 8, 1, 64 * 2304, 128, 64, 160),     # the merge's states and selected blocks in several chunks
])
def test_decode_bf16_stats(lib, tail, B, Hq, Hkv, N, d, block, k):
    # the decode reading the bf16 copies of kmean, kvar and vsum / block: its
    # scores against the oracle's taylor2 score of the bf16-rounded oracle
    # statistics, the selection bit-exact against the oracle's top-k of the
    # GPU's scores, the output against the float64 oracle (exact statistics)
    g = torch.Generator(device=DEV)
    g.manual_seed(300 + N + k)
    q = torch.randn(B, Hq, d, generator=g, device=DEV).to(torch.bfloat16)
    Kc = (torch.randn(B, Hkv, N // block, block, d, generator=g, device=DEV)
          + 0.7 * torch.randn(B, Hkv, N // block, 1, d, generator=g, device=DEV)).reshape(B, Hkv, N, d).to(torch.bfloat16)
    Vc = torch.randn(B, Hkv, N, d, generator=g, device=DEV).to(torch.bfloat16)
    st = bd.block_pool(None, Kc, Vc, block, variance=True, centroids_bf16=True,
                       residual=(tail == "residual_linear"))
    s = 1 / math.sqrt(d)
    o, idx, sc = bd.decode_fwd(q, Kc, Vc, bd.decode_stats_bf16(st), block, k, s, tail=tail)
    torch.cuda.synchronize()
    assert_no_device_error()
    check_topk_exact(idx, sc, k)
    ost = oracle.block_pool(None, np64(Kc), np64(Vc), block, variance=True)
    ref_sc = oracle.decode_route_scores(np64(q), _bf16_round(ost["kmean"]), _bf16_round(ost["kvar"]), s)
    # a float32 and a float64 mean can round to neighbouring bf16 values: one
    # ulp (2^-8 relative) of one channel moves a score by ~1e-4
    assert_stats_close(sc, ref_sc, "decode scores (bf16 statistics)", rtol=1e-4)
    selection_agreement(np64(sc), ref_sc, k, gap_rel=1e-3)
    ref_o, _, _ = oracle.decode_attention(np64(q), np64(Kc), np64(Vc), block, k, s, tail=tail,
                                          block_idx=idx.cpu().numpy())
    assert_tol(np64(o), ref_o, BF16_TOL, f"decode {tail} (bf16 statistics)")


def test_decode_bf16_stats_requires_the_bf16_copies(lib):
    q = torch.zeros(1, 4, 128, device=DEV, dtype=torch.bfloat16)
    Kc = torch.zeros(1, 1, 1024, 128, device=DEV, dtype=torch.bfloat16)
    st = bd.block_pool(None, Kc, Kc, 64, variance=True, centroids_bf16=True)
    view = bd.decode_stats_bf16(st)
    del view["vmean_bf16"]
    with pytest.raises(bd.SparseAttnError) as e:
        bd.decode_fwd(q, Kc, Kc, view, 64, 4, 0.1, tail="zero_order")
    assert e.value.status == bd.SA_ERR_INVALID_ARG
    # without the zero-order tail the value means are not needed
    bd.decode_fwd(q, Kc, Kc, view, 64, 4, 0.1, tail="drop")
    torch.cuda.synchronize()
    assert_no_device_error()


def test_block_pool_sexp(lib):
    # SPLA's all-token state Σ_n exp(k_n) v_nᵀ: tensor-core path (bf16, d = 128,
    # φ(k) rounded to bf16) and CUDA-core path (fp32)
    for dtype, d, tol in ((torch.bfloat16, 128, 5e-3), (torch.float32, 64, 1e-5)):
        Q, K, V = _gauss(2, 2, 1024, d, dtype, 17)
        st = bd.block_pool(None, K, V, 64, residual=True)
        ref = np.einsum("bhnc,bhne->bhce", np.exp(np64(K)), np64(V))
        assert_stats_close(st["sexp"], ref, f"sexp {dtype}", rtol=tol)


def test_residual_linear_prefill_is_rejected(lib):
    Q = torch.zeros(1, 1, 256, 128, device=DEV, dtype=torch.bfloat16)
    st = bd.block_pool(Q, Q, Q, 128, residual=True)
    idx, _ = bd.route(st, (1, 1, 256, 128, 128), "dot", 1)
    with pytest.raises(bd.SparseAttnError) as e:
        bd.sparse_attn_fwd(Q, Q, Q, idx, 128, "residual_linear", st, 0.1)
    assert e.value.status == bd.SA_ERR_UNSUPPORTED


# --------------------------------------------------------------------------
# FP8 e4m3 sparse branch
# --------------------------------------------------------------------------

FP8_TOL = (6e-2, 6e-3)


def _e4m3_values(codes: torch.Tensor) -> np.ndarray:
    return codes.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


@pytest.mark.parametrize("N,block", [(4096, 128), (4736, 128), (1000, 128), (2048, 64)])
def test_quantize_e4m3_bit_exact(lib, N, block):
    g = torch.Generator(device=DEV)
    g.manual_seed(N)
    X = (torch.randn(2, 3, N, 128, generator=g, device=DEV) * 3).to(torch.bfloat16)
    X[0, 1, :block] = 0          # an all-zero block gets scale 1
    codes, scales, smax = bd.quantize_e4m3(X, block, want_max=True)
    torch.cuda.synchronize()
    Xn = np64(X)
    nblk = (N + block - 1) // block
    pad = nblk * block - N
    Xp = np.concatenate([Xn, np.zeros((2, 3, pad, 128))], axis=2) if pad else Xn
    deq, ref_codes, ref_sigma = oracle.quantise_blocks_e4m3(Xp, block)
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_sigma)
    np.testing.assert_array_equal(_e4m3_values(codes), ref_codes[:, :, :N])
    np.testing.assert_array_equal(smax.cpu().numpy(), ref_sigma.max(axis=2))


def _fp8_case(Q, K, V, k, tail):
    """The e4m3 kernel against the oracle's quantised forward (SLA2 §2C: Q, K,
    V and the centroid tiles quantised per block, float64 attention, exact P).
    What is left is the e4m3 rounding of P (at most 2^-4 relative per element),
    checked elementwise against the bound it implies."""
    B, H, N, d = Q.shape
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, 128, centroids_bf16=True)
    idx, sc = bd.route(st, (B, H, N, d, 128), "dot", k, want_scores=True)
    ops = bd.fp8_operands(Q, K, V, st)
    O = bd.sparse_attn_fwd_fp8(ops, (B, H, N, d, 128), idx, tail, s)
    torch.cuda.synchronize()
    assert_no_device_error()
    args = (np64(Q), np64(K), np64(V), idx.cpu().numpy(), 128, tail, s)
    emu = oracle.fp8_attention(*args)
    emu_abs = oracle.fp8_attention(*args, absolute_values=True)
    return assert_fp8_bound(np64(O), emu, emu_abs, f"fp8 {tail} k={k}")


@pytest.mark.parametrize("tail", ["zero_order", "drop"])
@pytest.mark.parametrize("k", [0, 1, 4, 32])
def test_fp8_video_small(lib, tail, k):
    w = wl.WORKLOADS["fp8"]
    inp = wl.prefill_inputs(w, DEV, H=2, N=4096)
    _fp8_case(inp["Q"], inp["K"], inp["V"], k, tail)


@pytest.mark.parametrize("tail", ["zero_order", "drop"])
@pytest.mark.parametrize("nb,k", [(37, 5), (133, 13)])
def test_fp8_ragged(lib, tail, nb, k):
    Q, K, V = _gauss(2, 2, nb * 128, 128, torch.bfloat16, 70 + nb)
    _fp8_case(Q, K, V, k, tail)


# --------------------------------------------------------------------------
# sparse feature attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("d,kf", [(128, 16), (128, 1), (64, 8), (128, 32)])
def test_sfa_encode_bit_exact(lib, d, kf):
    g = torch.Generator(device=DEV)
    g.manual_seed(30 + kf)
    # rounded to a coarse grid so that equal magnitudes (the tie rule) occur
    X = (torch.randn(3, 257, d, generator=g, device=DEV) * 4).round().div(4).to(torch.bfloat16)
    vals, idx, dense = bd.sfa_encode(X, kf)
    torch.cuda.synchronize()
    rv, ri = oracle.sfa_codes(np64(X), kf)
    np.testing.assert_array_equal(idx.cpu().numpy().astype(np.int64), ri)
    np.testing.assert_array_equal(np64(vals), rv)
    np.testing.assert_array_equal(np64(dense), oracle.sfa_densify(rv, ri, d))
    back = bd.sfa_densify(vals, idx, d)
    torch.cuda.synchronize()
    assert torch.equal(back, dense)


@pytest.mark.parametrize("d,block,N,kf", [(128, 128, 1024, 16), (128, 128, 1152, 32), (64, 64, 640, 8)])
def test_sfa_attention(lib, d, block, N, kf):
    Q, K, V = _gauss(1, 2, N, d, torch.bfloat16, 40 + N)
    _, _, Qs = bd.sfa_encode(Q, kf)
    _, _, Ks = bd.sfa_encode(K, kf)
    s = 1 / math.sqrt(d)
    O = bd.sfa_attn_fwd(Qs, Ks, V, block, s)
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle.sfa_attention(np64(Q), np64(K), np64(V), kf, s)
    assert_tol(np64(O), ref, BF16_TOL, f"sfa d={d} kf={kf}")


# --------------------------------------------------------------------------
# backward
# --------------------------------------------------------------------------

@pytest.mark.parametrize("tail", ["zero_order", "drop"])
def test_backward_batched_heads(lib, tail):
    # several sequences and heads: the (batch, head) indexing of the tensor
    # maps, the query lists and the pseudo-key ranges of the tcgen05 backward
    B, H, nb, k, d, block = 2, 3, 10, 3, 128, 128
    N = nb * block
    Q, K, V = _gauss(B, H, N, d, torch.bfloat16, 91)
    g = torch.Generator(device=DEV)
    g.manual_seed(92)
    dO = torch.randn(B, H, N, d, generator=g, device=DEV).to(torch.bfloat16)
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, block, centroids_bf16=True)
    idx, _ = bd.route(st, (B, H, N, d, block), "dot", k)
    L = torch.empty(B, H, N, device=DEV, dtype=torch.float32)
    O = bd.sparse_attn_fwd(Q, K, V, idx, block, tail, st, s, lse=L)
    grads = bd.sparse_attn_bwd(Q, K, V, O, dO, idx, block, tail, st, s)
    grads_lse = bd.sparse_attn_bwd(Q, K, V, O, dO, idx, block, tail, st, s, lse=L)
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle.sparse_attention_backward(np64(Q), np64(K), np64(V), idx.cpu().numpy(), block, tail, s, np64(dO))
    for got_set, what in ((grads, "recomputed lse"), (grads_lse, "forward's lse")):
        for got, r, name in zip(got_set, ref, ("dQ", "dK", "dV")):
            assert_tol(np64(got), r, (3e-2, 2e-3), f"batched backward ({what}) {tail} {name}")


@pytest.mark.parametrize("B,H,nb,k", [(1, 2, 9, 3), (1, 2, 37, 5), (1, 1, 133, 13), (1, 2, 20, 0), (1, 2, 8, 8),
                                      (2, 3, 10, 3)])
def test_backward_first_order(lib, B, H, nb, k):
    # PISA's hybrid order: inputs whose values follow the keys' in-block
    # deviations, so the first-order terms move the gradients well past the
    # tolerance (checked against the zero-order backward of the same inputs)
    block, d = 128, 128
    inp = wl.block_linear_inputs(B, H, nb, block, d, torch.bfloat16, 130 + nb + k, DEV)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    N = nb * block
    g = torch.Generator(device=DEV)
    g.manual_seed(131)
    dO = torch.randn(B, H, N, d, generator=g, device=DEV).to(torch.bfloat16)
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, block, centroids_bf16=True, first_order=True)
    idx, _ = bd.route(st, (B, H, N, d, block), "dot", k)
    L = torch.empty(B, H, N, device=DEV, dtype=torch.float32)
    O = bd.sparse_attn_fwd(Q, K, V, idx, block, "first_order", st, s, lse=L)
    grads = bd.sparse_attn_bwd(Q, K, V, O, dO, idx, block, "first_order", st, s)
    grads_lse = bd.sparse_attn_bwd(Q, K, V, O, dO, idx, block, "first_order", st, s, lse=L)
    torch.cuda.synchronize()
    assert_no_device_error()
    args = (np64(Q), np64(K), np64(V), idx.cpu().numpy(), block)
    ref = oracle.sparse_attention_backward(*args, "first_order", s, np64(dO))
    zo = oracle.sparse_attention_backward(*args, "zero_order", s, np64(dO))
    # the centroid logits use the bf16 block means: up to s Σ_c |q_c k̄_c| 2^-9
    # per logit, ~5e-3 in log2 units for these keys (centroids ~ N(0, 1))
    np.testing.assert_allclose(np64(L), oracle.sparse_attention_lse(np64(Q), np64(K), idx.cpu().numpy(), block,
                                                                    "first_order", s), rtol=0, atol=1e-2)
    for got_set, what in ((grads, "recomputed lse"), (grads_lse, "forward's lse")):
        for got, r, name in zip(got_set, ref, ("dQ", "dK", "dV")):
            sc = max(1.0, float(np.abs(r).max()))
            assert_tol(np64(got), r, (2e-2 * sc, 2e-3), f"first-order backward ({what}) {name}")
    if k < nb:
        assert max(float(np.abs(r - z).max()) for r, z in zip(ref, zo)) > 0.1


def test_backward_of_the_e4m3_forward_straight_through(lib):
    # SLA2 §2C: the forward of the sparse branch runs in e4m3, the backward in
    # 16 bits.  Straight-through: the bf16 backward at the unquantised
    # operands, δ = dO·O from the forward that ran.  The GPU backward given the
    # oracle's e4m3 forward output matches the oracle's straight-through
    # backward; dV (Pᵀ dO) does not depend on the forward's output at all.
    B, H, nb, k, d, block = 1, 2, 12, 3, 128, 128
    N = nb * block
    Q, K, V = _gauss(B, H, N, d, torch.bfloat16, 140)
    g = torch.Generator(device=DEV)
    g.manual_seed(141)
    dO = torch.randn(B, H, N, d, generator=g, device=DEV).to(torch.bfloat16)
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, block, centroids_bf16=True)
    idx, _ = bd.route(st, (B, H, N, d, block), "dot", k)
    O8 = bd.sparse_attn_fwd_fp8(bd.fp8_operands(Q, K, V, st), (B, H, N, d, block), idx, "zero_order", s)
    g8 = bd.sparse_attn_bwd(Q, K, V, O8, dO, idx, block, "zero_order", st, s)
    args = (np64(Q), np64(K), np64(V), idx.cpu().numpy(), block)
    emu = oracle.fp8_attention(*args, "zero_order", s)
    Oe = torch.as_tensor(emu).to(DEV, torch.bfloat16)
    ge = bd.sparse_attn_bwd(Q, K, V, Oe, dO, idx, block, "zero_order", st, s)
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle.sparse_attention_backward(*args, "zero_order", s, np64(dO), o_forward=emu)
    for got, r, name in zip(ge, ref, ("dQ", "dK", "dV")):
        assert_tol(np64(got), r, (3e-2, 2e-3), f"straight-through backward {name}")
    assert torch.equal(g8[2], ge[2])


@pytest.mark.parametrize("B,H,nb,k", [(1, 2, 9, 3), (1, 1, 37, 5), (1, 2, 20, 0), (1, 2, 8, 8), (2, 3, 10, 3)])
def test_backward_linear_mix(lib, B, H, nb, k):
    # SLA2's mixture: α per head and channel in (0.2, 0.9); the linear branch's
    # share of the gradients checked against the drop backward of α⊙dO
    block, d = 128, 128
    N = nb * block
    Q, K, V = _gauss(B, H, N, d, torch.bfloat16, 150 + nb + k)
    g = torch.Generator(device=DEV)
    g.manual_seed(151)
    dO = torch.randn(B, H, N, d, generator=g, device=DEV).to(torch.bfloat16)
    alpha = (0.2 + 0.7 * torch.rand(H, d, generator=g, device=DEV)).contiguous()
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, block, linear=True)
    idx, _ = bd.route(st, (B, H, N, d, block), "dot", k)
    O = bd.sparse_attn_fwd(Q, K, V, idx, block, "linear_mix", st, s, alpha=alpha)
    grads = bd.sparse_attn_bwd_linear_mix(Q, K, V, O, dO, idx, block, alpha, st, s)
    torch.cuda.synchronize()
    assert_no_device_error()
    args = (np64(Q), np64(K), np64(V), idx.cpu().numpy(), block)
    ref = oracle.sparse_attention_backward(*args, "linear_mix", s, np64(dO), alpha=np64(alpha))
    drop = oracle.sparse_attention_backward(*args, "drop", s, np64(dO) * np64(alpha)[None, :, None, :])
    for got, r, name in zip(grads, ref, ("dQ", "dK", "dV")):
        sc = max(1.0, float(np.abs(r).max()))
        assert_tol(np64(got), r, (2e-2 * sc, 2e-3), f"linear-mix backward {name}")
    if k < nb:
        assert max(float(np.abs(r - z).max()) for r, z in zip(ref, drop)) > 0.05


def test_backward_first_order_is_rejected_off_the_tensor_cores(lib):
    Q, K, V = _gauss(1, 1, 512, 64, torch.float32, 132)
    st = bd.block_pool(Q, K, V, 64, first_order=True)
    idx, _ = bd.route(st, (1, 1, 512, 64, 64), "dot", 2)
    O = bd.sparse_attn_fwd(Q, K, V, idx, 64, "first_order", st, 0.125)
    with pytest.raises(bd.SparseAttnError) as e:
        bd.sparse_attn_bwd(Q, K, V, O, O, idx, 64, "first_order", st, 0.125)
    assert e.value.status == bd.SA_ERR_UNSUPPORTED


@pytest.mark.parametrize("tail", ["zero_order", "drop"])
@pytest.mark.parametrize("nb,k", [(12, 3), (133, 13), (20, 0), (8, 8)])
def test_forward_lse_and_backward_lse(lib, tail, nb, k):
    # sa_sparse_attn_fwd_lse: O unchanged, lse2 against the oracle's row
    # log-sum-exp; sa_sparse_attn_bwd_lse: gradients against the oracle
    B, H, N, d, block = 1, 2, nb * 128, 128, 128
    Q, K, V = _gauss(B, H, N, d, torch.bfloat16, 80 + nb + k)
    g = torch.Generator(device=DEV)
    g.manual_seed(81)
    dO = torch.randn(B, H, N, d, generator=g, device=DEV).to(torch.bfloat16)
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, block, centroids_bf16=True)
    idx, _ = bd.route(st, (B, H, N, d, block), "dot", k)
    O_plain = bd.sparse_attn_fwd(Q, K, V, idx, block, tail, st, s)
    L = torch.empty(B, H, N, device=DEV, dtype=torch.float32)
    O = bd.sparse_attn_fwd(Q, K, V, idx, block, tail, st, s, lse=L)
    dQ, dK, dV = bd.sparse_attn_bwd(Q, K, V, O, dO, idx, block, tail, st, s, lse=L)
    torch.cuda.synchronize()
    assert_no_device_error()
    assert torch.equal(O, O_plain)
    ref_l = oracle.sparse_attention_lse(np64(Q), np64(K), idx.cpu().numpy(), block, tail, s)
    got_l = L.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isfinite(got_l), np.isfinite(ref_l))
    fin = np.isfinite(ref_l)
    # log2 units: the approximate exponentials (≤ 1e-4 relative per term) and
    # the bf16 centroids move it by well under 2e-3
    np.testing.assert_allclose(got_l[fin], ref_l[fin], rtol=0, atol=2e-3)
    rQ, rK, rV = oracle.sparse_attention_backward(np64(Q), np64(K), np64(V), idx.cpu().numpy(), block, tail, s,
                                                  np64(dO))
    for got, ref, name in ((dQ, rQ, "dQ"), (dK, rK, "dK"), (dV, rV, "dV")):
        assert_tol(np64(got), ref, (3e-2, 2e-3), f"backward with lse {tail} {name}")


@pytest.mark.parametrize("tail", ["zero_order", "drop"])
@pytest.mark.parametrize("dtype,d,block,nb,k", [
    (torch.float32, 64, 64, 9, 2),
    (torch.bfloat16, 128, 128, 12, 3),
    (torch.bfloat16, 128, 128, 133, 13),    # two centroid tiles, the second ragged
    (torch.bfloat16, 128, 128, 20, 0),      # zero-order: centroids only; drop: no key at all
    (torch.bfloat16, 128, 128, 8, 8),       # every block selected: the centroid tile fully masked
    (torch.bfloat16, 128, 64, 10, 0),
    (torch.bfloat16, 64, 128, 6, 6),        # every block selected
])
def test_backward(lib, tail, dtype, d, block, nb, k):
    B, H, N = 1, 2, nb * block
    Q, K, V = _gauss(B, H, N, d, dtype, 60 + nb + k)
    g = torch.Generator(device=DEV)
    g.manual_seed(61)
    dO = torch.randn(B, H, N, d, generator=g, device=DEV).to(dtype)
    s = 1 / math.sqrt(d)
    st = bd.block_pool(Q, K, V, block, centroids_bf16=(dtype == torch.bfloat16))
    idx, _ = bd.route(st, (B, H, N, d, block), "dot", k)
    O = bd.sparse_attn_fwd(Q, K, V, idx, block, tail, st, s)
    dQ, dK, dV = bd.sparse_attn_bwd(Q, K, V, O, dO, idx, block, tail, st, s)
    torch.cuda.synchronize()
    assert_no_device_error()
    # the oracle differentiates its own float64 forward at the same inputs;
    # the GPU uses its (rounded) forward output O for δ = dO·O
    rQ, rK, rV = oracle.sparse_attention_backward(np64(Q), np64(K), np64(V), idx.cpu().numpy(), block, tail, s,
                                                  np64(dO))
    tol = (1e-4, 1e-5) if dtype == torch.float32 else (3e-2, 2e-3)
    for got, ref, name in ((dQ, rQ, "dQ"), (dK, rK, "dK"), (dV, rV, "dV")):
        assert_tol(np64(got), ref, tol, f"backward {tail} {name}")
