"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times: the whole step runs on the device, then sampled query blocks
(prefill) or sampled (sequence, KV head) groups (decode) are recomputed by the
oracle with the GPU's own selection, and the selection itself is checked
bit-exactly against the oracle's top-k of the GPU's scores."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_approximate_b200 import binding as bd
from block_sparse_approximate_b200 import workloads as wl
from block_sparse_approximate_b200.pipeline import DecodeStep, Fp8PrefillStep, PrefillStep
from tests._parity import (BF16_TOL, assert_fp8_bound, assert_no_device_error, assert_tol, check_topk_exact,
                           np64, selection_agreement)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sample_blocks(H, nqb, n, seed):
    rng = np.random.default_rng(seed)
    picks = {(0, h, nqb - 1 if h % 2 else 0) for h in range(min(H, 4))}   # first/last blocks
    while len(picks) < n:
        picks.add((0, int(rng.integers(H)), int(rng.integers(nqb))))
    return sorted(picks)


@pytest.mark.parametrize("name", ["video_dit", "video_dit_pisa", "sla2_mix"])
def test_prefill_full_size_sampled(lib, name):
    w = wl.WORKLOADS[name]
    inp = wl.prefill_inputs(w, DEV)
    step = PrefillStep(w, inp, want_scores=True)
    O = step()
    torch.cuda.synchronize()
    assert_no_device_error()
    buf = step.buf
    check_topk_exact(buf.block_idx, buf.scores, w.k)
    ref_sc = oracle.route_scores(np64(buf.stats["qmean"]), np64(buf.stats["kmean"]), w.route,
                                 proj_q=None if "proj_q" not in inp else np64(inp["proj_q"]),
                                 proj_k=None if "proj_k" not in inp else np64(inp["proj_k"]),
                                 covnorm=None if "covnorm" not in buf.stats else np64(buf.stats["covnorm"]),
                                 scale=w.scale, block=w.block)
    assert selection_agreement(np64(buf.scores[0, :2]), ref_sc[0, :2], w.k) >= 0.95
    picks = _sample_blocks(w.H, w.nb, 12, 1)
    heads = sorted({h for _, h, _ in picks})
    hmap = {h: r for r, h in enumerate(heads)}
    idx = buf.block_idx[:, heads].cpu().numpy()
    sub = {n: inp[n][:, heads].cpu().float().numpy() for n in ("Q", "K", "V")}
    alpha = None if "alpha" not in inp else np64(inp["alpha"])[heads]
    ref = oracle.sparse_attention(sub["Q"], sub["K"], sub["V"], idx, w.block, w.tail, w.scale,
                                  alpha=alpha, qblocks=[(b, hmap[h], i) for b, h, i in picks])
    got = np.stack([np64(O[b, h, i * w.block:(i + 1) * w.block]) for b, h, i in picks])
    mx, mn = assert_tol(got, ref, BF16_TOL, name)
    print(f"parity {name}: max-abs {mx:.3e} mean-abs {mn:.3e} over {len(picks)} sampled query blocks")


@pytest.mark.parametrize("name,stats_dtype", [("decode", "bf16"), ("decode", "f32"), ("decode_rla", "bf16")])
def test_decode_full_size_sampled(lib, name, stats_dtype):
    w = wl.WORKLOADS[name]
    inp = wl.decode_inputs(w, DEV)
    sb = stats_dtype == "bf16"
    st = bd.block_pool(None, inp["Kcache"], inp["Vcache"], w.block, variance=True,
                       residual=(w.tail == "residual_linear"), centroids_bf16=sb)
    step = DecodeStep(w, inp, bd.decode_stats_bf16(st) if sb else st)
    o = step()
    torch.cuda.synchronize()
    assert_no_device_error()
    check_topk_exact(step.idx, step.scores, w.k)
    pairs = [(0, 0), (7, 3), (15, 7)]
    g = w.H // w.Hkv
    q = np64(inp["q"])
    errs = []
    for b, kh in pairs:
        Kh = inp["Kcache"][b:b + 1, kh:kh + 1].cpu().float().numpy()
        Vh = inp["Vcache"][b:b + 1, kh:kh + 1].cpu().float().numpy()
        qg = q[b:b + 1, kh * g:(kh + 1) * g]
        ref_o, _, ref_sc = oracle.decode_attention(qg, Kh, Vh, w.block, w.k, w.scale, tail=w.tail,
                                                   block_idx=step.idx[b:b + 1, kh:kh + 1].cpu().numpy())
        if sb:
            # the scores of the bf16-rounded statistics; a float32 and a
            # float64 mean can round to neighbouring bf16 values (~1e-4 in a score)
            ost = oracle.block_pool(None, Kh, Vh, w.block, variance=True)
            r16 = lambda x: torch.as_tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
            ref_sc = oracle.decode_route_scores(qg, r16(ost["kmean"]), r16(ost["kvar"]), w.scale)
            selection_agreement(np64(step.scores[b, kh]), ref_sc[0, 0], w.k, gap_rel=1e-3)
        else:
            selection_agreement(np64(step.scores[b, kh]), ref_sc[0, 0], w.k)  # asserts on clear gaps
        errs.append(assert_tol(np64(o[b, kh * g:(kh + 1) * g]), ref_o[0], BF16_TOL, f"decode b={b} g={kh}"))
    print(f"parity {name} ({stats_dtype} statistics): max-abs {max(e[0] for e in errs):.3e} "
          f"mean-abs {np.mean([e[1] for e in errs]):.3e} over {len(pairs)} (sequence, KV head) pairs")


def _fp8_full_size_run():
    w = wl.WORKLOADS["fp8"]
    inp = wl.prefill_inputs(w, DEV)
    step = Fp8PrefillStep(w, inp)
    O = step()
    torch.cuda.synchronize()
    assert_no_device_error()
    picks = _sample_blocks(w.H, w.nb, 12, 3)
    heads = sorted({h for _, h, _ in picks})
    hmap = {h: r for r, h in enumerate(heads)}
    idx = step.buf.block_idx[:, heads].cpu().numpy()
    sub = {n: inp[n][:, heads].cpu().float().numpy() for n in ("Q", "K", "V")}
    qb = [(b, hmap[h], i) for b, h, i in picks]
    got = np.stack([np64(O[b, h, i * w.block:(i + 1) * w.block]) for b, h, i in picks])
    return w, got, (sub["Q"], sub["K"], sub["V"], idx, w.block, w.tail, w.scale), qb


def test_fp8_full_size_sampled(lib):
    # e4m3 sparse branch against the oracle's quantised forward, within the
    # bound of P's e4m3 rounding and the bf16 store
    _, got, args, qb = _fp8_full_size_run()
    emu = oracle.fp8_attention(*args, qblocks=qb)
    emu_abs = oracle.fp8_attention(*args, qblocks=qb, absolute_values=True)
    assert_fp8_bound(got, emu, emu_abs, "fp8 full size vs quantised forward")
    ref = oracle.sparse_attention(*args, qblocks=qb)
    err, err_emu = np.abs(got - ref), np.abs(emu - ref)
    print(f"fp8 vs unquantised float64 oracle: max-abs {err.max():.3e} mean-abs {err.mean():.3e} "
          f"(the exact e4m3 forward: {err_emu.max():.3e} / {err_emu.mean():.3e})")


@pytest.mark.xfail(strict=True, reason="e4m3 format limit on these inputs: rounding Q, K, V to e4m3 with P "
                   "kept exact already moves the output 0.34 max-abs / 0.020 mean-abs from the "
                   "unquantised oracle (V alone: 0.10 / 0.004)")
def test_fp8_full_size_within_fp8_tolerance_of_unquantised_oracle(lib):
    # the e4m3 workload's stated tolerance against the unquantised float64
    # oracle: max-abs 6e-2, mean-abs 6e-3
    _, got, args, qb = _fp8_full_size_run()
    ref = oracle.sparse_attention(*args, qblocks=qb)
    assert_tol(got, ref, (6e-2, 6e-3), "fp8 full size vs unquantised oracle")


def test_sfa_full_size_sampled(lib):
    w = wl.WORKLOADS["sfa"]
    inp = wl.prefill_inputs(w, DEV)
    kf = w.extra["kf"]
    _, _, Qs = bd.sfa_encode(inp["Q"], kf)
    _, _, Ks = bd.sfa_encode(inp["K"], kf)
    O = bd.sfa_attn_fwd(Qs, Ks, inp["V"], w.block, w.scale)
    torch.cuda.synchronize()
    assert_no_device_error()
    rng = np.random.default_rng(5)
    rows = np.sort(np.concatenate([[0, w.N - 1], rng.choice(w.N, 30, replace=False)]))
    for h in (0, w.H - 1):
        sub = {n: inp[n][:, h:h + 1].cpu().float().numpy() for n in ("Q", "K", "V")}
        ref = oracle.sfa_attention(sub["Q"], sub["K"], sub["V"], kf, w.scale, rows=rows)
        assert_tol(np64(O[:, h:h + 1, rows]), ref, BF16_TOL, f"sfa head {h}")


def test_backward_full_size_heads(lib):
    # the video_dit backward on the GPU (all 12 heads); the oracle recomputes
    # two whole heads (every dQ, dK, dV entry of them)
    w = wl.WORKLOADS["video_dit"]
    inp = wl.prefill_inputs(w, DEV)
    step = PrefillStep(w, inp)
    O = step()
    g = torch.Generator(device=DEV)
    g.manual_seed(99)
    dO = torch.randn(O.shape, generator=g, device=DEV).to(O.dtype)
    dQ, dK, dV = bd.sparse_attn_bwd(inp["Q"], inp["K"], inp["V"], O, dO, step.buf.block_idx, w.block, w.tail,
                                    step.buf.stats, w.scale)
    # the same through the forward's log-sum-exp (as bench.py times it)
    L = torch.empty(O.shape[:3], device=DEV, dtype=torch.float32)
    O2 = bd.sparse_attn_fwd(inp["Q"], inp["K"], inp["V"], step.buf.block_idx, w.block, w.tail, step.buf.stats,
                            w.scale, lse=L)
    grads_lse = bd.sparse_attn_bwd(inp["Q"], inp["K"], inp["V"], O2, dO, step.buf.block_idx, w.block, w.tail,
                                   step.buf.stats, w.scale, lse=L)
    torch.cuda.synchronize()
    assert_no_device_error()
    assert torch.equal(O2, O)
    for h in (0, w.H - 1):
        sl = slice(h, h + 1)
        sub = {n: inp[n][:, sl].cpu().float().numpy() for n in ("Q", "K", "V")}
        rQ, rK, rV = oracle.sparse_attention_backward(sub["Q"], sub["K"], sub["V"],
                                                      step.buf.block_idx[:, sl].cpu().numpy(), w.block, w.tail,
                                                      w.scale, np64(dO[:, sl]))
        for got, ref, name in ((dQ, rQ, "dQ"), (dK, rK, "dK"), (dV, rV, "dV")):
            # bf16 storage of O enters δ = dO·O (≈2^-9 relative per entry), and a
            # key's dK / dV sums ds·q / p·dO over every row of every query block
            # that selected it (thousands of rows here), so the bound scales with
            # the gradient's own size
            scale_ref = max(1.0, float(np.abs(ref).max()))
            assert_tol(np64(got[:, sl]), ref, (2e-2 * scale_ref, 2e-3), f"backward head {h} {name}")
        for got, ref, name in zip(grads_lse, (rQ, rK, rV), ("dQ", "dK", "dV")):
            scale_ref = max(1.0, float(np.abs(ref).max()))
            assert_tol(np64(got[:, sl]), ref, (2e-2 * scale_ref, 2e-3), f"backward (forward's lse) head {h} {name}")
