"""Benchmark of the block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the prefill hot path over the video-DiT workload
(B=1, H=12, N=32768 on an 8x64x64 grid, d=128, bf16, block 128, dot router,
keep 10% of KV blocks, zero-order tail): block statistics -> router ->
sparse attention.  Inputs (302 MB) are larger than L2 (126 MB) and are
generated on the device before timing.  Rank 0 prints one JSON line.

With N > 1 (torchrun, one process per GPU) every rank runs its own,
independently seeded problem of the same size: the path shards by (batch,
head) with no exchange, so the scaling is weak and no collective touches the
data path (NCCL only carries the timing max).

--impl reference times the CPU oracle (float64 numpy) on a bounded sample of
the same workload on the host cores (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_approximate_b200 import workloads as wl  # noqa: E402

WORKLOAD = "video_dit"
METRIC = "sparse-attn prefill dense-equivalent TFLOPS (block_pool+route+sparse_attn_fwd step)"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one
# attn_tc_kernel launch on the video_dit workload, from an ncu capture, keyed by
# the SHA-256 of the attention kernel's sources at capture time.  When the
# sources change the figure no longer describes the kernel and is reported as
# null until it is captured again.
ATTN_TRAFFIC = {"sources": ("csrc/attn_tc.cu", "csrc/tc_util.cuh", "csrc/common.cuh"),
                "sha256": "d73ebb7f 77c2c6eb 20b529c1", "bytes": 386.42e6}


def attn_traffic_bytes():
    import hashlib
    pkg = os.path.join(ROOT, "block_sparse_approximate_b200")
    got = []
    for rel in ATTN_TRAFFIC["sources"]:
        try:
            with open(os.path.join(pkg, rel), "rb") as f:
                got.append(hashlib.sha256(f.read()).hexdigest()[:8])
        except OSError:
            return None
    return ATTN_TRAFFIC["bytes"] if " ".join(got) == ATTN_TRAFFIC["sha256"] else None


def dense_flops(w) -> float:
    return 4.0 * w.B * w.H * float(w.N) * w.N * w.d


def algorithmic_attn_flops(w) -> float:
    """FLOPs the method performs in the attention kernel: every query row takes
    4·d FLOPs (QKᵀ and PV) per exact key (k blocks × block tokens) and per
    zero-order pseudo-key (nb − k unselected blocks); the first-order tail adds
    the row's (s q)ᵀ H̄, 2·d² FLOPs."""
    tail = w.tail in ("zero_order", "first_order")
    keys = w.k * w.block + ((w.nb - w.k) if tail else 0)
    fo = 2.0 * w.d * w.d if (w.tail == "first_order" and w.k < w.nb) else 0.0
    return (4.0 * w.d * keys + fo) * w.B * w.H * float(w.N)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        self.marks = []

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(", ") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            if len(r) >= 9:
                for n, v in zip(names, r[5:9]):
                    if v.strip() == "Active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest of the ranks' x (a device time): every rank calls it in the
    same order.  ``device`` is where the one-element reduction tensor lives
    (cuda for NCCL, cpu for gloo)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w, rank: int):
    """Rank r's problem: the same shapes, seed + 1000 r (independent problems,
    no exchange between ranks)."""
    return wl.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank}) if rank else w


def job_value(w, world: int, ms_step: float) -> float:
    """Whole-job dense-equivalent TFLOPS: every rank ran one step of w in at
    most ms_step (the max over ranks)."""
    return world * dense_flops(w) / (ms_step * 1e-3) / 1e12


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# --------------------------------------------------------------------------

def oracle_sample(w, inp_cpu: dict, n_blocks: int, seed: int = 0):
    """Runs the oracle's full path (stats of one head, route scores, top-k,
    attention) for n_blocks query blocks of one head; returns (seconds,
    dense-equivalent FLOPs of those query blocks)."""
    import oracle
    rng = np.random.default_rng(seed)
    h = int(rng.integers(w.H))
    Q = inp_cpu["Q"][:, h:h + 1].float().numpy()
    K = inp_cpu["K"][:, h:h + 1].float().numpy()
    V = inp_cpu["V"][:, h:h + 1].float().numpy()
    blocks = sorted(rng.choice(w.nb, n_blocks, replace=False).tolist())
    t0 = time.perf_counter()
    st = oracle.block_pool(Q, K, V, w.block)
    sc = oracle.route_scores(st["qmean"][:, :, blocks], st["kmean"], "dot")
    idx_sel = oracle.topk_from_scores(sc, w.k)                  # [1,1,n,k]
    idx = np.zeros((1, 1, w.nb, w.k), dtype=np.int64)
    idx[0, 0, blocks] = idx_sel[0, 0]
    oracle.sparse_attention(Q, K, V, idx, w.block, w.tail, w.scale,
                            qblocks=[(0, 0, i) for i in blocks])
    dt = time.perf_counter() - t0
    # the stats of one head serve all its query blocks: charge them pro rata
    return dt, 4.0 * w.block * n_blocks * float(w.N) * w.d


def cpu_baseline(w, inp_cpu: dict, budget_s: float = 15.0) -> dict:
    import oracle  # noqa: F401  (test infrastructure: only this leg runs it)
    n = 2
    dt, fl = oracle_sample(w, inp_cpu, n)
    while dt < budget_s / 4 and n < w.nb:
        n = min(w.nb, n * 2)
        dt, fl = oracle_sample(w, inp_cpu, n, seed=n)
    return {"value": fl / dt / 1e12, "unit": "TFLOPS", "cores": torch.get_num_threads(),
            "kind": "oracle",
            "sample": f"{n} query blocks of one head of {w.name} (of {w.H * w.nb}), full oracle path "
                      f"(stats, route, top-k, float64 attention), {dt:.1f} s; value = dense-equivalent "
                      f"FLOPs of the sample / time"}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = wl.WORKLOADS[WORKLOAD]
    inp = wl.prefill_inputs(w, "cpu")
    per_step = []
    flops = 0.0
    for i in range(args.warmup + args.steps):
        dt, fl = oracle_sample(w, inp, 2, seed=i)
        if i >= args.warmup:
            per_step.append(dt)
            flops += fl
    tot = sum(per_step)
    val = flops / tot / 1e12
    cores = torch.get_num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                                            "block": w.block, "route": w.route, "keep_pct": w.keep_pct,
                                            "tail": w.tail, "sample_per_step": "2 query blocks"},
            "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                             "sample": "each step: the oracle's full path for 2 query blocks of one head"},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------

def time_decode(steps: int = 50, warmup: int = 5, batch=None, name: str = "decode", stats_dtype: str = "bf16"):
    """Decode workload timing (separate from the prefill step): GB/s of the
    bytes the method moves per decode step.  ``batch`` shrinks the number of
    sequences (for bounded profiler captures).  ``decode_rla`` is the same
    caches with SPLA's residual linear tail.  ``stats_dtype``: the block
    statistics the decode reads, "bf16" (kmean, kvar, vsum / block as bf16
    copies) or "f32"."""
    from block_sparse_approximate_b200 import binding as bd
    from block_sparse_approximate_b200.pipeline import DecodeStep
    w = wl.WORKLOADS[name]
    rla = w.tail == "residual_linear"
    if batch:
        w = wl.Workload(**{**w.__dict__, "B": int(batch)})
    inp = wl.decode_inputs(w, "cuda")
    sb = stats_dtype == "bf16"
    st = bd.block_pool(None, inp["Kcache"], inp["Vcache"], w.block, variance=True, residual=rla, centroids_bf16=sb)
    step = DecodeStep(w, inp, bd.decode_stats_bf16(st) if sb else st)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        step()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    B, Hkv, nb, d = w.B, w.Hkv, w.nb, w.d
    kv = 2.0 * B * Hkv * w.k * w.block * d * 2          # selected K and V, bf16
    # kmean, kvar (route) and vsum (zero-order tail), bf16 or fp32, read once
    # each; the residual linear tail reads S_all (d×d fp32 per KV head) instead of vsum
    esz = 2.0 if sb else 4.0
    stats = (2.0 if rla else 3.0) * B * Hkv * nb * d * esz + (4.0 * B * Hkv * d * d if rla else 0.0)
    qo = 2.0 * B * w.H * d * 2
    byts = kv + stats + qo
    hbm, _, _, src = _peaks()
    del inp, st, step
    torch.cuda.empty_cache()
    return {"workload": name, "stats": stats_dtype, "ms": ms, "bytes_per_step": byts, "gbs": byts / ms / 1e6,
            "hbm_peak_gbs": hbm, "frac": byts / ms / 1e6 / hbm, "peak_source": src}


def _time_prefill_variant(step, attn_call, steps: int, warmup: int):
    """Times ``step`` (whole step) and ``attn_call`` (the attention launch alone)."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        step()
    e.record()
    torch.cuda.synchronize()
    ms_step = s.elapsed_time(e) / steps
    s.record()
    for _ in range(steps):
        attn_call()
    e.record()
    torch.cuda.synchronize()
    return ms_step, s.elapsed_time(e) / steps


def fp8_gemm_peak(n: int = 8192, reps: int = 10):
    """Dense e4m3 throughput of this GPU, measured here: a library GEMM
    (torch._scaled_mm, e4m3 x e4m3 -> bf16, n^3, 2·n^3 FLOPs) timed with CUDA
    events, best of `reps` after warm-up — the burst figure, like the driver's
    bf16 one.  Returns (TFLOP/s, source) or (None, reason)."""
    try:
        g = torch.Generator(device="cuda")
        g.manual_seed(0)
        a = torch.randn(n, n, generator=g, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, generator=g, device="cuda").to(torch.float8_e4m3fn).t()
        one = torch.ones((), device="cuda", dtype=torch.float32)
        mm = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            mm()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mm()
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12, f"measured here: torch._scaled_mm e4m3 {n}^3, best of {reps}"
    except Exception as e:  # no e4m3 GEMM in this torch build
        return None, f"e4m3 GEMM unavailable ({type(e).__name__})"


def time_fp8(steps: int = 10, warmup: int = 3):
    """The e4m3 sparse branch on the fp8 workload (video_dit shapes, seed 3)."""
    from block_sparse_approximate_b200 import binding as bd
    from block_sparse_approximate_b200.pipeline import Fp8PrefillStep
    w = wl.WORKLOADS["fp8"]
    inp = wl.prefill_inputs(w, "cuda")
    step = Fp8PrefillStep(w, inp)
    step()
    attn = lambda: bd.sparse_attn_fwd_fp8(step.ops, step.shape, step.buf.block_idx, w.tail, w.scale,
                                          out=step.buf.out)
    ms_step, attn_ms = _time_prefill_variant(step, attn, steps, warmup)
    _, bf16, _, src = _peaks()
    fl = algorithmic_attn_flops(w)
    ach = fl / (attn_ms * 1e-3) / 1e12
    peak, peak_src = fp8_gemm_peak()
    if peak is None:
        peak, peak_src = 2 * bf16, f"2 x {src} bf16 burst (nominal e4m3/bf16 ratio; {peak_src})"
    out = {"workload": w.name, "ms_per_step": ms_step, "attn_ms": attn_ms, "executed_tflops": ach,
           "dense_equiv_tflops": dense_flops(w) / (ms_step * 1e-3) / 1e12,
           "peak_tflops": peak, "frac": ach / peak, "peak_source": peak_src,
           "step": "block_pool + route + e4m3 quantisation of Q, K, V and centroids + sparse_attn_fwd_fp8"}
    del inp, step
    torch.cuda.empty_cache()
    return out


def time_pisa(steps: int = 10, warmup: int = 3):
    """PISA's full method on the video_dit inputs (same seed): covariance-aware
    routing and the hybrid-order tail; the step (block_pool with H̄ and M_j +
    route + attention) and the attention launch alone."""
    from block_sparse_approximate_b200 import binding as bd
    from block_sparse_approximate_b200.pipeline import PrefillStep
    w = wl.WORKLOADS["video_dit_pisa"]
    inp = wl.prefill_inputs(w, "cuda")
    step = PrefillStep(w, inp)
    step()
    attn = lambda: bd.sparse_attn_fwd(inp["Q"], inp["K"], inp["V"], step.buf.block_idx, w.block, w.tail,
                                      step.buf.stats, w.scale, out=step.buf.out)
    ms_step, attn_ms = _time_prefill_variant(step, attn, steps, warmup)
    _, bf16, _, src = _peaks()
    fl = algorithmic_attn_flops(w)
    ach = fl / (attn_ms * 1e-3) / 1e12
    out = {"workload": w.name, "ms_per_step": ms_step, "attn_ms": attn_ms, "executed_tflops": ach,
           "dense_equiv_tflops": dense_flops(w) / (ms_step * 1e-3) / 1e12,
           "peak_tflops": bf16, "frac": ach / bf16, "peak_source": f"{src} bf16 burst",
           "step": "block_pool (+ H̄ and M_j on the tensor cores) + route (cov) + sparse_attn_fwd (first_order)"}
    del inp, step
    torch.cuda.empty_cache()
    return out


def time_sfa(steps: int = 10, warmup: int = 3):
    """Sparse feature attention: top-16 feature codes of Q and K (zero-filled
    rows written by the encoder) and the online-softmax attention over every
    KV tile.  FLOPs counted as dense attention (4·N²·d per head): the tensor
    cores run the zero-filled operands at full width."""
    from block_sparse_approximate_b200 import binding as bd
    w = wl.WORKLOADS["sfa"]
    inp = wl.prefill_inputs(w, "cuda")
    kf = w.extra["kf"]
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    lib = bd.load()
    shape = bd.Shape(w.B, w.H, w.N, w.d, w.block)
    ws = torch.empty(max(int(lib.sa_sfa_workspace_size(shape)), 256), device="cuda", dtype=torch.uint8)
    qv = torch.empty(Q.shape[:-1] + (kf,), device="cuda", dtype=torch.bfloat16)
    qi = torch.empty(Q.shape[:-1] + (kf,), device="cuda", dtype=torch.uint8)
    kv, ki = torch.empty_like(qv), torch.empty_like(qi)
    Qs, Ks, O = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(Q)
    rows = Q.numel() // w.d

    def encode():
        st = bd._stream(None)
        bd._check("sa_sfa_encode", lib.sa_sfa_encode(Q.data_ptr(), rows, w.d, kf, qv.data_ptr(), qi.data_ptr(),
                                                     Qs.data_ptr(), st))
        bd._check("sa_sfa_encode", lib.sa_sfa_encode(K.data_ptr(), rows, w.d, kf, kv.data_ptr(), ki.data_ptr(),
                                                     Ks.data_ptr(), st))

    def attn():
        bd._check("sa_sfa_attn_fwd", lib.sa_sfa_attn_fwd(Qs.data_ptr(), Ks.data_ptr(), V.data_ptr(), bd.SA_BF16,
                                                         shape, float(w.scale), O.data_ptr(), ws.data_ptr(),
                                                         ws.numel(), bd._stream(None)))

    def step():
        encode()
        attn()

    ms_step, attn_ms = _time_prefill_variant(step, attn, steps, warmup)
    _, bf16, _, src = _peaks()
    fl = dense_flops(w)
    ach = fl / (attn_ms * 1e-3) / 1e12
    # the method's own work ("Scaling Attention via Feature Sparsity" §2): the
    # scores cost a (kf/d)² fraction of the dense scores (2·N²·kf²/d per
    # head, the expected overlap of two random supports being kf²/d), the
    # value product stays dense (2·N²·d per head)
    method = 2.0 * w.B * w.H * float(w.N) ** 2 * (kf * kf / w.d + w.d)
    out = {"workload": w.name, "kf": kf, "ms_per_step": ms_step, "attn_ms": attn_ms, "encode_ms": ms_step - attn_ms,
           "executed_tflops": ach, "peak_tflops": bf16, "frac": ach / bf16, "peak_source": f"{src} bf16 burst",
           "method_flops": method, "method_tflops": method / (attn_ms * 1e-3) / 1e12,
           "note": "executed = dense-counted (zero-filled operands at full width); method = (kf/d)^2-counted scores "
                   "+ dense P.V",
           "step": "sfa_encode (Q, K) + sfa_attn_fwd over every KV tile"}
    del inp, Q, K, V, Qs, Ks, O
    torch.cuda.empty_cache()
    return out


def backward_flops(w, with_lse: bool = False) -> float:
    """FLOPs the backward executes over the exact and pseudo-keys of every
    query row: per (row, key) the dQ pass forms 2·d (scores) + 2·d (dP) +
    2·d (dQ) and the key-side passes again 2·d (scores) + 2·d (dP) + 2·d (dV) +
    2·d (dK); without the forward's log-sum-exp the dQ kernel first recomputes
    the scores once more (2·d): 14·d or 16·d per (row, key)."""
    keys = w.k * w.block + ((w.nb - w.k) if w.tail in ("zero_order", "first_order") else 0)
    fl = (14.0 if with_lse else 16.0) * w.d * keys * w.B * w.H * float(w.N)
    if w.tail == "first_order":
        # PISA's first-order terms: H̄ dO_t (twice: for δ's shift and for dQ),
        # G = s Σ λ q dOᵀ, and the dK, dV products with G: 5 × 2·d² per row
        fl += 10.0 * w.d * w.d * w.B * w.H * float(w.N)
    return fl


def time_backward(steps: int = 3, warmup: int = 3, name: str = "video_dit"):
    """Backward of the video_dit prefill (zero-order tail; "video_dit_pisa":
    PISA's first-order tail): forward step once (with the rows' log-sum-exp,
    sa_sparse_attn_fwd_lse), then sa_sparse_attn_bwd_lse timed on the saved
    inputs, output, log-sum-exp and a random dO; sa_sparse_attn_bwd (which
    recomputes the log-sum-exp) is timed beside it."""
    import ctypes
    from block_sparse_approximate_b200 import binding as bd
    from block_sparse_approximate_b200.pipeline import PrefillStep
    w = wl.WORKLOADS[name]
    inp = wl.prefill_inputs(w, "cuda")
    step = PrefillStep(w, inp)
    O = step()
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    dO = torch.randn(O.shape, generator=g, device="cuda").to(O.dtype)
    lib = bd.load()
    shape = bd.Shape(w.B, w.H, w.N, w.d, w.block)
    ws = torch.empty(int(lib.sa_sparse_attn_bwd_workspace_size(shape, w.k)), device="cuda", dtype=torch.uint8)
    f = dict(device="cuda", dtype=torch.float32)
    dQ, dK, dV = torch.empty(O.shape, **f), torch.empty(O.shape, **f), torch.empty(O.shape, **f)
    buf = step.buf
    L = torch.empty(O.shape[:3], **f)
    bd.sparse_attn_fwd(inp["Q"], inp["K"], inp["V"], buf.block_idx, w.block, w.tail, buf.stats, w.scale, out=O,
                       lse=L)

    def bwd_lse():
        bd._check("sa_sparse_attn_bwd_lse", lib.sa_sparse_attn_bwd_lse(
            inp["Q"].data_ptr(), inp["K"].data_ptr(), inp["V"].data_ptr(), O.data_ptr(), dO.data_ptr(),
            L.data_ptr(), bd.SA_BF16, shape, buf.block_idx.data_ptr(), int(w.k), bd.TAIL[w.tail],
            ctypes.byref(step.cst), float(w.scale), dQ.data_ptr(), dK.data_ptr(), dV.data_ptr(), ws.data_ptr(),
            ws.numel(), bd._stream(None)))

    def bwd():
        bd._check("sa_sparse_attn_bwd", lib.sa_sparse_attn_bwd(
            inp["Q"].data_ptr(), inp["K"].data_ptr(), inp["V"].data_ptr(), O.data_ptr(), dO.data_ptr(),
            bd.SA_BF16, shape, buf.block_idx.data_ptr(), int(w.k), bd.TAIL[w.tail], ctypes.byref(step.cst),
            float(w.scale), dQ.data_ptr(), dK.data_ptr(), dV.data_ptr(), ws.data_ptr(), ws.numel(),
            bd._stream(None)))

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(steps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / steps

    ms_recompute = timed(bwd)
    ms = timed(bwd_lse)
    fl = backward_flops(w, with_lse=True)
    _, bf16, _, src = _peaks()
    ach = fl / (ms * 1e-3) / 1e12
    out = {"workload": w.name, "tail": w.tail, "ms": ms, "tflops": ach, "peak_tflops": bf16, "frac": ach / bf16,
           "peak_source": f"{src} bf16 burst", "entry": "sa_sparse_attn_bwd_lse (the forward's log-sum-exp given)",
           "ms_recompute_lse": ms_recompute,
           "tflops_recompute_lse": backward_flops(w) / (ms_recompute * 1e-3) / 1e12,
           "kernels": "bf16 tcgen05: dQ (+ δ; the lse pass only without the forward's lse); key-major dK/dV of the pseudo-keys (16 query ranges, reduced in order), then of the exact keys with the pseudo-key share added" + ("; first-order terms through H̄ on mma.sync (δ shift, G = s Σ λ q dOᵀ in ordered partial sums, the dQ, dK, dV updates)" if w.tail == "first_order" else ""),
           "flops_per_call": fl}
    del inp, step, O, dO, dQ, dK, dV, ws, L
    torch.cuda.empty_cache()
    return out


def linear_mix_flops(w) -> float:
    """Per query block: exact softmax part 4·d·(k·B)·B, the A_i accumulation
    2·d²·(k·B) and the final relu(Q)(H_tot − A_i) 2·d²·B."""
    per_qblk = 4.0 * w.d * w.k * w.block * w.block + 2.0 * w.d * w.d * w.k * w.block + 2.0 * w.d * w.d * w.block
    return per_qblk * w.B * w.H * w.nb


def time_sla2(steps: int = 2, warmup: int = 1):
    """The SLA2 mix workload (H=40, N=65536, proj router, linear mix)."""
    from block_sparse_approximate_b200 import binding as bd
    from block_sparse_approximate_b200.pipeline import PrefillStep
    w = wl.WORKLOADS["sla2_mix"]
    inp = wl.prefill_inputs(w, "cuda")
    step = PrefillStep(w, inp)
    step()

    def attn():
        import ctypes
        buf = step.buf
        bd._check("sa_sparse_attn_fwd",
                  step.lib.sa_sparse_attn_fwd(inp["Q"].data_ptr(), inp["K"].data_ptr(), inp["V"].data_ptr(),
                                              step.dtype, step.shape, buf.block_idx.data_ptr(), int(w.k),
                                              bd.TAIL[w.tail], inp["alpha"].data_ptr(), ctypes.byref(step.cst),
                                              float(w.scale), buf.out.data_ptr(),
                                              torch.cuda.current_stream().cuda_stream))
    ms_step, attn_ms = _time_prefill_variant(step, attn, steps, warmup)
    _, bf16, _, src = _peaks()
    fl = linear_mix_flops(w)
    ach = fl / (attn_ms * 1e-3) / 1e12
    out = {"workload": w.name, "ms_per_step": ms_step, "attn_ms": attn_ms, "executed_tflops": ach,
           "dense_equiv_tflops": dense_flops(w) / (ms_step * 1e-3) / 1e12,
           "peak_tflops": bf16, "frac": ach / bf16, "peak_source": f"{src} bf16 burst"}
    del inp, step
    torch.cuda.empty_cache()
    return out


def time_backward_linear_mix(steps: int = 2, warmup: int = 3):
    """Backward of the SLA2 mix workload (H=40, N=65536, linear mix):
    sa_sparse_attn_bwd_linear_mix on the step's inputs, output and a random dO.
    FLOPs: the softmax branch's drop backward recomputing its log-sum-exp,
    16·d per (row, selected key), plus the linear branch's products, 14·d² per
    row (h_j; H_U·φ(q) twice; dH_U; the dq product; the dk, dv products)."""
    import ctypes
    from block_sparse_approximate_b200 import binding as bd
    from block_sparse_approximate_b200.pipeline import PrefillStep
    w = wl.WORKLOADS["sla2_mix"]
    inp = wl.prefill_inputs(w, "cuda")
    step = PrefillStep(w, inp)
    O = step()
    g = torch.Generator(device="cuda")
    g.manual_seed(98)
    dO = torch.randn(O.shape, generator=g, device="cuda").to(O.dtype)
    lib = bd.load()
    shape = bd.Shape(w.B, w.H, w.N, w.d, w.block)
    ws = torch.empty(int(lib.sa_sparse_attn_bwd_linear_mix_workspace_size(shape, w.k)), device="cuda",
                     dtype=torch.uint8)
    f = dict(device="cuda", dtype=torch.float32)
    dQ, dK, dV = torch.empty(O.shape, **f), torch.empty(O.shape, **f), torch.empty(O.shape, **f)
    buf = step.buf

    def bwd():
        bd._check("sa_sparse_attn_bwd_linear_mix", lib.sa_sparse_attn_bwd_linear_mix(
            inp["Q"].data_ptr(), inp["K"].data_ptr(), inp["V"].data_ptr(), O.data_ptr(), dO.data_ptr(), bd.SA_BF16,
            shape, buf.block_idx.data_ptr(), int(w.k), inp["alpha"].data_ptr(), ctypes.byref(step.cst),
            float(w.scale), dQ.data_ptr(), dK.data_ptr(), dV.data_ptr(), ws.data_ptr(), ws.numel(),
            bd._stream(None)))

    for _ in range(warmup):
        bwd()
    torch.cuda.synchronize()
    s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s_.record()
    for _ in range(steps):
        bwd()
    e_.record()
    torch.cuda.synchronize()
    ms = s_.elapsed_time(e_) / steps
    fl = (16.0 * w.d * w.k * w.block + 14.0 * w.d * w.d) * w.B * w.H * float(w.N)
    _, bf16, _, src = _peaks()
    ach = fl / (ms * 1e-3) / 1e12
    out = {"workload": w.name, "tail": w.tail, "ms": ms, "tflops": ach, "peak_tflops": bf16, "frac": ach / bf16,
           "peak_source": f"{src} bf16 burst", "entry": "sa_sparse_attn_bwd_linear_mix", "flops_per_call": fl,
           "kernels": "softmax branch: tcgen05 drop backward of alpha*dO with the branch's delta; linear branch on "
                      "mma.sync (per-block h_j, per-query-block H_U, dH_U, key-major dh_j)"}
    del inp, step, O, dO, dQ, dK, dV, ws
    torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local):
    from block_sparse_approximate_b200 import binding as bd
    from block_sparse_approximate_b200.pipeline import PrefillStep
    torch.cuda.set_device(local)
    bd.load()
    if args.only in ("decode", "decode_rla"):
        if rank == 0:
            print(json.dumps({args.only: time_decode(args.steps, args.warmup, args.decode_batch, args.only,
                                                     args.decode_stats)}), flush=True)
        return 0
    if args.only == "fp8":
        if rank == 0:
            print(json.dumps({"fp8": time_fp8(args.steps, args.warmup)}), flush=True)
        return 0
    if args.only == "sla2":
        if rank == 0:
            print(json.dumps({"sla2_mix": time_sla2(args.steps, args.warmup)}), flush=True)
        return 0
    if args.only == "backward":
        if rank == 0:
            print(json.dumps({"backward": time_backward(args.steps, args.warmup),
                              "backward_first_order": time_backward(args.steps, args.warmup, "video_dit_pisa"),
                              "backward_linear_mix": time_backward_linear_mix(min(args.steps, 2), 3)}),
                  flush=True)
        return 0
    if args.only == "sfa":
        if rank == 0:
            print(json.dumps({"sfa": time_sfa(args.steps, args.warmup)}), flush=True)
        return 0
    if args.only == "pisa":
        if rank == 0:
            print(json.dumps({"pisa": time_pisa(args.steps, args.warmup)}), flush=True)
        return 0
    w = wl.WORKLOADS[WORKLOAD]
    wr = rank_workload(w, rank)
    inp = wl.prefill_inputs(wr, "cuda")
    step = PrefillStep(wr, inp)
    clocks = ClockSampler(local) if rank == 0 else None

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # timed region: K steps, attention kernel bracketed by events on the
    # launching stream (torch's current stream, which the step launches on)
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    lib = step.lib

    def attn_only():
        import ctypes
        buf = step.buf
        bd._check("sa_sparse_attn_fwd",
                  lib.sa_sparse_attn_fwd(inp["Q"].data_ptr(), inp["K"].data_ptr(), inp["V"].data_ptr(),
                                         step.dtype, step.shape, buf.block_idx.data_ptr(), int(wr.k),
                                         bd.TAIL[wr.tail], None, ctypes.byref(step.cst),
                                         float(wr.scale), buf.out.data_ptr(), stream.cuda_stream))

    def pool_route():
        import ctypes
        buf = step.buf
        s = stream.cuda_stream
        bd._check("sa_block_pool", lib.sa_block_pool(inp["Q"].data_ptr(), inp["K"].data_ptr(),
                                                     inp["V"].data_ptr(), step.dtype, step.shape,
                                                     ctypes.byref(step.cst), s))
        bd._check("sa_route", lib.sa_route(ctypes.byref(step.cst), step.shape, bd.ROUTE[wr.route],
                                           None, None, float(wr.scale), int(wr.k),
                                           buf.block_idx.data_ptr(), None, s))

    _barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.mark()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        pool_route()
        ev[i][0].record(stream)
        attn_only()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    if clocks:
        clocks.mark()
    ms_total = t0.elapsed_time(t1)
    ms_total = _max_over_ranks(ms_total, world)
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms_step = ms_total / args.steps

    # end to end: pinned host inputs -> device, step, output -> host.  Every
    # step copies its Q, K, V in and its O out inside the timed region.  Two
    # buffer sets and three streams let step i's inputs cross PCIe while step
    # i - 1 computes and step i - 2's output comes back (the copies of one
    # step still precede its kernels, and the output copy follows them); the
    # same loop on one stream (no overlap) is reported beside it.
    e2e = None
    if not args.no_e2e:
        names = ("Q", "K", "V")
        host = {n: inp[n].cpu().pin_memory() for n in names}
        inp2 = {n: (torch.empty_like(v) if n in names else v) for n, v in inp.items()}
        steps2 = (step, PrefillStep(wr, inp2))
        inps = (inp, inp2)
        hostO = [torch.empty(step.buf.out.shape, dtype=step.buf.out.dtype).pin_memory() for _ in range(2)]
        s_in, s_cp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def pipelined(n):
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_cp[b])           # step i - 2 has read this buffer's inputs
                    for nm in names:
                        inps[b][nm].copy_(host[nm], non_blocking=True)
                    ev_in[b].record(s_in)
                s_cp.wait_event(ev_in[b])
                if i >= 2:
                    s_cp.wait_event(ev_out[b])              # step i - 2's output has left this buffer
                steps2[b](stream=s_cp)
                ev_cp[b].record(s_cp)
                s_out.wait_event(ev_cp[b])
                with torch.cuda.stream(s_out):
                    hostO[b].copy_(steps2[b].buf.out, non_blocking=True)
                    ev_out[b].record(s_out)

        def serial(n):
            for _ in range(n):
                for nm in names:
                    inp[nm].copy_(host[nm], non_blocking=True)
                step()
                hostO[0].copy_(step.buf.out, non_blocking=True)

        n_e2e = max(3, min(args.steps, 10))
        times = {}
        for name, fn in (("pipelined", pipelined), ("serial", serial)):
            fn(2)
            torch.cuda.synchronize()
            _barrier(world)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            s_in.wait_stream(torch.cuda.current_stream())
            fn(n_e2e)
            torch.cuda.current_stream().wait_stream(s_out)
            torch.cuda.current_stream().wait_stream(s_cp)
            e1.record(stream)
            torch.cuda.synchronize()
            times[name] = _max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        e2e_ms = times["pipelined"]
        e2e = {"value": job_value(w, world, e2e_ms), "unit": "TFLOPS",
               "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": sum(inp[n].numel() * inp[n].element_size() for n in names),
               "d2h_bytes_per_step": step.buf.out.numel() * step.buf.out.element_size(),
               "steps": n_e2e,
               "overlap": "two buffer sets, three streams: step i's copy-in, step i-1's kernels and "
                          "step i-2's copy-out run concurrently",
               "serial_ms_per_step": times["serial"],
               "serial_value": job_value(w, world, times["serial"])}
        del steps2, inp2
        torch.cuda.empty_cache()

    decode = decode_f32 = decode_rla = fp8 = sla2 = pisa = sfa = backward = backward_fo = backward_lm = None
    if rank == 0 and args.only == "all" and not args.no_decode:
        del step
        torch.cuda.empty_cache()
        decode = time_decode(batch=args.decode_batch)
        decode_f32 = time_decode(batch=args.decode_batch, stats_dtype="f32")
        decode_rla = time_decode(batch=args.decode_batch, name="decode_rla")
        fp8 = time_fp8()
        sla2 = time_sla2()
        pisa = time_pisa()
        sfa = time_sfa()
        backward = time_backward()
        backward_fo = time_backward(name="video_dit_pisa")
        backward_lm = time_backward_linear_mix()
    ck = clocks.stop() if clocks else None

    if rank != 0:
        return 0
    hbm, bf16, bf16_sus, src = _peaks()
    attn_flops = algorithmic_attn_flops(w)
    achieved = attn_flops / (attn_ms * 1e-3) / 1e12
    cpu = None
    if not args.no_cpu:
        inp_cpu = {n: inp[n].cpu() for n in ("Q", "K", "V")}
        cpu = cpu_baseline(w, inp_cpu)
    line = {
        "metric": METRIC, "value": job_value(w, world, ms_step), "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "grid": list(w.grid), "d": w.d,
                   "block": w.block, "route": w.route, "keep_pct": w.keep_pct, "topk": w.k,
                   "tail": w.tail, "parallelism": f"replicas x{world} (independent problems)",
                   "l2": "inputs larger than L2 (302 MB vs 126 MB)"},
        "attn_ms": attn_ms,
        "executed_tflops": achieved,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                     "frac": achieved / bf16, "traffic": attn_traffic_bytes(),
                     "traffic_unit": "bytes per launch",
                     "kernel": "sparse_attn_fwd", "peak_source": f"{src} bf16 dense (burst)"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * PrefillStepLaunches(w),
        "clocks": ck,
        "decode": decode,
        "decode_f32_stats": decode_f32,
        "decode_rla": decode_rla,
        "fp8": fp8,
        "sla2_mix": sla2,
        "pisa": pisa,
        "sfa": sfa,
        "backward": backward,
        "backward_first_order": backward_fo,
        "backward_linear_mix": backward_lm,
    }
    print(json.dumps(line), flush=True)
    return 0


def PrefillStepLaunches(w) -> int:
    return 3 + (1 if w.tail == "linear_mix" else 0)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "decode_rla", "fp8", "sla2", "pisa", "sfa",
                                       "backward"],
                    default="all",
                    help="prefill: the timed step only; decode / fp8 / sla2 / pisa (covariance routing + "
                         "first-order tail): only that workload's timing")
    ap.add_argument("--decode-stats", choices=["bf16", "f32"], default="bf16",
                    help="element type of the block statistics the decode reads (--only decode / decode_rla)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="sequences in the decode workload (default: the full 16)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = _dist()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
