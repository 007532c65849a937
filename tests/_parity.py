"""Shared helpers of the GPU parity tests: tolerance checks and the glue that
runs the library's pipeline and the oracle on the same seeded inputs."""
import numpy as np
import torch

import oracle
from block_sparse_approximate_b200 import binding as bd

# bf16 outputs against the float64 oracle: max-abs and mean-abs bounds
BF16_TOL = (2e-2, 2e-3)
# fp32 outputs: the kernels accumulate in fp32 with MUFU exp2 (relative error
# ~2^-22) over at most a few thousand terms
FP32_TOL = (1e-4, 1e-5)


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_no_device_error():
    assert bd.device_error() == 0, "a kernel gave up on a bounded wait"


def assert_tol(got, ref, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mx, mn = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= tol[0] and mn <= tol[1], (f"{what}: max-abs {mx:.3e} (tol {tol[0]}), mean-abs {mn:.3e} "
                                           f"(tol {tol[1]}), max |ref| {float(np.abs(ref).max()):.3e}")
    return mx, mn


def assert_stats_close(got: torch.Tensor, ref: np.ndarray, what: str, rtol=1e-4):
    g = np64(got)
    scale = max(1.0, float(np.abs(ref).max()))
    err = float(np.abs(g - ref).max())
    assert err <= rtol * scale + 1e-5, f"{what}: max err {err:.3e} (scale {scale:.2f})"


def check_topk_exact(idx_gpu: torch.Tensor, scores_gpu: torch.Tensor, k: int):
    """The kept indices equal the oracle's top-k of the GPU's own scores (bit-exact)."""
    ref = oracle.topk_from_scores(np64(scores_gpu), k)
    got = idx_gpu.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(got, ref)


def selection_agreement(scores_gpu: np.ndarray, scores_ref: np.ndarray, k: int, gap_rel=1e-4):
    """Rows where the oracle's own top-k is separated from the (k+1)-th score by
    more than gap_rel (relative) must select the same set from both score
    tables; returns the fraction of rows that agree overall."""
    sg = scores_gpu.reshape(-1, scores_gpu.shape[-1])
    sr = scores_ref.reshape(-1, scores_ref.shape[-1])
    nb = sr.shape[1]
    if k == 0 or k == nb:
        return 1.0
    agree = 0
    for r in range(sr.shape[0]):
        a = set(oracle.topk_from_scores(sg[r], k).tolist())
        b = set(oracle.topk_from_scores(sr[r], k).tolist())
        srt = np.sort(sr[r])[::-1]
        gap = srt[k - 1] - srt[k]
        if gap > gap_rel * max(1.0, abs(srt[k - 1])):
            assert a == b, f"row {r}: selections differ although the score gap is {gap:.3e}"
        agree += a == b
    return agree / sr.shape[0]


# e4m3 rounds to nearest even with 3 mantissa bits: the relative error of a
# rounded normal value is at most 2^-4
E4M3_REL = 2.0 ** -4


def assert_fp8_bound(got, emu, emu_abs, what=""):
    """|got - emu| <= 2^-4 Σp|v|/l (P rounded to e4m3) + 2^-8 |emu| (bf16
    output) + 2e-3 (fp32 sums, e4m3 subnormals of tiny p), elementwise."""
    got = np.asarray(got, dtype=np.float64)
    bound = E4M3_REL * np.asarray(emu_abs) + 2.0 ** -8 * np.abs(emu) + 2e-3
    err = np.abs(got - emu)
    worst = float((err / bound).max())
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert worst <= 1.0, f"{what}: error reaches {worst:.2f} of the e4m3 rounding bound (max-abs {err.max():.3e})"
    return float(err.max()), float(err.mean())
