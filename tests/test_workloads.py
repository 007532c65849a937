"""The seeded synthetic input generators (no method arithmetic)."""
import math

import torch

from block_sparse_approximate_b200 import workloads as wl


def test_keep_counts():
    assert wl.WORKLOADS["video_dit"].k == 26
    assert wl.WORKLOADS["sla2_mix"].k == 26
    assert wl.WORKLOADS["tiny"].k == 4
    assert wl.WORKLOADS["decode"].k == 64
    assert wl.WORKLOADS["video_dit"].nb == 256 and wl.WORKLOADS["sla2_mix"].nb == 512


def test_prefill_inputs_deterministic_and_shaped():
    w = wl.WORKLOADS["video_dit"]
    a = wl.prefill_inputs(w, H=2, N=4096)
    b = wl.prefill_inputs(w, H=2, N=4096)
    for n in ("Q", "K", "V"):
        assert a[n].shape == (1, 2, 4096, 128) and a[n].dtype == torch.bfloat16
        assert torch.equal(a[n], b[n])
    # field: 8 unit sinusoids (variance 1/2 each, sum var 4) + noise var 0.5
    var = a["Q"].float().var().item()
    assert 3.0 < var < 6.0
    # V ~ N(0,1)
    assert abs(a["V"].float().var().item() - 1.0) < 0.05
    # smooth part: neighbouring tokens along x are strongly correlated
    q = a["Q"].float()[0, 0]
    c = torch.corrcoef(torch.stack([q[:-1].flatten(), q[1:].flatten()]))[0, 1].item()
    assert c > 0.6


def test_mix_parameters():
    w = wl.WORKLOADS["sla2_mix"]
    a = wl.prefill_inputs(w, H=3, N=4096)
    assert a["alpha"].shape == (3, 128)
    assert 0.2 <= a["alpha"].min().item() and a["alpha"].max().item() <= 0.9
    assert abs(a["proj_q"].std().item() - 1 / math.sqrt(128)) < 0.005


def test_decode_inputs():
    w = wl.WORKLOADS["decode"]
    a = wl.decode_inputs(w, B=2, N=4096, Hkv=2)
    assert a["q"].shape == (2, 8, 128)
    assert a["Kcache"].shape == (2, 2, 4096, 128) and a["Kcache"].dtype == torch.bfloat16
    k = a["Kcache"].float().reshape(2, 2, 64, 64, 128)
    # block offsets of variance 0.5 on top of N(0,1) tokens
    assert abs(k.mean(dim=3).var().item() - (0.5 + 1 / 64)) < 0.05
    assert abs(k.var(dim=3).mean().item() - 1.0) < 0.05
