"""Pins of the oracle's e4m3 forward (SLA2 §2C, low-precision sparse branch)
beyond the format itself: the zero-order tail's centroids, and how far the
quantised forward lies from the unquantised one on the e4m3 workload.

The centroid path of ``oracle.fp8_attention`` rounds each block's key mean
k̄_j and value mean vsum_j / B to bfloat16 and then to e4m3 with one absmax
scale per group of 128 blocks.  The worked example below is built so that
every one of those steps has a value whose rounding was derived by hand: a
dropped bf16 rounding, a scale taken over the wrong group (or over all
blocks) or vsum_j used in place of vsum_j / B each changes the output, and
the test checks that each such mistake would be caught.
"""
import numpy as np

import oracle

# block size, channels, blocks: 130 blocks make two centroid groups (128 + 2)
BLK, D, NB = 4, 2, 130
S = 0.5
P = (1 + 2.0 ** -4 + 2.0 ** -12) / 64   # bf16 drops the 2^-12 bit; e4m3 then meets a tie


def _blocks(vals):
    """[1,1,NB*BLK,D] with every token of block j equal to vals[j]."""
    X = np.zeros((NB, D))
    for j, v in vals.items():
        X[j] = v
    return np.repeat(X, BLK, axis=0)[None, None]


def _case():
    Q = np.tile(np.array([0.875, 0.0]), (NB * BLK, 1))[None, None]   # absmax 0.875 = 448 * 2^-9
    # block 0 is the selected block; the others are the zero-order tail.
    # centroid group 0 (blocks 0..127): absmax 7 -> scale 2^-6;
    # group 1 (blocks 128, 129): absmax 14 -> scale 2^-5
    K = _blocks({0: (7.0, -3.5), 2: (P, 0.0), 3: (3 * 2.0 ** -15, 0.0), 128: (0.0, 14.0),
                 129: (3 * 2.0 ** -15, 0.0)})
    V = _blocks({0: (7.0, 0.0), 2: (P, 0.0), 3: (0.0, 3 * 2.0 ** -15), 128: (14.0, 0.0),
                 129: (0.0, 3 * 2.0 ** -15)})
    idx = np.arange(NB).reshape(1, 1, NB, 1)   # query block 0 selects key block 0
    return Q, K, V, idx


# The hand-quantised centroids (block 0 and the zero blocks are e4m3-exact):
#  key means, group 0, scale 2^-6:
#    P -> bf16 (1 + 2^-4)/64 -> x 64 = 1.0625, halfway between e4m3 1 and
#         1.125, ties to even -> 1 -> 2^-6            (no bf16 step: 1.125/64)
#    3*2^-15 -> x 64 = 3*2^-9, the subnormal code 3 -> exact
#                                         (under 2^-5: 1.5*2^-9 -> 2*2^-9 -> 2^-13)
#  key means, group 1, scale 2^-5:
#    3*2^-15 -> x 32 = 1.5*2^-9, a tie between the subnormal codes 1 and 2,
#         to even -> 2*2^-9 -> 2^-13                   (under 2^-6: exact 3*2^-15)
#  value means: the same values in the value slots, so the same roundings.
K_HAT = {0: (7.0, -3.5), 2: (2.0 ** -6, 0.0), 3: (3 * 2.0 ** -15, 0.0), 128: (0.0, 14.0),
         129: (2.0 ** -13, 0.0)}
V_HAT = {0: (7.0, 0.0), 2: (2.0 ** -6, 0.0), 3: (0.0, 3 * 2.0 ** -15), 128: (14.0, 0.0),
         129: (0.0, 2.0 ** -13)}


def _expected(k_hat, v_hat):
    """PISA's zero-order attention on blocks holding the quantised centroids:
    constant blocks make each block mean its value, so sparse_attention sees
    exactly the tail terms the quantised forward must use."""
    Q, _, _, idx = _case()
    return oracle.sparse_attention(Q, _blocks(k_hat), _blocks(v_hat), idx, BLK, "zero_order", S,
                                   qblocks=[(0, 0, 0)])


def test_fp8_zero_order_centroids_worked_example():
    Q, K, V, idx = _case()
    got = oracle.fp8_attention(Q, K, V, idx, BLK, "zero_order", S, qblocks=[(0, 0, 0)])
    want = _expected(K_HAT, V_HAT)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)
    # the probes are live: the unquantised forward differs
    plain = oracle.sparse_attention(Q, K, V, idx, BLK, "zero_order", S, qblocks=[(0, 0, 0)])
    assert np.abs(plain - got).max() > 1e-6


def test_fp8_zero_order_worked_example_catches_plausible_mistakes():
    Q, K, V, idx = _case()
    got = oracle.fp8_attention(Q, K, V, idx, BLK, "zero_order", S, qblocks=[(0, 0, 0)])
    wrong = {
        # the bf16 step skipped: P rounds straight to 1.125 * 2^-6
        "no bf16 rounding of k̄": ({**K_HAT, 2: (1.125 * 2.0 ** -6, 0.0)}, V_HAT),
        "no bf16 rounding of v̄": (K_HAT, {**V_HAT, 2: (1.125 * 2.0 ** -6, 0.0)}),
        # one scale (2^-5) for every centroid instead of one per 128 blocks
        "one scale for all key centroids": ({**K_HAT, 3: (2.0 ** -13, 0.0)}, V_HAT),
        "one scale for all value centroids": (K_HAT, {**V_HAT, 3: (0.0, 2.0 ** -13)}),
        # group 1 quantised with group 0's scale
        "group 1 under group 0's scale": ({**K_HAT, 129: (3 * 2.0 ** -15, 0.0)}, V_HAT),
        # the block sum used as the value mean
        "vsum for vsum / B": (K_HAT, {j: tuple(BLK * np.array(v)) if j else v for j, v in V_HAT.items()}),
    }
    for name, (kh, vh) in wrong.items():
        assert np.abs(_expected(kh, vh) - got).max() > 1e-9, name


def test_fp8_zero_order_is_exact_on_representable_centroids():
    # random e4m3 values on power-of-two scales, blocks of pairs (c + e, c - e)
    # so that every block mean c is itself e4m3-exact under its group's scale:
    # every quantisation step is then lossless and the quantised forward
    # equals the float64 zero-order attention (three centroid groups)
    rng = np.random.default_rng(80)
    blk, d, nb = 4, 8, 300
    grid = np.array([0.0, 0.25, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0])   # c, c ± e stay on e4m3 values
    def make():
        c = rng.choice(grid, size=(nb, 1, d)) * rng.choice([-1, 1], size=(nb, 1, d))
        e = rng.choice([0.0, 0.5, 1.0], size=(nb, 1, d))
        X = np.concatenate([c + e, c - e, c + e, c - e], axis=1)          # block mean c
        X[:, 0, 0], X[:, 1, 0] = 7.0, 7.0                                  # block absmax 7 (scale 2^-6)
        X[:, 2, 0], X[:, 3, 0] = 7.0, 7.0
        X[::128, :, 1] = 7.0                                               # group absmax 7 as well
        return (X.reshape(1, 1, nb * blk, d) * 2.0 ** -4)
    Q, K, V = make(), make(), make()
    idx = np.stack([np.sort(rng.choice(nb, 5, replace=False)) for _ in range(nb)])[None, None]
    qb = [(0, 0, i) for i in (0, 7, 131, 299)]
    for X in (K, V):   # every block mean is e4m3-exact under its group's scale
        means = X.reshape(1, 1, nb, blk, d).mean(axis=3)
        np.testing.assert_array_equal(oracle.quantise_blocks_e4m3(means, 128)[0], means)
    a = oracle.fp8_attention(Q, K, V, idx, blk, "zero_order", 0.3, qblocks=qb)
    b = oracle.sparse_attention(Q, K, V, idx, blk, "zero_order", 0.3, qblocks=qb)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_e4m3_forward_is_far_from_the_unquantised_one_on_the_fp8_workload():
    """The e4m3 rounding of Q, K and V alone, with P kept exact, moves the
    output of the e4m3 workload (video-DiT shapes, smooth Q and K fields whose
    logits spread over ~25 per row) further than max-abs 6e-2 from the
    unquantised forward; the value rounding alone already does.  This is a
    property of the format on these inputs (3 mantissa bits: up to 2^-4
    relative error per operand), measured here on a sample of one head."""
    from block_sparse_approximate_b200 import workloads as wl
    w = wl.WORKLOADS["fp8"]
    inp = wl.prefill_inputs(w, "cpu", H=1)
    Q, K, V = (inp[n].float().numpy() for n in ("Q", "K", "V"))
    st = oracle.block_pool(Q, K, V, w.block)
    idx = oracle.topk_from_scores(oracle.route_scores(st["qmean"], st["kmean"], "dot"), w.k)
    qb = [(0, 0, i) for i in np.random.default_rng(0).choice(w.nb, 8, replace=False)]
    ref = oracle.sparse_attention(Q, K, V, idx, w.block, w.tail, w.scale, qblocks=qb)
    emu = oracle.fp8_attention(Q, K, V, idx, w.block, w.tail, w.scale, qblocks=qb)
    v_only = oracle.sparse_attention(Q, K, oracle.quantise_blocks_e4m3(V, w.block)[0], idx, w.block, w.tail,
                                     w.scale, qblocks=qb)
    err, err_v = np.abs(emu - ref), np.abs(v_only - ref)
    assert err.max() > 6e-2 and err.mean() > 6e-3, (err.max(), err.mean())
    assert err_v.max() > 6e-2, err_v.max()
    # this sample measures 0.37 / 0.019 (all three operands) and 0.069 / 0.0036 (V alone)
    assert err.max() < 0.5 and err.mean() < 0.03
