"""CPU checks of the seeded input recipe shared by the tests, the bench and
smoke(): every block is reproducible from its own seed, bf16 inputs are the
round-to-nearest-even of the fp32 draw, the outlier workload scales exactly
floor(0.01 L) key rows per (b, kv head) by 8, and the decode workload's lengths
cross the multiple of w_pretrained where the recipe says."""
import math

import numpy as np

from rope_context_extension_jet_b200 import inputs as I


def small(outlier_frac=0.0, dtype="bf16"):
    return I.PrefillWorkload("t", 7, dtype, 2, 4, 2, 32, 1000, 256, 50, 1e4, outlier_frac=outlier_frac)


def test_inputs_are_reproducible():
    w = small(0.01)
    a, b = I.prefill_inputs(w), I.prefill_inputs(w)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_each_block_comes_from_its_own_seed():
    for dtype in ("bf16", "fp32"):
        w = small(dtype=dtype)
        q, k, v = I.prefill_inputs(w)
        for arr, base, nheads in ((q, 1000, w.Hq), (k, 2000, w.Hkv), (v, 3000, w.Hkv)):
            for b in range(w.B):
                for h in range(nheads):
                    c = b * nheads + h
                    x = np.random.default_rng([base + w.index, c]).standard_normal((w.L, w.d), dtype=np.float32)
                    want = I.to_bf16_bits(x) if dtype == "bf16" else x
                    np.testing.assert_array_equal(arr[b, h], want)


def test_outlier_rows_are_exactly_one_percent_scaled_by_eight():
    w = small(0.01)
    mask = I.outlier_rows(w)
    assert mask.shape == (w.B, w.Hkv, w.L)
    assert (mask.sum(axis=2) == math.floor(0.01 * w.L)).all()
    _, k, _ = I.prefill_inputs(w)
    for b in range(w.B):
        for h in range(w.Hkv):
            c = b * w.Hkv + h
            x = np.random.default_rng([2000 + w.index, c]).standard_normal((w.L, w.d), dtype=np.float32)
            x[mask[b, h]] *= np.float32(8.0)
            np.testing.assert_array_equal(k[b, h], I.to_bf16_bits(x))
    # the other tensors do not depend on the outliers
    q0, _, v0 = I.prefill_inputs(small(0.0))
    q1, _, v1 = I.prefill_inputs(w)
    np.testing.assert_array_equal(q0, q1)
    np.testing.assert_array_equal(v0, v1)


def test_decode_lengths_cross_the_group_boundary_mid_pass():
    w = I.D
    lens = [w.length_at(t) for t in range(w.steps)]
    assert lens[0] == 131041 and lens[-1] == 131104 and lens[-1] <= w.Lcap
    g = [max(1, -(-L // w.w_pretrained)) for L in lens]
    assert g[:32] == [4] * 32 and g[32:] == [5] * 32


def test_sampled_rows_cover_the_edges():
    w = I.C4
    rows = I.sampled_rows(w, heads=[0])
    i = set(rows[:, 2].tolist())
    assert set(range(64)) <= i and set(range(w.L - 64, w.L)) <= i
    assert set(range(w.w0 - 2, w.w0 + 3)) <= i
    for m in range(w.w_pretrained, w.L, w.w_pretrained):
        assert set(range(m - 2, m + 3)) <= i
    assert (rows[:, 0] == 0).all() and (rows[:, 1] == 0).all()
    small_w = small()
    assert len(I.sampled_rows(small_w)) == small_w.B * small_w.Hq * small_w.L
