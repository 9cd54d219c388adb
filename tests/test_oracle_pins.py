"""Pins for the fp64 CPU oracle (CPU only; marked "not gpu").

Each test ties the oracle to something other than itself: hand-evaluated values
of G, Python's floor division, closed-form rotations, RoPE's relative-position
property, textbook numpy RoPE attention in the cases the pages say reduce to it,
the pages' inclusion-exclusion formulation, and (for decode over a standard
RoPE cache) complex-number RoPE and the composition of rotations.  The mutation tests at the end
plant plausible mistakes in copies of the oracle source and check that the pins
catch every one of them.

Page: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
(gist.science/it/paper/2607.07740), Metodologia 1 and 2.
"""
import math
import os
import tempfile

import numpy as np
import pytest

import oracle
import textbook as tb

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "group_size.txt")


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


# ----------------------------------------------------------------------------- battery
# Every pin is a function (lib) -> None that raises AssertionError on failure, so
# the same battery runs against the real oracle and against planted mutants.

def pin_group_size_table(lib):
    for L, w, G in _golden_rows():
        assert oracle.group_size(L, w, lib=lib) == G, (L, w, G)


def pin_remote_position(lib):
    for G in range(1, 8):
        for x in range(0, 300):
            assert oracle.remote_position(x, G, lib=lib) == x // G
        # each aliased position is shared by exactly G consecutive positions
        vals = [oracle.remote_position(x, G, lib=lib) for x in range(G * 20)]
        assert all(vals.count(p) == G for p in range(20))


def pin_rotation_closed_form(lib):
    # d = 4, rope_theta = 1e4: theta_0 = 1, theta_1 = 1e4^(-1/2) = 0.01 exactly.
    e = np.eye(4)
    y = oracle.rotate(e[0], 1, 1e4, lib=lib)
    np.testing.assert_allclose(y, [math.cos(1.0), 0.0, math.sin(1.0), 0.0], atol=1e-15)
    y = oracle.rotate(e[2], 1, 1e4, lib=lib)
    np.testing.assert_allclose(y, [-math.sin(1.0), 0.0, math.cos(1.0), 0.0], atol=1e-15)
    y = oracle.rotate(e[1], 3, 1e4, lib=lib)
    np.testing.assert_allclose(y, [0.0, math.cos(0.03), 0.0, math.sin(0.03)], atol=1e-15)
    y = oracle.rotate(e[3], 3, 1e4, lib=lib)
    np.testing.assert_allclose(y, [0.0, -math.sin(0.03), 0.0, math.cos(0.03)], atol=1e-15)


def pin_rotation_algebra(lib):
    rng = np.random.default_rng(7)
    for d, theta in ((8, 1e4), (64, 1e4), (128, 1e6)):
        x = rng.standard_normal(d)
        np.testing.assert_allclose(oracle.rotate(x, 0, theta, lib=lib), x, atol=0)
        for a, b in ((3, 5), (100, 27), (131000, 71)):
            # rotations compose additively (Metodologia 2, correction rotation)
            ab = oracle.rotate(oracle.rotate(x, a, theta, lib=lib), b, theta, lib=lib)
            np.testing.assert_allclose(ab, oracle.rotate(x, a + b, theta, lib=lib),
                                       rtol=0, atol=1e-9 * np.abs(x).max())
            y = oracle.rotate(x, a, theta, lib=lib)
            assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)


def pin_relative_invariance(lib):
    rng = np.random.default_rng(11)
    d, theta = 64, 1e4
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    for (a, b, s) in ((5, 2, 17), (40, 3, 1000), (1000, 999, 123456)):
        d0 = np.dot(oracle.rotate(q, a, theta, lib=lib), oracle.rotate(k, b, theta, lib=lib))
        d1 = np.dot(oracle.rotate(q, a + s, theta, lib=lib),
                    oracle.rotate(k, b + s, theta, lib=lib))
        assert abs(d0 - d1) <= 1e-9 * (abs(d0) + 1.0)
    # routed logits: local pairs invariant under any joint shift, remote pairs
    # under joint shifts by multiples of G (both aliased positions move by s).
    w0, G = 6, 3
    for i, j in ((10, 8), (30, 25), (40, 2), (21, 9)):
        l0 = oracle.pair_logit(q, k, i, j, w0, G, theta, lib=lib)
        if i - j < w0:
            for s in (1, 2, 7, 500):
                l1 = oracle.pair_logit(q, k, i + s, j + s, w0, G, theta, lib=lib)
                assert abs(l0 - l1) <= 1e-9 * (abs(l0) + 1.0)
        else:
            for s in (1, 4, 100):
                l1 = oracle.pair_logit(q, k, i + s * G, j + s * G, w0, G, theta, lib=lib)
                assert abs(l0 - l1) <= 1e-9 * (abs(l0) + 1.0)


def pin_routing_enumeration(lib):
    """Brute force over every pair with L <= 64: count the pairs routed to the exact
    branch (pair logit equal to the classic-RoPE logit and not to the aliased one)."""
    rng = np.random.default_rng(13)
    d, theta, G = 16, 1e4, 4
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    rq = {p: oracle.rotate(q, p, theta, lib=lib) for p in range(64)}
    rk = {p: oracle.rotate(k, p, theta, lib=lib) for p in range(64)}
    for L, w0 in ((64, 5), (40, 1), (33, 12), (64, 64)):
        local = 0
        for i in range(L):
            for j in range(i + 1):
                lg = oracle.pair_logit(q, k, i, j, w0, G, theta, lib=lib)
                ex = float(np.dot(rq[i], rk[j]))
                al = float(np.dot(rq[i // G], rk[j // G]))
                is_ex = abs(lg - ex) <= 1e-12 * (abs(ex) + 1)
                is_al = abs(lg - al) <= 1e-12 * (abs(al) + 1)
                assert is_ex or is_al, (i, j)
                if is_ex and not is_al:
                    local += 1
                if is_ex and is_al:
                    # only possible when both branches see the same relative offset
                    assert (i - j) == (i // G - j // G)
                    local += 1 if i - j < w0 else 0
        assert local == sum(min(i + 1, w0) for i in range(L)), (L, w0, local)


def _prefill_small(lib, L, w0, w_pre, Hq=4, Hkv=2, d=16, theta=1e4, seed=0, dtype="fp32", B=2):
    # two sequences, so the per-sequence offsets of q, k, v and out are pinned too
    q = _rand((B, Hq, L, d), seed)
    k = _rand((B, Hkv, L, d), seed + 1)
    v = _rand((B, Hkv, L, d), seed + 2)
    scale = 1.0 / math.sqrt(d)
    out = oracle.prefill(q, k, v, w0=w0, w_pretrained=w_pre, rope_theta=theta, scale=scale,
                         nthreads=2, lib=lib)
    kk = tb.repeat_kv(k.astype(np.float64), Hq // Hkv)
    vv = tb.repeat_kv(v.astype(np.float64), Hq // Hkv)
    return out, q.astype(np.float64), kk, vv, scale


def pin_reduction_g1(lib):
    # L <= w_pretrained -> G = 1: the method is classic RoPE attention for any w0
    for L, w0 in ((48, 0), (48, 5), (48, 48), (33, 7)):
        out, q, k, v, sc = _prefill_small(lib, L, w0, 64)
        ref, _ = tb.rope_attention(q, k, v, np.arange(L), 1e4, sc)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)


def pin_reduction_wide_window(lib):
    # w0 >= L -> every pair is local: classic RoPE attention whatever G is
    for L, w0, w_pre in ((48, 48, 16), (40, 100, 7), (64, 64, 9)):
        out, q, k, v, sc = _prefill_small(lib, L, w0, w_pre)
        ref, _ = tb.rope_attention(q, k, v, np.arange(L), 1e4, sc)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)


def pin_reduction_zero_window(lib):
    # w0 = 0 -> every pair is remote: classic RoPE attention at positions // G
    for L, w_pre in ((48, 16), (50, 7), (64, 20)):
        G = -(-L // w_pre)
        out, q, k, v, sc = _prefill_small(lib, L, 0, w_pre)
        ref, _ = tb.rope_attention(q, k, v, np.arange(L) // G, 1e4, sc)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)


def pin_inclusion_exclusion(lib):
    # the pages' three-pass LSE merge reaches the same routed output
    # w0 = 0: the window passes are empty (LSE -inf, weight 0) and B alone remains;
    # w0 >= L: C equals B and cancels, A alone remains
    for L, w0, w_pre in ((64, 8, 16), (64, 1, 20), (50, 13, 11), (37, 36, 5), (64, 63, 30),
                         (40, 0, 9), (40, 40, 9), (33, 1000, 7)):
        G = -(-L // w_pre)
        out, q, k, v, sc = _prefill_small(lib, L, w0, w_pre, seed=L + w0)
        ref = tb.inclusion_exclusion(q, k, v, w0, G, 1e4, sc)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-9)


def pin_decode_matches_prefill_row(lib):
    B, L, Hq, Hkv, d, w0, w_pre = 2, 45, 4, 2, 16, 6, 10
    q = _rand((B, Hq, L, d), 21)
    k = _rand((B, Hkv, L, d), 22)
    v = _rand((B, Hkv, L, d), 23)
    sc = 0.25
    rows = np.array([(b, h, L - 1) for b in range(B) for h in range(Hq)], dtype=np.int32)
    pre = oracle.prefill_rows(q, k, v, rows, w0=w0, w_pretrained=w_pre, rope_theta=1e4, scale=sc,
                              lib=lib)
    Lcap = L + 7
    kc = np.zeros((B, Hkv, Lcap, d), np.float32)
    vc = np.zeros((B, Hkv, Lcap, d), np.float32)
    kc[:, :, :L] = k
    vc[:, :, :L] = v
    kc[:, :, L:] = 1e3  # rows past L must be ignored
    dec = oracle.decode(np.ascontiguousarray(q[:, :, L - 1]), kc, vc, L, w0=w0, w_pretrained=w_pre,
                        rope_theta=1e4, scale=sc, lib=lib)
    np.testing.assert_allclose(dec.reshape(B * Hq, d), pre, rtol=0, atol=1e-13)


def pin_row_lse_textbook(lib):
    # each row's log-sum-exp equals textbook RoPE attention's, where the method
    # reduces to it: G = 1 (any window), w0 >= L, and w0 = 0 at positions // G
    L, Hq, Hkv, d, sc = 40, 4, 2, 16, 0.3
    q = _rand((1, Hq, L, d), 61)
    k = _rand((1, Hkv, L, d), 62)
    v = _rand((1, Hkv, L, d), 63)
    b, h, i = np.meshgrid(np.arange(1), np.arange(Hq), np.arange(L), indexing="ij")
    rows = np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1)
    kk = tb.repeat_kv(k.astype(np.float64), Hq // Hkv)
    vv = tb.repeat_kv(v.astype(np.float64), Hq // Hkv)
    for w0, w_pre, pos in ((7, 64, np.arange(L)), (L, 9, np.arange(L)), (0, 9, np.arange(L) // 5)):
        _, lse = oracle.prefill_rows(q, k, v, rows, w0=w0, w_pretrained=w_pre, rope_theta=1e4,
                                     scale=sc, with_lse=True, lib=lib)
        _, ref = tb.rope_attention(q.astype(np.float64), kk, vv, pos, 1e4, sc)
        np.testing.assert_allclose(lse, ref.reshape(-1), rtol=0, atol=1e-10)


def pin_rotate_rows_textbook(lib):
    # a standard RoPE cache built by the oracle equals the complex-number RoPE
    x = _rand((2, 37, 16), 31)
    got = oracle.rotate_rows(x, 1e4, lib=lib)
    ref = tb.rope_complex(x.astype(np.float64), np.arange(37), 1e4)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def _decode_case(L, Hq=4, Hkv=2, d=16, seed=40):
    q = _rand((1, Hq, d), seed)
    k = _rand((1, Hkv, L + 3, d), seed + 1)
    v = _rand((1, Hkv, L + 3, d), seed + 2)
    return q, k, v


def pin_rope_cache_decode_textbook(lib):
    # Decode over a standard RoPE cache (key row j stored rotated to j) against
    # textbook attention with the stored rows taken as they are: every pair
    # local (w0 >= L) -> query at i, keys as stored; every pair remote (w0 = 0)
    # -> query at f(i), stored key j moved by f(j) - j (complex RoPE handles the
    # negative angle).  The stored rows are arbitrary vectors here.
    L, sc, theta = 41, 0.3, 1e4
    q, kc, vc = _decode_case(L)
    group = 2
    i = L - 1
    for w0, w_pre in ((L, 9), (0, 9), (0, 41)):
        G = -(-L // w_pre)
        got = oracle.decode_rope_cache(q, kc, vc, L, w0=w0, w_pretrained=w_pre, rope_theta=theta,
                                       scale=sc, lib=lib)
        for h in range(q.shape[1]):
            kk = kc[0, h // group, :L].astype(np.float64)
            vv = vc[0, h // group, :L].astype(np.float64)
            if w0 >= L:
                qq = tb.rope_complex(q[0, h][None].astype(np.float64), np.array([i]), theta)
                keys = kk
            else:
                qq = tb.rope_complex(q[0, h][None].astype(np.float64), np.array([i // G]), theta)
                j = np.arange(L)
                keys = tb.rope_complex(kk, j // G - j, theta)
            ref, _ = tb.masked_attention(qq, keys, vv, sc, np.ones((1, L), bool))
            np.testing.assert_allclose(got[0, h], ref[0], rtol=0, atol=1e-10)


def pin_rope_cache_decode_composition(lib):
    # Rotations compose: decoding a RoPE cache built from raw keys equals
    # decoding the raw keys, for every window / group size (the cache is
    # rounded to fp32, hence the tolerance).
    L, sc, theta = 53, 0.25, 1e4
    q, k, v = _decode_case(L, seed=50)
    cache = tb.rope_complex(k.astype(np.float64), np.arange(k.shape[2]), theta).astype(np.float32)
    for w0, w_pre in ((5, 9), (0, 20), (17, 5), (60, 7), (1, 53)):
        kw = dict(w0=w0, w_pretrained=w_pre, rope_theta=theta, scale=sc, lib=lib)
        a = oracle.decode_rope_cache(q, cache, v, L, **kw)
        b = oracle.decode(q, k, v, L, **kw)
        np.testing.assert_allclose(a, b, rtol=0, atol=2e-5)


def pin_bf16_widening(lib):
    # bf16 inputs are the upper 16 bits of an fp32: the oracle on bf16 bits equals
    # the oracle on those values given as fp32 (numpy's own view of the bits)
    from rope_context_extension_jet_b200.inputs import bf16_bits_to_f32, to_bf16_bits
    L, d = 40, 16
    qb = to_bf16_bits(_rand((1, 2, L, d), 1))
    kb = to_bf16_bits(_rand((1, 2, L, d), 2))
    vb = to_bf16_bits(_rand((1, 2, L, d), 3))
    kw = dict(w0=5, w_pretrained=16, rope_theta=1e4, scale=0.25, lib=lib)
    a = oracle.prefill(qb, kb, vb, **kw)
    b = oracle.prefill(bf16_bits_to_f32(qb), bf16_bits_to_f32(kb), bf16_bits_to_f32(vb), **kw)
    np.testing.assert_array_equal(a, b)


PINS = [pin_group_size_table, pin_remote_position, pin_rotation_closed_form,
        pin_rotation_algebra, pin_relative_invariance, pin_routing_enumeration,
        pin_reduction_g1, pin_reduction_wide_window, pin_reduction_zero_window,
        pin_inclusion_exclusion, pin_decode_matches_prefill_row, pin_row_lse_textbook,
        pin_rotate_rows_textbook,
        pin_rope_cache_decode_textbook, pin_rope_cache_decode_composition, pin_bf16_widening]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.load())




def test_bf16_rounding_is_nearest_even():
    from rope_context_extension_jet_b200.inputs import bf16_bits_to_f32, to_bf16_bits
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> ties to even (1.0)
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 3.0e-3], np.float32)
    y = bf16_bits_to_f32(to_bf16_bits(x))
    assert y[0] == 1.0 and y[1] == 1.0 and y[2] == 1.0 + 2.0 ** -6 and y[3] == -2.5
    assert abs(y[4] - 3.0e-3) <= 3.0e-3 * 2.0 ** -8


# ----------------------------------------------------------------------------- mutants
# Plausible mistakes, planted in copies of the oracle source on the CPU.  Each must
# make at least one pin fail.  The snippets must exist verbatim in the source.
MUTANTS = {
    "floor_instead_of_ceil_for_G": ("if (g * w_pretrained < L) g += 1; /* ceiling */",
                                    "/* ceiling dropped */"),
    "window_boundary_le": ("if (i - j < (int64_t)c->w0) {", "if (i - j <= (int64_t)c->w0) {"),
    "query_not_aliased": ("rotate_cached(c, qraw, qm, jlo_remote_position(i, c->G));",
                          "rotate_cached(c, qraw, qm, i);"),
    "key_not_aliased": ("else rotate_cached(c, kraw, kr, fj);", "else rotate_cached(c, kraw, kr, j);"),
    "rotation_sign": ("y[m + h] = a * ss + b * cc;", "y[m + h] = -a * ss + b * cc;"),
    "interleaved_pairing": ("double a = x[m], b = x[m + h];\n        y[m] = a * cc - b * ss;\n"
                            "        y[m + h] = a * ss + b * cc;",
                            "double a = x[(2*m)%c->d], b = x[(2*m+1)%c->d];\n"
                            "        y[m] = a * cc - b * ss;\n        y[m + h] = a * ss + b * cc;"),
    "frequency_exponent": ("return pow(rope_theta, -2.0 * (double)m / (double)d);",
                           "return pow(rope_theta, -1.0 * (double)m / (double)d);"),
    "gqa_modulo": ("int kvh = h / group;", "int kvh = h % J->Hkv;"),
    "rope_cache_delta_sign": ("y[m] = a * cc + b * ss;\n        y[m + h] = -a * ss + b * cc;",
                              "y[m] = a * cc - b * ss;\n        y[m + h] = a * ss + b * cc;"),
    "rope_cache_local_rotated_again": ("if (c->rope_cache) memcpy(kr, kraw, sizeof(double) * (size_t)d);",
                                       "if (c->rope_cache) rotate_cached(c, kraw, kr, j);"),
    "rope_cache_moved_to_fj": ("if (c->rope_cache) unrotate_cached(c, kraw, kr, j - fj);",
                               "if (c->rope_cache) rotate_cached(c, kraw, kr, fj);"),
    "lse_without_max": ("if (lse) *lse = mx + log(sum);", "if (lse) *lse = log(sum);"),
    "local_query_aliased": ("            else rotate_cached(c, kraw, kr, j);\n            qq = qe;",
                            "            else rotate_cached(c, kraw, kr, j);\n            qq = qm;"),
    "scale_dropped": ("logit[j] = c->scale * a;", "logit[j] = a;"),
    "decode_query_at_L_minus_2": ("rows[3 * r + 1] = h; rows[3 * r + 2] = L - 1;",
                                  "rows[3 * r + 1] = h; rows[3 * r + 2] = L - 2;"),
    "prefill_G_from_L_minus_1": ("J.c.G = jlo_group_size(L, w_pretrained);\n    J.c.scale = scale; "
                                 "J.c.in_dtype = in_dtype; J.c.npos = npos;\n",
                                 "J.c.G = jlo_group_size(L - 1, w_pretrained);\n    J.c.scale = scale; "
                                 "J.c.in_dtype = in_dtype; J.c.npos = npos;\n"),
    "decode_G_from_Lcap": ("J.c.G = jlo_group_size(L, w_pretrained);\n    J.c.scale = scale; J.c.in_dtype = in_dtype; "
                           "J.c.npos = L; J.c.rope_cache = rope_cache;",
                           "J.c.G = jlo_group_size(Lcap, w_pretrained);\n    J.c.scale = scale; J.c.in_dtype = in_dtype; "
                           "J.c.npos = L; J.c.rope_cache = rope_cache;"),
    "decode_query_of_sequence_0": ("size_t q_off = J->q_is_decode ? ((size_t)b * J->Hq + h) * d",
                                   "size_t q_off = J->q_is_decode ? ((size_t)0 * J->Hq + h) * d"),
    "prefill_query_of_sequence_0": (": (((size_t)b * J->Hq + h) * J->L + i) * d;",
                                    ": (((size_t)0 * J->Hq + h) * J->L + i) * d;"),
    "keys_of_sequence_0": ("size_t kv_off = ((size_t)b * J->Hkv + kvh) * (size_t)J->Lkv * d;",
                           "size_t kv_off = ((size_t)0 * J->Hkv + kvh) * (size_t)J->Lkv * d;"),
    "bf16_widened_one_bit_low": ("uint32_t bits = ((uint32_t)((const uint16_t*)base)[idx]) << 16;",
                                 "uint32_t bits = ((uint32_t)((const uint16_t*)base)[idx]) << 15;"),
    "dropped_self_key": ("for (int64_t j = 0; j <= i; ++j) {\n        size_t off = kv_off + (size_t)j * d;\n"
                         "        for (int t = 0; t < d; ++t) kraw[t]",
                         "for (int64_t j = 0; j < i; ++j) {\n        size_t off = kv_off + (size_t)j * d;\n"
                         "        for (int t = 0; t < d; ++t) kraw[t]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    src = open(oracle._SRC).read()
    old, new = MUTANTS[name]
    assert old in src, f"mutation anchor for {name} not found in the oracle source"
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load(oracle.build(force=True, src=path, out=os.path.join(td, "libm.so")))
        failed = []
        for pin in PINS:
            try:
                pin(lib)
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
        assert failed, f"no pin caught the planted mistake {name}"
