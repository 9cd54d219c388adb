"""GPU parity of jetlong_prefill against the fp64 CPU oracle (through the C ABI).

Small cases compare every output element; the 32K / 64K / 128K workloads are
run in full on the GPU and compared on the sampled rows the oracle computes
one by one.  Gates: bf16 max-abs <= 2e-2 and rel-L2 <= 5e-3; fp32 max-abs <= 1e-4.
"""
import numpy as np
import pytest

import oracle
import rope_context_extension_jet_b200 as jl
from rope_context_extension_jet_b200 import inputs as I
from helpers import check_gate, to_device, to_host_f64

pytestmark = pytest.mark.gpu


def run_prefill(w, q, k, v, poison=True):
    import torch
    qd, kd, vd = to_device(q), to_device(k), to_device(v)
    out = torch.empty_like(qd)
    if poison:
        out.fill_(float("nan"))
    jl.prefill(qd, kd, vd, out, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
               scale=w.scale)
    jl.device_status()
    return out


def full_case(w):
    q, k, v = I.prefill_inputs(w)
    out = to_host_f64(run_prefill(w, q, k, v))
    ref = oracle.prefill(q, k, v, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                         scale=w.scale)
    return check_gate(out, ref, w.dtype, w.name)


def small(name, dtype="bf16", B=1, Hq=4, Hkv=2, d=128, L=300, w_pre=100, w0=17, theta=1e6,
          outliers=0.0, index=20):
    return I.PrefillWorkload(name, index, dtype, B, Hq, Hkv, d, L, w_pre, w0, theta,
                             outlier_frac=outliers)


def test_pr1_full_output_fp32():
    """PR1: fp32, B=1, Hq=Hkv=2, d=64, L=512, G=4, w0=32 -- every output checked."""
    full_case(I.PR1)


RAGGED = [1, 2, 63, 64, 65, 127, 128, 129, 200, 513]


@pytest.mark.parametrize("L", RAGGED)
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_ragged_lengths(L, dtype):
    full_case(small(f"ragged-L{L}", dtype=dtype, L=L, w_pre=max(1, L // 3), w0=17, index=21))


W0_EDGES = [0, 1, 63, 64, 65, 127, 128, 129, 299, 300, 1000]


@pytest.mark.parametrize("w0", W0_EDGES)
def test_window_edges_bf16(w0):
    full_case(small(f"w0-{w0}", L=300, w_pre=100, w0=w0, index=22))


@pytest.mark.parametrize("w0", [0, 64, 129, 300])
def test_window_edges_fp32(w0):
    full_case(small(f"w0-{w0}-fp32", dtype="fp32", L=300, w_pre=100, w0=w0, index=23))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_head_dims(d, dtype):
    full_case(small(f"d{d}", dtype=dtype, d=d, L=700, w_pre=200, w0=150, index=24))


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (8, 1), (6, 3), (8, 8), (16, 2)])
def test_gqa_groups(Hq, Hkv):
    full_case(small(f"gqa{Hq}-{Hkv}", Hq=Hq, Hkv=Hkv, L=260, w_pre=64, w0=70, index=25))


def test_batch_and_theta():
    full_case(small("batch2-theta1e4", B=2, Hq=4, Hkv=4, L=400, w_pre=90, w0=33, theta=1e4,
                    index=26))


# Four (or eight) query heads per kv head with d = 128 take the CTA-pair kernel:
# the same edge cases again on that path.
@pytest.mark.parametrize("L", RAGGED)
def test_ragged_lengths_head_quads(L):
    full_case(small(f"quad-ragged-L{L}", Hq=4, Hkv=1, L=L, w_pre=max(1, L // 3), w0=17, index=29))


@pytest.mark.parametrize("w0", W0_EDGES)
def test_window_edges_head_quads(w0):
    full_case(small(f"quad-w0-{w0}", Hq=8, Hkv=2, L=300, w_pre=100, w0=w0, index=30))


def test_batch_and_theta_head_quads():
    full_case(small("quad-batch2-theta1e4", B=2, Hq=8, Hkv=2, L=700, w_pre=90, w0=133, theta=1e4,
                    index=31))


def test_outlier_keys_head_quads():
    full_case(small("quad-outliers", Hq=4, Hkv=1, L=1000, w_pre=500, w0=128, outliers=0.01, index=32))


def test_outlier_keys_small():
    full_case(small("outliers", L=1000, w_pre=500, w0=128, outliers=0.01, index=27))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_two_thousand_tokens_g4(dtype):
    full_case(small(f"L2048-{dtype}", dtype=dtype, Hq=4, Hkv=1, L=2048, w_pre=512, w0=300,
                    index=28))


def _sampled_case(w, heads):
    q, k, v = I.prefill_inputs(w)
    out = run_prefill(w, q, k, v)
    rows = I.sampled_rows(w, heads=heads)
    got = to_host_f64(out[rows[:, 0], rows[:, 1], rows[:, 2]])
    del out
    ref = oracle.prefill_rows(q, k, v, rows, w0=w.w0, w_pretrained=w.w_pretrained,
                              rope_theta=w.rope_theta, scale=w.scale)
    return check_gate(got, ref, w.dtype, w.name)


def test_c2_l32768_g1_sampled():
    _sampled_case(I.C2, heads=range(I.C2.Hq))


def test_c2_equals_plain_rope_attention_on_gpu():
    """G = 1: the w0 = 4096 output equals the w0 >= L output (plain RoPE attention)."""
    import torch
    w = I.C2
    q, k, v = I.prefill_inputs(w)
    a = run_prefill(w, q, k, v)
    b = run_prefill(w.with_(w0=w.L), q, k, v)
    torch.cuda.synchronize()
    diff = (a.float() - b.float()).abs().max().item()
    assert diff <= 2e-2, diff


def test_c3_l65536_g2_outliers_sampled():
    _sampled_case(I.C3, heads=[0, 5, 10, 15, 16, 21, 26, 31])


def test_c4_l131072_g4_sampled():
    _sampled_case(I.C4, heads=[0, 5, 10, 15, 16, 21, 26, 31])


def test_position_map_bit_exact():
    import torch
    for L, wp in ((1, 1), (512, 128), (513, 128), (131072, 32768), (131073, 32768), (1000, 7)):
        out = torch.full((L,), -1, dtype=torch.int32, device="cuda")
        jl.position_map(out, L, wp)
        G = oracle.group_size(L, wp)
        ref = np.array([oracle.remote_position(x, G) for x in range(0, L, max(1, L // 4096))])
        got = out.cpu().numpy()[:: max(1, L // 4096)]
        np.testing.assert_array_equal(got, ref)
        full = out.cpu().numpy()
        np.testing.assert_array_equal(full, np.arange(L) // G)


# ---------------------------------------------------------------- chunked prefill
# jetlong_prefill_chunk: the C query rows at positions [P, P + C) over cache rows
# [0, P + C); G from P + C.  Reference: the oracle's prefill rows i in [P, P + C)
# of the length-(P + C) sequence made of the same cache rows.

def chunk_case(name, P, C, Lcap, *, dtype="bf16", B=1, Hq=4, Hkv=1, d=128, w_pre=100, w0=17,
               theta=1e6, index=60, nan_tail=False, rows=None):
    import torch
    L = P + C
    w = I.PrefillWorkload(name, index, dtype, B, Hq, Hkv, d, Lcap, w_pre, w0, theta)
    q, k, v = I.prefill_inputs(w)
    qc = np.ascontiguousarray(q[:, :, P:L])
    kd, vd = to_device(k), to_device(v)
    if nan_tail and L < Lcap:
        kd[:, :, L:] = float("nan")
        vd[:, :, L:] = float("nan")
    out = torch.full_like(to_device(qc), float("nan"))
    jl.prefill_chunk(to_device(qc), kd, vd, P, out, w0=w0, w_pretrained=w_pre, rope_theta=theta,
                     scale=w.scale)
    jl.device_status()
    got = to_host_f64(out)
    if rows is None:
        bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(P, L), indexing="ij")
        rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    rows = np.asarray(rows, dtype=np.int32)
    ref = oracle.prefill_rows(np.ascontiguousarray(q[:, :, :L]), np.ascontiguousarray(k[:, :, :L]),
                              np.ascontiguousarray(v[:, :, :L]), rows, w0=w0, w_pretrained=w_pre,
                              rope_theta=theta, scale=w.scale)
    sel = got[rows[:, 0], rows[:, 1], rows[:, 2] - P]
    return check_gate(sel, ref, dtype, name)


CHUNKS = [(0, 300), (128, 256), (100, 77), (1000, 1), (999, 130), (300, 700), (5, 1200)]


@pytest.mark.parametrize("P,C", CHUNKS)
def test_chunk_head_quads(P, C):
    chunk_case(f"chunk-q-{P}-{C}", P, C, P + C + 40, index=61)


@pytest.mark.parametrize("P,C", [(128, 256), (100, 77), (999, 130)])
def test_chunk_head_pairs_and_single(P, C):
    chunk_case(f"chunk-p-{P}-{C}", P, C, P + C + 3, Hq=4, Hkv=2, index=62)
    chunk_case(f"chunk-s-{P}-{C}", P, C, P + C + 3, Hq=3, Hkv=3, index=63)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("P,C", [(0, 200), (150, 90), (511, 1)])
def test_chunk_fp32(d, P, C):
    chunk_case(f"chunk-f32-{d}-{P}-{C}", P, C, P + C + 5, dtype="fp32", Hq=2, Hkv=1, d=d, index=64)


@pytest.mark.parametrize("w0", [0, 1, 128, 5000])
def test_chunk_windows(w0):
    chunk_case(f"chunk-w0-{w0}", 700, 300, 1100, Hq=8, Hkv=2, w0=w0, w_pre=240, index=65)


def test_chunk_ignores_cache_rows_past_length():
    chunk_case("chunk-nan-tail", 600, 200, 1024, nan_tail=True, index=66)
    chunk_case("chunk-nan-tail-f32", 600, 200, 1024, dtype="fp32", Hq=2, d=64, nan_tail=True, index=66)


def test_chunk_of_one_row_equals_decode():
    import torch
    P, Lcap = 1536, 1600
    w = I.PrefillWorkload("chunk-vs-decode", 67, "bf16", 2, 8, 2, 128, Lcap, 400, 200, 1e6)
    q, k, v = I.prefill_inputs(w)
    qd, kd, vd = to_device(q), to_device(k), to_device(v)
    kw = dict(w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta, scale=w.scale)
    ch = jl.prefill_chunk(qd[:, :, P:P + 1].contiguous(), kd, vd, P, **kw)
    dec = jl.decode(qd[:, :, P].contiguous(), kd, vd, P + 1, **kw)
    torch.cuda.synchronize()
    check_gate(to_host_f64(ch[:, :, 0]), to_host_f64(dec), "bf16", "one-row chunk vs decode")


def test_chunk_of_128k_sequence_sampled():
    """The last 4096 rows of the 131072-token headline sequence as one chunk (G = 4)."""
    P, C = 131072 - 4096, 4096
    rng = np.random.default_rng(68)
    rows = [(0, h, P + int(r)) for h in (0, 9, 22, 31) for r in
            list(range(0, 8)) + list(range(C - 8, C)) + list(rng.integers(0, C, 8))]
    chunk_case("chunk-128k", P, C, P + C, B=1, Hq=32, Hkv=8, d=128, w_pre=32768, w0=4096, index=69,
               rows=rows)


# ---------------------------------------------------------------- variable-length batch + LSE
# jetlong_prefill_varlen: sequence b of a padded batch uses rows [0, lens[b]) and
# its own G; reference: the oracle's prefill of that sequence alone.  The LSE
# (natural log of each row's softmax denominator) is a scaled-logit quantity, so
# it takes the output gates' max-abs bound: 2e-2 for bf16 (fp16 logit operands),
# 1e-4 for fp32.

def varlen_case(name, lens, *, dtype="bf16", Hq=4, Hkv=1, d=128, w_pre=100, w0=17, theta=1e6,
                index=70, pad=5, nan_qk_padding=False, launches=None):
    import torch
    B, Lmax = len(lens), max(lens) + pad
    w = I.PrefillWorkload(name, index, dtype, B, Hq, Hkv, d, Lmax, w_pre, w0, theta)
    q, k, v = I.prefill_inputs(w)
    qd, kd = to_device(q), to_device(k)
    if nan_qk_padding:  # padding rows of q and k may hold anything (those of v must be finite)
        for b, Lb in enumerate(lens):
            qd[b, :, Lb:] = float("nan")
            kd[b, :, Lb:] = float("nan")
    out = torch.full_like(qd, float("nan"))
    before = jl.launch_count()
    out, lse = jl.prefill_varlen(qd, kd, to_device(v), lens, out, w0=w0, w_pretrained=w_pre,
                                 rope_theta=theta, scale=w.scale, with_lse=True)
    jl.device_status()
    if launches is not None:
        assert jl.launch_count() - before == launches
    got, got_lse = to_host_f64(out), lse.double().cpu().numpy()
    tol = 2e-2 if dtype == "bf16" else 1e-4
    for b, Lb in enumerate(lens):
        hh, ii = np.meshgrid(np.arange(Hq), np.arange(Lb), indexing="ij")
        rows = np.stack([np.zeros(hh.size, np.int32), hh.ravel(), ii.ravel()], axis=1)
        sl = lambda a: np.ascontiguousarray(a[b:b + 1, :, :Lb])
        ref, ref_lse = oracle.prefill_rows(sl(q), sl(k), sl(v), rows, w0=w0, w_pretrained=w_pre,
                                           rope_theta=theta, scale=w.scale, with_lse=True)
        check_gate(got[b, :, :Lb].reshape(-1, d), ref, dtype, f"{name} seq {b}")
        assert np.abs(got_lse[b, :, :Lb].reshape(-1) - ref_lse).max() <= tol, f"{name} lse seq {b}"
        assert np.isnan(got[b, :, Lb:]).all(), "rows past a sequence's length must stay untouched"


@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (4, 2), (3, 3)])
def test_varlen_bf16(Hq, Hkv):
    varlen_case(f"varlen-{Hq}-{Hkv}", [1000, 37, 513, 1, 130], Hq=Hq, Hkv=Hkv, w_pre=120, w0=64, index=71)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_fp32(d):
    varlen_case(f"varlen-f32-{d}", [300, 1, 129], dtype="fp32", Hq=2, Hkv=1, d=d, w_pre=50, w0=20,
                index=72)


def test_varlen_lengths_cross_group_sizes():
    # w_pretrained = 256: G = 1, 2, 4, 5 for the four sequences
    varlen_case("varlen-G", [256, 257, 1024, 1025], Hq=8, Hkv=2, w_pre=256, w0=100, index=73)


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 2), (2, 2)])
def test_varlen_one_launch_for_64_sequences(Hq, Hkv):
    # bf16: one range scan, one key rotation and one prefill launch per 64
    # sequences (70 here: two of each), every sequence with its own length and
    # G; NaN in the padding rows of q and k must not reach any output
    rng = np.random.default_rng(74)
    lens = [int(x) for x in rng.integers(1, 300, size=70)]
    lens[3], lens[40] = 300, 129
    varlen_case("varlen-70", lens, Hq=Hq, Hkv=Hkv, w_pre=64, w0=40, index=74, nan_qk_padding=True,
                launches=6)


# ---------------------------------------------------------------- inclusion-exclusion form
# jetlong_prefill_ie: the pages' three passes merged with their LSEs; the
# reference is the same oracle (the merge is exact), at the same gates.

def ie_case(name, *, dtype="bf16", B=1, Hq=4, Hkv=1, d=128, L=600, w_pre=100, w0=17, theta=1e6, index=80):
    w = I.PrefillWorkload(name, index, dtype, B, Hq, Hkv, d, L, w_pre, w0, theta)
    q, k, v = I.prefill_inputs(w)
    out = jl.prefill_ie(to_device(q), to_device(k), to_device(v), w0=w0, w_pretrained=w_pre,
                        rope_theta=theta, scale=w.scale)
    jl.device_status()
    ref = oracle.prefill(q, k, v, w0=w0, w_pretrained=w_pre, rope_theta=theta, scale=w.scale)
    return check_gate(to_host_f64(out), ref, dtype, name)


@pytest.mark.parametrize("w0", [0, 1, 17, 128, 300, 598, 599, 5000])
def test_ie_windows_head_quads(w0):
    # w0 = L - 1 = 599 and L - 2: passes B and C nearly coincide and their
    # difference is small, the case where rounding the passes would show
    ie_case(f"ie-q-{w0}", w0=w0, index=81)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (3, 3)])
def test_ie_other_groups(Hq, Hkv):
    ie_case(f"ie-g-{Hq}-{Hkv}", Hq=Hq, Hkv=Hkv, L=513, w0=130, index=82)


@pytest.mark.parametrize("d", [64, 128])
def test_ie_fp32(d):
    ie_case(f"ie-f32-{d}", dtype="fp32", Hq=2, Hkv=1, d=d, L=300, w0=40, w_pre=64, index=83)


def test_ie_equals_one_pass_at_128k_sampled():
    """The headline workload in the three-pass form: sampled rows against the oracle."""
    w = I.C4
    q, k, v = I.prefill_inputs(w)
    out = jl.prefill_ie(to_device(q), to_device(k), to_device(v), w0=w.w0, w_pretrained=w.w_pretrained,
                        rope_theta=w.rope_theta, scale=w.scale)
    jl.device_status()
    rows = I.sampled_rows(w, heads=[0, 11, 22, 31])
    got = to_host_f64(out[rows[:, 0], rows[:, 1], rows[:, 2]])
    del out
    ref = oracle.prefill_rows(q, k, v, rows, w0=w.w0, w_pretrained=w.w_pretrained,
                              rope_theta=w.rope_theta, scale=w.scale)
    check_gate(got, ref, "bf16", "ie-128k")


# ---------------------------------------------------------------- host buffers, overlapped copies
@pytest.mark.parametrize("L,nchunks,Hq,Hkv,dtype", [(1000, 3, 4, 1, "bf16"), (777, 16, 4, 2, "bf16"), (2000, 5, 4, 1, "bf16"),
                                                    (300, 2, 2, 1, "fp32"), (129, 8, 4, 1, "bf16")])
def test_streamed_prefill_from_host(L, nchunks, Hq, Hkv, dtype):
    import torch
    w = I.PrefillWorkload(f"stream-{L}-{nchunks}", 90, dtype, 1, Hq, Hkv, 128, L, 200, 50, 1e6)
    q, k, v = I.prefill_inputs(w)

    def host(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.contiguous().pin_memory()

    qh, kh, vh = host(q), host(k), host(v)
    outh = torch.full_like(qh, float("nan")).pin_memory()
    qd, kd, vd = (torch.empty_like(x, device="cuda") for x in (qh, kh, vh))
    outd = torch.empty_like(qd)
    jl.prefill_streamed(qh, kh, vh, outh, qd, kd, vd, outd, w0=w.w0, w_pretrained=w.w_pretrained,
                        rope_theta=w.rope_theta, scale=w.scale, nchunks=nchunks)
    torch.cuda.current_stream().synchronize()
    jl.device_status()
    ref = oracle.prefill(q, k, v, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                         scale=w.scale)
    check_gate(outh.double().numpy(), ref, dtype, w.name)
