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
