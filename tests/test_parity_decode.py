"""GPU parity of jetlong_decode against the fp64 CPU oracle (through the C ABI),
plus decode/prefill cross-consistency.  Gates as in the prefill tests."""
import numpy as np
import pytest

import oracle
import rope_context_extension_jet_b200 as jl
from rope_context_extension_jet_b200 import inputs as I
from helpers import check_gate, to_device, to_host_f64

pytestmark = pytest.mark.gpu


def small_decode(name, dtype="bf16", B=2, Hq=8, Hkv=2, d=128, L0=2999, Lcap=3008, steps=4,
                 w_pre=700, w0=64, theta=1e6, index=40):
    return I.DecodeWorkload(name, index, dtype, B, Hq, Hkv, d, L0, Lcap, steps, w_pre, w0, theta)


def run_decode(w, qs, kc, vc, steps, ws=None):
    import torch
    kcd, vcd = to_device(kc), to_device(vc)
    if ws is None:
        ws = torch.empty(jl.decode_workspace_size(w.B, w.Hq, w.Hkv, w.Lcap, w.d), dtype=torch.uint8,
                         device="cuda")
    outs = {}
    for t in steps:
        qd = to_device(np.ascontiguousarray(qs[t]))
        out = torch.full_like(qd, float("nan"))
        jl.decode(qd, kcd, vcd, w.length_at(t), out, w0=w.w0, w_pretrained=w.w_pretrained,
                  rope_theta=w.rope_theta, scale=w.scale, workspace=ws)
        outs[t] = out
    jl.device_status()
    return {t: to_host_f64(o) for t, o in outs.items()}


def check_steps(w, steps):
    qs, kc, vc = I.decode_inputs(w)
    got = run_decode(w, qs, kc, vc, steps)
    for t in steps:
        ref = oracle.decode(np.ascontiguousarray(qs[t]), kc, vc, w.length_at(t), w0=w.w0,
                            w_pretrained=w.w_pretrained, rope_theta=w.rope_theta, scale=w.scale)
        check_gate(got[t], ref, w.dtype, f"{w.name} step {t}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("L0", [0, 1, 30, 31, 32, 33, 700, 1400, 2999])
def test_decode_lengths(dtype, L0):
    check_steps(small_decode(f"dec-L{L0 + 1}", dtype=dtype, L0=L0, steps=1), [0])


@pytest.mark.parametrize("w0", [0, 1, 64, 1000, 5000])
def test_decode_windows(w0):
    check_steps(small_decode(f"dec-w0-{w0}", w0=w0, L0=2100, steps=1, index=41), [0])


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 8, 128), (8, 1, 128), (6, 2, 64), (4, 4, 64), (12, 4, 128)])
def test_decode_shapes(Hq, Hkv, d):
    check_steps(small_decode(f"dec-{Hq}-{Hkv}-{d}", Hq=Hq, Hkv=Hkv, d=d, L0=1500, steps=1,
                             index=42), [0])


def test_decode_crosses_group_boundary_small():
    # w_pre = 1000: lengths 2999 -> 3002 cross 3 * 1000 (G 3 -> 4) inside the steps
    w = small_decode("dec-cross", L0=2998, Lcap=3008, steps=4, w_pre=1000, w0=100, index=43)
    assert jl.group_size(w.length_at(0), 1000) == 3 and jl.group_size(w.length_at(3), 1000) == 4
    check_steps(w, [0, 1, 2, 3])


def test_decode_full_size_g4_to_g5():
    """B=8, Hq=32, Hkv=8, d=128, cache 131136 rows; steps 31 (G=4) and 32 (G=5)."""
    w = I.D
    assert jl.group_size(w.length_at(31), w.w_pretrained) == 4
    assert jl.group_size(w.length_at(32), w.w_pretrained) == 5
    check_steps(w, [31, 32])


def test_decode_matches_prefill_last_row():
    import torch
    w = I.PrefillWorkload("dec-vs-pre", 44, "bf16", 1, 8, 2, 128, 1537, 400, 200, 1e6)
    q, k, v = I.prefill_inputs(w)
    qd, kd, vd = to_device(q), to_device(k), to_device(v)
    pre = jl.prefill(qd, kd, vd, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                     scale=w.scale)
    dec = jl.decode(qd[:, :, -1].contiguous(), kd, vd, w.L, w0=w.w0, w_pretrained=w.w_pretrained,
                    rope_theta=w.rope_theta, scale=w.scale)
    torch.cuda.synchronize()
    check_gate(to_host_f64(dec), to_host_f64(pre[:, :, -1]), "bf16", "decode vs prefill row L-1")


def test_workspace_contents_do_not_matter():
    import torch
    w = small_decode("dec-ws", L0=2500, steps=1, index=45)
    qs, kc, vc = I.decode_inputs(w)
    ws = torch.empty(jl.decode_workspace_size(w.B, w.Hq, w.Hkv, w.Lcap, w.d), dtype=torch.uint8,
                     device="cuda")
    ws.fill_(0xFF)
    a = run_decode(w, qs, kc, vc, [0], ws=ws)[0]
    ws.fill_(0x5A)
    b = run_decode(w, qs, kc, vc, [0], ws=ws)[0]
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_cache_rows_past_length_are_ignored(dtype):
    """Rows >= L of the caches may hold anything (here NaN): the output must not see them."""
    import torch
    w = small_decode("dec-nan-tail", dtype=dtype, L0=1000, Lcap=1100, steps=1, index=46)
    qs, kc, vc = I.decode_inputs(w)
    L = w.length_at(0)
    kd, vd = to_device(kc), to_device(vc)
    kd[:, :, L:] = float("nan")
    vd[:, :, L:] = float("nan")
    qd = to_device(np.ascontiguousarray(qs[0]))
    out = jl.decode(qd, kd, vd, L, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                    scale=w.scale)
    jl.device_status()
    ref = oracle.decode(np.ascontiguousarray(qs[0]), kc, vc, L, w0=w.w0,
                        w_pretrained=w.w_pretrained, rope_theta=w.rope_theta, scale=w.scale)
    check_gate(to_host_f64(out), ref, dtype, "decode with NaN rows past L")


# ---------------------------------------------------------------- standard RoPE cache
# jetlong_decode_rope_cache: key row j is stored rotated to its exact position
# j (built here by the oracle from the seeded raw keys, rounded to the input
# dtype); the reference is the oracle's decode over the same stored rows.

def rope_cache_of(kc, w):
    rot = oracle.rotate_rows(kc, w.rope_theta)
    return I.to_bf16_bits(rot.astype(np.float32)) if w.dtype == "bf16" else rot.astype(np.float32)


def check_rope_cache_steps(w, steps):
    import torch
    qs, kc, vc = I.decode_inputs(w)
    kr = rope_cache_of(kc, w)
    krd, vcd = to_device(kr), to_device(vc)
    ws = torch.empty(jl.decode_workspace_size(w.B, w.Hq, w.Hkv, w.Lcap, w.d), dtype=torch.uint8,
                     device="cuda")
    for t in steps:
        qd = to_device(np.ascontiguousarray(qs[t]))
        out = torch.full_like(qd, float("nan"))
        jl.decode_rope_cache(qd, krd, vcd, w.length_at(t), out, w0=w.w0, w_pretrained=w.w_pretrained,
                             rope_theta=w.rope_theta, scale=w.scale, workspace=ws)
        jl.device_status()
        ref = oracle.decode_rope_cache(np.ascontiguousarray(qs[t]), kr, vc, w.length_at(t), w0=w.w0,
                                       w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                                       scale=w.scale)
        check_gate(to_host_f64(out), ref, w.dtype, f"{w.name} rope-cache step {t}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("L0,w0", [(0, 64), (31, 64), (700, 64), (2999, 64), (2100, 0), (2100, 5000),
                                   (1500, 1)])
def test_rope_cache_decode_small(dtype, L0, w0):
    check_rope_cache_steps(small_decode(f"rc-{dtype}-L{L0 + 1}-w{w0}", dtype=dtype, L0=L0, w0=w0,
                                        steps=1, index=47), [0])


def test_rope_cache_decode_crosses_group_boundary():
    w = small_decode("rc-cross", L0=2998, Lcap=3008, steps=4, w_pre=1000, w0=100, index=48)
    check_rope_cache_steps(w, [0, 1, 2, 3])


def test_rope_cache_decode_full_size_g4_to_g5():
    """B=8, Hq=32, Hkv=8, d=128, cache 131136 rows stored rotated; steps 31 (G=4) and 32 (G=5)."""
    check_rope_cache_steps(I.D, [31, 32])


def test_rope_cache_decode_matches_raw_cache_decode():
    # the same attention reached two ways on the GPU: raw keys rotated in the
    # kernel, or stored rotated keys corrected by f(j) - j
    import torch
    w = small_decode("rc-vs-raw", L0=2500, w_pre=600, w0=300, steps=1, index=49)
    qs, kc, vc = I.decode_inputs(w)
    kr = rope_cache_of(kc, w)
    qd = to_device(np.ascontiguousarray(qs[0]))
    kw = dict(w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta, scale=w.scale)
    a = jl.decode_rope_cache(qd, to_device(kr), to_device(vc), w.length_at(0), **kw)
    b = jl.decode(qd, to_device(kc), to_device(vc), w.length_at(0), **kw)
    torch.cuda.synchronize()
    check_gate(to_host_f64(a), to_host_f64(b), "bf16", "rope-cache decode vs raw-cache decode")
