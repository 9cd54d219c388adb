"""Allocation-free decode (jetlong_decode_noalloc), called through the C ABI.

Some callers cannot allocate device memory (a serving runtime whose caching
allocator must not grow, code in a host callback, a framework that hands the
library only the step's tensors), so they cannot pass jetlong_decode a
workspace.  jetlong_decode_noalloc keeps that scratch in a fixed device array
inside the library.  These tests check that two calls in a row -- the second
one finding the first one's leftovers in the shared array -- give the same
output as jetlong_decode and as the fp64 oracle within the parity gate of the
input type (bf16 and fp32), and that a problem too large for the array is
refused before anything is launched.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import oracle
import rope_context_extension_jet_b200 as jl
from rope_context_extension_jet_b200 import inputs as I
from helpers import check_gate, to_device, to_host_f64

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, q, kc, vc, out, w, L, stream):
    return lib.jetlong_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
        ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        w.B, w.Hq, w.Hkv, L, w.Lcap, w.d, w.w0, w.w_pretrained, w.rope_theta, w.scale,
        jl.BF16 if w.dtype == "bf16" else jl.FP32, ctypes.c_void_p(stream.cuda_stream))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_noalloc_matches_workspace_decode_two_calls_in_a_row(dtype):
    import torch
    lib = jl.load_library()
    w = I.DecodeWorkload("noalloc", 60, dtype, 2, 8, 2, 128, 2990, 3008, 2, 1000, 64, 1e6)
    qs, kc, vc = I.decode_inputs(w)
    kcd, vcd = to_device(kc), to_device(vc)
    stream = torch.cuda.current_stream()
    ws = torch.empty(jl.decode_workspace_size(w.B, w.Hq, w.Hkv, w.Lcap, w.d), dtype=torch.uint8,
                     device="cuda")
    for t in range(w.steps):  # two calls in a row; L = 2991, 2992 (G = 3)
        L = w.length_at(t)
        qd = to_device(np.ascontiguousarray(qs[t]))
        ref = torch.empty_like(qd)
        jl.decode(qd, kcd, vcd, L, ref, w0=w.w0, w_pretrained=w.w_pretrained,
                  rope_theta=w.rope_theta, scale=w.scale, workspace=ws, stream=stream)
        got = torch.full_like(qd, float("nan"))
        st = _call_noalloc(lib, qd, kcd, vcd, got, w, L, stream)
        assert st == 0, lib.jetlong_last_error().decode()
        jl.device_status(stream)
        check_gate(to_host_f64(got), to_host_f64(ref), dtype, f"no-alloc decode call {t}")
        exact = oracle.decode(np.ascontiguousarray(qs[t]), kc, vc, L, w0=w.w0, w_pretrained=w.w_pretrained,
                              rope_theta=w.rope_theta, scale=w.scale)
        check_gate(to_host_f64(got), exact, dtype, f"no-alloc decode call {t} against the oracle")


def test_noalloc_rejects_problem_larger_than_its_array():
    import torch
    lib = jl.load_library()
    # B*Hq partial states of (d + 2) floats already exceed the 4 MiB array with one split.
    w = I.DecodeWorkload("noalloc-big", 61, "bf16", 256, 32, 8, 128, 63, 64, 1, 1000, 64, 1e6)
    q = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((w.B, w.Hkv, w.Lcap, w.d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    out = torch.zeros_like(q)
    torch.cuda.synchronize()
    before = jl.launch_count()
    st = _call_noalloc(lib, q, kc, vc, out, w, w.length_at(0), torch.cuda.current_stream())
    assert st == 1  # JETLONG_ERR_INVALID_ARG
    assert "scratch" in lib.jetlong_last_error().decode()
    assert jl.launch_count() == before
