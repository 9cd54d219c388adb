"""CPU checks of the Python binding: it exports every entry point, rejects
mismatched tensors before any pointer reaches the library (a wrong shape or
element type would make a kernel read or write out of bounds), and has no CPU
fallback (host tensors raise instead of being computed on the host)."""
import pytest
import torch

import rope_context_extension_jet_b200 as jl
from rope_context_extension_jet_b200 import _build

KW = dict(w0=4, w_pretrained=8, rope_theta=1e4)


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    jl.load_library()


def t(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def test_all_lists_every_entry_point():
    for name in ("prefill", "prefill_chunk", "prefill_varlen", "prefill_ie", "prefill_streamed",
                 "decode", "decode_rope_cache", "decode_noalloc", "position_map", "group_size"):
        assert name in jl.__all__ and callable(getattr(jl, name))


@pytest.mark.parametrize("call", [
    lambda: jl.prefill(t(1, 2, 16, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), **KW),
    lambda: jl.prefill_chunk(t(1, 2, 4, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 12, **KW),
    lambda: jl.prefill_varlen(t(1, 2, 16, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), [10], **KW),
    lambda: jl.prefill_ie(t(1, 2, 16, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), **KW),
    lambda: jl.decode(t(1, 2, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 16, **KW),
    lambda: jl.decode_rope_cache(t(1, 2, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 16, **KW),
    lambda: jl.decode_noalloc(t(1, 2, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 16, **KW),
])
def test_host_tensors_raise_instead_of_a_cpu_fallback(call):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        call()


@pytest.mark.parametrize("call", [
    lambda: jl.prefill(t(1, 2, 16, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), t(1, 2, 8, 64), **KW),
    lambda: jl.prefill(t(1, 2, 16, 64), t(1, 1, 16, 64), t(1, 1, 16, 64),
                       t(1, 2, 16, 64, dtype=torch.float32), **KW),
    lambda: jl.prefill_chunk(t(1, 2, 4, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 12, t(1, 2, 16, 64), **KW),
    lambda: jl.prefill_varlen(t(1, 2, 16, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), [10], t(1, 2, 15, 64),
                              **KW),
    lambda: jl.prefill_ie(t(1, 2, 16, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), t(2, 2, 16, 64), **KW),
    lambda: jl.decode(t(1, 2, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 16, t(1, 3, 64), **KW),
    lambda: jl.decode_noalloc(t(1, 2, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 16, t(2, 64), **KW),
])
def test_out_must_match_q(call):
    with pytest.raises(ValueError, match="out must match q"):
        call()


@pytest.mark.parametrize("call", [
    lambda: jl.prefill(t(1, 2, 16, 64), t(1, 1, 16, 64, dtype=torch.float32), t(1, 1, 16, 64), **KW),
    lambda: jl.prefill_chunk(t(1, 2, 4, 64), t(1, 1, 16, 64), t(1, 1, 16, 64, dtype=torch.float32), 12,
                             **KW),
    lambda: jl.prefill_ie(t(1, 2, 16, 64, dtype=torch.float32), t(1, 1, 16, 64), t(1, 1, 16, 64), **KW),
    lambda: jl.decode(t(1, 2, 64, dtype=torch.float32), t(1, 1, 16, 64), t(1, 1, 16, 64), 16, **KW),
    lambda: jl.decode_noalloc(t(1, 2, 64), t(1, 1, 16, 64), t(1, 1, 16, 64, dtype=torch.float32), 16,
                              **KW),
])
def test_mixed_element_types_are_rejected(call):
    with pytest.raises(TypeError, match="must share a dtype"):
        call()


@pytest.mark.parametrize("call", [
    lambda: jl.decode(t(1, 2, 64), t(1, 1, 16, 128), t(1, 1, 16, 128), 16, **KW),
    lambda: jl.decode(t(2, 2, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 16, **KW),
    lambda: jl.decode_rope_cache(t(1, 2, 64), t(1, 1, 16, 64), t(1, 1, 8, 64), 8, **KW),
    lambda: jl.decode_noalloc(t(1, 2, 16, 64), t(1, 1, 16, 64), t(1, 1, 16, 64), 16, **KW),
])
def test_decode_cache_shapes_must_match_q(call):
    with pytest.raises(ValueError, match="must be \\[B, Hq, d\\]|the caches must be|same shape"):
        call()


def test_streamed_shapes_must_match():
    qh, kh = t(1, 2, 16, 64), t(1, 1, 16, 64)
    with pytest.raises(ValueError, match="k_host must be"):
        jl.prefill_streamed(qh, t(1, 1, 12, 64), t(1, 1, 12, 64), t(1, 2, 16, 64), t(1, 2, 16, 64),
                            t(1, 1, 12, 64), t(1, 1, 12, 64), t(1, 2, 16, 64), **KW)
    with pytest.raises(ValueError, match="out_dev must match"):
        jl.prefill_streamed(qh, kh, kh.clone(), t(1, 2, 16, 64), t(1, 2, 16, 64), kh.clone(), kh.clone(),
                            t(1, 2, 8, 64), **KW)
