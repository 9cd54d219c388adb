"""Failure detection without a GPU fault: a kernel's bounded wait that expires
sets the library's device error word and returns; the host reads it as
JETLONG_ERR_TIMEOUT, and the context stays usable.  The expiry is made by a
self-test kernel waiting on a barrier nothing arrives at (~1 ms limit)."""
import numpy as np
import pytest

import oracle
import rope_context_extension_jet_b200 as jl
from rope_context_extension_jet_b200 import inputs as I
from helpers import check_gate, to_device, to_host_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_cleared():
    jl.device_status()  # clean state
    jl.selftest_wait_timeout()
    with pytest.raises(jl.JetLongError) as ei:
        jl.device_status()
    assert ei.value.status == 4  # JETLONG_ERR_TIMEOUT
    assert "bounded device wait" in str(ei.value)
    jl.device_status()  # cleared by the read


def test_context_usable_after_timeout():
    jl.selftest_wait_timeout()
    with pytest.raises(jl.JetLongError):
        jl.device_status()
    w = I.PrefillWorkload("after-timeout", 80, "bf16", 1, 4, 2, 128, 300, 100, 40, 1e6)
    q, k, v = I.prefill_inputs(w)
    out = jl.prefill(to_device(q), to_device(k), to_device(v), w0=w.w0,
                     w_pretrained=w.w_pretrained, rope_theta=w.rope_theta, scale=w.scale)
    jl.device_status()
    ref = oracle.prefill(q, k, v, w0=w.w0, w_pretrained=w.w_pretrained,
                         rope_theta=w.rope_theta, scale=w.scale)
    check_gate(to_host_f64(out), ref, "bf16", "prefill after a reported timeout")
