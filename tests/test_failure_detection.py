"""Failure detection without a GPU fault: a kernel's bounded wait that expires
sets the library's device error word and returns; the host reads it as
JETLONG_ERR_TIMEOUT, and the context stays usable.  The expiry is made by a
self-test kernel waiting on a barrier nothing arrives at (~1 ms limit), and in
the attention kernels themselves by the one-shot test hook
(jetlong_debug_inject_timeout): the launch withholds one barrier arrival and
limits every wait to ~1 ms.  The recovery call after each expiry is not armed,
which also shows the hook is consumed by one call."""
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


# The attention kernels' own bounded waits, made to expire by the one-shot test
# hook: the launch withholds one barrier arrival and limits every wait to ~1 ms.
LIMIT = 2_000_000  # SM cycles, ~1 ms
PAIR_CODES = {0x331, 0x332, 0x333} | set(range(0x401, 0x403)) | set(range(0x411, 0x418)) | {0x421} \
    | set(range(0x431, 0x435))
ONE_CTA_CODES = {0x331, 0x332, 0x333} | set(range(0x301, 0x303)) | set(range(0x311, 0x31c)) \
    | set(range(0x321, 0x325))
DECODE_CODES = {0x111, 0x112, 0x113}


def _timeout_code():
    with pytest.raises(jl.JetLongError) as ei:
        jl.device_status()
    assert ei.value.status == 4, str(ei.value)  # JETLONG_ERR_TIMEOUT
    msg = str(ei.value)
    return int(msg[msg.index("code 0x") + 5:].split(")")[0], 16)


@pytest.mark.parametrize("Hq,Hkv,codes", [(8, 2, PAIR_CODES), (4, 2, ONE_CTA_CODES)],
                         ids=["pair-kernel", "one-cta-kernel"])
def test_prefill_kernel_wait_expires_and_context_recovers(Hq, Hkv, codes):
    jl.device_status()  # clean state
    w = I.PrefillWorkload("inject-prefill", 81, "bf16", 1, Hq, Hkv, 128, 300, 100, 40, 1e6)
    q, k, v = I.prefill_inputs(w)
    qd, kd, vd = to_device(q), to_device(k), to_device(v)
    kw = dict(w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta, scale=w.scale)
    jl.debug_inject_timeout(jl.INJECT_PREFILL_KEY_TILE, LIMIT)
    jl.prefill(qd, kd, vd, **kw)
    assert _timeout_code() in codes
    jl.device_status()  # the read cleared the word
    # the next launch on the same context allocates tensor memory again and is
    # correct: the expired launch released everything it held
    out = jl.prefill(qd, kd, vd, **kw)
    jl.device_status()
    ref = oracle.prefill(q, k, v, **kw)
    check_gate(to_host_f64(out), ref, "bf16", "prefill after an expired kernel wait")


def test_decode_kernel_wait_expires_and_context_recovers():
    jl.device_status()
    w = I.DecodeWorkload("inject-decode", 82, "bf16", 2, 8, 2, 128, 1500, 1536, 1, 400, 64, 1e6)
    qs, kc, vc = I.decode_inputs(w)
    qd, kcd, vcd = to_device(np.ascontiguousarray(qs[0])), to_device(kc), to_device(vc)
    kw = dict(w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta, scale=w.scale)
    L = w.length_at(0)
    jl.debug_inject_timeout(jl.INJECT_DECODE_COPY, LIMIT)
    jl.decode(qd, kcd, vcd, L, **kw)
    assert _timeout_code() in DECODE_CODES
    jl.device_status()
    out = jl.decode(qd, kcd, vcd, L, **kw)
    jl.device_status()
    ref = oracle.decode(np.ascontiguousarray(qs[0]), kc, vc, L, **kw)
    check_gate(to_host_f64(out), ref, "bf16", "decode after an expired kernel wait")
