"""Input range of the bf16 tensor-core paths (GPU, against the fp64 oracle).

The Q K^T operands of the bf16 kernels are the rotated vectors rounded to fp16,
whose range ends at 65504 and whose normal range starts at 6.1e-5, while bf16
inputs span 1e-38 .. 3.4e38.  The prefill scales all queries and all keys of a
call by powers of two chosen from the data (a range scan before the kernel);
the decode scales each query head, and each key row of a block whose fp16
logits would not be finite (or of every block, for extreme queries), and both
undo the scales in the softmax.  These cases put q or k
far outside fp16's range, in both directions, with the other operand scaled the
opposite way so the logits keep the size of N(0,1) attention logits: the method
places no limit on the magnitude of q and k (Jet-Long, gist.science/it/paper/
2607.07740, Metodologia 1), so the outputs must pass the same bf16 gates as the
ordinary workloads.  Every kernel that rounds to fp16 is covered: the CTA-pair
prefill (four query heads per kv head), the one-CTA prefill (one or two heads,
d = 64 and 128) and the bf16 decode (raw and RoPE'd caches).
"""
import numpy as np
import pytest

import oracle
import rope_context_extension_jet_b200 as jl
from rope_context_extension_jet_b200 import inputs as I
from helpers import check_gate, to_device, to_host_f64

pytestmark = pytest.mark.gpu

FP16_MAX = 65504.0
FP16_MIN_NORMAL = 2.0 ** -14


def scaled(bits, factor, rows=None):
    """bf16 bits times `factor` (all rows, or a boolean mask over the row axis),
    rounded back to bf16."""
    x = I.bf16_bits_to_f32(bits).astype(np.float64)
    if rows is None:
        x = x * factor
    else:
        x[rows] = x[rows] * factor
    return I.to_bf16_bits(x.astype(np.float32))


def absmax(bits):
    return float(np.abs(I.bf16_bits_to_f32(bits)).max())


def absmin_nonzero(bits):
    a = np.abs(I.bf16_bits_to_f32(bits))
    return float(a[a > 0].min())


# (name, q factor, k factor): the logits of q * a and k * b equal those of
# q * (a b) and k, so a * b stays near 1
CASES = [
    ("q_2e17_k_2e-17", 2.0 ** 17, 2.0 ** -17),       # q up to ~6e5: overflows fp16 unscaled
    ("q_7.5e4_k_1.33e-5", 7.5e4, 1.0 / 7.5e4),       # q up to ~3e5, factors not powers of two
    ("k_2e16_q_2e-16", 2.0 ** -16, 2.0 ** 16),        # k up to ~3e5
    ("k_2e-20_q_2e20", 2.0 ** 20, 2.0 ** -20),        # k below fp16's subnormals, q far above its max
    ("both_1e-3", 1e-3, 1e-3),                        # every value ~1e-3: near-uniform softmax
]

KERNELS = [  # (Hq, Hkv, d): pair kernel, one-CTA with two and one heads, one-CTA d = 64
    (8, 2, 128), (4, 2, 128), (2, 2, 128), (4, 2, 64),
]


def prefill_case(name, Hq, Hkv, d, fq, fk, L=300, w_pre=100, w0=40, index=30, outlier_rows=None):
    w = I.PrefillWorkload(name, index, "bf16", 1, Hq, Hkv, d, L, w_pre, w0, 1e6)
    q, k, v = I.prefill_inputs(w)
    q = scaled(q, fq)
    k = scaled(k, fk, outlier_rows)
    return w, q, k, v


def run_prefill(w, q, k, v):
    import torch
    qd, kd, vd = to_device(q), to_device(k), to_device(v)
    out = torch.full_like(qd, float("nan"))
    jl.prefill(qd, kd, vd, out, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
               scale=w.scale)
    jl.device_status()
    return to_host_f64(out)


@pytest.mark.parametrize("Hq,Hkv,d", KERNELS)
@pytest.mark.parametrize("name,fq,fk", CASES)
def test_prefill_operands_outside_fp16_range(name, fq, fk, Hq, Hkv, d):
    w, q, k, v = prefill_case(name, Hq, Hkv, d, fq, fk)
    if fq > 1e3:
        assert absmax(q) > FP16_MAX
    if fk > 1e3:
        assert absmax(k) > FP16_MAX
    if fk < 1e-5:
        assert absmax(k) < FP16_MIN_NORMAL  # every key would be an fp16 subnormal
    ref = oracle.prefill(q, k, v, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                         scale=w.scale)
    check_gate(run_prefill(w, q, k, v), ref, "bf16", f"{name} Hq={Hq} Hkv={Hkv} d={d}")


@pytest.mark.parametrize("Hq,Hkv,d", KERNELS)
def test_prefill_key_rows_far_apart_in_one_tile(Hq, Hkv, d):
    # 1% of the key rows 2^10 larger than the rest (each key tile then holds
    # keys 2^10 apart and one scale), queries 2^10 smaller: the large keys' logits
    # are N(0,1)-sized, the others near 0 but still resolved
    w = I.PrefillWorkload("mixed", 31, "bf16", 1, Hq, Hkv, d, 300, 100, 40, 1e6)
    rng = np.random.default_rng(31)
    rows = np.zeros((1, Hkv, w.L), dtype=bool)
    for h in range(Hkv):
        rows[0, h, rng.permutation(w.L)[:3]] = True
    w, q, k, v = prefill_case("mixed", Hq, Hkv, d, 2.0 ** -10, 2.0 ** 10, index=31, outlier_rows=rows)
    ref = oracle.prefill(q, k, v, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                         scale=w.scale)
    check_gate(run_prefill(w, q, k, v), ref, "bf16", f"mixed key rows Hq={Hq} Hkv={Hkv} d={d}")


def test_prefill_chunk_and_varlen_large_queries():
    # the chunked and variable-length entry points run the same kernels
    w, q, k, v = prefill_case("chunk-range", 8, 2, 128, 2.0 ** 17, 2.0 ** -17, L=500, index=32)
    P = 300
    qd = to_device(np.ascontiguousarray(q[:, :, P:]))
    out = jl.prefill_chunk(qd, to_device(k), to_device(v), P, w0=w.w0, w_pretrained=w.w_pretrained,
                           rope_theta=w.rope_theta, scale=w.scale)
    jl.device_status()
    rows = np.array([(0, h, i) for h in range(w.Hq) for i in range(P, w.L)], dtype=np.int32)
    ref = oracle.prefill_rows(q, k, v, rows, w0=w.w0, w_pretrained=w.w_pretrained,
                              rope_theta=w.rope_theta, scale=w.scale)
    check_gate(to_host_f64(out).reshape(-1, w.d), ref, "bf16", "chunk with q up to 6e5")


# ---------------------------------------------------------------- decode

def decode_case(name, fq, fk, Hq=8, Hkv=2, rope_cache=False, index=41):
    import torch
    w = I.DecodeWorkload(name, index, "bf16", 2, Hq, Hkv, 128, 1500, 1536, 1, 400, 64, 1e6)
    qs, kc, vc = I.decode_inputs(w)
    q = scaled(np.ascontiguousarray(qs[0]), fq)
    kc = scaled(kc, fk)
    L = w.length_at(0)
    if rope_cache:
        rot = oracle.rotate_rows(kc, w.rope_theta)
        kc = I.to_bf16_bits(rot.astype(np.float32))
    ws = torch.empty(jl.decode_workspace_size(w.B, w.Hq, w.Hkv, w.Lcap, w.d), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    fn = jl.decode_rope_cache if rope_cache else jl.decode
    fn(to_device(q), to_device(kc), to_device(vc), L, out, w0=w.w0, w_pretrained=w.w_pretrained,
       rope_theta=w.rope_theta, scale=w.scale, workspace=ws)
    jl.device_status()
    ref_fn = oracle.decode_rope_cache if rope_cache else oracle.decode
    ref = ref_fn(q, kc, vc, L, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                 scale=w.scale)
    return q, kc, to_host_f64(out), ref


@pytest.mark.parametrize("Hq", [8, 16, 2])
@pytest.mark.parametrize("name,fq,fk", CASES)
def test_decode_operands_outside_fp16_range(name, fq, fk, Hq):
    q, kc, got, ref = decode_case(name, fq, fk, Hq=Hq)
    if fq > 1e3:
        assert absmax(q) > FP16_MAX
    if fk > 1e3:
        assert absmax(kc) > FP16_MAX
    check_gate(got, ref, "bf16", f"decode {name} Hq={Hq}")


@pytest.mark.parametrize("name,fq,fk", CASES[:3])
def test_rope_cache_decode_operands_outside_fp16_range(name, fq, fk):
    _, _, got, ref = decode_case(name, fq, fk, rope_cache=True, index=42)
    check_gate(got, ref, "bf16", f"rope-cache decode {name}")
