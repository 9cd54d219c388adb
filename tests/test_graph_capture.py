"""CUDA graph capture of the library's calls: after one call of each kind on
the device (which creates the library's per-device resources: the rotated-
operand pool, the error word, the range slots), a bf16 prefill and a decode
step are captured into one graph with torch.cuda.graph and replayed twice on
new inputs copied into the same buffers; every replay is checked against the
fp64 oracle with the usual gates.  Nothing here changes what the kernels
compute; it shows that the calls contain no operation a stream capture
refuses and that a replayed graph recomputes from its buffers' current
contents (the range scan and the key rotation included)."""
import numpy as np
import pytest

import oracle
import rope_context_extension_jet_b200 as jl
from rope_context_extension_jet_b200 import inputs as I
from helpers import check_gate, to_device, to_host_f64

pytestmark = pytest.mark.gpu


def test_prefill_and_decode_replayed_from_a_cuda_graph():
    import torch
    # GQA 4 (the CTA-pair prefill kernel), G = 2 at this length
    pw = [I.PrefillWorkload(f"graph-prefill-{r}", 95 + r, "bf16", 1, 8, 2, 128, 700, 400, 96, 1e6)
          for r in range(3)]
    dw = [I.DecodeWorkload(f"graph-decode-{r}", 97 + r, "bf16", 2, 8, 2, 128, 999, 1024, 1, 400, 64, 1e6)
          for r in range(3)]
    pin = [I.prefill_inputs(w) for w in pw]
    din = [I.decode_inputs(w) for w in dw]
    q, k, v = (to_device(a) for a in pin[0])
    out = torch.empty_like(q)
    dq = to_device(np.ascontiguousarray(din[0][0][0]))
    kc, vc = to_device(din[0][1]), to_device(din[0][2])
    dout = torch.empty_like(dq)
    w, d = pw[0], dw[0]
    ws = torch.empty(jl.decode_workspace_size(d.B, d.Hq, d.Hkv, d.Lcap, d.d), dtype=torch.uint8, device="cuda")
    L = d.length_at(0)

    def step(stream):
        jl.prefill(q, k, v, out, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta, scale=w.scale,
                   stream=stream)
        jl.decode(dq, kc, vc, L, dout, w0=d.w0, w_pretrained=d.w_pretrained, rope_theta=d.rope_theta,
                  scale=d.scale, workspace=ws, stream=stream)

    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        step(side)  # first calls on this device: resources exist before the capture
    side.synchronize()
    jl.device_status()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(side)
    for r in (1, 2):
        q.copy_(to_device(pin[r][0]))
        k.copy_(to_device(pin[r][1]))
        v.copy_(to_device(pin[r][2]))
        dq.copy_(to_device(np.ascontiguousarray(din[r][0][0])))
        kc.copy_(to_device(din[r][1]))
        vc.copy_(to_device(din[r][2]))
        out.fill_(float("nan"))
        dout.fill_(float("nan"))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        jl.device_status()
        pq, pk, pv = pin[r]
        ref = oracle.prefill(pq, pk, pv, w0=w.w0, w_pretrained=w.w_pretrained, rope_theta=w.rope_theta,
                             scale=w.scale)
        check_gate(to_host_f64(out), ref, "bf16", f"graph replay {r}: prefill")
        qs, kcache, vcache = din[r]
        dref = oracle.decode(np.ascontiguousarray(qs[0]), kcache, vcache, L, w0=d.w0, w_pretrained=d.w_pretrained,
                             rope_theta=d.rope_theta, scale=d.scale)
        check_gate(to_host_f64(dout), dref, "bf16", f"graph replay {r}: decode")
    del graph
