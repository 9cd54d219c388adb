"""Shared helpers for the parity tests: host<->device marshalling and the gates."""
from __future__ import annotations

import numpy as np

# Gates on the attention output (fixed before any kernel existed):
#   bf16 inputs: max |gpu - oracle| <= 2e-2 and ||gpu - oracle||_2 / ||oracle||_2 <= 5e-3
#   fp32 inputs: max |gpu - oracle| <= 1e-4
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
FP32_MAX_ABS = 1e-4


def to_device(a: np.ndarray, device="cuda"):
    """uint16 arrays are bf16 bit patterns; float32 arrays stay fp32."""
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    if a.dtype == np.float32:
        return torch.from_numpy(a).to(device)
    raise TypeError(a.dtype)


def to_host_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def check_gate(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    if dtype == "fp32":
        assert max_abs <= FP32_MAX_ABS, f"{what}: fp32 max-abs {max_abs:.3e} > {FP32_MAX_ABS}"
        return {"max_abs": max_abs}
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= BF16_MAX_ABS, f"{what}: bf16 max-abs {max_abs:.3e} > {BF16_MAX_ABS}"
    assert rel <= BF16_REL_L2, f"{what}: bf16 rel-L2 {rel:.3e} > {BF16_REL_L2}"
    return {"max_abs": max_abs, "rel_l2": rel}
