"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds no part of the attention method: it only draws i.i.d. normal
tensors with numpy, rounds them to bf16 (round-to-nearest-even on the bit
pattern) where the workload is bf16, and scales a seeded 1% of key rows by 8
for the outlier-key workload.  Both the CUDA path and the CPU oracle consume
exactly these arrays.

Workload shapes follow the pages' setting (Qwen3-style grouped-query attention,
head dim 128, a 32K native window extended to 128K): "Jet-Long: Efficient
Long-Context Extension with Dynamic Bifocal RoPE", Risultati Sperimentali.

Recipe (workload index n; block c = b * heads + h, one [L, d] block per head):
  q ~ N(0,1): block c drawn by default_rng([1000 + n, c]).standard_normal(float32);
  k ~ N(0,1): default_rng([2000 + n, c]) per (b, kv-head);
  v ~ N(0,1): default_rng([3000 + n, c]) per (b, kv-head);
  outlier keys: default_rng([4000, c]).permutation(L)[:floor(0.01 L)] are the rows
  of kv block c multiplied by 8 before rounding.
Blocks are independent streams, so they are drawn in parallel threads.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    index: int
    dtype: str  # "bf16" or "fp32"
    B: int
    Hq: int
    Hkv: int
    d: int
    L: int
    w_pretrained: int
    w0: int
    rope_theta: float
    outlier_frac: float = 0.0
    outlier_scale: float = 8.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "PrefillWorkload":
        return replace(self, **kw)


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    index: int
    dtype: str
    B: int
    Hq: int
    Hkv: int
    d: int
    L0: int      # valid cache rows before the first step
    Lcap: int    # allocated cache rows
    steps: int   # step t attends rows [0, L0 + 1 + t)
    w_pretrained: int
    w0: int
    rope_theta: float

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def length_at(self, t: int) -> int:
        return self.L0 + 1 + t

    def with_(self, **kw) -> "DecodeWorkload":
        return replace(self, **kw)


# The five workloads: a small fp32 case with every output checked, three bf16
# prefills at 32K / 64K / 128K and a B=8 decode whose length crosses 4 * 32768
# inside its 64 steps (G goes 4 -> 5 at step 32).
PR1 = PrefillWorkload("prefill-fp32-L512-G4", 0, "fp32", 1, 2, 2, 64, 512, 128, 32, 1e4)
C2 = PrefillWorkload("prefill-bf16-L32768-G1", 1, "bf16", 1, 16, 8, 128, 32768, 32768, 4096, 1e6)
C3 = PrefillWorkload("prefill-bf16-L65536-G2-outliers", 2, "bf16", 1, 32, 8, 128, 65536, 32768,
                     4096, 1e6, outlier_frac=0.01)
C4 = PrefillWorkload("prefill-bf16-L131072-G4", 3, "bf16", 1, 32, 8, 128, 131072, 32768, 4096, 1e6)
D = DecodeWorkload("decode-bf16-B8-L131041..131104-G4to5", 4, "bf16", 8, 32, 8, 128,
                   131040, 131136, 64, 32768, 4096, 1e6)

WORKLOADS = {"PR1": PR1, "C2": C2, "C3": C3, "C4": C4, "D": D}


def _blocks(seed: int, nblocks: int, shape, dtype: str, transform=None) -> np.ndarray:
    """nblocks independent N(0,1) blocks (block c from default_rng([seed, c])),
    optionally transformed per block, then rounded to bf16 bits or kept fp32."""
    out = np.empty((nblocks,) + tuple(shape), dtype=np.uint16 if dtype == "bf16" else np.float32)

    def one(c):
        x = np.random.default_rng([seed, c]).standard_normal(shape, dtype=np.float32)
        if transform is not None:
            transform(c, x)
        out[c] = to_bf16_bits(x) if dtype == "bf16" else x

    with ThreadPoolExecutor(max_workers=min(16, max(1, os.cpu_count() or 1))) as ex:
        list(ex.map(one, range(nblocks)))
    return out


def outlier_rows(w: PrefillWorkload) -> np.ndarray:
    """Boolean [B, Hkv, L] mask of the key rows scaled for the outlier workload."""
    mask = np.zeros((w.B * w.Hkv, w.L), dtype=bool)
    n_out = int(math.floor(w.outlier_frac * w.L))
    if n_out:
        for c in range(w.B * w.Hkv):
            mask[c, np.random.default_rng([4000, c]).permutation(w.L)[:n_out]] = True
    return mask.reshape(w.B, w.Hkv, w.L)


def prefill_inputs(w: PrefillWorkload):
    """(q, k, v): q [B,Hq,L,d], k/v [B,Hkv,L,d]; uint16 bf16 bits or float32."""
    q = _blocks(1000 + w.index, w.B * w.Hq, (w.L, w.d), w.dtype).reshape(w.B, w.Hq, w.L, w.d)
    transform = None
    if w.outlier_frac > 0:
        mask = outlier_rows(w).reshape(w.B * w.Hkv, w.L)

        def transform(c, x):
            x[mask[c]] *= np.float32(w.outlier_scale)
    k = _blocks(2000 + w.index, w.B * w.Hkv, (w.L, w.d), w.dtype, transform)
    k = k.reshape(w.B, w.Hkv, w.L, w.d)
    v = _blocks(3000 + w.index, w.B * w.Hkv, (w.L, w.d), w.dtype).reshape(w.B, w.Hkv, w.L, w.d)
    return q, k, v


def decode_inputs(w: DecodeWorkload):
    """(q_steps, kcache, vcache): q_steps [steps,B,Hq,d]; caches [B,Hkv,Lcap,d].

    Rows [0, L0) are the cache before the first step; row L0 + t holds the raw
    key/value of the token appended at step t (the caller's append).
    """
    q = _blocks(1000 + w.index, w.steps, (w.B, w.Hq, w.d), w.dtype)
    kc = _blocks(2000 + w.index, w.B * w.Hkv, (w.Lcap, w.d), w.dtype).reshape(w.B, w.Hkv, w.Lcap, w.d)
    vc = _blocks(3000 + w.index, w.B * w.Hkv, (w.Lcap, w.d), w.dtype).reshape(w.B, w.Hkv, w.Lcap, w.d)
    return q, kc, vc


def sampled_rows(w: PrefillWorkload, heads=None, n_random: int = 128, seed: int = 5000) -> np.ndarray:
    """Query rows checked at sizes where the oracle cannot do every row.

    Per (b, h): rows 0..63, w0-2..w0+2, +-2 around every multiple of
    w_pretrained, the last 64 rows and n_random seeded rows.  Returns an
    [n, 3] int32 array of (b, h, i) triples.  All rows when L <= 4096.
    """
    L = w.L
    if L <= 4096:
        base = np.arange(L)
    else:
        s = set(range(min(64, L)))
        s.update(x for x in range(w.w0 - 2, w.w0 + 3) if 0 <= x < L)
        for m in range(w.w_pretrained, L + 1, w.w_pretrained):
            s.update(x for x in range(m - 2, m + 3) if 0 <= x < L)
        s.update(range(max(0, L - 64), L))
        rng = np.random.default_rng(seed + w.index)
        s.update(int(x) for x in rng.integers(0, L, size=n_random))
        base = np.array(sorted(s), dtype=np.int64)
    heads = range(w.Hq) if heads is None else heads
    trip = [(b, h, int(i)) for b in range(w.B) for h in heads for i in base]
    return np.array(trip, dtype=np.int32).reshape(-1, 3)
