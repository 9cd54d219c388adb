"""TEST INFRASTRUCTURE ONLY -- the fp64 CPU oracle for Jet-Long bifocal RoPE attention.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``rope_context_extension_jet_b200``) never imports it and shares no code with it.

The arithmetic lives in ``jetlong_oracle.c`` (plain C, fp64, one explicit RoPE
rotation per (query, key) pair).  This module only compiles it with gcc and
marshals numpy arrays through ctypes.

Method source: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
RoPE" (gist.science/it/paper/2607.07740), Metodologia 1 (local window w0 with
classic RoPE; remote positions f(x) = floor(x/G), G = max(1, ceil(L/w_pretrained)))
and Metodologia 2 (rotations compose additively; one exact distance-routed
softmax).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "jetlong_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libjetlong_oracle.so")

IN_BF16 = 0
IN_FP32 = 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle C file into a shared library (gcc, IEEE fp64, no fast-math)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           "-fno-fast-math", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building if needed) the oracle library; returns the ctypes handle."""
    global _lib
    with _lock:
        if path is None and _lib is not None:
            return _lib
        p = path or build()
        lib = ctypes.CDLL(p)
        i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.jlo_group_size.restype = i64
        lib.jlo_group_size.argtypes = [i64, i64]
        lib.jlo_remote_position.restype = i64
        lib.jlo_remote_position.argtypes = [i64, i64]
        lib.jlo_rotate.restype = None
        lib.jlo_rotate.argtypes = [vp, vp, i32, i64, dbl]
        lib.jlo_pair_logit.restype = dbl
        lib.jlo_pair_logit.argtypes = [vp, vp, i32, i64, i64, i64, i64, dbl]
        lib.jlo_prefill_rows.restype = i32
        lib.jlo_prefill_rows.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                         dbl, dbl, vp, i64, vp, i32]
        lib.jlo_prefill_rows_lse.restype = i32
        lib.jlo_prefill_rows_lse.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                             dbl, dbl, vp, i64, vp, vp, i32]
        for fn in (lib.jlo_decode, lib.jlo_decode_rope_cache):
            fn.restype = i32
            fn.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, i32, dbl, dbl, vp, i32]
        lib.jlo_rotate_rows.restype = i32
        lib.jlo_rotate_rows.argtypes = [vp, i32, i64, i64, i32, dbl, vp]
        if path is None:
            _lib = lib
        return lib


def _as_input(a: np.ndarray):
    """bf16 inputs travel as uint16 bit patterns, fp32 as float32; both C-contiguous."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, IN_BF16
    if a.dtype == np.float32:
        return a, IN_FP32
    raise TypeError(f"oracle inputs must be uint16 (bf16 bits) or float32, got {a.dtype}")


def group_size(L: int, w_pretrained: int, lib=None) -> int:
    return int((lib or load()).jlo_group_size(L, w_pretrained))


def remote_position(x: int, G: int, lib=None) -> int:
    return int((lib or load()).jlo_remote_position(x, G))


def rotate(x: np.ndarray, p: int, rope_theta: float, lib=None) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    (lib or load()).jlo_rotate(x.ctypes.data, y.ctypes.data, x.shape[-1], int(p), float(rope_theta))
    return y


def pair_logit(q, k, i, j, w0, G, rope_theta, lib=None) -> float:
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    return float((lib or load()).jlo_pair_logit(q.ctypes.data, k.ctypes.data, q.shape[-1],
                                                int(i), int(j), int(w0), int(G), float(rope_theta)))


def prefill_rows(q, k, v, rows, *, w0, w_pretrained, rope_theta, scale, nthreads=0, lib=None,
                 with_lse=False):
    """Routed attention outputs (fp64, [n, d]) for the (b, h, i) triples in ``rows``
    (and, with ``with_lse``, each row's log sum_j exp(scale * logit) as [n]).

    q: [B,Hq,L,d], k/v: [B,Hkv,L,d] as uint16 bf16 bits or float32.
    """
    q, dq = _as_input(q)
    k, dk = _as_input(k)
    v, dv = _as_input(v)
    if not (dq == dk == dv):
        raise TypeError("q, k, v must share one input dtype")
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    out = np.empty((rows.shape[0], d), dtype=np.float64)
    lse = np.empty(rows.shape[0], dtype=np.float64)
    st = (lib or load()).jlo_prefill_rows_lse(q.ctypes.data, k.ctypes.data, v.ctypes.data, dq,
                                              B, Hq, Hkv, L, d, int(w0), int(w_pretrained),
                                              float(rope_theta), float(scale),
                                              rows.ctypes.data, rows.shape[0], out.ctypes.data,
                                              lse.ctypes.data, int(nthreads))
    if st != 0:
        raise ValueError(f"oracle prefill_rows failed with status {st}")
    return (out, lse) if with_lse else out


def prefill(q, k, v, *, w0, w_pretrained, rope_theta, scale, nthreads=0, lib=None):
    """Full routed attention output [B,Hq,L,d] (fp64); for small L only."""
    B, Hq, L, d = q.shape
    b, h, i = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L), indexing="ij")
    rows = np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1)
    out = prefill_rows(q, k, v, rows, w0=w0, w_pretrained=w_pretrained, rope_theta=rope_theta,
                       scale=scale, nthreads=nthreads, lib=lib)
    return out.reshape(B, Hq, L, d)


def rotate_rows(x, rope_theta, lib=None) -> np.ndarray:
    """Row j of every [rows, d] plane of x rotated to position j (fp64): a
    standard RoPE key cache built from raw keys."""
    x, dx = _as_input(x)
    d, nrows = x.shape[-1], x.shape[-2]
    nplanes = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    out = np.empty(x.shape, dtype=np.float64)
    st = (lib or load()).jlo_rotate_rows(x.ctypes.data, dx, nplanes, nrows, d, float(rope_theta),
                                         out.ctypes.data)
    if st != 0:
        raise ValueError(f"oracle rotate_rows failed with status {st}")
    return out


def decode_rope_cache(q, kcache, vcache, L, *, w0, w_pretrained, rope_theta, scale, nthreads=0,
                      lib=None):
    """Decode output [B,Hq,d] (fp64) over a standard RoPE cache: key row j is
    stored rotated to its exact position j."""
    return decode(q, kcache, vcache, L, w0=w0, w_pretrained=w_pretrained, rope_theta=rope_theta,
                  scale=scale, nthreads=nthreads, lib=lib, _fn="jlo_decode_rope_cache")


def decode(q, kcache, vcache, L, *, w0, w_pretrained, rope_theta, scale, nthreads=0, lib=None,
           _fn="jlo_decode"):
    """Decode output [B,Hq,d] (fp64) for a query at position L-1 over cache rows [0, L)."""
    q, dq = _as_input(q)
    kcache, dk = _as_input(kcache)
    vcache, dv = _as_input(vcache)
    if not (dq == dk == dv):
        raise TypeError("q and caches must share one input dtype")
    B, Hq, d = q.shape
    Hkv, Lcap = kcache.shape[1], kcache.shape[2]
    out = np.empty((B, Hq, d), dtype=np.float64)
    st = getattr(lib or load(), _fn)(q.ctypes.data, kcache.ctypes.data, vcache.ctypes.data, dq,
                                    B, Hq, Hkv, int(L), Lcap, d, int(w0), int(w_pretrained),
                                    float(rope_theta), float(scale), out.ctypes.data, int(nthreads))
    if st != 0:
        raise ValueError(f"oracle decode failed with status {st}")
    return out
