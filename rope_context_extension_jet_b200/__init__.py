"""Jet-Long dynamic bifocal RoPE attention for NVIDIA B200 -- Python binding.

Thin ctypes binding of ``libjetlong.so`` (C ABI declared in ``include/jetlong.h``).
Functions keep the C names without the ``jetlong_`` prefix.  This module only
marshals arguments: torch tensors supply device pointers and the current CUDA
stream; every step of the attention runs in the library's CUDA kernels.  There
is no fallback: if the library is missing the calls raise.

Method: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
(gist.science/it/paper/2607.07740), Metodologia 1 (local window w0 with classic
RoPE; remote pairs at f(x) = floor(x/G), G = max(1, ceil(L/w_pretrained))) and
Metodologia 2 (rotations applied on the fly to an untouched cache; one exact
distance-routed softmax).
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

__all__ = [
    "BF16", "FP32", "JetLongError", "load_library", "group_size", "position_map", "prefill",
    "prefill_chunk", "prefill_varlen", "prefill_ie", "prefill_streamed", "decode_workspace_size",
    "decode", "decode_rope_cache", "decode_noalloc", "device_status", "last_error", "launch_count",
    "DECODE_NOALLOC_SCRATCH_BYTES", "selftest_wait_timeout", "debug_inject_timeout",
    "INJECT_PREFILL_KEY_TILE", "INJECT_DECODE_COPY", "debug_rope_phase", "debug_tile_plan", "debug_ex2", "debug_rope_keys",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libjetlong.so")

BF16 = 0
FP32 = 1
_STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT"}

_lock = threading.Lock()
_lib = None


class JetLongError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"jetlong {_STATUS.get(status, status)}: {message}")
        self.status = status


def load_library(path: str | None = None):
    """Load libjetlong.so (built in-tree by ``python -m rope_context_extension_jet_b200._build``)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with "
                               "`python -m rope_context_extension_jet_b200._build`")
        lib = ctypes.CDLL(p)
        vp, i32, i64, sz, dbl, flt = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_size_t, ctypes.c_double, ctypes.c_float)
        lib.jetlong_group_size.restype = i64
        lib.jetlong_group_size.argtypes = [i64, i64]
        lib.jetlong_position_map.restype = i32
        lib.jetlong_position_map.argtypes = [vp, i64, i64, vp]
        lib.jetlong_prefill.restype = i32
        lib.jetlong_prefill.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                        dbl, flt, i32, vp]
        lib.jetlong_prefill_ie_workspace_size.restype = sz
        lib.jetlong_prefill_ie_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        lib.jetlong_prefill_ie.restype = i32
        lib.jetlong_prefill_ie.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, dbl, flt,
                                           i32, vp, sz, vp]
        lib.jetlong_prefill_streamed.restype = i32
        lib.jetlong_prefill_streamed.argtypes = [vp] * 8 + [i32, i32, i32, i32, i32, i32, i32, dbl, flt,
                                                            i32, i32, vp]
        lib.jetlong_prefill_varlen.restype = i32
        lib.jetlong_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, vp, i32, i32, i32,
                                               i32, dbl, flt, i32, vp]
        lib.jetlong_prefill_chunk.restype = i32
        lib.jetlong_prefill_chunk.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                              i32, i32, dbl, flt, i32, vp]
        lib.jetlong_decode_workspace_size.restype = sz
        lib.jetlong_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        for fn in (lib.jetlong_decode, lib.jetlong_decode_rope_cache):
            fn.restype = i32
            fn.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                           dbl, flt, i32, vp, sz, vp]
        lib.jetlong_decode_noalloc.restype = i32
        lib.jetlong_decode_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                               i32, dbl, flt, i32, vp]
        lib.jetlong_selftest_wait_timeout.restype = i32
        lib.jetlong_selftest_wait_timeout.argtypes = [vp]
        lib.jetlong_debug_inject_timeout.restype = i32
        lib.jetlong_debug_inject_timeout.argtypes = [i32, ctypes.c_longlong]
        lib.jetlong_debug_rope_phase.restype = i32
        lib.jetlong_debug_rope_phase.argtypes = [vp, i64, i32, dbl, i32, vp, vp]
        lib.jetlong_debug_tile_plan.restype = i32
        lib.jetlong_debug_tile_plan.argtypes = [i32, i32, i32, i32, vp, vp, vp]
        lib.jetlong_debug_ex2.restype = i32
        lib.jetlong_debug_ex2.argtypes = [vp, i64, vp, vp]
        lib.jetlong_debug_rope_keys.restype = i32
        lib.jetlong_debug_rope_keys.argtypes = [vp, i32, i32, i32, i32, dbl, vp, vp, ctypes.POINTER(ctypes.c_int), vp]
        lib.jetlong_device_status.restype = i32
        lib.jetlong_device_status.argtypes = [vp]
        lib.jetlong_last_error.restype = ctypes.c_char_p
        lib.jetlong_last_error.argtypes = []
        lib.jetlong_launch_count.restype = ctypes.c_uint64
        lib.jetlong_launch_count.argtypes = []
        if path is None:
            _lib = lib
        return lib


def _check(status: int, lib=None):
    if status != 0:
        lib = lib or load_library()
        raise JetLongError(status, lib.jetlong_last_error().decode())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")


def _dev(t, name):
    import torch
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device} but the library runs on the current device "
                         f"cuda:{torch.cuda.current_device()} (select it with torch.cuda.device)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _like(t, ref, name, ref_name):
    """The library writes ``t`` with ``ref``'s shape and element type."""
    if tuple(t.shape) != tuple(ref.shape) or t.dtype != ref.dtype:
        raise ValueError(f"{name} must match {ref_name}: shape {tuple(ref.shape)}, dtype {ref.dtype} "
                         f"(got {tuple(t.shape)}, {t.dtype})")


def _same_dtype(*named):
    if len({t.dtype for t, _ in named}) != 1:
        raise TypeError(", ".join(n for _, n in named) + " must share a dtype")


def last_error() -> str:
    return load_library().jetlong_last_error().decode()


def launch_count() -> int:
    return int(load_library().jetlong_launch_count())


def group_size(L: int, w_pretrained: int) -> int:
    """G = max(1, ceil(L / w_pretrained)); -1 for invalid arguments."""
    return int(load_library().jetlong_group_size(int(L), int(w_pretrained)))


def position_map(out, L: int, w_pretrained: int, stream=None):
    """Write floor(x / G) for x in [0, L) into the int32 CUDA tensor ``out``."""
    import torch
    if out.dtype != torch.int32 or out.numel() < L:
        raise ValueError("out must be an int32 tensor with at least L elements")
    lib = load_library()
    _check(lib.jetlong_position_map(_dev(out, "out"), int(L), int(w_pretrained), _stream(stream)),
           lib)
    return out


def prefill(q, k, v, out=None, *, w0: int, w_pretrained: int, rope_theta: float,
            scale: float | None = None, stream=None):
    """Routed causal attention over raw q [B,Hq,L,d], k/v [B,Hkv,L,d] (bf16 or fp32)."""
    import torch
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, L, d] matching q")
    _same_dtype((q, "q"), (k, "k"), (v, "v"))
    if out is None:
        out = torch.empty_like(q)
    _like(out, q, "out", "q")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    lib = load_library()
    _check(lib.jetlong_prefill(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"),
                               B, Hq, Hkv, L, d, int(w0), int(w_pretrained), float(rope_theta),
                               float(scale), _dtype_code(q), _stream(stream)), lib)
    return out


def prefill_chunk(q, kcache, vcache, P: int, out=None, *, w0: int, w_pretrained: int,
                  rope_theta: float, scale: float | None = None, stream=None):
    """Chunked prefill: raw queries q [B,Hq,C,d] at positions [P, P+C) over cache
    rows [0, P+C) of kcache/vcache [B,Hkv,Lcap,d]; G from P + C."""
    import torch
    B, Hq, C, d = q.shape
    _, Hkv, Lcap, _ = kcache.shape
    if vcache.shape != kcache.shape or kcache.shape[0] != B or kcache.shape[3] != d:
        raise ValueError("kcache and vcache must be [B, Hkv, Lcap, d] matching q")
    _same_dtype((q, "q"), (kcache, "kcache"), (vcache, "vcache"))
    if out is None:
        out = torch.empty_like(q)
    _like(out, q, "out", "q")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    lib = load_library()
    _check(lib.jetlong_prefill_chunk(_dev(q, "q"), _dev(kcache, "kcache"), _dev(vcache, "vcache"),
                                     _dev(out, "out"), B, Hq, Hkv, int(P), C, Lcap, d, int(w0),
                                     int(w_pretrained), float(rope_theta), float(scale),
                                     _dtype_code(q), _stream(stream)), lib)
    return out


def prefill_ie(q, k, v, out=None, *, w0: int, w_pretrained: int, rope_theta: float,
               scale: float | None = None, workspace=None, stream=None):
    """The pages' three-pass inclusion-exclusion form of the prefill (same
    result as ``prefill``; for comparing the two forms)."""
    import torch
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, L, d] matching q")
    _same_dtype((q, "q"), (k, "k"), (v, "v"))
    if out is None:
        out = torch.empty_like(q)
    _like(out, q, "out", "q")
    lib = load_library()
    need = int(lib.jetlong_prefill_ie_workspace_size(B, Hq, L, d, _dtype_code(q)))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    _check(lib.jetlong_prefill_ie(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), B, Hq,
                                  Hkv, L, d, int(w0), int(w_pretrained), float(rope_theta),
                                  float(scale), _dtype_code(q), _dev(workspace, "workspace"),
                                  workspace.numel() * workspace.element_size(), _stream(stream)), lib)
    return out


def _host(t, name):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def prefill_streamed(q_host, k_host, v_host, out_host, q_dev, k_dev, v_dev, out_dev, *, w0: int,
                     w_pretrained: int, rope_theta: float, scale: float | None = None, nchunks: int = 16,
                     stream=None):
    """Prefill from (page-locked) host tensors into ``out_host`` with the transfers
    overlapped with the compute, chunk by chunk; ``*_dev`` are device tensors of
    the same shapes used as staging.  Asynchronous on ``stream``."""
    B, Hq, L, d = q_host.shape
    Hkv = k_host.shape[1]
    for t, n in ((q_dev, "q_dev"), (out_dev, "out_dev"), (out_host, "out_host")):
        if t.shape != q_host.shape or t.dtype != q_host.dtype:
            raise ValueError(f"{n} must match q_host's shape and dtype")
    for t, n in ((k_dev, "k_dev"), (v_dev, "v_dev"), (v_host, "v_host")):
        if t.shape != k_host.shape or t.dtype != k_host.dtype:
            raise ValueError(f"{n} must match k_host's shape and dtype")
    if k_host.shape[0] != B or k_host.shape[2] != L or k_host.shape[3] != d:
        raise ValueError("k_host must be [B, Hkv, L, d] matching q_host")
    _same_dtype((q_host, "q_host"), (k_host, "k_host"))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    lib = load_library()
    _check(lib.jetlong_prefill_streamed(_host(q_host, "q_host"), _host(k_host, "k_host"),
                                        _host(v_host, "v_host"), _host(out_host, "out_host"),
                                        _dev(q_dev, "q_dev"), _dev(k_dev, "k_dev"), _dev(v_dev, "v_dev"),
                                        _dev(out_dev, "out_dev"), B, Hq, Hkv, L, d, int(w0),
                                        int(w_pretrained), float(rope_theta), float(scale),
                                        _dtype_code(q_host), int(nchunks), _stream(stream)), lib)
    return out_host


def prefill_varlen(q, k, v, lens, out=None, *, w0: int, w_pretrained: int, rope_theta: float,
                   scale: float | None = None, with_lse: bool = False, stream=None):
    """Variable-length batch in padded tensors q/out [B,Hq,Lmax,d], k/v
    [B,Hkv,Lmax,d]; sequence b uses rows [0, lens[b]) and its own G.  With
    ``with_lse`` also returns the per-row natural-log LSE [B,Hq,Lmax] (fp32;
    rows past a sequence's length are left as allocated)."""
    import numpy as _np
    import torch
    B, Hq, Lmax, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, Lmax, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, Lmax, d] matching q")
    _same_dtype((q, "q"), (k, "k"), (v, "v"))
    lens = _np.ascontiguousarray(_np.asarray(lens, dtype=_np.int32).reshape(-1))
    if lens.shape[0] != B:
        raise ValueError("lens must have one length per sequence")
    if out is None:
        out = torch.empty_like(q)
    _like(out, q, "out", "q")
    lse = torch.empty((B, Hq, Lmax), dtype=torch.float32, device=q.device) if with_lse else None
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    lib = load_library()
    _check(lib.jetlong_prefill_varlen(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"),
                                      lse.data_ptr() if lse is not None else None, B, Hq, Hkv,
                                      lens.ctypes.data, Lmax, d, int(w0), int(w_pretrained),
                                      float(rope_theta), float(scale), _dtype_code(q),
                                      _stream(stream)), lib)
    return (out, lse) if with_lse else out


def _decode_shapes(q, kcache, vcache):
    if q.dim() != 3 or kcache.dim() != 4:
        raise ValueError("q must be [B, Hq, d] and the caches [B, Hkv, Lcap, d]")
    if vcache.shape != kcache.shape:
        raise ValueError("kcache and vcache must have the same shape")
    if kcache.shape[0] != q.shape[0] or kcache.shape[3] != q.shape[2]:
        raise ValueError("the caches must be [B, Hkv, Lcap, d] with q's B and d")
    _same_dtype((q, "q"), (kcache, "kcache"), (vcache, "vcache"))


def decode_workspace_size(B: int, Hq: int, Hkv: int, Lcap: int, d: int) -> int:
    return int(load_library().jetlong_decode_workspace_size(B, Hq, Hkv, Lcap, d))


def decode_rope_cache(q, kcache, vcache, L: int, out=None, *, w0: int, w_pretrained: int,
                      rope_theta: float, scale: float | None = None, workspace=None, stream=None):
    """One decode step over a standard RoPE cache (key row j stored rotated to
    position j): jetlong_decode_rope_cache."""
    return decode(q, kcache, vcache, L, out, w0=w0, w_pretrained=w_pretrained,
                  rope_theta=rope_theta, scale=scale, workspace=workspace, stream=stream,
                  _entry="jetlong_decode_rope_cache")


def decode(q, kcache, vcache, L: int, out=None, *, w0: int, w_pretrained: int,
           rope_theta: float, scale: float | None = None, workspace=None, stream=None,
           _entry: str = "jetlong_decode"):
    """One decode step: raw q [B,Hq,d] at position L-1 over cache rows [0, L)."""
    import torch
    _decode_shapes(q, kcache, vcache)
    B, Hq, d = q.shape
    _, Hkv, Lcap, _ = kcache.shape
    if out is None:
        out = torch.empty_like(q)
    _like(out, q, "out", "q")
    need = decode_workspace_size(B, Hq, Hkv, Lcap, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    lib = load_library()
    _check(getattr(lib, _entry)(_dev(q, "q"), _dev(kcache, "kcache"), _dev(vcache, "vcache"),
                              _dev(out, "out"), B, Hq, Hkv, int(L), Lcap, d, int(w0),
                              int(w_pretrained), float(rope_theta), float(scale),
                              _dtype_code(q), _dev(workspace, "workspace"),
                              workspace.numel() * workspace.element_size(), _stream(stream)), lib)
    return out


# Size of the library's fixed decode scratch array (JETLONG_DECODE_NOALLOC_SCRATCH_BYTES).
DECODE_NOALLOC_SCRATCH_BYTES = 4 << 20


def decode_noalloc(q, kcache, vcache, L: int, out=None, *, w0: int, w_pretrained: int,
                   rope_theta: float, scale: float | None = None, stream=None):
    """Decode step for callers that cannot allocate device memory.

    Same result as ``decode`` but without a workspace: the library keeps the
    split partials in its own fixed device array (shared by all calls on a
    device, so calls that overlap on the GPU race).  ``out`` should be
    preallocated by such callers; problems too large for the array raise
    JetLongError(INVALID_ARG).
    """
    import torch
    _decode_shapes(q, kcache, vcache)
    B, Hq, d = q.shape
    _, Hkv, Lcap, _ = kcache.shape
    if out is None:
        out = torch.empty_like(q)
    _like(out, q, "out", "q")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    lib = load_library()
    _check(lib.jetlong_decode_noalloc(_dev(q, "q"), _dev(kcache, "kcache"), _dev(vcache, "vcache"),
                                      _dev(out, "out"), B, Hq, Hkv, int(L), Lcap, d, int(w0),
                                      int(w_pretrained), float(rope_theta), float(scale),
                                      _dtype_code(q), _stream(stream)), lib)
    return out


def selftest_wait_timeout(stream=None):
    """Launch the bounded-wait self test; the next device_status() raises TIMEOUT."""
    lib = load_library()
    _check(lib.jetlong_selftest_wait_timeout(_stream(stream)), lib)


# Sites of the failure-detection test hook (JETLONG_INJECT_*).
INJECT_PREFILL_KEY_TILE = 1
INJECT_DECODE_COPY = 2


def debug_inject_timeout(site: int, wait_cycles: int):
    """Arm the one-shot test hook: the next prefill or decode call of this thread
    withholds one barrier arrival (``site``) with every bounded wait limited to
    ``wait_cycles`` SM cycles, so its waits expire and the following
    device_status() raises TIMEOUT (jetlong_debug_inject_timeout)."""
    lib = load_library()
    _check(lib.jetlong_debug_inject_timeout(int(site), int(wait_cycles)), lib)


def debug_rope_phase(pos, d: int, rope_theta: float, accurate: bool, stream=None):
    """(cos, sin) of pos[i] * theta_m as the kernels form them: float32 CUDA
    tensor [n, d/2, 2] (test hook jetlong_debug_rope_phase).  pos: int32 CUDA
    tensor holding uint32 positions."""
    import torch
    if pos.dtype != torch.int32:
        raise TypeError("pos must be int32 (uint32 bit patterns)")
    out = torch.empty((pos.numel(), d // 2, 2), dtype=torch.float32, device=pos.device)
    lib = load_library()
    _check(lib.jetlong_debug_rope_phase(_dev(pos, "pos"), pos.numel(), int(d), float(rope_theta),
                                        1 if accurate else 0, _dev(out, "out"), _stream(stream)), lib)
    return out


def debug_tile_plan(P: int, C: int, w0: int, max_kb: int, stream=None):
    """The prefill's tile plan (nR, kE0, nkb) per query block and the class of
    every tile (0 remote, 1 local, 2 both; -1 past nkb): test hook
    jetlong_debug_tile_plan.  Returns (plan [nqb, 3] int32, cls [nqb, max_kb] int8)."""
    import torch
    nqb = (C + 127) // 128
    plan = torch.empty((nqb, 3), dtype=torch.int32, device="cuda")
    cls = torch.full((nqb, max_kb), -1, dtype=torch.int8, device="cuda")
    lib = load_library()
    _check(lib.jetlong_debug_tile_plan(int(P), int(C), int(w0), int(max_kb), _dev(plan, "plan"), _dev(cls, "cls"),
                                       _stream(stream)), lib)
    return plan, cls


def debug_ex2(y, stream=None):
    """2^y as the one-CTA prefill's softmax forms part of its exponentials on the
    FMA pipe (test hook jetlong_debug_ex2).  y: float32 CUDA tensor with an even
    number of elements; returns a tensor of the same shape."""
    import torch
    if y.dtype != torch.float32 or y.numel() % 2:
        raise TypeError("y must be float32 with an even number of elements")
    y = y.contiguous()
    out = torch.empty_like(y)
    lib = load_library()
    _check(lib.jetlong_debug_ex2(_dev(y, "y"), y.numel(), _dev(out, "out"), _stream(stream)), lib)
    return out


def debug_rope_keys(k, G: int, rope_theta: float, remote: bool = True, stream=None):
    """The bf16 prefill's key rotation pass on its own (test hook
    jetlong_debug_rope_keys): k, a bf16 CUDA tensor [planes, L, d], rotated to
    positions j and floor(j / G) times the prefill's key scale 2^e.  Returns
    (kl, kr or None, e); kl and kr are fp16 tensors of k's shape."""
    import ctypes as ct
    import torch
    if k.dtype != torch.bfloat16 or k.dim() != 3:
        raise TypeError("k must be a bf16 tensor [planes, L, d]")
    k = k.contiguous()
    kl = torch.empty(k.shape, dtype=torch.float16, device=k.device)
    kr = torch.empty_like(kl) if remote else None
    ex = ct.c_int(0)
    lib = load_library()
    _check(lib.jetlong_debug_rope_keys(_dev(k, "k"), k.shape[0], k.shape[1], k.shape[2], int(G), float(rope_theta),
                                       _dev(kl, "kl"), _dev(kr, "kr") if remote else None, ct.byref(ex),
                                       _stream(stream)), lib)
    return kl, kr, int(ex.value)


def device_status(stream=None):
    """Synchronise the stream and raise if a kernel's bounded wait expired."""
    lib = load_library()
    _check(lib.jetlong_device_status(_stream(stream)), lib)
