"""CPU checks of the C-ABI library: it builds, loads, exports every declared
symbol, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import oracle
import rope_context_extension_jet_b200 as jl
from rope_context_extension_jet_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jetlong.h")


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return jl.load_library()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(jetlong_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("jetlong_group_size", "jetlong_position_map", "jetlong_prefill",
              "jetlong_decode_workspace_size", "jetlong_decode", "jetlong_last_error"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in declared_symbols():
        assert hasattr(lib, s), f"{s} declared in jetlong.h but not exported"


def test_exports_are_c_linkage(lib):
    out = os.popen(f"nm -D --defined-only {jl.LIB_PATH}").read()
    for s in declared_symbols():
        assert re.search(rf"\bT {s}$", out, flags=re.M), s


def test_group_size_matches_golden(lib):
    path = os.path.join(ROOT, "tests", "golden", "group_size.txt")
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        L, w, G = (int(x) for x in line.split())
        assert jl.group_size(L, w) == G
        assert jl.group_size(L, w) == oracle.group_size(L, w)
    assert jl.group_size(-1, 5) == -1 and jl.group_size(5, 0) == -1


NULL = ctypes.c_void_p(0)
P = ctypes.c_void_p(1 << 20)  # a 16-byte aligned non-null value; never dereferenced


def _prefill(lib, **kw):
    a = dict(q=P, k=P, v=P, out=P, B=1, Hq=4, Hkv=2, L=64, d=128, w0=8, wp=32, theta=1e6,
             scale=0.088, dtype=0)
    a.update(kw)
    return lib.jetlong_prefill(a["q"], a["k"], a["v"], a["out"], a["B"], a["Hq"], a["Hkv"], a["L"],
                               a["d"], a["w0"], a["wp"], a["theta"], a["scale"], a["dtype"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(q=NULL), 1), (dict(out=NULL), 1), (dict(k=ctypes.c_void_p((1 << 20) + 2)), 1),
    (dict(B=0), 1), (dict(Hq=0), 1), (dict(Hkv=3), 1), (dict(L=0), 1), (dict(w0=-1), 1),
    (dict(wp=0), 1), (dict(theta=1.0), 1), (dict(theta=float("nan")), 1), (dict(scale=0.0), 1),
    (dict(scale=float("inf")), 1), (dict(dtype=7), 1), (dict(d=96), 2), (dict(d=0), 1),
])
def test_prefill_rejects_bad_arguments_on_host(lib, kw, status):
    before = jl.launch_count()
    assert _prefill(lib, **kw) == status
    assert jl.launch_count() == before  # nothing launched
    assert jl.last_error() != ""


def _decode(lib, **kw):
    a = dict(q=P, kc=P, vc=P, out=P, B=2, Hq=8, Hkv=2, L=100, Lcap=128, d=128, w0=8, wp=32,
             theta=1e6, scale=0.088, dtype=0, ws=P, wsb=1 << 30)
    a.update(kw)
    return lib.jetlong_decode(a["q"], a["kc"], a["vc"], a["out"], a["B"], a["Hq"], a["Hkv"],
                              a["L"], a["Lcap"], a["d"], a["w0"], a["wp"], a["theta"], a["scale"],
                              a["dtype"], a["ws"], a["wsb"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(kc=NULL), 1), (dict(ws=NULL), 1), (dict(L=0), 1), (dict(L=129), 1), (dict(wsb=16), 1),
    (dict(Hkv=3), 1), (dict(d=80), 2), (dict(w0=-2), 1), (dict(scale=-1.0), 1),
])
def test_decode_rejects_bad_arguments_on_host(lib, kw, status):
    before = jl.launch_count()
    assert _decode(lib, **kw) == status
    assert jl.launch_count() == before


def test_decode_workspace_size(lib):
    assert jl.decode_workspace_size(8, 32, 8, 131136, 128) > 0
    assert jl.decode_workspace_size(8, 32, 8, 131136, 96) == 0
    assert jl.decode_workspace_size(8, 30, 8, 131136, 128) == 0
    # monotone in the cache capacity
    assert jl.decode_workspace_size(1, 4, 1, 1000, 64) <= jl.decode_workspace_size(1, 4, 1, 9000, 64)


def test_position_map_rejects_bad_arguments(lib):
    assert lib.jetlong_position_map(NULL, 10, 4, NULL) == 1
    assert lib.jetlong_position_map(P, 0, 4, NULL) == 1
    assert lib.jetlong_position_map(P, 10, 0, NULL) == 1


def _chunk(lib, **kw):
    a = dict(q=P, kc=P, vc=P, out=P, B=1, Hq=4, Hkv=1, P0=100, C=28, Lcap=128, d=128, w0=8, wp=32,
             theta=1e6, scale=0.088, dtype=0)
    a.update(kw)
    return lib.jetlong_prefill_chunk(a["q"], a["kc"], a["vc"], a["out"], a["B"], a["Hq"], a["Hkv"],
                                     a["P0"], a["C"], a["Lcap"], a["d"], a["w0"], a["wp"], a["theta"],
                                     a["scale"], a["dtype"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(q=NULL), 1), (dict(vc=NULL), 1), (dict(P0=-1), 1), (dict(C=0), 1), (dict(C=29), 1),
    (dict(Lcap=0), 1), (dict(Hkv=3), 1), (dict(d=96), 2), (dict(wp=0), 1), (dict(dtype=5), 1),
    (dict(out=ctypes.c_void_p((1 << 20) + 8)), 1),
])
def test_prefill_chunk_rejects_bad_arguments_on_host(lib, kw, status):
    before = jl.launch_count()
    assert _chunk(lib, **kw) == status
    assert jl.launch_count() == before
    assert jl.last_error() != ""


@pytest.mark.parametrize("kw,status", [
    (dict(kc=NULL), 1), (dict(ws=NULL), 1), (dict(L=0), 1), (dict(L=129), 1), (dict(wsb=16), 1),
    (dict(Hkv=3), 1), (dict(d=80), 2),
])
def test_decode_rope_cache_rejects_bad_arguments_on_host(lib, kw, status):
    a = dict(q=P, kc=P, vc=P, out=P, B=2, Hq=8, Hkv=2, L=100, Lcap=128, d=128, w0=8, wp=32,
             theta=1e6, scale=0.088, dtype=0, ws=P, wsb=1 << 30)
    a.update(kw)
    before = jl.launch_count()
    st = lib.jetlong_decode_rope_cache(a["q"], a["kc"], a["vc"], a["out"], a["B"], a["Hq"], a["Hkv"],
                                       a["L"], a["Lcap"], a["d"], a["w0"], a["wp"], a["theta"],
                                       a["scale"], a["dtype"], a["ws"], a["wsb"], NULL)
    assert st == status
    assert jl.launch_count() == before


@pytest.mark.parametrize("lens,kw,status", [
    ([10, 20], dict(), None), ([0, 20], dict(), 1), ([10, 65], dict(), 1), (None, dict(), 1),
    ([10, 20], dict(q=NULL), 1), ([10, 20], dict(lse=ctypes.c_void_p((1 << 20) + 2)), 1),
    ([10, 20], dict(d=96), 2),
])
def test_prefill_varlen_rejects_bad_arguments_on_host(lib, lens, kw, status):
    a = dict(q=P, k=P, v=P, out=P, lse=NULL, B=2, Hq=4, Hkv=2, Lmax=64, d=128, w0=8, wp=32,
             theta=1e6, scale=0.088, dtype=0)
    a.update(kw)
    arr = (ctypes.c_int32 * 2)(*lens) if lens is not None else None
    if status is None:
        return  # valid arguments would launch; covered by the GPU tests
    before = jl.launch_count()
    st = lib.jetlong_prefill_varlen(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"],
                                    a["Hkv"], arr, a["Lmax"], a["d"], a["w0"], a["wp"], a["theta"],
                                    a["scale"], a["dtype"], NULL)
    assert st == status
    assert jl.launch_count() == before


def test_prefill_ie_workspace_and_arguments(lib):
    # three fp32 pass outputs and three fp32 LSE arrays, each segment 256-byte aligned
    assert lib.jetlong_prefill_ie_workspace_size(1, 4, 600, 128, 0) == 3 * (4 * 600 * 128 * 4 + 9728)
    assert lib.jetlong_prefill_ie_workspace_size(1, 4, 600, 128, 1) == 3 * (4 * 600 * 128 * 4 + 9728)
    assert lib.jetlong_prefill_ie_workspace_size(1, 4, 600, 96, 0) == 0
    before = jl.launch_count()
    args = [P, P, P, P, 1, 4, 2, 64, 128, 8, 32, 1e6, 0.088, 0]
    assert lib.jetlong_prefill_ie(*args, NULL, 1 << 30, NULL) == 1          # null workspace
    assert lib.jetlong_prefill_ie(*args, P, 16, NULL) == 1                  # too small
    args[5] = 3
    assert lib.jetlong_prefill_ie(*args, P, 1 << 30, NULL) == 1             # Hq % Hkv
    assert jl.launch_count() == before


def _streamed(lib, **kw):
    a = dict(qh=P, kh=P, vh=P, oh=P, qd=P, kd=P, vd=P, od=P, B=1, Hq=4, Hkv=2, L=300, d=128, w0=8,
             wp=32, theta=1e6, scale=0.088, dtype=0, nch=4)
    a.update(kw)
    return lib.jetlong_prefill_streamed(a["qh"], a["kh"], a["vh"], a["oh"], a["qd"], a["kd"], a["vd"],
                                        a["od"], a["B"], a["Hq"], a["Hkv"], a["L"], a["d"], a["w0"],
                                        a["wp"], a["theta"], a["scale"], a["dtype"], a["nch"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(qh=NULL), 1), (dict(oh=NULL), 1), (dict(kd=NULL), 1), (dict(od=NULL), 1), (dict(L=0), 1),
    (dict(nch=0), 1), (dict(Hkv=3), 1), (dict(d=96), 2), (dict(theta=0.5), 1), (dict(dtype=5), 1),
])
def test_prefill_streamed_rejects_bad_arguments_on_host(lib, kw, status):
    before = jl.launch_count()
    assert _streamed(lib, **kw) == status
    assert jl.launch_count() == before
    assert jl.last_error() != ""


def _noalloc(lib, **kw):
    a = dict(q=P, kc=P, vc=P, out=P, B=2, Hq=8, Hkv=2, L=100, Lcap=128, d=128, w0=8, wp=32,
             theta=1e6, scale=0.088, dtype=0)
    a.update(kw)
    return lib.jetlong_decode_noalloc(a["q"], a["kc"], a["vc"], a["out"], a["B"], a["Hq"], a["Hkv"],
                                      a["L"], a["Lcap"], a["d"], a["w0"], a["wp"], a["theta"],
                                      a["scale"], a["dtype"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(q=NULL), 1), (dict(vc=ctypes.c_void_p((1 << 20) + 8)), 1), (dict(L=0), 1),
    (dict(L=129), 1), (dict(Hkv=3), 1), (dict(d=80), 2), (dict(wp=0), 1), (dict(scale=float("nan")), 1),
])
def test_decode_noalloc_rejects_bad_arguments_on_host(lib, kw, status):
    before = jl.launch_count()
    assert _noalloc(lib, **kw) == status
    assert jl.launch_count() == before
    assert jl.last_error() != ""


def test_injection_hook_arguments(lib):
    # failure-detection test hook: unknown sites and out-of-range limits are refused
    assert lib.jetlong_debug_inject_timeout(3, 2_000_000) == 1
    assert lib.jetlong_debug_inject_timeout(-1, 2_000_000) == 1
    assert lib.jetlong_debug_inject_timeout(1, 9_999) == 1
    assert lib.jetlong_debug_inject_timeout(2, 4_000_000_001) == 1
    assert "wait_cycles" in lib.jetlong_last_error().decode()
    assert lib.jetlong_debug_inject_timeout(1, 2_000_000) == 0
    assert lib.jetlong_debug_inject_timeout(0, 0) == 0  # disarmed again
