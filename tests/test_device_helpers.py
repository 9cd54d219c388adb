"""GPU unit tests of the attention kernels' device helpers, each run on its own
through a test hook and checked against an independent host computation.

* RoPE phase (jetlong_debug_rope_phase): the kernels form the angle of pair m
  at position p as an exact fixed-point fraction of a turn, then take sin / cos
  (sincospif, or __sincosf in the hot loops).  Checked against long-double
  cos / sin of frac(p theta_m / 2 pi) for positions up to 2^31 - 1, with stated
  bounds: 1e-6 (accurate) and 2e-6 (fast) absolute.  A plain fp32 p * theta_m
  would be off by radians there.  Rotations compose additively (Jet-Long,
  gist.science/it/paper/2607.07740, Metodologia 2), which is what lets the
  kernels step angles row by row from these values.
* Tile plan (jetlong_debug_tile_plan): every (query block, key block) tile's
  class against brute-force classification of its causal pairs (local iff
  i - j < w0, Metodologia 1), and the plan's two phases against the sets of key
  blocks holding remote and local pairs.
* Key rotation pass (jetlong_debug_rope_keys): the bf16 prefill rotates each
  call's keys once, to j and to floor(j / G), times its power-of-two key scale,
  into fp16 copies its kernels load.  Checked against the oracle's fp64
  rotation of the same bf16 keys (row by row at those positions) within fp16
  rounding plus the fast sine's error, and the scale's exponent against
  13 - floor(log2 max|k|) from numpy.
* Softmax exponential on the FMA pipe (jetlong_debug_ex2): 2^y as a quarter of
  the one-CTA prefill's exponentials are formed, against numpy's exp2 in fp64
  over the softmax's range (relative error <= 1e-4, well below the 2^-9 of
  the bf16 P it feeds), with -inf and values below -127 giving exactly 0 and
  NaN staying NaN.
"""
import numpy as np
import pytest

import rope_context_extension_jet_b200 as jl

pytestmark = pytest.mark.gpu


def _ref_cos_sin(pos, d, theta):
    ld = np.longdouble
    assert np.finfo(ld).nmant >= 63, "needs x86 extended precision for the reference"
    m = np.arange(d // 2, dtype=ld)
    th = np.power(ld(theta), -ld(2) * m / ld(d))
    two_pi = ld("6.283185307179586476925286766559")
    turns = np.asarray(pos, dtype=ld)[:, None] * (th / two_pi)[None, :]
    frac = turns - np.floor(turns)
    ang = frac * two_pi
    return np.cos(ang).astype(np.float64), np.sin(ang).astype(np.float64)


def _positions():
    rng = np.random.default_rng(90)
    p = np.concatenate([np.arange(0, 1024), np.array([131071, 131072, 131103, 2 ** 20, 2 ** 24 + 1, 2 ** 30,
                                                      2 ** 31 - 2, 2 ** 31 - 1]),
                        rng.integers(0, 2 ** 31, size=4000)]).astype(np.int64)
    return p


@pytest.mark.parametrize("d,theta", [(128, 1e6), (64, 1e4), (128, 1e4)])
@pytest.mark.parametrize("accurate,bound", [(True, 1e-6), (False, 2e-6)])
def test_rope_phase_against_long_double(d, theta, accurate, bound):
    import torch
    pos = _positions()
    got = jl.debug_rope_phase(torch.from_numpy(pos.astype(np.uint32).view(np.int32)).cuda(), d, theta, accurate)
    jl.device_status()
    got = got.double().cpu().numpy()
    rc, rs = _ref_cos_sin(pos, d, theta)
    err = max(np.abs(got[..., 0] - rc).max(), np.abs(got[..., 1] - rs).max())
    assert err <= bound, f"phase error {err:.3e} > {bound}"
    # the large positions are where a plain fp32 product p * theta_m would fail
    big = pos >= 2 ** 30
    assert np.abs(got[big, :, 0] - rc[big]).max() <= bound


def _brute_classes(P, C, w0):
    L = P + C
    nqb = (C + 127) // 128
    out = []
    for qb in range(nqb):
        i = np.arange(P + qb * 128, min(P + qb * 128 + 128, L))[:, None]
        row = {}
        for kb in range((i.max() // 128) + 1):
            j = np.arange(kb * 128, min(kb * 128 + 128, L))[None, :]
            causal = j <= i
            dist = (i - j)[causal]
            loc, rem = bool(np.any(dist < w0)), bool(np.any(dist >= w0))
            row[kb] = 2 if (loc and rem) else (1 if loc else 0)
        out.append(row)
    return out


@pytest.mark.parametrize("P,C,w0", [(0, 5000, 0), (0, 5000, 1), (0, 5000, 127), (0, 5000, 128), (0, 5000, 129),
                                    (0, 5000, 300), (0, 5000, 4096), (0, 5000, 4999), (0, 5000, 6000),
                                    (1000, 700, 64), (37, 129, 5), (0, 1, 0), (0, 1, 1), (4095, 2, 4096)])
def test_tile_plan_against_brute_force(P, C, w0):
    L = P + C
    max_kb = (L + 127) // 128
    plan, cls = jl.debug_tile_plan(P, C, w0, max_kb)
    jl.device_status()
    plan, cls = plan.cpu().numpy(), cls.cpu().numpy()
    ref = _brute_classes(P, C, min(w0, L))
    for qb, row in enumerate(ref):
        nR, kE0, nkb = (int(x) for x in plan[qb])
        assert nkb == len(row), (qb, nkb, len(row))
        for kb, c in row.items():
            assert cls[qb, kb] == c, (qb, kb, int(cls[qb, kb]), c)
        remote = {kb for kb, c in row.items() if c in (0, 2)}
        local = {kb for kb, c in row.items() if c in (1, 2)}
        assert remote == set(range(nR)), (qb, nR, sorted(remote))
        assert local == set(range(kE0, nkb)), (qb, kE0, nkb, sorted(local))


def test_softmax_exp2_on_fma_pipe():
    import torch
    rng = np.random.default_rng(91)
    y = np.concatenate([np.linspace(-125.5, 8.0, 400001), rng.uniform(-30.0, 0.0, 100000),
                        np.arange(-125, 9, dtype=np.float64), np.arange(-125, 8) + 0.5,
                        np.array([0.0, -0.0, -1e-7, -0.5, 0.5, 7.999])]).astype(np.float32)
    if y.size % 2:
        y = np.append(y, np.float32(-1.0))
    got = jl.debug_ex2(torch.from_numpy(y).cuda())
    jl.device_status()
    got = got.double().cpu().numpy()
    ref = np.exp2(y.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= 1e-4, f"relative error {rel.max():.3e} at y = {y[rel.argmax()]}"
    # below the normal range of the result: tiny, and exactly 0 from -127 down
    low = np.array([-126.0, -126.4, -126.6, -127.0, -128.0, -1000.0, -np.inf, np.nan], dtype=np.float32)
    gl = jl.debug_ex2(torch.from_numpy(low).cuda()).double().cpu().numpy()
    jl.device_status()
    assert np.all(np.abs(gl[:3]) <= 2.0 ** -125)
    assert np.all(gl[3:7] == 0.0), gl
    assert np.isnan(gl[7])


@pytest.mark.parametrize("planes,L,d,G,theta", [(2, 3000, 128, 4, 1e6), (3, 1500, 64, 3, 1e4), (1, 700, 128, 1, 1e6),
                                               (1, 20000, 128, 5, 1e6)])
def test_key_rotation_pass_against_oracle(planes, L, d, G, theta):
    import torch
    from oracle import rotate, rotate_rows
    rng = np.random.default_rng(92 + G)
    k = (rng.standard_normal((planes, L, d)) * 3.0).astype(np.float32)
    kd = torch.from_numpy(k).to(torch.bfloat16).cuda()
    kl, kr, e = jl.debug_rope_keys(kd, G, theta, remote=G > 1)
    jl.device_status()
    kb = kd.float().cpu().numpy().astype(np.float64)  # the bf16 values the pass reads
    mx = np.abs(kb).max()
    assert e == 13 - int(np.floor(np.log2(mx)))
    scale = 2.0 ** e
    ref_l = rotate_rows(kb.astype(np.float32), theta) * scale  # bf16 values are exact in fp32
    checks = [(kl, ref_l, "exact positions")]
    if G > 1:
        ref_r = np.stack([np.stack([rotate(kb[z, j], j // G, theta) for j in range(L)]) for z in range(planes)]) * scale
        checks.append((kr, ref_r, "aliased positions"))
    # fp16 rounding (half an ulp, 2^-11 relative) plus the fast sine's ~5e-7
    # absolute error on each factor of a pair (|x| + |y| <= 2 max|k|)
    for got, ref, what in checks:
        g = got.double().cpu().numpy()
        bound = 2.0 ** -11 * np.abs(ref) + 2e-6 * 2 * mx * scale + 1e-7
        err = np.abs(g - ref) - bound
        assert err.max() <= 0, f"{what}: worst excess {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}"
