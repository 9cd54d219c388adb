"""Textbook numpy attention used to pin the oracle (tests only).

Written independently of the oracle's C code: RoPE here is multiplication of
complex numbers z_m = x_m + i x_{m+d/2} by exp(i p theta_m), and attention is
dense softmax(scale * Q K^T + mask) V with numpy matrix products.  Grouped-query
attention is expressed by explicitly repeating K/V heads.
"""
from __future__ import annotations

import numpy as np


def rope_complex(x: np.ndarray, pos: np.ndarray, rope_theta: float) -> np.ndarray:
    """x [..., L, d] -> rotated copy; pos [L] integer positions."""
    d = x.shape[-1]
    h = d // 2
    freqs = np.power(float(rope_theta), -np.arange(h, dtype=np.float64) * (2.0 / d))
    z = x[..., :h].astype(np.float64) + 1j * x[..., h:].astype(np.float64)
    zr = z * np.exp(1j * np.outer(np.asarray(pos, dtype=np.float64), freqs))
    return np.concatenate([zr.real, zr.imag], axis=-1)


def masked_attention(q, k, v, scale, allowed):
    """Dense attention for one head. q [L,d], k/v [L,d], allowed [L,L] bool.

    Returns (out [L,d], lse [L]); rows without any allowed key get out = 0 and
    lse = -inf.
    """
    s = scale * (q @ k.T)
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=-1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(s - m_safe[:, None])
    p = np.where(allowed, p, 0.0)
    l = p.sum(axis=-1)
    out = (p @ v) / np.where(empty, 1.0, l)[:, None]
    lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, l)))
    return out, lse


def causal(L):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    return j <= i


def window(L, w0):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    return (j <= i) & (i - j < w0)


def repeat_kv(x, group):
    return np.repeat(x, group, axis=1)


def rope_attention(q, k, v, pos, rope_theta, scale, allowed=None):
    """Standard RoPE causal attention for [B,H,L,d] inputs (K/V already per q head)."""
    B, H, L, d = q.shape
    allowed = causal(L) if allowed is None else allowed
    qr = rope_complex(q, pos, rope_theta)
    kr = rope_complex(k, pos, rope_theta)
    out = np.empty((B, H, L, d))
    lse = np.empty((B, H, L))
    for b in range(B):
        for h in range(H):
            out[b, h], lse[b, h] = masked_attention(qr[b, h], kr[b, h], v[b, h], scale,
                                                    allowed)
    return out, lse


def inclusion_exclusion(q, k, v, w0, G, rope_theta, scale):
    """The pages' three-pass formulation, merged with log-sum-exp weights.

    A: local window, classic positions; B: full causal, positions // G;
    C: local window, positions // G.  out = (e^lA O_A + e^lB O_B - e^lC O_C) /
    (e^lA + e^lB - e^lC), all weights taken relative to max(lA, lB).
    """
    L = q.shape[2]
    pos = np.arange(L)
    oa, la = rope_attention(q, k, v, pos, rope_theta, scale, window(L, w0))
    ob, lb = rope_attention(q, k, v, pos // G, rope_theta, scale, causal(L))
    oc, lc = rope_attention(q, k, v, pos // G, rope_theta, scale, window(L, w0))
    m = np.maximum(la, lb)
    wa = np.exp(la - m)
    wb = np.exp(lb - m)
    wc = np.exp(lc - m)
    num = wa[..., None] * oa + wb[..., None] * ob - wc[..., None] * oc
    den = wa + wb - wc
    return num / den[..., None]
