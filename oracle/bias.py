"""Additive ALiBi bias on top of a compact mask, float64 (oracle; test infrastructure).

Written from the Ascend CANN "Mask Compression" page (the ALiBi paragraphs):
the ALiBi mask is a per-head coefficient (slope) times a bias matrix, plus
the triangular mask; the slopes are passed in. The page's figures of the
bias matrices are lost, so the bias of visible pair (i, j) is read as:

* LINEAR (right-aligned, MASK_TYPE_ALIBI_COMPRESS): slope_h * (j - i), zero on
  the diagonal and decreasing to the left (standard ALiBi);
* SQRT (MASK_TYPE_ALIBI_COMPRESS_SQRT, "the bias changed to its square root"):
  -slope_h * sqrt(|i - j|);
* LEFT (left-aligned, MASK_TYPE_ALIBI_COMPRESS_LEFT_ALIGN): slope_h * j.

LEFT and LINEAR differ by slope_h * i in every row, which the softmax
removes: same output, lse larger by slope_h * i. The boolean visibility still
comes from the mask description (the triangular part of the page's mask is
one such description). Masked pairs take no bias.
"""
from __future__ import annotations

import numpy as np

from . import masks
from .attention import _f64, attention_rows

LINEAR, SQRT, LEFT = 1, 2, 3


def bias_rows(kind: int, slope: float, rows, Nk: int) -> np.ndarray:
    """[len(rows), Nk] bias of one head."""
    i = np.asarray(rows, dtype=np.float64)[:, None]
    j = np.arange(Nk, dtype=np.float64)[None, :]
    if kind == LINEAR:
        return slope * (j - i)
    if kind == SQRT:
        return -slope * np.sqrt(np.abs(i - j))
    if kind == LEFT:
        return slope * np.broadcast_to(j, (i.shape[0], Nk)).copy()
    raise ValueError(f"unknown bias kind {kind}")


def attention_bias(q, k, v, mask, kind: int, slopes, rows=None, heads=None):
    """Masked attention with the additive bias; shapes as attention.attention."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    slopes = np.asarray(slopes, dtype=np.float64)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    rows = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(Hq)) if heads is None else list(heads)
    out = np.zeros((B, len(heads), len(rows), v.shape[-1]))
    lse = np.zeros((B, len(heads), len(rows)))
    for b in range(B):
        for hi, h in enumerate(heads):
            hm = 0 if mask.Hm == 1 else h
            vis = mask.visible_rows(b, hm, rows) if hasattr(mask, "visible_rows") else \
                masks.visible_rows(mask, b, hm, rows)
            o, s = attention_rows(q[b, h, rows], k[b, h // G], v[b, h // G], vis,
                                  bias_rows(kind, float(slopes[h]), rows, Nk))
            out[b, hi], lse[b, hi] = o, s
    return out, lse


def alibi_slopes(H: int) -> np.ndarray:
    """The usual geometric ALiBi slopes 2^(-8 h / H), h = 1..H (a workload
    choice: the page passes slopes in and does not fix them)."""
    return np.array([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)])
