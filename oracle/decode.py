"""Selected-key attention for a few query rows (decode), float64 (oracle; test infrastructure).

Written from "vulkan : selected-key flash attention for QSA block selection"
(the pull request's overview and kernel description) and the workload list's
block-selection rule:

* each (batch b, key/value head g, query row i) has a list of key-block
  indices (blocks of 64 keys); entries of -1 are empty and a block listed
  twice counts once (the kernel skips invalid and duplicate entries, as the
  CPU path does);
* the list is shared by the query heads of that key/value head (one subgroup
  per query head of the K/V head);
* the queries are the last Nq positions of the sequence, so query row i
  sits at absolute position i + Nk - Nq and sees key j only when
  j <= i + Nk - Nq. With Nq == Nk this is the forward pass's rule for block
  selection (element-wise causal inside the diagonal block);
* key j is visible to row i exactly when its block is listed and the causal
  rule holds; a row with no visible key outputs 0 and lse = -inf.

Attention itself is attention.attention_rows (the forward oracle).
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from .attention import _f64, attention_rows

BLOCK = 64


def visible_row(sel_row, i: int, Nq: int, Nk: int) -> np.ndarray:
    """Boolean [Nk] visibility of query row i under one selection list."""
    vis = np.zeros(Nk, dtype=bool)
    for entry in sel_row:
        e = int(entry)
        if e < 0:
            continue
        vis[e * BLOCK:min((e + 1) * BLOCK, Nk)] = True
    last = i + Nk - Nq  # the row's absolute position: keys after it are hidden
    if last < 0:
        vis[:] = False
    else:
        vis[last + 1:] = False
    return vis


def decode_attention(q, k, v, sel, rows: Optional[Sequence[int]] = None):
    """q [B, Hq, Nq, d], k/v [B, Hkv, Nk, d], sel int [B, Hkv, Nq, sel_k].

    Returns (out [B, Hq, len(rows), d], lse [B, Hq, len(rows)]) in float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    sel = np.asarray(sel)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    if G * Hkv != Hq:
        raise ValueError("Hq must be a multiple of Hkv")
    if np.any(sel >= (Nk + BLOCK - 1) // BLOCK) or np.any(sel < -1):
        raise ValueError("selection entries must be -1 or a block index below ceil(Nk / 64)")
    rows = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((B, Hq, len(rows), v.shape[-1]))
    lse = np.zeros((B, Hq, len(rows)))
    for b in range(B):
        for g in range(Hkv):
            vis = np.stack([visible_row(sel[b, g, i], int(i), Nq, Nk) for i in rows]) if len(rows) else \
                np.zeros((0, Nk), dtype=bool)
            for h in range(g * G, (g + 1) * G):
                o, s = attention_rows(q[b, h, rows], k[b, g], v[b, g], vis)
                out[b, h], lse[b, h] = o, s
    return out, lse


def visible_dense(sel, b: int, g: int, Nq: int, Nk: int) -> np.ndarray:
    """Boolean [Nq, Nk] visibility of one (batch, key/value head)."""
    sel = np.asarray(sel)
    return np.stack([visible_row(sel[b, g, i], i, Nq, Nk) for i in range(Nq)]) if Nq else \
        np.zeros((0, Nk), dtype=bool)
