"""Gradients of exact masked attention in float64 (oracle; test infrastructure).

The FlashMask author response puts training first among the mask's uses; the
pages give no backward formulas, so this is the derivative of the forward
definition in ``attention.py`` by the chain rule, for a loss whose gradient
with respect to ``out`` is ``dout`` (the loss does not use lse):

    P_ij    = exp(s_ij - lse_i) on visible pairs, 0 elsewhere
    dV_j    = sum_i P_ij dout_i
    dP_ij   = dout_i . v_j
    Delta_i = sum_j P_ij dP_ij
    dS_ij   = P_ij (dP_ij - Delta_i)
    dQ_i    = sum_j dS_ij k_j / sqrt(d)
    dK_j    = sum_i dS_ij q_i / sqrt(d)

Key/value head g receives the sums over its query heads g*G .. g*G+G-1
(G = Hq / Hkv, contiguous groups as in the forward). A row with no visible key
has P = 0 and contributes nothing. Every sum over i splits over disjoint sets
of rows, so the contributions of a subset of rows are exact partial sums.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

from . import masks
from .attention import _f64, attention_rows


def head_backward(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, vis: np.ndarray, dout_rows: np.ndarray):
    """Gradient contributions of some query rows of one head.

    q_rows, dout_rows [R, d]; k, v [Nk, d]; vis [R, Nk] bool (each row's full
    key range). Returns dq_rows [R, d] (exact for these rows) and the rows'
    contributions dk, dv [Nk, d].
    """
    d = q_rows.shape[1]
    _, lse = attention_rows(q_rows, k, v, vis)
    s = (q_rows @ k.T) / math.sqrt(d)
    live = vis & np.isfinite(lse)[:, None]
    p = np.where(live, np.exp(s - np.where(np.isfinite(lse), lse, 0.0)[:, None]), 0.0)
    dp = dout_rows @ v.T
    delta = (p * dp).sum(axis=1)
    ds = p * (dp - delta[:, None])
    dq = (ds @ k) / math.sqrt(d)
    dk = (ds.T @ q_rows) / math.sqrt(d)
    dv = p.T @ dout_rows
    return dq, dk, dv


def _visible(mask, b, hm, rows):
    if hasattr(mask, "visible_rows"):  # e.g. sparse_modes.SparseMode
        return mask.visible_rows(b, hm, rows)
    return masks.visible_rows(mask, b, hm, rows)


def attention_backward(q, k, v, mask, dout, rows: Optional[Sequence[int]] = None,
                       heads: Optional[Sequence[int]] = None, batches: Optional[Sequence[int]] = None):
    """Gradients for q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d], dout [B,Hq,Nq,d].

    Returns (dq [len(batches), len(heads), len(rows), d], dk, dv
    [len(batches), Hkv, Nk, d]). ``rows`` and ``heads`` restrict the sums to a
    sample: dq is exact for the listed rows, and dk/dv hold the contributions
    of the listed (row, head) pairs only, which is the exact gradient of every
    key column that no other row of those heads sees.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    rows = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(Hq)) if heads is None else list(heads)
    batches = list(range(B)) if batches is None else list(batches)
    dq = np.zeros((len(batches), len(heads), len(rows), d))
    dk = np.zeros((len(batches), Hkv, Nk, d))
    dv = np.zeros((len(batches), Hkv, Nk, v.shape[-1]))
    for bi, b in enumerate(batches):
        vis_cache = {}
        for hi, h in enumerate(heads):
            hm = 0 if mask.Hm == 1 else h
            if hm not in vis_cache:
                vis_cache[hm] = _visible(mask, b, hm, rows)
            g = h // G
            dq_h, dk_h, dv_h = head_backward(q[b, h, rows], k[b, g], v[b, g], vis_cache[hm], dout[b, h, rows])
            dq[bi, hi] = dq_h
            dk[bi, g] += dk_h
            dv[bi, g] += dv_h
    return dq, dk, dv
