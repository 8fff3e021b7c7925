"""Exact masked attention in float64 (oracle; test infrastructure).

Definition followed (the forward pass the FlashMask author response and the
Binary Block Masking abstract accelerate, written out plainly):

    s_ij = (q_i . k_j) / sqrt(d)                 for the visible j of row i
    out_i = sum_j exp(s_ij - m_i) v_j / l_i,     m_i = max_j s_ij, l_i = sum_j exp(s_ij - m_i)
    lse_i = m_i + ln(l_i)                        (natural logarithm)

A row with no visible key outputs zeros and lse = -inf (the selected-key pull
request's split-K note: an empty part must never produce exp(-inf - -inf)).
Query head h reads key/value head h // (Hq / Hkv) (contiguous GQA groups, as in
the pull request's "query heads of that K/V head"). The mask head is 0 when the
description has one head, else h.

Inputs are used exactly as given: bf16 or fp32 values are widened to float64.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

from . import masks


def _f64(t) -> np.ndarray:
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def attention_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, vis: np.ndarray, bias=None):
    """Attention of some query rows of one head.

    q_rows [R, d], k [Nk, d], v [Nk, dv] in float64, vis [R, Nk] bool;
    bias: optional [R, Nk] float64 added to the scores of visible pairs.
    Returns (out [R, dv], lse [R]).
    """
    d = q_rows.shape[1]
    s = (q_rows @ k.T) / math.sqrt(d)
    if bias is not None:
        s = s + bias
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], -np.inf)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    w = np.exp(s - m_safe[:, None])  # exp(-inf) = 0 for masked keys
    l = w.sum(axis=1)
    out = (w @ v) / np.where(empty, 1.0, l)[:, None]
    out[empty] = 0.0
    lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, l)))
    return out, lse


def attention(q, k, v, mask, rows: Optional[Sequence[int]] = None,
              heads: Optional[Sequence[int]] = None, batches: Optional[Sequence[int]] = None):
    """Masked attention for q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d].

    ``rows``, ``heads`` and ``batches`` restrict the computation to a sample;
    the result has shape [len(batches), len(heads), len(rows), d] (and lse
    without the last axis). All arithmetic is float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    rows = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(Hq)) if heads is None else list(heads)
    batches = list(range(B)) if batches is None else list(batches)
    out = np.zeros((len(batches), len(heads), len(rows), v.shape[-1]))
    lse = np.zeros((len(batches), len(heads), len(rows)))
    for bi, b in enumerate(batches):
        vis_cache = {}
        for hi, h in enumerate(heads):
            hm = 0 if mask.Hm == 1 else h
            if hm not in vis_cache:
                if hasattr(mask, "visible_rows"):  # e.g. sparse_modes.SparseMode
                    vis_cache[hm] = mask.visible_rows(b, hm, rows)
                else:
                    vis_cache[hm] = masks.visible_rows(mask, b, hm, rows)
            o, s = attention_rows(q[b, h, rows], k[b, h // G], v[b, h // G], vis_cache[hm])
            out[bi, hi], lse[bi, hi] = o, s
    return out, lse
