"""Dense visibility of a compact mask description (oracle; test infrastructure).

Conventions (readings of the pages, stated once here):

* Column-wise row intervals (FlashMask's compact representation, named in the
  FlashMask author response, "Response to Weaknesses and Questions"): for key
  column j, query rows i with LTS[j] <= i < LTE[j] or UTS[j] <= i < UTE[j] are
  masked. Half-open; an interval whose start >= end is empty. Bounds must lie in
  [0, Nq].
* Band (Ascend sparseMode page, "sparseMode 0: defaultMask" and "sparseMode 4"):
  the pair (i, j) is computed iff -preTokens <= j - i <= nextTokens, both ends
  inclusive, origin at the upper left. With Nq == Nk this equals sparseMode 4.
* Block selection (selected-key flash attention pull request, kernel
  description): for query block i // 64 a list of key blocks; entries equal to
  -1 are ignored, duplicates count once. Inside a selected block the usual
  causal rule j <= i applies.

Masked means "not attended": attenMask True = masked (Ascend sparseMode page,
attenMask paragraph).
"""
from __future__ import annotations

import numpy as np

COLWISE, BAND, BLOCKSEL = 0, 1, 2
SEL_BLOCK = 64


def check(mask) -> None:
    """Reject descriptions outside the documented ranges (raises ValueError)."""
    if mask.kind == COLWISE:
        for name in ("lts", "lte", "uts", "ute"):
            a = getattr(mask, name)
            if a is None:
                continue
            a = np.asarray(a)
            if a.shape != (mask.B, mask.Hm, mask.Nk):
                raise ValueError(f"{name} has shape {a.shape}")
            if a.size and (a.min() < 0 or a.max() > mask.Nq):
                raise ValueError(f"{name} outside [0, Nq]")
    elif mask.kind == BLOCKSEL:
        nkb = -(-mask.Nk // SEL_BLOCK)
        sel = np.asarray(mask.sel)
        if sel.size and (sel.min() < -1 or sel.max() >= nkb):
            raise ValueError("selection entry outside [-1, ceil(Nk/64))")
    elif mask.kind != BAND:
        raise ValueError(f"unknown mask kind {mask.kind}")


def _interval(mask, name_s, name_e, b, hm):
    s, e = getattr(mask, name_s), getattr(mask, name_e)
    if s is None or e is None:  # a missing pair is the empty interval
        z = np.zeros(mask.Nk, np.int64)
        return z, z
    return np.asarray(s)[b, hm].astype(np.int64), np.asarray(e)[b, hm].astype(np.int64)


def visible_rows(mask, b: int, hm: int, rows) -> np.ndarray:
    """Boolean [len(rows), Nk]: True where query row i may attend to key j."""
    check(mask)
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(mask.Nk, dtype=np.int64)[None, :]
    if mask.kind == COLWISE:
        lts, lte = _interval(mask, "lts", "lte", b, hm)
        uts, ute = _interval(mask, "uts", "ute", b, hm)
        in_lt = (lts[None, :] <= i) & (i < lte[None, :])
        in_ut = (uts[None, :] <= i) & (i < ute[None, :])
        return ~(in_lt | in_ut)
    if mask.kind == BAND:
        diff = j - i
        return (diff >= -int(mask.pre_tokens)) & (diff <= int(mask.next_tokens))
    # BLOCKSEL
    sel = np.asarray(mask.sel)[b, hm]
    out = np.zeros((i.shape[0], mask.Nk), dtype=bool)
    for r, row in enumerate(i[:, 0]):
        chosen = {int(x) for x in sel[row // SEL_BLOCK] if x >= 0}
        kb = j[0] // SEL_BLOCK
        out[r] = np.isin(kb, list(chosen)) & (j[0] <= row)
    return out


def visible_dense(mask, b: int = 0, hm: int = 0) -> np.ndarray:
    """Boolean [Nq, Nk] visibility of one (batch, mask head)."""
    return visible_rows(mask, b, hm, np.arange(mask.Nq))


def visible_pairs(mask, b: int = 0, hm: int = 0, row_chunk: int = 2048) -> int:
    """Number of visible (i, j) pairs of one (batch, mask head), by expansion."""
    total = 0
    for r0 in range(0, mask.Nq, row_chunk):
        rows = np.arange(r0, min(r0 + row_chunk, mask.Nq))
        total += int(visible_rows(mask, b, hm, rows).sum())
    return total
