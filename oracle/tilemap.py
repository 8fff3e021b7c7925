"""Reference tile map: per-tile SKIP / FULL / PARTIAL and compacted k-tile lists.

Oracle, test infrastructure. It follows Binary Block Masking ("Efficiently
Dispatching Flash Attention For Partially Filled Attention Masks", abstract):
the attention matrix is cut into tiles, tiles with no visible pair are not
processed, tiles with only visible pairs need no per-element mask, and the rest
apply the element mask. The FlashMask author response (paragraph on FlashInfer's
block-sparse wrapper) gives the reason: only the necessary tiles are computed.

Map layout (all per batch b and mask head hm, BQ x BK tiles, nQT = ceil(Nq/BQ),
nKT = ceil(Nk/BK)):

* ``kminmax`` int32 [B, Hm, nKT, 8] -- over the valid columns of k-tile kt:
  LTS min, LTS max, LTE min, LTE max, UTS min, UTS max, UTE min, UTE max,
  after writing every empty interval (start >= end) as start = Nq, end = 0.
  That choice makes an empty column block "covers" (its start is the largest
  possible, its end the smallest) and leaves "clear" to the non-empty columns,
  so plain min/max give the per-column answer. The band
  kind is first written as column bounds: UT = [0, clamp(j - next, 0, Nq)),
  LT = [clamp(j + pre + 1, 0, Nq), Nq). Zero for the block-selected kind.
* ``tile_class`` uint8 [B, Hm, nQT, nKT] -- bits 0-1: 0 SKIP, 1 FULL, 2 PARTIAL.
  Block-selected kind only: bit 4 + 2*qs + ks is set when the 64x64 sub-block
  (query sub-block qs, key sub-block ks of the tile) holds a visible pair.
* ``tile_list`` int32 [B, Hm, nQT, nKT] -- the non-SKIP kt in ascending order,
  then -1.
* ``tile_count`` int32 [B, Hm, nQT].
* ``order`` int32 [B*Hm*nQT] -- flat (b, hm, qt) indices sorted by count,
  largest first, ties by index (longest-processing-time-first schedule).

Rule R for the interval kinds, with r0 = qt*BQ, r1 = min(r0 + BQ, Nq):
SKIP if (LTS max <= r0 and LTE min >= r1) or (UTS max <= r0 and UTE min >= r1);
else FULL if (LTS min >= r1 or LTE max <= r0) and (UTS min >= r1 or UTE max <= r0);
else PARTIAL. It is conservative: a tile that is uniform only through a mix of
the two intervals is PARTIAL, which is still exact because PARTIAL applies the
element mask.

Block-selected kind: a 64x64 sub-block (qs, ks) is empty when ks is not in the
list of query block qs or ks > qs, full when listed and ks < qs, diagonal when
listed and ks == qs. A tile is SKIP when all its valid sub-blocks are empty,
FULL when all are full, PARTIAL otherwise.
"""
from __future__ import annotations

import numpy as np

from . import masks

SKIP, FULL, PARTIAL = 0, 1, 2


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


def column_bounds(mask, b: int, hm: int):
    """(lts, lte, uts, ute) as int64 arrays over the key columns; empty -> (Nq, 0)."""
    Nq, Nk = mask.Nq, mask.Nk
    j = np.arange(Nk, dtype=np.int64)
    if mask.kind == masks.BAND:
        pre, nxt = int(mask.pre_tokens), int(mask.next_tokens)
        uts = np.zeros(Nk, np.int64)
        ute = np.clip(j - nxt, 0, Nq)
        lts = np.clip(j + pre + 1, 0, Nq)
        lte = np.full(Nk, Nq, np.int64)
    else:
        lts, lte = masks._interval(mask, "lts", "lte", b, hm)
        uts, ute = masks._interval(mask, "uts", "ute", b, hm)
    out = []
    for s, e in ((lts, lte), (uts, ute)):
        empty = s >= e
        out.append(np.where(empty, Nq, s))
        out.append(np.where(empty, 0, e))
    return tuple(out)


def kminmax(mask, BK: int) -> np.ndarray:
    masks.check(mask)
    nkt = cdiv(mask.Nk, BK)
    res = np.zeros((mask.B, mask.Hm, nkt, 8), np.int32)
    if mask.kind == masks.BLOCKSEL:
        return res
    for b in range(mask.B):
        for hm in range(mask.Hm):
            cols = column_bounds(mask, b, hm)
            for kt in range(nkt):
                c0, c1 = kt * BK, min(kt * BK + BK, mask.Nk)
                for a, arr in enumerate(cols):
                    res[b, hm, kt, 2 * a] = arr[c0:c1].min()
                    res[b, hm, kt, 2 * a + 1] = arr[c0:c1].max()
    return res


def _classify_intervals(mask, BQ: int, BK: int) -> np.ndarray:
    mm = kminmax(mask, BK)
    nqt, nkt = cdiv(mask.Nq, BQ), cdiv(mask.Nk, BK)
    cls = np.zeros((mask.B, mask.Hm, nqt, nkt), np.uint8)
    for b in range(mask.B):
        for hm in range(mask.Hm):
            for qt in range(nqt):
                r0, r1 = qt * BQ, min(qt * BQ + BQ, mask.Nq)
                for kt in range(nkt):
                    lts_min, lts_max, lte_min, lte_max, uts_min, uts_max, ute_min, ute_max = mm[b, hm, kt]
                    lt_covers = lts_max <= r0 and lte_min >= r1
                    ut_covers = uts_max <= r0 and ute_min >= r1
                    if lt_covers or ut_covers:
                        cls[b, hm, qt, kt] = SKIP
                        continue
                    lt_clear = lts_min >= r1 or lte_max <= r0
                    ut_clear = uts_min >= r1 or ute_max <= r0
                    cls[b, hm, qt, kt] = FULL if (lt_clear and ut_clear) else PARTIAL
    return cls


def _classify_blocksel(mask, BQ: int, BK: int) -> np.ndarray:
    sb = masks.SEL_BLOCK
    nqt, nkt = cdiv(mask.Nq, BQ), cdiv(mask.Nk, BK)
    nqs_valid, nks_valid = cdiv(mask.Nq, sb), cdiv(mask.Nk, sb)
    sel = np.asarray(mask.sel)
    cls = np.zeros((mask.B, mask.Hm, nqt, nkt), np.uint8)
    for b in range(mask.B):
        for hm in range(mask.Hm):
            for qt in range(nqt):
                for kt in range(nkt):
                    states, bits = [], 0
                    for qsl in range(BQ // sb):
                        qs = qt * BQ // sb + qsl
                        if qs >= nqs_valid:
                            continue
                        chosen = {int(x) for x in sel[b, hm, qs] if x >= 0}
                        for ksl in range(BK // sb):
                            ks = kt * BK // sb + ksl
                            if ks >= nks_valid:
                                continue
                            if ks not in chosen or ks > qs:
                                states.append("empty")
                            else:
                                states.append("full" if ks < qs else "diag")
                                bits |= 1 << (4 + 2 * qsl + ksl)
                    if all(s == "empty" for s in states):
                        c = SKIP
                    elif all(s == "full" for s in states):
                        c = FULL
                    else:
                        c = PARTIAL
                    cls[b, hm, qt, kt] = c | bits
    return cls


def classify(mask, BQ: int, BK: int) -> np.ndarray:
    masks.check(mask)
    if mask.kind == masks.BLOCKSEL:
        return _classify_blocksel(mask, BQ, BK)
    return _classify_intervals(mask, BQ, BK)


def compact(cls: np.ndarray):
    """Ascending list of the non-SKIP k-tiles of every q-tile, -1 padded, and counts."""
    B, Hm, nqt, nkt = cls.shape
    lst = np.full((B, Hm, nqt, nkt), -1, np.int32)
    cnt = np.zeros((B, Hm, nqt), np.int32)
    for b in range(B):
        for hm in range(Hm):
            for qt in range(nqt):
                kts = [kt for kt in range(nkt) if (cls[b, hm, qt, kt] & 3) != SKIP]
                lst[b, hm, qt, : len(kts)] = kts
                cnt[b, hm, qt] = len(kts)
    return lst, cnt


def lpt_order(cnt: np.ndarray) -> np.ndarray:
    flat = cnt.reshape(-1)
    idx = sorted(range(flat.size), key=lambda e: (-int(flat[e]), e))
    return np.asarray(idx, dtype=np.int32)


def tile_map(mask, BQ: int, BK: int) -> dict:
    """The full reference map (see the module docstring for the layout)."""
    cls = classify(mask, BQ, BK)
    lst, cnt = compact(cls)
    return {
        "kminmax": kminmax(mask, BK),
        "tile_class": cls,
        "tile_list": lst,
        "tile_count": cnt,
        "order": lpt_order(cnt),
    }
