"""Dense visibility of the Ascend sparse modes (oracle; test infrastructure).

Written from the Ascend CANN "sparseMode introduction" page (one paragraph
per mode) and its worked examples. Rows are queries i in [0, Sq), columns keys j in
[0, Skv); True means the pair is computed (attenMask False). Each mode is
coded from its own sentence, independently of the library's conversion of
the mode into a compact mask description:

* 0 defaultMask: the band -preTokens <= j - i <= nextTokens, origin at the
  upper-left corner.
* 2 leftUpCausal: the lower triangle from the upper-left vertex, j <= i.
* 3 rightDownCausal: the lower triangle from the lower-right vertex,
  j - i <= Skv - Sq.
* 4 band, start point at the lower-right corner:
  -preTokens <= (j - i) - (Skv - Sq) <= nextTokens.
* 5 prefix (6 is the same with a compressed attenMask input): rightDownCausal
  with a full Sq x N block added on the left, N = prefix[b] per batch:
  visible iff j < N or j - i <= Skv - Sq.
* 7 / 8 varlen, long sequence split externally: B = 1 holds packed sequences;
  actual_seq_qlen / actual_seq_kvlen are cumulative ends. Pairs from different
  sequences are never computed. Inside a sequence of lengths (lq, lk):
  mode 7 is rightDownCausal, except the last non-empty sequence, which is the
  band from the lower-right vertex with (preTokens, nextTokens); mode 8 is
  leftUpCausal, except the first non-empty sequence, which is that band.

Mode 1 (a full Sq x Skv attenMask) has no compact form and is not covered.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

MODES = (0, 2, 3, 4, 5, 6, 7, 8)


@dataclasses.dataclass
class SparseMode:
    mode: int
    B: int
    Nq: int
    Nk: int
    pre_tokens: int = 0
    next_tokens: int = 0
    prefix: Optional[Sequence[int]] = None  # modes 5, 6: one length per batch
    seq_q: Optional[Sequence[int]] = None   # modes 7, 8: cumulative query ends (actual_seq_qlen)
    seq_kv: Optional[Sequence[int]] = None  # modes 7, 8: cumulative key ends (actual_seq_kvlen)
    Hm: int = 1
    name: str = "sparse_mode"

    def visible_rows(self, b: int, hm: int, rows) -> np.ndarray:
        return visible_rows(self, b, rows)


def _segments(ends: Sequence[int]):
    starts = [0] + [int(x) for x in ends[:-1]]
    return list(zip(starts, [int(x) for x in ends]))


def _band(dj, lq, lk, pre, nxt):
    """Band from the lower-right vertex of an lq x lk block, dj = j - i."""
    return (dj - (lk - lq) >= -pre) & (dj - (lk - lq) <= nxt)


def visible_rows(m: SparseMode, b: int, rows) -> np.ndarray:
    """Boolean [len(rows), Nk]: True where query row i computes key j."""
    if m.mode not in MODES:
        raise ValueError(f"sparse mode {m.mode} is not covered")
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(m.Nk, dtype=np.int64)[None, :]
    dj = j - i
    d = m.Nk - m.Nq
    pre, nxt = int(m.pre_tokens), int(m.next_tokens)
    if m.mode == 0:
        return (dj >= -pre) & (dj <= nxt)
    if m.mode == 2:
        return dj <= 0
    if m.mode == 3:
        return dj <= d
    if m.mode == 4:
        return _band(dj, m.Nq, m.Nk, pre, nxt)
    if m.mode in (5, 6):
        n = int(m.prefix[b])
        return (j < n) | (dj <= d)
    # 7 / 8: packed sequences in batch 0
    if m.B != 1:
        raise ValueError("varlen modes take B = 1")
    qs, ks = _segments(m.seq_q), _segments(m.seq_kv)
    if len(qs) != len(ks):
        raise ValueError("actual_seq_qlen and actual_seq_kvlen differ in length")
    nonempty = [s for s, ((q0, q1), (k0, k1)) in enumerate(zip(qs, ks)) if q1 > q0 and k1 > k0]
    band_seq = (nonempty[-1] if m.mode == 7 else nonempty[0]) if nonempty else -1
    out = np.zeros((i.shape[0], m.Nk), dtype=bool)
    for s, ((q0, q1), (k0, k1)) in enumerate(zip(qs, ks)):
        in_seq = (i >= q0) & (i < q1) & (j >= k0) & (j < k1)
        li, lj = i - q0, j - k0
        lq, lk = q1 - q0, k1 - k0
        if s == band_seq:
            rule = _band(lj - li, lq, lk, pre, nxt)
        elif m.mode == 7:
            rule = (lj - li) <= (lk - lq)
        else:
            rule = lj <= li
        out |= in_seq & rule
    return out


def visible_dense(m: SparseMode, b: int = 0) -> np.ndarray:
    return visible_rows(m, b, np.arange(m.Nq))
