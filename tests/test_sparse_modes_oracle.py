"""The oracle's Ascend sparse modes against closed forms and the page's examples.

Pins (Ascend CANN "sparseMode introduction" page):
* square shapes: modes 2 and 3 are the plain causal triangle and mode 4 is
  mode 0 (the page: the lower-right and upper-left origins coincide);
* per-row visible counts in closed form for modes 0, 2, 3, 4 and 5 on
  rectangular shapes;
* the varlen examples of modes 7 and 8: a long sequence split across two
  devices, whose two pieces must recombine into the unsplit mask;
* pairs from different packed sequences are never visible (brute force).
"""
import numpy as np
import pytest

from oracle import sparse_modes as SM


def counts(m, b=0):
    return SM.visible_dense(m, b).sum(axis=1)


@pytest.mark.parametrize("n", [1, 7, 64, 100])
def test_square_modes_reduce_to_causal_and_band(n):
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    causal = j <= i
    assert np.array_equal(SM.visible_dense(SM.SparseMode(2, 1, n, n)), causal)
    assert np.array_equal(SM.visible_dense(SM.SparseMode(3, 1, n, n)), causal)
    for pre, nxt in ((5, 0), (0, 3), (40, -2), (3, 3)):
        assert np.array_equal(SM.visible_dense(SM.SparseMode(4, 1, n, n, pre, nxt)),
                              SM.visible_dense(SM.SparseMode(0, 1, n, n, pre, nxt)))


@pytest.mark.parametrize("nq,nk", [(5, 9), (9, 5), (64, 200), (200, 64), (17, 17)])
def test_rectangular_row_counts_in_closed_form(nq, nk):
    d = nk - nq
    rows = np.arange(nq)
    # mode 2: keys 0..i; mode 3: keys 0..i+d
    assert np.array_equal(counts(SM.SparseMode(2, 1, nq, nk)), np.clip(rows + 1, 0, nk))
    assert np.array_equal(counts(SM.SparseMode(3, 1, nq, nk)), np.clip(rows + d + 1, 0, nk))
    for pre, nxt in ((4, 1), (0, 0), (50, -3), (2, 7)):
        # mode 0: j in [i - pre, i + nxt]; mode 4: the same shifted by d
        for mode, shift in ((0, 0), (4, d)):
            lo = np.clip(rows + shift - pre, 0, nk)
            hi = np.clip(rows + shift + nxt + 1, 0, nk)
            assert np.array_equal(counts(SM.SparseMode(mode, 1, nq, nk, pre, nxt)), np.maximum(hi - lo, 0))
    for n in (0, 3, nk // 2, nk):
        m = SM.SparseMode(5, 2, nq, nk, prefix=[n, 0])
        assert np.array_equal(counts(m, 0), np.maximum(np.clip(rows + d + 1, 0, nk), n))
        assert np.array_equal(counts(m, 1), np.clip(rows + d + 1, 0, nk))
        assert np.array_equal(SM.visible_dense(SM.SparseMode(6, 2, nq, nk, prefix=[n, 0]), 0),
                              SM.visible_dense(m, 0))


def test_mode7_split_example_recombines():
    """The page's mode-7 example: a batch whose second sequence (4 queries x 6
    keys, rightDownCausal) is split by query rows over two devices. Card 1
    holds sequence lengths q (3, 2), kv (3, 6) with the last sequence as the
    band preTokens 6, nextTokens -2; card 2 keeps sparseMode 3 on pieces with q
    (2, 5, 4), kv (6, 5, 4), written here as mode 7 whose last (square)
    sequence takes a band that equals its rightDownCausal triangle. The first
    card's band rows and the second card's first rows must be rows 0-1 and 2-3
    of the unsplit 4 x 6 rightDownCausal."""
    full = SM.visible_dense(SM.SparseMode(3, 1, 4, 6))
    card1 = SM.SparseMode(7, 1, 5, 9, pre_tokens=6, next_tokens=-2, seq_q=[3, 5], seq_kv=[3, 9])
    v1 = SM.visible_dense(card1)
    assert np.array_equal(v1[0:3, 0:3], SM.visible_dense(SM.SparseMode(3, 1, 3, 3)))
    assert np.array_equal(v1[3:5, 3:9], full[0:2])
    assert not v1[0:3, 3:].any() and not v1[3:5, 0:3].any()
    card2 = SM.SparseMode(7, 1, 11, 15, pre_tokens=4, next_tokens=0, seq_q=[2, 7, 11], seq_kv=[6, 11, 15])
    v2 = SM.visible_dense(card2)
    assert np.array_equal(v2[0:2, 0:6], full[2:4])


def test_mode8_split_example_recombines():
    """The page's mode-8 example: a 5 x 4 leftUpCausal sequence split by query
    rows. Card 1 keeps sparseMode 2 on pieces q (3, 2), kv (3, 4), written here
    as mode 8 whose first (square) sequence takes a band equal to its
    leftUpCausal triangle; its second sequence is rows 0-1 of the 5 x 4 block.
    Card 2 holds q (3, 5, 4), kv (4, 5, 4) with its first sequence as the band
    preTokens 4, nextTokens 1: rows 2-4."""
    full = SM.visible_dense(SM.SparseMode(2, 1, 5, 4))
    card1 = SM.SparseMode(8, 1, 5, 7, pre_tokens=3, next_tokens=0, seq_q=[3, 5], seq_kv=[3, 7])
    v1 = SM.visible_dense(card1)
    # card 1's first sequence is the band (3 x 3, pre 3, next 0): the square causal triangle
    assert np.array_equal(v1[0:3, 0:3], np.tril(np.ones((3, 3), bool)))
    assert np.array_equal(v1[3:5, 3:7], full[0:2])
    card2 = SM.SparseMode(8, 1, 12, 13, pre_tokens=4, next_tokens=1, seq_q=[3, 8, 12], seq_kv=[4, 9, 13])
    v2 = SM.visible_dense(card2)
    assert np.array_equal(v2[0:3, 0:4], full[2:5])


def test_packed_sequences_are_independent():
    rng = np.random.default_rng(3)
    for mode in (7, 8):
        lq = rng.integers(0, 9, size=5)
        lk = rng.integers(1, 9, size=5)
        sq, sk = np.cumsum(lq), np.cumsum(lk)
        m = SM.SparseMode(mode, 1, int(sq[-1]), int(sk[-1]), pre_tokens=3, next_tokens=1, seq_q=sq, seq_kv=sk)
        v = SM.visible_dense(m)
        q_of = np.repeat(np.arange(5), lq)
        k_of = np.repeat(np.arange(5), lk)
        cross = q_of[:, None] != k_of[None, :]
        assert not v[cross].any()
        # inside each non-band sequence: the mode's triangle on the block
        nonempty = [s for s in range(5) if lq[s] and lk[s]]
        band = nonempty[-1] if mode == 7 else nonempty[0]
        for s in nonempty:
            if s == band:
                continue
            q0, k0 = int(sq[s] - lq[s]), int(sk[s] - lk[s])
            block = v[q0:q0 + lq[s], k0:k0 + lk[s]]
            ref = SM.visible_dense(SM.SparseMode(3 if mode == 7 else 2, 1, int(lq[s]), int(lk[s])))
            assert np.array_equal(block, ref)
