"""Pins of the decode (selected-key, few query rows) oracle, oracle/decode.py.

* With Nq == Nk and every row of a 64-query block given that block's list,
  the visibility equals the forward oracle's block-selection mask, which is
  pinned against kron(selection, ones) & tril elsewhere;
* q = 0: out is the mean of the visible values and lse = ln(count), with the
  visible set counted by scalar loops over the definition (block listed,
  key at or before the row's absolute position);
* -1 entries, duplicates and the order of a list change nothing (bit-exact);
* a single visible key gives out = v_j; rows with no visible key give
  out = 0, lse = -inf;
* planted mistakes (top-left instead of bottom-right causal alignment, -1
  read as block 0) fail one of these.
"""
import math

import numpy as np
import pytest

from mask_aware_block_mfa_b200 import workloads as W
from oracle import decode as OD
from oracle import masks as OM


def _qkv(rng, B, Hq, Hkv, Nq, Nk, d):
    return (rng.standard_normal((B, Hq, Nq, d)), rng.standard_normal((B, Hkv, Nk, d)),
            rng.standard_normal((B, Hkv, Nk, d)))


def test_equals_forward_block_selection_when_square():
    rng = np.random.default_rng(0)
    N = 300
    m = W.blocksel_topk(rng, 1, N, 3)
    sel_rows = np.repeat(m.sel[0, 0], 64, axis=0)[:N]               # row i takes its block's list
    sel = sel_rows[None, None]                                       # [B=1, Hkv=1, Nq, sel_k]
    assert np.array_equal(OD.visible_dense(sel, 0, 0, N, N), OM.visible_dense(m, 0))


def _count_loops(sel_row, i, Nq, Nk):
    listed = set(int(e) for e in sel_row if e >= 0)
    return sum(1 for j in range(Nk) if (j // 64) in listed and j <= i + Nk - Nq)


@pytest.mark.parametrize("Nq,Nk", [(1, 1000), (5, 777), (16, 64), (3, 2)])
def test_zero_query_closed_form(Nq, Nk):
    rng = np.random.default_rng(1)
    q, k, v = _qkv(rng, 2, 4, 2, Nq, Nk, 8)
    q[:] = 0.0
    nb = (Nk + 63) // 64
    sel = rng.integers(-1, nb, size=(2, 2, Nq, 6))
    out, lse = OD.decode_attention(q, k, v, sel)
    for b in range(2):
        for h in range(4):
            g = h // 2
            for i in range(Nq):
                n = _count_loops(sel[b, g, i], i, Nq, Nk)
                if n == 0:
                    assert np.isneginf(lse[b, h, i]) and not out[b, h, i].any()
                    continue
                listed = set(int(e) for e in sel[b, g, i] if e >= 0)
                js = [j for j in range(Nk) if (j // 64) in listed and j <= i + Nk - Nq]
                np.testing.assert_allclose(out[b, h, i], v[b, g, js].mean(axis=0), atol=1e-13)
                assert math.isclose(lse[b, h, i], math.log(n), abs_tol=1e-13)


def test_pads_duplicates_and_order_change_nothing():
    rng = np.random.default_rng(2)
    q, k, v = _qkv(rng, 1, 8, 2, 4, 1500, 16)
    base = np.array([[[[3, 7, 20, 0], [1, 2, 3, 4], [23, 22, 5, 9], [0, 11, 12, 13]]] * 2])
    noisy = np.concatenate([base[..., ::-1], base[..., :2], np.full(base.shape[:-1] + (3,), -1)], axis=-1)
    a = OD.decode_attention(q, k, v, base)
    b = OD.decode_attention(q, k, v, noisy)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_single_key_and_empty_rows():
    rng = np.random.default_rng(3)
    q, k, v = _qkv(rng, 1, 2, 1, 3, 129, 4)
    # row 0 sits at position 126: block 1 is keys 64..127 -> 63 visible; block 2 (key 128) hidden
    sel = np.array([[[[2, -1], [-1, -1], [1, -1]]]])
    out, lse = OD.decode_attention(q, k, v, sel)
    assert np.isneginf(lse[0, :, 0]).all() and not out[0, :, 0].any()   # block 2 = key 128 > 126
    assert np.isneginf(lse[0, :, 1]).all()
    assert np.isfinite(lse[0, :, 2]).all()
    sel1 = np.array([[[[2, -1], [2, -1], [2, -1]]]])
    out1, lse1 = OD.decode_attention(q, k, v, sel1)
    np.testing.assert_allclose(out1[0, :, 2], np.broadcast_to(v[0, 0, 128], (2, 4)), atol=1e-15)
    s = q[0, :, 2] @ k[0, 0, 128] / 2.0
    np.testing.assert_allclose(lse1[0, :, 2], s, atol=1e-14)


def test_out_of_range_entries_are_rejected():
    rng = np.random.default_rng(4)
    q, k, v = _qkv(rng, 1, 1, 1, 1, 100, 4)
    with pytest.raises(ValueError):
        OD.decode_attention(q, k, v, np.array([[[[2]]]]))


@pytest.mark.parametrize("mutation", ["top_left", "pad_as_block0"])
def test_planted_mistakes_are_caught(monkeypatch, mutation):
    orig = OD.visible_row

    def mutant(sel_row, i, Nq, Nk):
        if mutation == "top_left":
            return orig(sel_row, i, Nk, Nk)              # causal rule without the Nk - Nq shift
        return orig([0 if e < 0 else e for e in sel_row], i, Nq, Nk)

    monkeypatch.setattr(OD, "visible_row", mutant)
    check = (lambda: test_zero_query_closed_form(5, 777)) if mutation == "top_left" else \
        test_pads_duplicates_and_order_change_nothing
    with pytest.raises(AssertionError):
        check()
