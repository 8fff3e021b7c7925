"""Pins of the oracle tile map against the dense expansion and closed forms.

Binary Block Masking's contract (abstract of "Efficiently Dispatching Flash
Attention For Partially Filled Attention Masks"): a skipped tile holds no
visible pair, a tile processed without the element mask holds only visible
pairs. Both are checked by brute force over the dense mask; the lists must
cover every visible pair exactly once.
"""
import numpy as np
import pytest

from mask_aware_block_mfa_b200 import workloads as W
from oracle import masks as OM
from oracle import tilemap as OT


def _cases():
    rng = np.random.default_rng(11)
    return [
        ("doc", W.make_mask("doc8k", N=1024)),
        ("doc_ragged", W.make_mask("tiny_doc_fp32", N=500)),
        ("shared", W.make_mask("shared_question8k", N=2048)),
        ("band", W.band(1, 1000, 200, 0)),
        ("band_neg", W.band(2, 777, 300, -64)),
        ("band_negpre", W.band(1, 600, -40, 170)),
        ("random", W.random_colwise(rng, 2, 1, 300, 260)),
        ("random_hm", W.random_colwise(rng, 1, 3, 200, 333)),
        ("blocksel", W.blocksel_topk(rng, 1, 1024, 4)),
        ("blocksel_rand", W.random_blocksel(rng, 2, 700, 650, 5)),
    ]


CASES = _cases()


@pytest.mark.parametrize("name,m", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("BQ,BK", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_tile_classes_are_sound(name, m, BQ, BK):
    tm = OT.tile_map(m, BQ, BK)
    cls, lst, cnt = tm["tile_class"], tm["tile_list"], tm["tile_count"]
    nqt, nkt = OT.cdiv(m.Nq, BQ), OT.cdiv(m.Nk, BK)
    assert cls.shape == (m.B, m.Hm, nqt, nkt)
    for b in range(m.B):
        for hm in range(m.Hm):
            vis = OM.visible_dense(m, b, hm)
            covered = 0
            for qt in range(nqt):
                listed = [int(x) for x in lst[b, hm, qt] if x >= 0]
                assert listed == sorted(set(listed))                # strictly ascending
                assert len(listed) == cnt[b, hm, qt]
                assert (lst[b, hm, qt, cnt[b, hm, qt]:] == -1).all()
                for kt in range(nkt):
                    blk = vis[qt * BQ:(qt + 1) * BQ, kt * BK:(kt + 1) * BK]
                    c = cls[b, hm, qt, kt] & 3
                    if c == OT.SKIP:
                        assert not blk.any(), (qt, kt)
                        assert kt not in listed
                    else:
                        assert kt in listed
                        covered += int(blk.sum())
                    if c == OT.FULL:
                        assert blk.all(), (qt, kt)
                    if m.kind == OM.BLOCKSEL:
                        for qsl in range(BQ // 64):
                            for ksl in range(BK // 64):
                                sub = blk[qsl * 64:(qsl + 1) * 64, ksl * 64:(ksl + 1) * 64]
                                bit = (cls[b, hm, qt, kt] >> (4 + 2 * qsl + ksl)) & 1
                                assert bit == int(sub.any())
                    else:
                        assert cls[b, hm, qt, kt] >> 2 == 0
            assert covered == int(vis.sum())


@pytest.mark.parametrize("name", ["doc8k", "doc32k", "shared_question8k"])
def test_rule_is_exact_on_block_aligned_masks(name):
    """Block-aligned causal documents at 64x64: PARTIAL exactly when the tile is mixed."""
    m = W.make_mask(name, N=4096)
    cls = OT.tile_map(m, 64, 64)["tile_class"][0, 0]
    vis = OM.visible_dense(m)
    for qt in range(64):
        for kt in range(64):
            blk = vis[qt * 64:(qt + 1) * 64, kt * 64:(kt + 1) * 64]
            mixed = blk.any() and not blk.all()
            assert (cls[qt, kt] == OT.PARTIAL) == mixed


def test_kminmax_closed_forms():
    """Causal documents: UTE over k-tile kt spans [c0, c1 - 1]; LTS is the document end."""
    m = W.make_mask("doc8k", N=2048)
    mm = OT.kminmax(m, 128)[0, 0]
    ends = np.zeros(2048, np.int64)
    for (s, e) in m.docs[0]:
        ends[s:e] = e
    for kt in range(16):
        c0, c1 = kt * 128, kt * 128 + 128
        # column 0's UT [0, 0) is empty and is written as start = Nq, end = 0
        assert mm[kt, 4] == 0 and mm[kt, 5] == (2048 if kt == 0 else 0)
        assert mm[kt, 6] == c0 and mm[kt, 7] == c1 - 1
        last = ends[c0:c1] == 2048                      # the last document's LT is empty
        lts = np.where(last, 2048, ends[c0:c1])
        lte = np.where(last, 0, 2048)
        assert mm[kt, 0] == lts.min() and mm[kt, 1] == lts.max()
        assert mm[kt, 2] == lte.min() and mm[kt, 3] == lte.max()
    # band (pre, next): UTE = clamp(j - next), LTS = clamp(j + pre + 1)
    b = W.band(1, 1000, 300, -64)
    mm = OT.kminmax(b, 64)[0, 0]
    for kt in range(16):
        c0, c1 = kt * 64, min(kt * 64 + 64, 1000)
        assert mm[kt, 6] == min(c0 + 64, 1000) and mm[kt, 7] == min(c1 - 1 + 64, 1000)
        lo, hi = min(c0 + 301, 1000), min(c1 - 1 + 301, 1000)
        assert mm[kt, 0] == lo and mm[kt, 1] == hi


def test_lpt_order_properties():
    m = W.make_mask("doc32k", N=4096)
    tm = OT.tile_map(m, 64, 128)
    order, cnt = tm["order"], tm["tile_count"].reshape(-1)
    assert sorted(order.tolist()) == list(range(cnt.size))
    c = cnt[order]
    assert (np.diff(c) <= 0).all()
    for a in range(len(order) - 1):
        if c[a] == c[a + 1]:
            assert order[a] < order[a + 1]


def test_band_skip_fraction_matches_geometry():
    """pre = 2048, next = 0 at 128x128: a q-tile lists its 17 (or fewer at the start) k-tiles."""
    m = W.band(1, 16384, 2048, 0)
    tm = OT.tile_map(m, 128, 128)
    cnt = tm["tile_count"][0, 0]
    assert cnt.max() == 17 and cnt[0] == 1 and cnt[20] == 17
