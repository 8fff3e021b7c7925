"""Selected-key decode on the GPU (mfa_decode through the C ABI) against the oracle.

Every case compares out and lse of every row with oracle/decode.py on the same
bf16 inputs (tolerances of the forward pass). Lists carry -1 pads and
duplicates; some rows see no key (their list is empty, lists only blocks after
the row's position, or the row sits before the start of the sequence); the
split-K path runs with parts that end up empty.
"""
import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W
from oracle import decode as OD

from .gpu_util import compare_attention

pytestmark = pytest.mark.gpu


def _inputs(seed, Bsz, Hq, Hkv, Nq, Nk, d, sel_k, pads=2, dups=2):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Bsz, Hq, Nq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(Bsz, Hkv, Nk, d, generator=g).to(torch.bfloat16)
    v = torch.randn(Bsz, Hkv, Nk, d, generator=g).to(torch.bfloat16)
    sel = W.decode_selection(np.random.default_rng(seed), Bsz, Hkv, Nq, Nk, sel_k, pads=pads, dups=dups)
    return q, k, v, sel


def run(q, k, v, sel, n_split=0):
    dec = B.Decode(n_split)
    out, lse = dec(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(sel).cuda())
    return out.float().cpu(), lse.cpu(), dec.status()


CASES = [
    # d, G, Nq, Nk, sel_k, n_split
    (128, 4, 1, 5000, 16, 0),
    (256, 4, 1, 9000, 32, 0),
    (256, 8, 3, 4100, 24, 1),
    (128, 16, 2, 3000, 8, 5),
    (128, 1, 4, 777, 20, 3),
    (256, 2, 16, 2000, 40, 0),
    (128, 8, 70, 64, 4, 2),     # rows 0..5 sit before the sequence start: no key
    (256, 4, 5, 3000, 40, 0),   # 20 rows of 40 slots, 6 per CTA: rows split over up to 8 CTAs
    (128, 2, 300, 2500, 8, 0),  # 1200 rows of 8 slots: every CTA takes 9 whole rows, no partials
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "d%d_g%d_nq%d_nk%d_k%d_s%d" % c)
def test_decode_matches_oracle(case):
    d, G, Nq, Nk, sel_k, n_split = case
    Hkv = 2
    pads = dups = min(2, sel_k // 4)
    q, k, v, sel = _inputs(sum(case) % 1000, 2, Hkv * G, Hkv, Nq, Nk, d, sel_k, pads=pads, dups=dups)
    out, lse, err = run(q, k, v, sel, n_split)
    assert err == 0
    ref_out, ref_lse = OD.decode_attention(q, k, v, sel)
    compare_attention(out, lse, ref_out, ref_lse)


def test_decode_empty_lists_and_partial_block():
    """Rows sit at positions 997, 998, 999 of a 1000-key cache. Row 0 lists
    nothing; row 1 lists only the last block (keys 960-999, of which it sees
    960-998) twice; row 2 lists only pads."""
    q, k, v, sel = _inputs(5, 1, 4, 1, 3, 1000, 128, 6)
    sel[0, 0, 0] = -1
    sel[0, 0, 1] = [15, 15, -1, -1, -1, -1]
    sel[0, 0, 2] = [-1] * 6
    out, lse, err = run(q, k, v, sel, 4)
    assert err == 0
    ref_out, ref_lse = OD.decode_attention(q, k, v, sel)
    compare_attention(out, lse, ref_out, ref_lse)
    assert torch.isneginf(lse[0, :, 0]).all() and torch.isneginf(lse[0, :, 2]).all()
    assert (out[0, :, 0] == 0).all() and (out[0, :, 2] == 0).all()
    assert torch.isfinite(lse[0, :, 1]).all()


def test_decode_split_counts_agree():
    q, k, v, sel = _inputs(6, 2, 8, 2, 2, 6000, 256, 40, pads=5, dups=3)
    ref = OD.decode_attention(q, k, v, sel)
    for n_split in (1, 2, 7, 40):              # 40 parts: most of them empty (-FLT_MAX partials)
        out, lse, err = run(q, k, v, sel, n_split)
        assert err == 0
        compare_attention(out, lse, *ref)


def test_decode_out_of_range_entry_flagged_and_ignored():
    q, k, v, sel = _inputs(7, 1, 4, 1, 1, 640, 128, 5, pads=1, dups=0)   # 10 blocks
    clean = sel.copy()
    sel[0, 0, 0, np.argmax(sel[0, 0, 0] < 0)] = 10                       # one past the last block
    out, lse, err = run(q, k, v, sel, 1)
    assert err & B.DEVERR_SEL
    compare_attention(out, lse, *OD.decode_attention(q, k, v, clean))


def test_decode_full_size_workload():
    """The bench's decode workload (B=8, GQA 4, d=256, 64K cache, 32 blocks),
    every row of a sample of (batch, head) pairs."""
    q, k, v, sel = W.make_decode_problem("decode_sel64k")
    out, lse, err = run(q, k, v, sel)
    assert err == 0
    ref_out, ref_lse = OD.decode_attention(q[:2], k[:2], v[:2], sel[:2])
    compare_attention(out[:2], lse[:2], ref_out, ref_lse)


def test_decode_longest_lists():
    """Lists of the maximum length (256 entries, 16 pads and 16 duplicates) over
    a cache of 20000 keys (313 blocks, ragged last block), with the automatic
    split and with 3 parts."""
    q, k, v, sel = _inputs(9, 2, 8, 2, 2, 20000, 256, 256, pads=16, dups=16)
    ref = OD.decode_attention(q, k, v, sel)
    for n_split in (0, 3):
        out, lse, err = run(q, k, v, sel, n_split)
        assert err == 0
        compare_attention(out, lse, *ref)


def test_decode_slot_ranges_over_many_rows_and_waves():
    """2000 rows of 256 slots (at most 64 blocks in a 4096-key cache, so most
    slots are pads or duplicates): the automatic split gives every CTA 8 whole
    rows, 250 CTAs in two waves; one row in 7 is compared (the oracle is the
    given the same rows)."""
    q, k, v, sel = _inputs(11, 1, 4, 2, 1000, 4096, 128, 256, pads=100, dups=40)
    out, lse, err = run(q, k, v, sel)
    assert err == 0
    rows = list(range(0, 1000, 7))
    ref_out, ref_lse = OD.decode_attention(q, k, v, sel, rows=rows)
    compare_attention(out[:, :, rows], lse[:, :, rows], ref_out, ref_lse)


def test_decode_parts_starting_on_pads_duplicates_and_hidden_blocks():
    """Every part's first slot decides whether its first block is loaded
    before the list is deduplicated. With 4 parts of 2 slots, row 0's parts
    start on a kept block, on a duplicate of an earlier slot, on a pad and on
    a block after the row's position; row 1's on a pad, on an entry out of
    range (flagged and ignored), on a duplicate and on a pad. With 3 parts of
    3 slots, two of them start on kept blocks that follow other entries."""
    q, k, v, sel = _inputs(12, 1, 4, 1, 40, 2000, 256, 8, pads=0, dups=0)
    # 2000 keys: blocks 0-31; rows 0 and 1 sit at positions 1960 and 1961, so
    # block 31 (keys 1984-1999) is after both.
    sel[0, 0, 0] = [3, 7, 3, 9, -1, 12, 31, 30]
    sel[0, 0, 1] = [-1, 4, 32, 5, 5, 6, -1, -1]
    clean = sel.copy()
    clean[0, 0, 1, 2] = -1
    for n_split in (4, 3):
        out, lse, err = run(q, k, v, sel, n_split)
        assert err & B.DEVERR_SEL
        compare_attention(out, lse, *OD.decode_attention(q, k, v, clean))
