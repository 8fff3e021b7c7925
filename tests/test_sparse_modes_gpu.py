"""Ascend sparse modes on the GPU against the oracle's reading of each mode.

The column-wise bounds that mfa_mask_from_sparse_mode's kernel writes for the
prefix and varlen modes are expanded with the oracle's column-wise rule and
compared bit-exactly with the oracle's own visibility of the mode; the
attention computed through the tile map and the forward pass is compared
element by element with the oracle (tolerances as in test_fwd_gpu).
Shapes are rectangular (Sq != Skv), not multiples of the tiles, and the
packed sequences include an empty one and the band sequence.
"""
import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W
from oracle import masks as OM
from oracle import sparse_modes as SM

from .gpu_util import compare_attention, compare_map, oracle_rows

pytestmark = pytest.mark.gpu

CASES = [
    # name, mode, B, Nq, Nk, pre, next, prefix, seq_q, seq_kv
    ("prefix_wide", 5, 2, 300, 500, 0, 0, [37, 0], None, None),
    ("prefix_tall", 6, 2, 500, 300, 0, 0, [400, 123], None, None),
    ("varlen7", 7, 1, 310, 510, 500, -30, None, np.cumsum([100, 0, 150, 60]), np.cumsum([120, 40, 150, 200])),
    ("varlen8", 8, 1, 201, 187, 20, 5, None, np.cumsum([70, 130, 1]), np.cumsum([90, 64, 33])),
    ("page_mode7_card1", 7, 1, 5, 9, 6, -2, None, [3, 5], [3, 9]),
    ("right_down", 3, 1, 200, 700, 0, 0, None, None, None),
    ("band_lower_right", 4, 1, 700, 200, 100, -5, None, None, None),
    ("left_up", 2, 1, 333, 129, 0, 0, None, None, None),
]


def make(case):
    _, mode, Bn, nq, nk, pre, nxt, prefix, sq, skv = case
    dev = B.SparseModeMask(mode, Bn, nq, nk, pre, nxt, prefix=prefix, seq_q=sq, seq_kv=skv)
    ref = SM.SparseMode(mode, Bn, nq, nk, pre, nxt, prefix=prefix, seq_q=sq, seq_kv=skv)
    return dev, ref


@pytest.mark.parametrize("case", [c for c in CASES if c[1] >= 5], ids=lambda c: c[0])
def test_colwise_bounds_reproduce_the_mode(case):
    dev, ref = make(case)
    torch.cuda.synchronize()
    assert dev.kind == W.MASK_COLWISE
    lts, lte, uts, ute = (dev.bounds[i, :dev.B].cpu().numpy() for i in range(4))
    desc = W.MaskDesc(W.MASK_COLWISE, dev.B, 1, dev.Nq, dev.Nk, lts, lte, uts, ute)
    for b in range(dev.B):
        assert np.array_equal(OM.visible_dense(desc, b), SM.visible_dense(ref, b)), f"batch {b}"


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_attention_matches_the_oracle(case):
    dev, ref = make(case)
    _, mode, Bn, nq, nk = case[:5]
    g = torch.Generator().manual_seed(40 + mode)
    q = torch.randn(Bn, 4, nq, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(Bn, 2, nk, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(Bn, 2, nk, 128, generator=g).to(torch.bfloat16)
    prob = W.Problem(case[0], q, k, v, ref, 0)
    for bq, bk in ((64, 128), (128, 64)):
        att = B.Attention(dev, bq, bk)
        att.build()
        out, lse = att(q.cuda(), k.cuda(), v.cuda())
        assert B.device_status(att.tmap) == 0
        if dev.kind == W.MASK_COLWISE:
            lts, lte, uts, ute = (dev.bounds[i, :dev.B].cpu().numpy() for i in range(4))
            as_desc = W.MaskDesc(W.MASK_COLWISE, dev.B, 1, nq, nk, lts, lte, uts, ute)
        else:
            as_desc = W.MaskDesc(W.MASK_BAND, Bn, 1, nq, nk, pre_tokens=dev.desc.pre_tokens,
                                 next_tokens=dev.desc.next_tokens)
        compare_map({key: val.cpu().numpy() for key, val in att.tmap.arrays().items()}, as_desc, bq, bk)
        ref_out, ref_lse = oracle_rows(prob, None)
        compare_attention(out.float().cpu(), lse.cpu(), ref_out, ref_lse)


def test_varlen_prefill_full_size_sampled():
    """The bench's varlen_prefill16k workload (sparseMode 7, Nq 8000 x Nk 16384,
    32 query heads over 8 key/value heads) at the bench's 64 x 128 tiles:
    sampled rows of a few heads against the oracle's mode expansion."""
    import bench
    prob = W.make_problem("varlen_prefill16k")
    m = prob.mask
    bq, bk = bench.BLOCKS["varlen_prefill16k"]
    dev = B.SparseModeMask(**m.fields())
    att = B.Attention(dev, bq, bk)
    att.build()
    out, lse = att(prob.q.cuda(), prob.k.cuda(), prob.v.cuda())
    assert B.device_status(att.tmap) == 0
    rng = np.random.default_rng(23)
    rows = np.unique(np.concatenate([[0, 63, 64, m.Nq - 1], rng.choice(m.Nq, 60, replace=False)]))
    heads = [0, 13, 31]
    ref = SM.SparseMode(**m.fields())
    prob_o = W.Problem("varlen_prefill16k", prob.q, prob.k, prob.v, ref, prob.seed)
    ref_out, ref_lse = oracle_rows(prob_o, rows, heads)
    compare_attention(out.float().cpu()[:, heads][:, :, rows], lse.cpu()[:, heads][:, :, rows], ref_out, ref_lse)
