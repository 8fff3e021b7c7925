"""GPU tile map vs the oracle: bit-exact on every array, every mask kind."""
import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W

from .gpu_util import compare_map

pytestmark = pytest.mark.gpu


def _masks():
    rng = np.random.default_rng(21)
    return [
        ("doc_small", W.make_mask("doc8k", N=1024)),
        ("doc_ragged", W.make_mask("tiny_doc_fp32", N=1000)),
        ("tiny", W.make_mask("tiny_doc_fp32")),
        ("shared", W.make_mask("shared_question8k", N=2048)),
        ("band", W.band(2, 1500, 300, 0)),
        ("band_neg", W.band(1, 777, 300, -64)),
        ("band_huge", W.band(1, 600, 2 ** 40, -(2 ** 40))),
        ("random", W.random_colwise(rng, 2, 1, 300, 260)),
        ("random_hm", W.random_colwise(rng, 1, 3, 200, 333)),
        ("blocksel", W.blocksel_topk(rng, 1, 1024, 4)),
        ("blocksel_rand", W.random_blocksel(rng, 2, 700, 650, 5)),
    ]


MASKS = _masks()


@pytest.mark.parametrize("name,mask", MASKS, ids=[m[0] for m in MASKS])
@pytest.mark.parametrize("bq,bk", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_tile_map_bit_exact(name, mask, bq, bk):
    dm = B.DeviceMask(mask)
    tm = B.TileMap(mask.B, mask.Hm, mask.Nq, mask.Nk, bq, bk)
    B.build_tile_map(dm, tm)
    assert B.device_status(tm) == 0
    compare_map({k: v.cpu().numpy() for k, v in tm.arrays().items()}, mask, bq, bk)


@pytest.mark.parametrize("name,bq,bk", [("doc8k", 64, 128), ("shared_question8k", 64, 128), ("band16k", 128, 128),
                                         ("band16k_neg", 128, 128), ("doc32k", 64, 128), ("blocksel32k", 64, 64),
                                         ("tiny_doc_fp32", 128, 64)])
def test_tile_map_full_size(name, bq, bk):
    mask = W.make_mask(name)
    dm = B.DeviceMask(mask)
    tm = B.TileMap(mask.B, mask.Hm, mask.Nq, mask.Nk, bq, bk)
    B.build_tile_map(dm, tm)
    assert B.device_status(tm) == 0
    compare_map({k: v.cpu().numpy() for k, v in tm.arrays().items()}, mask, bq, bk)


def test_out_of_range_bounds_flagged():
    mask = W.make_mask("tiny_doc_fp32", N=256)
    mask.lte = mask.lte.copy()
    mask.lte[0, 0, 10] = 300
    dm = B.DeviceMask(mask)
    tm = B.TileMap(1, 1, 256, 256, 64, 64)
    B.build_tile_map(dm, tm)
    assert B.device_status(tm) & B.DEVERR_BOUNDS
    sel = W.blocksel_topk(np.random.default_rng(0), 1, 256, 2)
    sel.sel[0, 0, 2, 0] = 9
    dm = B.DeviceMask(sel)
    B.build_tile_map(dm, tm)
    assert B.device_status(tm) == B.DEVERR_SEL


def test_rebuild_clears_error_word():
    mask = W.make_mask("tiny_doc_fp32", N=256)
    tm = B.TileMap(1, 1, 256, 256, 64, 64)
    tm.arrays()["err"].fill_(5)
    B.build_tile_map(B.DeviceMask(mask), tm)
    assert B.device_status(tm) == 0
    torch.cuda.synchronize()
