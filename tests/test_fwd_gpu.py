"""GPU forward pass vs the float64 oracle, element by element.

Small problems are compared on every row (they span several tiles and end in
ragged tails); the named full-size workloads, in the launch configuration the
benchmark times, are compared on sampled rows of sampled heads.
Tolerances: max |out - ref| <= 2e-2, mean <= 2e-3, |lse - ref| <= 1e-3 on rows
with a visible key; rows without one must give exactly out = 0, lse = -inf.
"""
import zlib

import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W

from .gpu_util import compare_attention, compare_map, oracle_rows, run_gpu, sample_rows

pytestmark = pytest.mark.gpu


def small_problem(mask, Hq, Hkv, d, seed, Nq=None, Nk=None, dtype=torch.bfloat16):
    Nq = mask.Nq if Nq is None else Nq
    Nk = mask.Nk if Nk is None else Nk
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(mask.B, Hq, Nq, d, generator=g).to(dtype)
    k = torch.randn(mask.B, Hkv, Nk, d, generator=g).to(dtype)
    v = torch.randn(mask.B, Hkv, Nk, d, generator=g).to(dtype)
    return W.Problem("small", q, k, v, mask, seed)


def check_full(prob, bq, bk):
    out, lse, arrays, err = run_gpu(prob, bq, bk)
    assert err == 0
    compare_map(arrays, prob.mask, bq, bk)
    ref_out, ref_lse = oracle_rows(prob, None)
    return compare_attention(out, lse, ref_out, ref_lse)


RNG = np.random.default_rng(5)
CASES = [
    # name, mask, Hq, Hkv, d, block sizes
    ("doc_gqa", W.make_mask("doc8k", N=1024), 8, 2, 128, [(64, 128), (128, 128), (64, 64), (128, 64)]),
    ("doc_ragged", W.make_mask("tiny_doc_fp32", N=1000), 4, 2, 128, [(64, 128), (128, 64)]),
    ("shared", W.make_mask("shared_question8k", N=2048), 4, 2, 128, [(64, 128)]),
    ("band", W.band(2, 1500, 300, 0), 2, 2, 128, [(128, 128), (128, 64)]),
    ("band_neg", W.band(1, 900, 400, -64), 2, 2, 128, [(128, 128)]),
    ("band_negpre", W.band(1, 700, -40, 170), 2, 1, 128, [(128, 128), (64, 64)]),
    ("blocksel", W.blocksel_topk(RNG, 1, 1024, 4), 4, 2, 128, [(64, 64), (64, 128), (128, 128)]),
    ("blocksel_rand", W.random_blocksel(RNG, 1, 700, 700, 5), 2, 1, 128, [(64, 64), (128, 128)]),
    ("random_hm", W.random_colwise(RNG, 1, 4, 700, 700), 4, 2, 128, [(128, 128), (128, 64)]),
    ("doc_d64", W.make_mask("doc8k", N=1024), 4, 2, 64, [(64, 128), (128, 64)]),
    ("band_d64", W.band(1, 777, 100, 3), 2, 2, 64, [(128, 128)]),
]


@pytest.mark.parametrize("name,mask,Hq,Hkv,d,blocks", CASES, ids=[c[0] for c in CASES])
def test_fwd_small_all_rows(name, mask, Hq, Hkv, d, blocks):
    prob = small_problem(mask, Hq, Hkv, d, seed=zlib.crc32(name.encode()) % 1000)
    for bq, bk in blocks:
        check_full(prob, bq, bk)


FP32_CASES = [
    # fp32 inputs are computed in fp32 on the CUDA cores; output is fp32
    ("doc_fp32", W.make_mask("doc8k", N=1024), 4, 2, [(64, 128), (128, 64), (128, 128)]),
    ("ragged_fp32", W.make_mask("tiny_doc_fp32", N=700), 2, 2, [(128, 64), (128, 128)]),
    ("band_fp32", W.band(1, 600, 100, -5), 2, 1, [(64, 64), (128, 128)]),
    ("blocksel_fp32", W.random_blocksel(np.random.default_rng(3), 1, 640, 640, 4), 2, 2, [(128, 64)]),
]


@pytest.mark.parametrize("name,mask,Hq,Hkv,blocks", FP32_CASES, ids=[c[0] for c in FP32_CASES])
def test_fwd_fp32_all_rows(name, mask, Hq, Hkv, blocks):
    prob = small_problem(mask, Hq, Hkv, 64, seed=zlib.crc32(name.encode()) % 1000, dtype=torch.float32)
    for bq, bk in blocks:
        out, lse, arrays, err = run_gpu(prob, bq, bk)
        assert err == 0
        ref_out, ref_lse = oracle_rows(prob, None)
        compare_attention(out, lse, ref_out, ref_lse)


def test_fwd_fp32_d128_and_per_head_masks():
    rng = np.random.default_rng(12)
    mask = W.random_colwise(rng, 1, 3, 300, 280)
    prob = small_problem(mask, 3, 1, 128, seed=1, Nq=300, Nk=280, dtype=torch.float32)
    for bq, bk in [(64, 128), (128, 64)]:
        out, lse, _, err = run_gpu(prob, bq, bk)
        assert err == 0
        ref_out, ref_lse = oracle_rows(prob, None)
        compare_attention(out, lse, ref_out, ref_lse)


def test_fwd_rectangular_nq_ne_nk():
    rng = np.random.default_rng(9)
    mask = W.random_colwise(rng, 1, 1, 500, 900)
    prob = small_problem(mask, 4, 2, 128, seed=3, Nq=500, Nk=900)
    check_full(prob, 64, 128)


def test_fwd_no_keys():
    """Nk = 0: every row sees nothing."""
    mask = W.MaskDesc(W.MASK_COLWISE, 1, 1, 200, 0)
    prob = small_problem(mask, 4, 2, 128, seed=2, Nq=200, Nk=0)
    out, lse, _, err = run_gpu(prob, 64, 128)
    assert err == 0
    assert torch.isneginf(lse).all() and (out == 0).all()


def test_fwd_all_rows_masked():
    prob = small_problem(W.band(1, 300, 10, -400), 2, 2, 128, seed=4)
    out, lse, _, err = run_gpu(prob, 128, 128)
    assert err == 0
    assert torch.isneginf(lse).all() and (out == 0).all()


@pytest.mark.parametrize("layout", ["offset16", "bnhd"])
def test_fwd_output_layouts(layout):
    """The epilogue writes 32-byte pieces of a row when out and its strides are
    32-byte aligned and 16-byte pieces otherwise: an out that starts 16 bytes
    past an aligned address takes the second path, a [B, N, H, D] view (rows of
    one head H * D apart) the first one with a non-contiguous row stride."""
    mask = W.make_mask("doc8k", N=1024)
    prob = small_problem(mask, 4, 2, 128, seed=12)
    att = B.Attention(prob.mask, 64, 128)
    att.build()
    q, k, v = (t.to("cuda") for t in (prob.q, prob.k, prob.v))
    Bn, Hq, Nq, d = q.shape
    if layout == "offset16":
        buf = torch.zeros(q.numel() + 8, dtype=torch.bfloat16, device="cuda")
        out = buf[8:].view(Bn, Hq, Nq, d)
        assert out.data_ptr() % 32 == 16
    else:
        out = torch.zeros(Bn, Nq, Hq, d, dtype=torch.bfloat16, device="cuda").permute(0, 2, 1, 3)
    lse = torch.empty(Bn, Hq, Nq, dtype=torch.float32, device="cuda")
    att(q, k, v, out, lse)
    assert B.device_status(att.tmap) == 0
    ref_out, ref_lse = oracle_rows(prob, None)
    compare_attention(out.float().cpu(), lse.cpu(), ref_out, ref_lse)


def test_fwd_rows_without_keys_inside_visible_tiles():
    """Causal mask in which queries 100..109 see no key at all while the other
    rows of their tiles do. Those rows run through PARTIAL and FULL tiles with a
    running max of -inf (every score of the row is -inf, so each exponential is
    taken against a reference of 0); they must still give out = 0 and
    lse = -inf, and the rows around them must be unaffected."""
    N = 600
    j = np.arange(N, dtype=np.int32)
    uts = np.zeros((1, 1, N), np.int32)
    ute = j.reshape(1, 1, N).copy()                    # causal: rows < j masked
    lts = np.maximum(100, j).astype(np.int32).reshape(1, 1, N)
    lte = np.full((1, 1, N), 110, np.int32)
    lte = np.where(j.reshape(1, 1, N) < 110, lte, lts)  # rows [max(100, j), 110) masked
    mask = W.MaskDesc(W.MASK_COLWISE, 1, 1, N, N, lts, lte.astype(np.int32), uts, ute, name="holes")
    prob = small_problem(mask, 4, 2, 128, seed=21)
    for bq, bk in ((64, 128), (128, 64)):
        out, lse, arrays, err = run_gpu(prob, bq, bk)
        assert err == 0
        compare_map(arrays, prob.mask, bq, bk)
        ref_out, ref_lse = oracle_rows(prob, None)
        assert np.isneginf(ref_lse[:, :, 100:110]).all() and np.isfinite(ref_lse[:, :, 110:]).all()
        compare_attention(out, lse, ref_out, ref_lse)


def test_fwd_deterministic():
    prob = small_problem(W.make_mask("doc8k", N=1024), 4, 2, 128, seed=6)
    a, la, _, _ = run_gpu(prob, 64, 128)
    b, lb, _, _ = run_gpu(prob, 64, 128)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_fwd_zero_query_closed_form():
    """q = 0 makes every visible score 0: out is the mean of the visible v rows."""
    mask = W.make_mask("shared_question8k", N=1024)
    prob = small_problem(mask, 2, 1, 128, seed=8)
    prob.q.zero_()
    out, lse, _, err = run_gpu(prob, 64, 128)
    assert err == 0
    ref_out, ref_lse = oracle_rows(prob, None)
    compare_attention(out, lse, ref_out, ref_lse)


# Full-size named workloads in the benchmark's launch configuration.
FULL = [("tiny_doc_fp32", 128, 64), ("doc8k", 64, 128), ("shared_question8k", 64, 128), ("band16k", 128, 128),
        ("band16k_neg", 128, 128), ("doc32k", 64, 128), ("blocksel32k", 64, 64)]


@pytest.mark.parametrize("name,bq,bk", FULL, ids=[f[0] for f in FULL])
def test_fwd_full_size_sampled(name, bq, bk):
    prob = W.make_problem(name)
    out, lse, arrays, err = run_gpu(prob, bq, bk)
    assert err == 0
    compare_map(arrays, prob.mask, bq, bk)
    rng = np.random.default_rng(17)
    Bsz, Hq, _, N, _ = prob.shape
    rows = sample_rows(N, 96, rng)
    heads = sorted(set([0, Hq - 1] + [int(x) for x in rng.choice(Hq, 2, replace=False)]))
    ref_out, ref_lse = oracle_rows(prob, rows, heads)
    got_out = out[:, heads][:, :, rows]
    got_lse = lse[:, heads][:, :, rows]
    compare_attention(got_out, got_lse, ref_out, ref_lse)
    if name == "band16k_neg":   # 64 rows per (b, h) see no key
        assert torch.isneginf(lse[:, :, :64]).all() and torch.isfinite(lse[:, :, 64:]).all()


def test_fwd_blocksel_longest_lists():
    """Selection lists of the maximum length (256 entries per 64-query block),
    uniform over all 266 key blocks of 17000 keys: -1 pads, duplicates and
    entries above the diagonal (ignored), and a ragged last block."""
    rng = np.random.default_rng(31)
    mask = W.random_blocksel(rng, 1, 17000, 17000, 256, p_pad=0.3)
    prob = small_problem(mask, 2, 1, 128, 31)
    rows = sample_rows(17000, 64, np.random.default_rng(3))
    ref_out, ref_lse = oracle_rows(prob, rows)
    for bq, bk in ((64, 64), (128, 128)):
        out, lse, arrays, err = run_gpu(prob, bq, bk)
        assert err == 0
        compare_map(arrays, mask, bq, bk)
        compare_attention(out[:, :, rows], lse[:, :, rows], ref_out, ref_lse)


def test_binding_checks_raw_pointer_arguments():
    """Arguments passed as plain device pointers (lse, slopes, selection lists)
    are checked for dtype and shape before the call: a short buffer would be
    written past its end."""
    mask = W.band(1, 256, 64, 0)
    prob = small_problem(mask, 2, 1, 128, 4)
    att = B.Attention(mask, 128, 128)
    att.build()
    q, k, v = (t.cuda() for t in (prob.q, prob.k, prob.v))
    with pytest.raises(ValueError, match="lse"):
        att(q, k, v, lse=torch.empty(1, 2, 255, device="cuda"))
    with pytest.raises(ValueError, match="lse"):
        att(q, k, v, lse=torch.empty(1, 2, 256, dtype=torch.float64, device="cuda"))
    with pytest.raises(ValueError, match="slopes"):
        att(q, k, v, bias=(B.BIAS_ALIBI, torch.ones(1, device="cuda")))
    dec = B.Decode()
    with pytest.raises(ValueError, match="sel"):
        dec(q[:, :, :1], k, v, torch.zeros(1, 2, 1, 4, dtype=torch.int32, device="cuda"))  # Hkv is 1, not 2
    out, lse = att(q, k, v)
    assert B.device_status(att.tmap) == 0 and torch.isfinite(lse).all()
