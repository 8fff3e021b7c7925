"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each check uses something independent: a closed form of the mask, a library
routine the masked problem reduces to (torch's scaled_dot_product_attention in
float64), a brute-force scalar loop on tiny inputs, or a statement printed on
the pages (the Ascend band examples in tests/golden). The mutation tests at the
end plant plausible mistakes in a copy of the oracle and check that a pin fails.
"""
import math
import os

import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import workloads as W
from oracle import attention as OA
from oracle import masks as OM

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# closed forms of the mask kinds
# ----------------------------------------------------------------------------

def closed_causal_docs(N, docs):
    blocks = [torch.tril(torch.ones(e - s, e - s, dtype=torch.bool)) for (s, e) in docs]
    return torch.block_diag(*blocks).numpy()


def closed_band(Nq, Nk, pre, nxt):
    ones = np.ones((Nq, Nk), dtype=bool)
    return np.triu(ones, k=-pre) & np.tril(ones, k=nxt)


def closed_shared_question(N, q_len, answers):
    vis = np.zeros((N, N), dtype=bool)
    vis[:q_len, :q_len] = np.tril(np.ones((q_len, q_len), dtype=bool))
    for (s, e) in answers:
        vis[s:e, :q_len] = True
        vis[s:e, s:e] = np.tril(np.ones((e - s, e - s), dtype=bool))
    return vis


def closed_blocksel(N, sel_rows):
    nb = -(-N // 64)
    blk = np.zeros((nb, nb), dtype=bool)
    for qb in range(nb):
        for kb in sel_rows[qb]:
            if kb >= 0:
                blk[qb, kb] = True
    dense = np.kron(blk, np.ones((64, 64), dtype=bool))[:N, :N]
    return dense & np.tril(np.ones((N, N), dtype=bool))


@pytest.mark.parametrize("name,N", [("tiny_doc_fp32", 512), ("doc8k", 1024), ("doc8k", 8192),
                                    ("doc32k", 2048)])
def test_causal_document_equals_block_diagonal_tril(name, N):
    m = W.make_mask(name, N=N)
    docs = m.docs[0]
    assert docs[0][0] == 0 and docs[-1][1] == N
    np.testing.assert_array_equal(OM.visible_dense(m), closed_causal_docs(N, docs))


def test_shared_question_equals_union_form():
    m = W.make_mask("shared_question8k", N=2048)
    q_len = m.docs[0][0][1]
    answers = m.docs[0][1:]
    assert 4 <= len(answers) <= 8
    np.testing.assert_array_equal(OM.visible_dense(m), closed_shared_question(2048, q_len, answers))


@pytest.mark.parametrize("pre,nxt,N", [(2048, 0, 3000), (4096, -64, 5000), (5, 3, 40), (0, 0, 17),
                                       (100, -99, 130), (-3, 7, 20)])
def test_band_equals_triangular_pair(pre, nxt, N):
    m = W.band(1, N, pre, nxt)
    np.testing.assert_array_equal(OM.visible_dense(m), closed_band(N, N, pre, nxt))


@pytest.mark.parametrize("N", [512, 1000])
def test_blocksel_equals_kron_and_tril(N):
    m = W.blocksel_topk(np.random.default_rng(7), 1, N, 4)
    np.testing.assert_array_equal(OM.visible_dense(m), closed_blocksel(N, m.sel[0, 0]))


def test_blocksel_ignores_pads_and_duplicates():
    N = 256
    sel = np.full((1, 1, 4, 4), -1, np.int32)
    sel[0, 0, 3] = [1, 1, -1, 3]          # duplicate 1, pad, the diagonal block
    sel[0, 0, 1] = [3, -1, -1, -1]        # above the diagonal: no visible pair
    m = W.MaskDesc(W.MASK_BLOCKSEL, 1, 1, N, N, sel=sel)
    vis = OM.visible_dense(m)
    assert not vis[64:128].any()
    assert vis[192:256, 64:128].all()
    np.testing.assert_array_equal(vis[192:256, 192:256], np.tril(np.ones((64, 64), dtype=bool)))
    assert vis.sum() == 64 * 64 + 64 * 65 // 2


def test_visible_pairs_closed_forms():
    m = W.make_mask("doc8k")
    lengths = [e - s for (s, e) in m.docs[0]]
    assert all(L % 64 == 0 for L in lengths) and sum(lengths) == 8192
    assert OM.visible_pairs(m) == sum(L * (L + 1) // 2 for L in lengths)
    # band with next = 0: row i sees min(i, pre) + 1 keys
    N, pre = 3000, 2048
    expect = sum(min(i, pre) + 1 for i in range(N))
    assert OM.visible_pairs(W.band(1, N, pre, 0)) == expect
    # next = -64: row i sees keys [i - pre, i - 64] clipped at 0 -> 64 empty rows
    N, pre, nxt = 5000, 4096, -64
    expect = sum(max(0, (i + nxt) - max(0, i - pre) + 1) for i in range(N))
    assert OM.visible_pairs(W.band(1, N, pre, nxt)) == expect


def test_ascend_band_examples_from_page():
    """The page's own cases: causal, band, negative next and negative pre."""
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "ascend_band_examples.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 5
    for case, pre, nxt, sq, skv, shape in rows:
        pre, nxt, sq, skv = int(pre), int(nxt), int(sq), int(skv)
        vis = OM.visible_dense(W.MaskDesc(W.MASK_BAND, 1, 1, sq, skv, pre_tokens=pre, next_tokens=nxt))
        if shape == "causal":
            np.testing.assert_array_equal(vis, np.tril(np.ones((sq, skv), dtype=bool)))
        elif shape == "band":
            assert pre < sq and nxt < skv and pre >= 0 and nxt >= 0
            width = vis.sum(axis=1)
            assert (width[pre:sq - nxt] == pre + nxt + 1).all()
        elif shape == "neg_next":
            assert pre >= abs(nxt) and abs(nxt) < skv     # the page's constraint
            assert not vis[: -nxt].any()                  # the first |next| rows see nothing
            assert vis[sq - 1].sum() == pre + nxt + 1
        elif shape == "neg_pre":
            assert nxt >= abs(pre) and abs(pre) < sq
            assert not vis[:, : -pre].any()               # the first |pre| keys see no query
            assert not np.diag(vis).any()                 # the diagonal itself is outside
            assert vis[0].sum() == nxt + pre + 1


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def _sdpa(q, k, v, vis):
    """torch's fused attention in float64 with a dense boolean mask (True = attend)."""
    qt = torch.from_numpy(q)[None, None]
    kt = torch.from_numpy(k)[None, None]
    vt = torch.from_numpy(v)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(vis)[None, None])[0, 0].numpy()


def test_all_visible_equals_library_attention():
    rng = np.random.default_rng(0)
    N, d = 96, 32
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    m = W.MaskDesc(W.MASK_COLWISE, 1, 1, N, N)   # no intervals: everything visible
    out, _ = OA.attention(q[None, None], k[None, None], v[None, None], m)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None])[0, 0].numpy()
    np.testing.assert_allclose(out[0, 0], ref, rtol=0, atol=1e-13)


@pytest.mark.parametrize("mk", ["doc", "band", "shared", "blocksel"])
def test_masked_equals_library_attention_with_dense_mask(mk):
    rng = np.random.default_rng(1)
    N, d = 320, 16
    if mk == "doc":
        m = W.make_mask("tiny_doc_fp32", N=N)
        vis = closed_causal_docs(N, m.docs[0])
    elif mk == "band":
        m = W.band(1, N, 40, 5)
        vis = closed_band(N, N, 40, 5)
    elif mk == "shared":
        m = W.colwise_shared_question(1, N, 64, [[(64, 192), (192, 320)]])
        vis = closed_shared_question(N, 64, [(64, 192), (192, 320)])
    else:
        m = W.blocksel_topk(rng, 1, N, 2)
        vis = closed_blocksel(N, m.sel[0, 0])
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    out, lse = OA.attention(q[None, None], k[None, None], v[None, None], m)
    assert vis.any(axis=1).all()
    np.testing.assert_allclose(out[0, 0], _sdpa(q, k, v, vis), rtol=0, atol=1e-12)
    # lse against torch.logsumexp of the library's masked scores
    s = torch.from_numpy(q) @ torch.from_numpy(k).T / math.sqrt(d)
    s = s.masked_fill(~torch.from_numpy(vis), -math.inf)
    np.testing.assert_allclose(lse[0, 0], torch.logsumexp(s, dim=1).numpy(), rtol=0, atol=1e-12)


def test_brute_force_scalar_loops():
    """Direct formula, no max subtraction, exact summation (math.fsum), tiny sizes."""
    rng = np.random.default_rng(2)
    for N, d, pre, nxt in [(7, 3, 2, 1), (12, 4, 20, 0), (9, 2, 3, -2)]:
        q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
        m = W.band(1, N, pre, nxt)
        out, lse = OA.attention(q[None, None], k[None, None], v[None, None], m)
        for i in range(N):
            js = [j for j in range(N) if -pre <= j - i <= nxt]
            if not js:
                assert lse[0, 0, i] == -math.inf and not out[0, 0, i].any()
                continue
            e = [math.exp(math.fsum(q[i, t] * k[j, t] for t in range(d)) / math.sqrt(d)) for j in js]
            z = math.fsum(e)
            for t in range(d):
                o = math.fsum(e[a] * v[j, t] for a, j in enumerate(js)) / z
                assert abs(o - out[0, 0, i, t]) < 1e-12
            assert abs(math.log(z) - lse[0, 0, i]) < 1e-12


def test_zero_query_closed_form():
    """q = 0: every visible key has score 0, so out = mean of visible v, lse = ln(count)."""
    rng = np.random.default_rng(3)
    m = W.make_mask("shared_question8k", N=1024)
    N, d = 1024, 8
    q = np.zeros((N, d))
    k, v = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    rows = rng.choice(N, 64, replace=False)
    out, lse = OA.attention(q[None, None], k[None, None], v[None, None], m, rows=rows)
    vis = closed_shared_question(N, m.docs[0][0][1], m.docs[0][1:])
    for r, i in enumerate(rows):
        js = np.nonzero(vis[i])[0]
        np.testing.assert_allclose(out[0, 0, r], v[js].mean(axis=0), atol=1e-13)
        assert abs(lse[0, 0, r] - math.log(len(js))) < 1e-13


def test_single_visible_key_and_empty_rows():
    """next = -64: rows 0..63 see nothing (0, -inf); row 64 sees only key 0."""
    rng = np.random.default_rng(4)
    N, d = 200, 8
    q, k, v = (rng.standard_normal((1, 2, N, d)) for _ in range(3))
    m = W.band(1, N, 4096, -64)
    out, lse = OA.attention(q, k, v, m)
    assert np.isneginf(lse[0, :, :64]).all() and (out[0, :, :64] == 0).all()
    assert np.isfinite(lse[0, :, 64:]).all()
    for h in range(2):
        np.testing.assert_array_equal(out[0, h, 64], v[0, h, 0])
        assert abs(lse[0, h, 64] - q[0, h, 64] @ k[0, h, 0] / math.sqrt(d)) < 1e-13


def test_one_hot_values_give_softmax_weights():
    """V = identity: out_ij is the weight of key j, so ln(out_ij) + lse_i = s_ij."""
    rng = np.random.default_rng(5)
    N, d = 48, 6
    q, k = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    v = np.eye(N)
    m = W.band(1, N, 10, 2)
    out, lse = OA.attention(q[None, None], k[None, None], v[None, None], m)
    vis = closed_band(N, N, 10, 2)
    s = q @ k.T / math.sqrt(d)
    np.testing.assert_allclose(out[0, 0].sum(axis=1), 1.0, atol=1e-13)
    assert (out[0, 0][~vis] == 0).all()
    rows = np.nonzero(vis)[0]
    np.testing.assert_allclose(np.log(out[0, 0][vis]) + lse[0, 0][rows], s[vis], atol=1e-12)


def test_gqa_head_mapping():
    """Query head h reads key/value head h // G: compare with repeated K/V and no GQA."""
    rng = np.random.default_rng(6)
    N, d, Hq, Hkv = 64, 8, 6, 2
    q = rng.standard_normal((1, Hq, N, d))
    k, v = rng.standard_normal((1, Hkv, N, d)), rng.standard_normal((1, Hkv, N, d))
    m = W.band(1, N, 9, 0)
    out, _ = OA.attention(q, k, v, m)
    for h in range(Hq):
        ref = _sdpa(q[0, h], k[0, h // 3], v[0, h // 3], closed_band(N, N, 9, 0))
        np.testing.assert_allclose(out[0, h], ref, atol=1e-12)


def test_bounds_outside_range_rejected():
    m = W.make_mask("tiny_doc_fp32", N=128)
    m.lte = m.lte.copy()
    m.lte[0, 0, 5] = 129
    with pytest.raises(ValueError):
        OM.visible_dense(m)
    s = W.blocksel_topk(np.random.default_rng(0), 1, 128, 2)
    s.sel[0, 0, 0, 0] = 2
    with pytest.raises(ValueError):
        OM.visible_dense(s)


# ----------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle must fail one of the pins above
# ----------------------------------------------------------------------------

def _mutant_visible_rows(mutation):
    orig = OM.visible_rows

    def f(mask, b, hm, rows):
        vis = orig(mask, b, hm, rows)
        i = np.asarray(rows)[:, None]
        j = np.arange(mask.Nk)[None, :]
        if mutation == "closed_interval" and mask.kind == OM.COLWISE:
            ute = np.asarray(mask.ute)[b, hm][None, :]
            vis = vis & ~(i == ute)              # treats the interval end as inclusive
        if mutation == "band_sign" and mask.kind == OM.BAND:
            diff = i - j                          # j - i written the wrong way round
            vis = (diff >= -mask.pre_tokens) & (diff <= mask.next_tokens)
        if mutation == "blocksel_no_causal" and mask.kind == OM.BLOCKSEL:
            vis = vis.copy()
            for r, row in enumerate(np.asarray(rows)):
                d0 = (row // 64) * 64
                if vis[r, d0]:                    # diagonal block selected: drop j <= i
                    vis[r, d0:d0 + 64] = True
        return vis
    return f


@pytest.mark.parametrize("mutation,check", [
    ("closed_interval", lambda: test_causal_document_equals_block_diagonal_tril("doc8k", 1024)),
    ("band_sign", lambda: test_band_equals_triangular_pair(5, 3, 40)),
    ("blocksel_no_causal", lambda: test_blocksel_equals_kron_and_tril(512)),
])
def test_planted_mask_mistakes_are_caught(monkeypatch, mutation, check):
    monkeypatch.setattr(OM, "visible_rows", _mutant_visible_rows(mutation))
    with pytest.raises(AssertionError):
        check()


def test_planted_attention_mistakes_are_caught(monkeypatch):
    orig = OA.attention_rows

    def no_scale(q_rows, k, v, vis):        # drops the 1/sqrt(d)
        return orig(q_rows * math.sqrt(q_rows.shape[1]), k, v, vis)

    monkeypatch.setattr(OA, "attention_rows", no_scale)
    with pytest.raises(AssertionError):
        test_all_visible_equals_library_attention()

    def lse_log2(q_rows, k, v, vis):         # lse in base 2 instead of natural log
        o, s = orig(q_rows, k, v, vis)
        return o, s / math.log(2)

    monkeypatch.setattr(OA, "attention_rows", lse_log2)
    with pytest.raises(AssertionError):
        test_zero_query_closed_form()
