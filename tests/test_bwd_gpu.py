"""Gradients on the GPU (mfa_bwd through the C ABI) against the float64 oracle.

Every case runs the tile map and the forward pass, then the backward pass
with a seeded bf16 output gradient, and compares dq, dk, dv element by element
with oracle/backward.py on the same bf16 inputs. Tolerances (relative to the
gradient's own scale; the derivation is the rounding of P and dS to bf16
before the tensor-core products, plus Delta from the bf16 output):
max |err| <= GRAD_MAX_REL * max |ref| and mean |err| <= GRAD_MEAN_REL * mean |ref|.
Exact zeros: keys that no query sees get dk = dv = 0 and rows with no visible
key get dq = 0.
"""
import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W
from oracle import backward as OB
from oracle import masks as OM
from oracle import sparse_modes as SM

pytestmark = pytest.mark.gpu

GRAD_MAX_REL = 1e-2
GRAD_MEAN_REL = 5e-3


def compare_grad(got, ref, name, exact_zero=None):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    if exact_zero is not None and exact_zero.any():
        assert (got[exact_zero] == 0).all(), f"{name}: must be exactly 0 where nothing contributes"
    diff = np.abs(got - ref)
    scale = float(np.abs(ref).max())
    if scale == 0.0:
        assert float(diff.max()) == 0.0, f"{name}: expected all zeros"
        return 0.0, 0.0
    max_rel = float(diff.max()) / scale
    mean_rel = float(diff.mean()) / float(np.abs(ref).mean())
    assert max_rel <= GRAD_MAX_REL, f"{name}: max error {max_rel:.3e} of max |ref|"
    assert mean_rel <= GRAD_MEAN_REL, f"{name}: mean error {mean_rel:.3e} of mean |ref|"
    return max_rel, mean_rel


def _randn(g, *shape):
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def run_bwd(dev_mask, q, k, v, dout, block_q=None):
    """Map, forward and backward. The forward packs two heads of a group into
    a 64-query tile, which needs an even group size; otherwise the map (shared
    by both passes) uses 128-query tiles."""
    G = q.shape[1] // k.shape[1]
    block_q = block_q or (64 if G % 2 == 0 else 128)
    att = B.Attention(dev_mask, block_q, 128)
    att.build()
    qc, kc, vc, dc = (t.cuda() for t in (q, k, v, dout))
    out, lse = att(qc, kc, vc)
    dq, dk, dv = att.backward(qc, kc, vc, out, lse, dc)
    assert B.device_status(att.tmap) == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


def check_all(mask, oracle_mask, q, k, v, dout, dev_mask=None):
    dq, dk, dv = run_bwd(mask if dev_mask is None else dev_mask, q, k, v, dout)
    rq, rk, rv = OB.attention_backward(q, k, v, oracle_mask, dout)
    vis = np.stack([_visible(oracle_mask, b) for b in range(q.shape[0])])  # [B, Nq, Nk]
    no_key = ~vis.any(axis=2)                         # rows without a visible key
    unseen = ~vis.any(axis=1)                         # keys no query sees
    zq = np.broadcast_to(no_key[:, None, :, None], rq.shape)
    zk = np.broadcast_to(unseen[:, None, :, None], rk.shape)
    r = {}
    r["dq"] = compare_grad(dq, rq, "dq", zq)
    r["dk"] = compare_grad(dk, rk, "dk", zk)
    r["dv"] = compare_grad(dv, rv, "dv", zk)
    return r


def _visible(mask, b):
    if hasattr(mask, "visible_rows"):
        return mask.visible_rows(b, 0, np.arange(mask.Nq))
    return OM.visible_dense(mask, b)


SMALL = [
    # name, mask factory, Hq, Hkv
    ("doc_g2", lambda: W.make_mask("doc8k", N=1000), 4, 2),
    ("doc_g4", lambda: W.make_mask("doc8k", N=1000), 8, 2),
    ("doc_g1", lambda: W.make_mask("doc8k", N=1000), 2, 2),
    ("shared_question", lambda: W.make_mask("shared_question8k", N=1024), 4, 1),
    ("band", lambda: W.band(1, 1000, 100, 0), 4, 2),
    ("band_neg_empty_rows", lambda: W.band(2, 777, 200, -64), 2, 1),
    ("blocksel", lambda: W.make_mask("blocksel32k", N=1024), 4, 2),
    ("random_colwise", lambda: W.random_colwise(np.random.default_rng(5), 1, 1, 640, 640), 4, 2),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c[0])
def test_bwd_small_all_elements(case):
    name, factory, Hq, Hkv = case
    mask = factory()
    g = torch.Generator().manual_seed(11)
    Bsz, Nq, Nk = mask.B, mask.Nq, mask.Nk
    q, k, v = _randn(g, Bsz, Hq, Nq, 128), _randn(g, Bsz, Hkv, Nk, 128), _randn(g, Bsz, Hkv, Nk, 128)
    dout = _randn(g, Bsz, Hq, Nq, 128)
    check_all(mask, mask, q, k, v, dout)


@pytest.mark.parametrize("block_q", [64, 128])
def test_bwd_map_tile_heights(block_q):
    """The same problem through a 64-row and a 128-row map (both halves of a
    128-row tile take its class)."""
    mask = W.make_mask("blocksel32k", N=896)
    g = torch.Generator().manual_seed(19)
    q, k, v = _randn(g, 1, 4, 896, 128), _randn(g, 1, 2, 896, 128), _randn(g, 1, 2, 896, 128)
    dout = _randn(g, 1, 4, 896, 128)
    dq, dk, dv = run_bwd(mask, q, k, v, dout, block_q=block_q)
    rq, rk, rv = OB.attention_backward(q, k, v, mask, dout)
    compare_grad(dq, rq, "dq")
    compare_grad(dk, rk, "dk")
    compare_grad(dv, rv, "dv")


def test_bwd_rectangular_band():
    mask = W.MaskDesc(W.MASK_BAND, 1, 1, 700, 1300, pre_tokens=300, next_tokens=600)
    g = torch.Generator().manual_seed(12)
    q, k, v = _randn(g, 1, 4, 700, 128), _randn(g, 1, 2, 1300, 128), _randn(g, 1, 2, 1300, 128)
    check_all(mask, mask, q, k, v, _randn(g, 1, 4, 700, 128))


def test_bwd_sparse_mode_varlen():
    sq, skv = np.cumsum([100, 0, 150, 60]), np.cumsum([120, 40, 150, 200])
    dev = B.SparseModeMask(7, 1, 310, 510, 500, -30, seq_q=sq, seq_kv=skv)
    ref = SM.SparseMode(7, 1, 310, 510, 500, -30, seq_q=sq, seq_kv=skv)
    g = torch.Generator().manual_seed(13)
    q, k, v = _randn(g, 1, 4, 310, 128), _randn(g, 1, 1, 510, 128), _randn(g, 1, 1, 510, 128)
    check_all(None, ref, q, k, v, _randn(g, 1, 4, 310, 128), dev_mask=dev)


def test_bwd_large_values_and_zero_output_gradient():
    mask = W.make_mask("doc8k", N=512)
    g = torch.Generator().manual_seed(14)
    q = (torch.randn(1, 2, 512, 128, generator=g) * 4).to(torch.bfloat16)   # peaked softmax
    k, v = _randn(g, 1, 1, 512, 128), _randn(g, 1, 1, 512, 128)
    check_all(mask, mask, q, k, v, _randn(g, 1, 2, 512, 128))
    dq, dk, dv = run_bwd(mask, q, k, v, torch.zeros(1, 2, 512, 128, dtype=torch.bfloat16))
    assert (dq == 0).all() and (dk == 0).all() and (dv == 0).all()


def test_bwd_no_queries_and_no_keys():
    g = torch.Generator().manual_seed(15)
    m0 = W.MaskDesc(W.MASK_BAND, 1, 1, 0, 300, pre_tokens=10, next_tokens=0)
    dq, dk, dv = run_bwd(m0, _randn(g, 1, 2, 0, 128), _randn(g, 1, 1, 300, 128), _randn(g, 1, 1, 300, 128),
                         _randn(g, 1, 2, 0, 128))
    assert dk.shape == (1, 1, 300, 128) and (dk == 0).all() and (dv == 0).all()
    m1 = W.MaskDesc(W.MASK_BAND, 1, 1, 200, 0, pre_tokens=10, next_tokens=0)
    dq, dk, dv = run_bwd(m1, _randn(g, 1, 2, 200, 128), _randn(g, 1, 1, 0, 128), _randn(g, 1, 1, 0, 128),
                         _randn(g, 1, 2, 200, 128))
    assert (dq == 0).all()


def test_bwd_key_gradients_are_deterministic():
    mask = W.make_mask("doc8k", N=1024)
    g = torch.Generator().manual_seed(16)
    q, k, v = _randn(g, 1, 4, 1024, 128), _randn(g, 1, 2, 1024, 128), _randn(g, 1, 2, 1024, 128)
    dout = _randn(g, 1, 4, 1024, 128)
    a = run_bwd(mask, q, k, v, dout)
    b = run_bwd(mask, q, k, v, dout)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # dq sums key tiles in whatever order their reductions reach memory
    assert float((a[0].float() - b[0].float()).abs().max()) <= GRAD_MAX_REL * float(a[0].float().abs().max())


@pytest.mark.parametrize("name", ["doc8k", "blocksel32k"])
def test_bwd_full_size_sampled(name):
    """Full-size workload with the bench's launch configuration: dq on sampled
    rows, dk/dv on sampled key columns of one key/value head (the oracle sums
    only the rows that see those keys, which is exact for them)."""
    prob = W.make_problem(name)
    Bsz, Hq, Hkv, N, d = prob.shape
    G = Hq // Hkv
    g = torch.Generator().manual_seed(17)
    dout = _randn(g, Bsz, Hq, N, d)
    dq, dk, dv = run_bwd(prob.mask, prob.q, prob.k, prob.v, dout)
    rng = np.random.default_rng(18)
    rows = np.unique(np.concatenate([[0, 63, 64, N - 1], rng.choice(N, 24, replace=False)]))
    heads = [0, Hq - 1]
    rq, _, _ = OB.attention_backward(prob.q, prob.k, prob.v, prob.mask, dout, rows=rows, heads=heads)
    compare_grad(dq[0][heads][:, rows], rq[0], "dq (sampled rows)")
    hkv = Hkv - 1
    cols = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.choice(N, 12, replace=False)]))
    vis = OM.visible_dense(prob.mask, 0)
    seeing = np.nonzero(vis[:, cols].any(axis=1))[0]
    _, rk, rv = OB.attention_backward(prob.q, prob.k, prob.v, prob.mask, dout, rows=seeing,
                                      heads=list(range(hkv * G, hkv * G + G)))
    compare_grad(dk[0, hkv][cols], rk[0, hkv][cols], "dk (sampled keys)")
    compare_grad(dv[0, hkv][cols], rv[0, hkv][cols], "dv (sampled keys)")
