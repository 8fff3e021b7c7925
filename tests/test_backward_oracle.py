"""Pins of the oracle's attention gradients (oracle/backward.py).

* central finite differences of L = sum(out * dout) through the forward
  oracle (itself pinned against closed forms and torch), on tiny problems with
  grouped heads, empty rows, every mask kind and a rectangular sparse mode;
* torch.autograd in float64 of a dense masked softmax written with torch ops;
* closed forms and invariants: sum_j dK_j = 0; constant values give dQ = dK = 0;
  q = 0 gives dV_j = sum over the rows that see j of dout_i / (visible count of i);
  rows with no visible key get dQ = 0; row subsets give exact partial sums;
* planted mistakes in a copy of the oracle each fail one of these pins.
"""
import math

import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import workloads as W
from oracle import attention as OA
from oracle import backward as OB
from oracle import masks as OM
from oracle import sparse_modes as SM


def _problem(rng, B, Hq, Hkv, Nq, Nk, d):
    q = rng.standard_normal((B, Hq, Nq, d))
    k = rng.standard_normal((B, Hkv, Nk, d))
    v = rng.standard_normal((B, Hkv, Nk, d))
    dout = rng.standard_normal((B, Hq, Nq, d))
    return q, k, v, dout


def _loss(q, k, v, mask, dout):
    out, _ = OA.attention(q, k, v, mask)
    return float((out * dout).sum())


def _finite_differences(q, k, v, mask, dout, h=1e-6):
    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        x = args[which]
        g = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            x0 = x[idx]
            x[idx] = x0 + h
            lp = _loss(*args, mask, dout)
            x[idx] = x0 - h
            lm = _loss(*args, mask, dout)
            x[idx] = x0
            g[idx] = (lp - lm) / (2 * h)
        grads.append(g)
    return grads


def _fd_cases():
    rng = np.random.default_rng(7)
    docs = W.colwise_causal_documents(1, 11, [W.docs_from_lengths([4, 5, 2])], "docs")
    band_neg = W.band(1, 10, 4, -2)                       # rows 0-1 see no key
    sel = np.full((1, 1, 3, 2), -1, np.int32)
    sel[0, 0, 0] = [0, -1]
    sel[0, 0, 1] = [0, 1]
    sel[0, 0, 2] = [1, 1]                                 # duplicate entry
    blocksel = W.MaskDesc(W.MASK_BLOCKSEL, 1, 1, 130, 130, sel=sel)
    varlen = SM.SparseMode(7, 1, 9, 15, pre_tokens=6, next_tokens=-2, seq_q=[4, 9], seq_kv=[6, 15])
    return [
        ("docs_gqa", docs, (1, 4, 2, 11, 11, 3)),
        ("band_empty_rows", band_neg, (2, 2, 1, 10, 10, 3)),
        ("blocksel", blocksel, (1, 1, 1, 130, 130, 1)),
        ("varlen_rect", varlen, (1, 2, 1, 9, 15, 3)),
    ], rng


@pytest.mark.parametrize("case", range(4))
def test_gradients_match_finite_differences(case):
    cases, rng = _fd_cases()
    name, mask, (B, Hq, Hkv, Nq, Nk, d) = cases[case]
    if mask.B != B:
        mask = W.band(B, Nq, mask.pre_tokens, mask.next_tokens)
    q, k, v, dout = _problem(np.random.default_rng(100 + case), B, Hq, Hkv, Nq, Nk, d)
    dq, dk, dv = OB.attention_backward(q, k, v, mask, dout)
    fq, fk, fv = _finite_differences(q, k, v, mask, dout)
    for got, ref in ((dq, fq), (dk, fk), (dv, fv)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=2e-7)
    assert np.abs(fq).max() > 1e-2 and np.abs(fk).max() > 1e-2 and np.abs(fv).max() > 1e-2


def _torch_dense(q, k, v, vis, dout):
    """Dense masked attention with torch ops in float64, differentiated by autograd."""
    qt, kt, vt = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    G = q.shape[1] // k.shape[1]
    ke, ve = kt.repeat_interleave(G, dim=1), vt.repeat_interleave(G, dim=1)
    s = qt @ ke.transpose(-1, -2) / math.sqrt(q.shape[-1])
    s = s.masked_fill(~torch.from_numpy(vis), -math.inf)
    out = torch.softmax(s, dim=-1) @ ve
    (out * torch.from_numpy(dout)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("mk", ["doc", "band", "shared"])
def test_gradients_match_float64_autograd(mk):
    N, d = 192, 16
    if mk == "doc":
        m = W.colwise_causal_documents(1, N, [W.docs_from_lengths([70, 64, 58])], "doc")
    elif mk == "band":
        m = W.band(1, N, 30, 4)
    else:
        m = W.colwise_shared_question(1, N, 64, [[(64, 128), (128, 192)]])
    vis = OM.visible_dense(m, 0)
    assert vis.any(axis=1).all()
    q, k, v, dout = _problem(np.random.default_rng(3), 1, 4, 2, N, N, d)
    dq, dk, dv = OB.attention_backward(q, k, v, m, dout)
    tq, tk, tv = _torch_dense(q, k, v, vis[None, None], dout)
    for got, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_key_gradients_sum_to_zero_and_constant_values():
    m = W.band(1, 50, 9, -3)
    q, k, v, dout = _problem(np.random.default_rng(4), 1, 4, 2, 50, 50, 8)
    _, dk, _ = OB.attention_backward(q, k, v, m, dout)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    v_const = np.broadcast_to(np.random.default_rng(5).standard_normal(8), v.shape).copy()
    dq, dk, _ = OB.attention_backward(q, k, v_const, m, dout)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)


def test_zero_query_value_gradient_closed_form():
    m = W.colwise_causal_documents(1, 40, [W.docs_from_lengths([13, 27])], "doc")
    q, k, v, dout = _problem(np.random.default_rng(6), 1, 2, 1, 40, 40, 4)
    q[:] = 0.0
    _, _, dv = OB.attention_backward(q, k, v, m, dout)
    vis = OM.visible_dense(m, 0)
    n = vis.sum(axis=1)
    ref = sum((vis / n[:, None]).T @ dout[0, h] for h in range(2))
    np.testing.assert_allclose(dv[0, 0], ref, atol=1e-12)


def test_empty_rows_and_row_subsets():
    m = W.band(1, 40, 6, -5)                               # rows 0-4 see no key
    q, k, v, dout = _problem(np.random.default_rng(8), 1, 2, 1, 40, 40, 4)
    dq, dk, dv = OB.attention_backward(q, k, v, m, dout)
    assert np.all(dq[0, :, :5] == 0.0)
    a, b = np.arange(0, 17), np.arange(17, 40)
    dqa, dka, dva = OB.attention_backward(q, k, v, m, dout, rows=a)
    dqb, dkb, dvb = OB.attention_backward(q, k, v, m, dout, rows=b)
    np.testing.assert_allclose(dka + dkb, dk, atol=1e-12)
    np.testing.assert_allclose(dva + dvb, dv, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([dqa, dqb], axis=2), dq, atol=1e-13)


# ----------------------------------------------------------------------------
# planted mistakes: each mutant of head_backward must fail a pin above
# ----------------------------------------------------------------------------

def _mutant(kind):
    def f(q_rows, k, v, vis, dout_rows):
        d = q_rows.shape[1]
        _, lse = OA.attention_rows(q_rows, k, v, vis)
        s = (q_rows @ k.T) / math.sqrt(d)
        live = vis & np.isfinite(lse)[:, None]
        p = np.where(live, np.exp(s - np.where(np.isfinite(lse), lse, 0.0)[:, None]), 0.0)
        dp = dout_rows @ v.T
        delta = (p * dp).sum(axis=1)
        ds = p * dp if kind == "no_delta" else p * (dp - delta[:, None])
        dq = (ds @ k) / math.sqrt(d)
        dk = ds.T @ q_rows if kind == "dk_no_scale" else (ds.T @ q_rows) / math.sqrt(d)
        dv = p @ dout_rows if kind == "dv_transposed" else p.T @ dout_rows
        return dq, dk, dv
    return f


@pytest.mark.parametrize("kind,check", [
    ("no_delta", lambda: test_key_gradients_sum_to_zero_and_constant_values()),
    ("dk_no_scale", lambda: test_gradients_match_finite_differences(0)),
    ("dv_transposed", lambda: test_zero_query_value_gradient_closed_form()),
])
def test_planted_backward_mistakes_are_caught(monkeypatch, kind, check):
    monkeypatch.setattr(OB, "head_backward", _mutant(kind))
    with pytest.raises(AssertionError):
        check()
