"""Pins of the ALiBi bias oracle (oracle/bias.py).

* slope 0 reproduces unbiased attention bit-exactly;
* LEFT and LINEAR give the same output, lse apart by slope * i;
* q = 0 on a causal row i: lse = ln sum_{t=0..i} e^(-slope t), the
  geometric series in closed form, and out = the weighted mean of v;
* SQRT against scalar loops with math.fsum (tiny);
* a planted sign error in the linear bias fails a pin.
"""
import math

import numpy as np
import pytest

from mask_aware_block_mfa_b200 import workloads as W
from oracle import attention as OA
from oracle import bias as OB


def _qkv(rng, Hq, Hkv, N, d):
    return (rng.standard_normal((1, Hq, N, d)), rng.standard_normal((1, Hkv, N, d)),
            rng.standard_normal((1, Hkv, N, d)))


def test_zero_slope_is_plain_attention():
    rng = np.random.default_rng(0)
    q, k, v = _qkv(rng, 4, 2, 100, 8)
    m = W.make_mask("doc8k", N=100)
    for kind in (OB.LINEAR, OB.SQRT, OB.LEFT):
        a = OB.attention_bias(q, k, v, m, kind, np.zeros(4))
        b = OA.attention(q, k, v, m)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_left_and_right_alignment_differ_by_a_row_constant():
    rng = np.random.default_rng(1)
    q, k, v = _qkv(rng, 4, 2, 90, 8)
    m = W.band(1, 90, 30, 5)
    slopes = OB.alibi_slopes(4)
    o1, l1 = OB.attention_bias(q, k, v, m, OB.LINEAR, slopes)
    o2, l2 = OB.attention_bias(q, k, v, m, OB.LEFT, slopes)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    i = np.arange(90)
    for h in range(4):
        np.testing.assert_allclose(l2[0, h] - l1[0, h], slopes[h] * i, atol=1e-10)


@pytest.mark.parametrize("slope", [0.5, 0.0625, 2.0])
def test_zero_query_geometric_series(slope):
    rng = np.random.default_rng(2)
    N = 70
    q, k, v = _qkv(rng, 1, 1, N, 4)
    q[:] = 0.0
    m = W.MaskDesc(W.MASK_BAND, 1, 1, N, N, pre_tokens=N, next_tokens=0)   # causal
    out, lse = OB.attention_bias(q, k, v, m, OB.LINEAR, [slope])
    r = math.exp(-slope)
    for i in (0, 1, 17, N - 1):
        closed = math.log((1.0 - r ** (i + 1)) / (1.0 - r))
        assert math.isclose(lse[0, 0, i], closed, rel_tol=0, abs_tol=1e-12)
        w = np.array([r ** (i - j) for j in range(i + 1)])
        np.testing.assert_allclose(out[0, 0, i], (w[:, None] * v[0, 0, :i + 1]).sum(0) / w.sum(), atol=1e-12)


def test_sqrt_bias_brute_force():
    rng = np.random.default_rng(3)
    N, d = 12, 3
    q, k, v = _qkv(rng, 2, 1, N, d)
    m = W.band(1, N, 4, 2)
    slopes = [0.3, 1.1]
    out, lse = OB.attention_bias(q, k, v, m, OB.SQRT, slopes)
    for h in range(2):
        for i in range(N):
            js = [j for j in range(N) if -4 <= j - i <= 2]
            s = [sum(q[0, h, i, t] * k[0, 0, j, t] for t in range(d)) / math.sqrt(d)
                 - slopes[h] * math.sqrt(abs(i - j)) for j in js]
            z = math.fsum(math.exp(x) for x in s)
            assert math.isclose(lse[0, h, i], math.log(z), abs_tol=1e-12)
            ref = [math.fsum(math.exp(s[a]) * v[0, 0, js[a], c] for a in range(len(js))) / z for c in range(d)]
            np.testing.assert_allclose(out[0, h, i], ref, atol=1e-12)


def test_planted_sign_error_is_caught(monkeypatch):
    orig = OB.bias_rows

    def flipped(kind, slope, rows, Nk):
        return -orig(kind, slope, rows, Nk) if kind == OB.LINEAR else orig(kind, slope, rows, Nk)

    monkeypatch.setattr(OB, "bias_rows", flipped)
    with pytest.raises(AssertionError):
        test_zero_query_geometric_series(0.5)
