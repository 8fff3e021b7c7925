"""Forward pass with an additive ALiBi bias on the GPU (mfa_fwd_bias) against
oracle/bias.py, every element, with the forward pass's tolerances: the three
bias kinds over column-wise, band (with rows that see nothing) and block
selection masks, at the tile shapes the bench uses."""
import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W
from oracle import bias as OBias

from .gpu_util import compare_attention

pytestmark = pytest.mark.gpu

KINDS = [(B.BIAS_ALIBI, OBias.LINEAR), (B.BIAS_ALIBI_SQRT, OBias.SQRT), (B.BIAS_ALIBI_LEFT, OBias.LEFT)]
MASKS = [
    ("doc", lambda: W.make_mask("doc8k", N=1000), (64, 128)),
    ("band_neg", lambda: W.band(1, 900, 200, -64), (128, 128)),
    ("blocksel", lambda: W.make_mask("blocksel32k", N=1024), (64, 64)),
    ("shared_q", lambda: W.make_mask("shared_question8k", N=1024), (128, 64)),
]


@pytest.mark.parametrize("mk", MASKS, ids=lambda m: m[0])
@pytest.mark.parametrize("kind", KINDS, ids=["linear", "sqrt", "left"])
def test_bias_matches_oracle(mk, kind):
    name, factory, (bq, bk) = mk
    mask = factory()
    Hq, Hkv = 4, 2
    g = torch.Generator().manual_seed(21)
    q = torch.randn(mask.B, Hq, mask.Nq, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(mask.B, Hkv, mask.Nk, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(mask.B, Hkv, mask.Nk, 128, generator=g).to(torch.bfloat16)
    slopes = OBias.alibi_slopes(Hq)
    att = B.Attention(mask, bq, bk)
    att.build()
    out, lse = att(q.cuda(), k.cuda(), v.cuda(),
                   bias=(kind[0], torch.tensor(slopes, dtype=torch.float32, device="cuda")))
    assert B.device_status(att.tmap) == 0
    ref_out, ref_lse = OBias.attention_bias(q, k, v, mask, kind[1], slopes)
    compare_attention(out.float().cpu(), lse.cpu(), ref_out, ref_lse)


def test_zero_slopes_match_the_plain_forward():
    mask = W.make_mask("doc8k", N=700)
    g = torch.Generator().manual_seed(22)
    q = torch.randn(1, 4, 700, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1, 2, 700, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1, 2, 700, 128, generator=g).to(torch.bfloat16).cuda()
    att = B.Attention(mask, 64, 128)
    att.build()
    o0, l0 = att(q, k, v)
    o1, l1 = att(q, k, v, bias=(B.BIAS_ALIBI, torch.zeros(4, dtype=torch.float32, device="cuda")))
    assert float((o0.float() - o1.float()).abs().max()) <= 1e-2
    assert float((l0 - l1).abs().max()) <= 1e-5


@pytest.mark.parametrize("kind", KINDS[:2], ids=["linear", "sqrt"])
def test_bias_full_size_sampled(kind):
    """doc32k (the bench's 64 x 128 tiles, 32 heads) with the bench's slopes
    2^(-8h/32): sampled rows of a few heads against the oracle."""
    import bench
    from .gpu_util import sample_rows
    prob = W.make_problem("doc32k")
    Bsz, Hq, Hkv, N, d = prob.shape
    bq, bk = bench.BLOCKS["doc32k"]
    slopes = OBias.alibi_slopes(Hq)
    att = B.Attention(prob.mask, bq, bk)
    att.build()
    out, lse = att(prob.q.cuda(), prob.k.cuda(), prob.v.cuda(),
                   bias=(kind[0], torch.tensor(slopes, dtype=torch.float32, device="cuda")))
    assert B.device_status(att.tmap) == 0
    rows = sample_rows(N, 48, np.random.default_rng(24))
    heads = [0, 7, 31]
    ref_out, ref_lse = OBias.attention_bias(prob.q, prob.k, prob.v, prob.mask, kind[1], slopes, rows=rows, heads=heads)
    compare_attention(out.float().cpu()[:, heads][:, :, rows], lse.cpu()[:, heads][:, :, rows], ref_out, ref_lse)
