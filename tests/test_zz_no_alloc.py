"""The allocation-free forward entry point, against the regular one.

mfa_fwd_noalloc is for callers that cannot allocate device memory (a plugin
inside an application that owns the GPU allocator, or code that must not
allocate at that point of its pipeline): it keeps the tile map in an array the
library holds. Here it must give the same result as mfa_build_tile_map +
mfa_fwd on caller-allocated buffers, on two calls in a row (the second call
reuses the array the first one left behind). This file is collected last so
that a run stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W

from .gpu_util import compare_attention

pytestmark = pytest.mark.gpu


def _problem(mask, Hq, Hkv, d, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(mask.B, Hq, mask.Nq, d, generator=g).to(dtype).cuda()
    k = torch.randn(mask.B, Hkv, mask.Nk, d, generator=g).to(dtype).cuda()
    v = torch.randn(mask.B, Hkv, mask.Nk, d, generator=g).to(dtype).cuda()
    return q, k, v


CASES = [
    ("doc", W.make_mask("doc8k", N=2048), 8, 2, 128, 64, 128, torch.bfloat16),
    ("band_neg", W.band(1, 1500, 300, -64), 2, 2, 128, 128, 128, torch.bfloat16),
    ("blocksel", W.blocksel_topk(np.random.default_rng(4), 1, 1024, 4), 4, 2, 128, 64, 64, torch.bfloat16),
    ("tiny_fp32", W.make_mask("tiny_doc_fp32"), 2, 2, 64, 128, 64, torch.float32),
]


@pytest.mark.parametrize("name,mask,Hq,Hkv,d,bq,bk,dtype", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_regular_path_on_two_calls(name, mask, Hq, Hkv, d, bq, bk, dtype):
    q, k, v = _problem(mask, Hq, Hkv, d, seed=31, dtype=dtype)
    ref = B.Attention(mask, bq, bk)
    ref.build()
    ref_out, ref_lse = ref(q, k, v)
    assert B.device_status(ref.tmap) == 0
    dmask = B.DeviceMask(mask)
    dev_err = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
        B.fwd_noalloc(q, k, v, dmask, bq, bk, out, lse, dev_err)
        torch.cuda.synchronize()
        assert int(dev_err.item()) == 0
        compare_attention(out.float().cpu(), lse.cpu(), ref_out.double().cpu().numpy(),
                          ref_lse.double().cpu().numpy())


def test_noalloc_rejects_maps_beyond_its_array():
    # 131072 x 131072 at 64 x 64 tiles needs a 2048 x 2048 map: over 16 MiB.
    lib = B.load()
    N = 131072
    assert lib.mfa_tile_map_bytes(1, 1, N, N, 64, 64) > B.NOALLOC_SCRATCH_BYTES
    mask = W.band(1, N, 64, 0)
    desc = B.MfaMaskDesc()
    desc.kind, desc.B, desc.Hm, desc.Nq, desc.Nk = mask.kind, 1, 1, N, N
    desc.pre_tokens, desc.next_tokens = 64, 0
    fake = B.MfaTensor()
    code = lib.mfa_fwd_noalloc(fake, fake, fake, desc, 64, 64, fake, None, None, None)
    assert code == B.MFA_ERR_UNSUPPORTED


def test_noalloc_matches_the_oracle():
    """One case checked against the float64 CPU oracle directly, so this file
    stands on its own and does not rely only on the regular path's parity."""
    from oracle import attention as OA
    mask = W.make_mask("doc8k", N=1536)
    q, k, v = _problem(mask, 4, 2, 128, seed=37)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    B.fwd_noalloc(q, k, v, B.DeviceMask(mask), 64, 128, out, lse)
    torch.cuda.synchronize()
    ref_out, ref_lse = OA.attention(q.cpu(), k.cpu(), v.cpu(), mask)
    compare_attention(out.float().cpu(), lse.cpu(), ref_out, ref_lse)


def test_noalloc_reports_device_errors_through_dev_err():
    """A column bound outside [0, Nq] is found by the map build on the device
    (MFA_DEVERR_BOUNDS, no fault); the bits reach the caller's dev_err. The
    next call with a valid mask clears them, and a call with dev_err = None
    skips the copy and still computes."""
    mask = W.make_mask("tiny_doc_fp32", N=256)
    bad = W.MaskDesc(**{**mask.__dict__})
    bad.lte = mask.lte.copy()
    bad.lte[0, 0, 5] = 256 + 7
    q, k, v = _problem(mask, 4, 2, 128, seed=41)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    dev_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.fwd_noalloc(q, k, v, B.DeviceMask(bad), 64, 64, out, lse, dev_err)
    torch.cuda.synchronize()
    assert int(dev_err.item()) & B.DEVERR_BOUNDS
    B.fwd_noalloc(q, k, v, B.DeviceMask(mask), 64, 64, out, lse, dev_err)
    torch.cuda.synchronize()
    assert int(dev_err.item()) == 0
    out2 = torch.full_like(q, float("nan"))
    B.fwd_noalloc(q, k, v, B.DeviceMask(mask), 64, 64, out2, lse, None)
    torch.cuda.synchronize()
    assert torch.equal(out2, out)
