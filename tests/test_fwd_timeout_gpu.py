"""The forward kernel's bounded waits, made to run out on purpose.

Every mbarrier wait of the bf16 forward pipeline gives up after a time limit,
after which the CTA unwinds and records MFA_DEVERR_TIMEOUT instead of hanging
(the selected-key pull request's "backend gating": decline or report, never
compute something wrong). mfa_test_arm_fwd_timeout makes the next launch
withhold one K tile, on which no copy will ever arrive, and shortens the limit:
one wait runs out, nothing faults, and the context stays usable.
"""
import time

import pytest
import torch

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W

from .gpu_util import compare_attention, oracle_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bq,bk", [(64, 128), (128, 64)])
def test_a_wait_that_runs_out_is_reported_and_the_next_call_is_exact(bq, bk):
    prob = W.make_problem("doc8k", N=1024, Hq=4, Hkv=2)
    q, k, v = (t.cuda() for t in (prob.q, prob.k, prob.v))
    att = B.Attention(prob.mask, bq, bk)
    att.build()
    out = torch.zeros_like(q)
    lse = torch.zeros(q.shape[:3], dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()

    B.arm_fwd_timeout_test(20_000)  # 20 ms
    t0 = time.perf_counter()
    att(q, k, v, out, lse)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    bits = B.device_status(att.tmap)
    assert bits & B.DEVERR_TIMEOUT, bits
    assert not bits & (B.DEVERR_BOUNDS | B.DEVERR_SEL | B.DEVERR_MAP), bits
    assert elapsed < 1.0, f"the shortened limit was not used ({elapsed:.3f} s)"

    # The same map, buffers and context: a rebuild clears the error word and
    # the forward pass is exact again.
    att.build()
    att(q, k, v, out, lse)
    assert B.device_status(att.tmap) == 0
    ref_out, ref_lse = oracle_rows(prob, None)
    compare_attention(out.float().cpu(), lse.cpu(), ref_out, ref_lse)


def test_the_hook_disarms_itself():
    prob = W.make_problem("doc8k", N=512, Hq=4, Hkv=2)
    q, k, v = (t.cuda() for t in (prob.q, prob.k, prob.v))
    att = B.Attention(prob.mask, 64, 128)
    att.build()
    B.arm_fwd_timeout_test(20_000)
    att(q, k, v)
    assert B.device_status(att.tmap) & B.DEVERR_TIMEOUT
    att.build()
    out, lse = att(q, k, v)
    assert B.device_status(att.tmap) == 0
    ref_out, ref_lse = oracle_rows(prob, None)
    compare_attention(out.float().cpu(), lse.cpu(), ref_out, ref_lse)
