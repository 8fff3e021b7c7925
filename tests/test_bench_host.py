"""Host-side pieces of bench.py: the visible-pair counts behind the metric."""
import numpy as np
import pytest

import bench
from mask_aware_block_mfa_b200 import workloads as W
from oracle import masks as OM


@pytest.mark.parametrize("name,N", [("tiny_doc_fp32", None), ("doc8k", 2048), ("shared_question8k", 2048),
                                    ("band16k", 3000), ("band16k_neg", 3000), ("doc32k", 4096),
                                    ("blocksel32k", 2048)])
def test_visible_pairs_match_oracle_expansion(name, N):
    m = W.make_mask(name, N=N)
    assert bench.visible_pairs(m) == sum(OM.visible_pairs(m, b) for b in range(m.B))


def test_full_size_counts_are_plausible():
    m = W.make_mask("doc8k")
    frac = bench.visible_pairs(m) / 8192 ** 2
    assert 0.02 < frac < 0.2
    m = W.make_mask("band16k")
    assert bench.visible_pairs(m) == 2 * sum(min(i, 2048) + 1 for i in range(16384))


def test_ncu_traffic_follows_the_kernel_digest():
    import bench
    digest = bench.kernel_digest()
    assert len(digest) == 16 and int(digest, 16) >= 0
    assert bench.ncu_traffic("no-such-workload") is None
    for name, (nbytes, dig) in bench.NCU_TRAFFIC.items():
        assert nbytes > 0 and len(dig) == 16
        assert bench.ncu_traffic(name) == (nbytes if dig == digest else None)
