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
    dec_digest = bench.kernel_digest(bench.DEC_KERNEL_SOURCES)
    for name, (nbytes, dig) in bench.DEC_NCU_TRAFFIC.items():
        assert nbytes > 0 and len(dig) == 16
        assert bench.ncu_traffic(name, bench.DEC_NCU_TRAFFIC, bench.DEC_KERNEL_SOURCES) == \
            (nbytes if dig == dec_digest else None)
    bwd_digest = bench.kernel_digest(bench.BWD_KERNEL_SOURCES)
    assert bwd_digest != digest
    for name, (nbytes, dig) in bench.BWD_NCU_TRAFFIC.items():
        assert nbytes > 0 and len(dig) == 16
        got = bench.ncu_traffic(name, bench.BWD_NCU_TRAFFIC, bench.BWD_KERNEL_SOURCES)
        assert got == (nbytes if dig == bwd_digest else None)


@pytest.mark.parametrize("N", [2048, 5000, None])
def test_varlen_prefill_pairs_match_the_oracle_modes(N):
    from oracle import sparse_modes as SM
    m = W.make_mask("varlen_prefill16k", N=N)
    assert m.Nq < m.Nk and m.seq_kv[-1] == m.Nk and m.seq_q[-1] == m.Nq
    ref = SM.SparseMode(**m.fields())
    assert bench.visible_pairs(m) == int(SM.visible_dense(ref).sum())
    # the band of the last sequence (pre = its key length, next = 0) equals its rightDownCausal triangle
    diag = W.SparseModeInput(**{**m.fields(), "pre_tokens": 0, "next_tokens": 0})
    lk = int(m.seq_kv[-1] - (m.seq_kv[-2] if len(m.seq_kv) > 1 else 0))
    assert m.pre_tokens == lk
    assert bench.visible_pairs(m) == bench.visible_pairs(W.SparseModeInput(**{**m.fields(), "pre_tokens": lk + 999}))
    assert bench.visible_pairs(diag) < bench.visible_pairs(m)


def test_varlen_prefill_problem_is_rectangular():
    p = W.make_problem("varlen_prefill16k", N=2048, Hq=4, Hkv=2)
    assert p.q.shape[2] == p.mask.Nq and p.k.shape[2] == p.v.shape[2] == p.mask.Nk == 2048


def test_decode_bytes_count_the_oracle_visibility():
    import torch
    from oracle import decode as OD
    rng = np.random.default_rng(9)
    sel = W.decode_selection(rng, 2, 2, 3, 1000, 8, pads=2, dups=2)
    q = torch.zeros(2, 8, 3, 128, dtype=torch.bfloat16)
    k = torch.zeros(2, 2, 1000, 128, dtype=torch.bfloat16)
    keys = sum(int(OD.visible_dense(sel, b, g, 3, 1000).sum()) for b in range(2) for g in range(2))
    expect = keys * 128 * 2 * 2 + 2 * q.numel() * 2 + 2 * 8 * 3 * 4 + sel.size * 4
    assert bench.decode_bytes(q, k, sel) == expect


def test_cpu_sample_sizing(monkeypatch):
    """timed_sample: a fixed count when asked, else units until the next would
    pass the budget (at least one, at most all)."""
    import bench
    clock = [0.0]
    monkeypatch.setattr(bench.time, "perf_counter", lambda: clock[0])

    def unit(cost):
        def run(_):
            clock[0] += cost
        return run

    assert bench.timed_sample(unit(1.0), 32, fixed=4) == (4, 4.0)
    assert bench.timed_sample(unit(1.0), 3, fixed=10) == (3, 3.0)
    assert bench.timed_sample(unit(4.0), 32, budget_s=15.0) == (3, 12.0)   # a fourth would reach 16 s
    assert bench.timed_sample(unit(40.0), 32, budget_s=15.0) == (1, 40.0)  # one unit even above the budget
    assert bench.timed_sample(unit(0.1), 5, budget_s=15.0)[0] == 5         # never more than all units
