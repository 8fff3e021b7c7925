"""Helpers shared by the GPU parity tests (device runs vs the CPU oracle)."""
import math

import numpy as np
import torch

from mask_aware_block_mfa_b200 import binding as B
from oracle import attention as OA
from oracle import tilemap as OT

# Tolerances of the bf16 forward pass against the float64 oracle.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def run_gpu(prob, block_q, block_k, stream=None):
    """Map + forward on cuda:0 for a workloads.Problem; returns (out, lse, map arrays, err)."""
    att = B.Attention(prob.mask, block_q, block_k)
    att.build(stream)
    q, k, v = (t.to("cuda") for t in (prob.q, prob.k, prob.v))
    out, lse = att(q, k, v, stream=stream)
    err = B.device_status(att.tmap, stream)
    arrays = {key: val.cpu().numpy() for key, val in att.tmap.arrays().items()}
    return out.float().cpu(), lse.cpu(), arrays, err


def compare_map(arrays, mask, block_q, block_k):
    ref = OT.tile_map(mask, block_q, block_k)
    for key in ("kminmax", "tile_class", "tile_list", "tile_count", "order"):
        got = arrays[key]
        exp = ref[key].reshape(got.shape)
        if not np.array_equal(got, exp.astype(got.dtype)):
            bad = np.argwhere(got != exp)
            raise AssertionError(f"{key}: {len(bad)} mismatches, first {bad[:5].tolist()}")


def compare_attention(out, lse, ref_out, ref_lse):
    """Element-wise parity on the rows given; empty rows must be exactly (0, -inf)."""
    out = out.double().numpy() if isinstance(out, torch.Tensor) else out
    lse = lse.double().numpy() if isinstance(lse, torch.Tensor) else lse
    empty = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), empty), "rows with no visible key differ"
    assert (out[empty] == 0).all(), "empty rows must output 0"
    diff = np.abs(out - ref_out)
    assert np.isfinite(out).all()
    max_abs, mean_abs = float(diff.max()) if diff.size else 0.0, float(diff.mean()) if diff.size else 0.0
    assert max_abs <= MAX_ABS, f"max abs error {max_abs}"
    assert mean_abs <= MEAN_ABS, f"mean abs error {mean_abs}"
    fin = ~empty
    if fin.any():
        lerr = float(np.abs(lse[fin] - ref_lse[fin]).max())
        assert lerr <= LSE_ABS, f"lse error {lerr}"
    return max_abs, mean_abs


def sample_rows(N, count, rng):
    """Row sample: the first and last rows, tile edges and uniform picks."""
    edges = [0, 1, 63, 64, 127, 128, N - 1, N - 2]
    rows = set(x for x in edges if 0 <= x < N)
    rows.update(int(x) for x in rng.choice(N, size=min(count, N), replace=False))
    return np.array(sorted(rows))


def visible_flops(mask, Hq, d):
    from oracle import masks as OM
    total = 0
    for b in range(mask.B):
        for hm in range(mask.Hm):
            total += OM.visible_pairs(mask, b, hm)
    per_head = Hq if mask.Hm == 1 else 1
    return 4.0 * d * total * per_head


def oracle_rows(prob, rows, heads=None):
    return OA.attention(prob.q, prob.k, prob.v, prob.mask, rows=rows, heads=heads)


__all__ = ["run_gpu", "compare_map", "compare_attention", "sample_rows", "oracle_rows", "visible_flops",
           "math"]
