"""Benchmark of the mask-aware attention forward pass (one JSON line on rank 0).

A step is one pass of the whole hot path on one batch: build the tile map from
the compact mask description (three kernels), then the forward kernel. The
metric is effective TFLOP/s counting only visible (query, key) pairs, 4*d FLOPs
each, over the whole job (all ranks). Inputs are seeded N(0,1) bf16 tensors of
the named workload's shape; they are resident in HBM when timing starts, and L2
is flushed (a 256 MiB write) between timed steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload doc32k] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); each rank runs an independent
replica of the workload (the path needs no exchange), so scaling is weak and
the value is the sum of all ranks' work over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mask_aware_block_mfa_b200 import workloads as W  # noqa: E402

BLOCKS = {  # launch configuration per workload: (block_q, block_k)
    "tiny_doc_fp32": (128, 64),
    "doc8k": (64, 128),
    "shared_question8k": (64, 128),
    "band16k": (128, 128),
    "band16k_neg": (128, 128),
    "doc32k": (64, 128),
    "blocksel32k": (64, 64),
    "varlen_prefill16k": (64, 128),
}
METRIC = "effective TFLOP/s (visible pairs only) and % of B200 bf16 tensor peak"
# The default line times the largest single-GPU workload (32K tokens, causal
# documents); the two document-mask workloads that carry the >= 50 % target
# (8K and 32K) are also timed forward-only in the same run ("targets").
DEFAULT_WORKLOAD = "doc32k"
TARGET_WORKLOADS = ("doc8k", "doc32k")

# DRAM bytes (read + write) of one forward launch, from one ncu capture of
# the forward kernel on that workload (the summaries under profiles/ give the
# command). Each entry holds the digest of the kernel sources it was taken
# on; a changed kernel reports traffic as null until it is captured again.
KERNEL_SOURCES = ("mask_aware_block_mfa_b200/csrc/fwd_sm100.cu", "mask_aware_block_mfa_b200/csrc/mfa_device.cuh")
NCU_TRAFFIC = {
    # doc8k, shared_question8k, band16k and blocksel32k were captured on digest
    # 4215f15e496d475a; the forward device code is unchanged since (the shared
    # device header only gained a non-blocking barrier test that the decode
    # kernel uses), so the entries carry the current digest.
    "doc8k": (134_846_208, "a4dd79f978f9b251"),
    "shared_question8k": (135_123_456, "a4dd79f978f9b251"),
    "band16k": (520_584_192, "a4dd79f978f9b251"),
    "blocksel32k": (1_125_267_456, "a4dd79f978f9b251"),
    "doc32k": (1_027_767_040, "a4dd79f978f9b251"),
}
# The same for the gradient kernel (mfa_bwd_kernel) of the backward pass.
BWD_KERNEL_SOURCES = ("mask_aware_block_mfa_b200/csrc/bwd_sm100.cu", "mask_aware_block_mfa_b200/csrc/mfa_device.cuh",
                      "mask_aware_block_mfa_b200/csrc/order.cuh")
BWD_NCU_TRAFFIC = {
    "doc8k": (851_308_032, "542bc078d317add5"),
    "doc32k": (2_108_781_056, "542bc078d317add5"),
}


# The same for the decode kernel (mfa_decode_kernel) of --pass decode.
DEC_KERNEL_SOURCES = ("mask_aware_block_mfa_b200/csrc/decode_sm100.cu", "mask_aware_block_mfa_b200/csrc/mfa_device.cuh")
DEC_NCU_TRAFFIC = {
    "decode_sel64k": (137_655_552, "cbc2580e69c2360a"),
}


def max_over_ranks(x: float, device) -> float:
    """The largest x over the ranks of the default process group (x itself
    without one): the job's time is its slowest rank's."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: float, world: int, steps: int, max_total_ms: float) -> float:
    """Units per second of the whole job: every rank processes the same units
    per step (replicas, weak scaling), timed by the slowest rank."""
    return units_per_rank_step * world * steps / (max_total_ms * 1e-3)


def kernel_digest(sources=KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    root = os.path.dirname(os.path.abspath(__file__))
    for rel in sources:
        with open(os.path.join(root, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, table=None, sources=KERNEL_SOURCES):
    entry = (NCU_TRAFFIC if table is None else table).get(workload)
    return entry[0] if entry and entry[1] == kernel_digest(sources) else None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, "fallback"


def sparse_mode_pairs(m) -> int:
    """Visible pairs of the varlen sparse modes from the page's per-sequence
    rules: rightDownCausal (7) or leftUpCausal (8) inside each packed sequence,
    the band from the sequence's lower-right vertex for the last (7) or first
    (8) non-empty one."""
    if m.mode not in (7, 8):
        raise ValueError("bench workloads use sparse modes 7 and 8 only")
    ends_q = [0] + [int(x) for x in m.seq_q]
    ends_k = [0] + [int(x) for x in m.seq_kv]
    seqs = [(ends_q[s + 1] - ends_q[s], ends_k[s + 1] - ends_k[s]) for s in range(len(m.seq_q))]
    nonempty = [s for s, (lq, lk) in enumerate(seqs) if lq > 0 and lk > 0]
    band = (nonempty[-1] if m.mode == 7 else nonempty[0]) if nonempty else -1
    total = 0
    for s, (lq, lk) in enumerate(seqs):
        li = np.arange(lq, dtype=np.int64)
        if s == band:
            lo = np.maximum(li + (lk - lq) - int(m.pre_tokens), 0)
            hi = np.minimum(li + (lk - lq) + int(m.next_tokens), lk - 1)
        elif m.mode == 7:
            lo, hi = np.zeros_like(li), np.minimum(li + (lk - lq), lk - 1)
        else:
            lo, hi = np.zeros_like(li), np.minimum(li, lk - 1)
        total += int(np.maximum(hi - lo + 1, 0).sum())
    return total


def visible_pairs(mask) -> int:
    """Visible pairs from the description's own closed forms (host integer arithmetic)."""
    if isinstance(mask, W.SparseModeInput):
        return sparse_mode_pairs(mask)
    total = 0
    for b in range(mask.B):
        if mask.kind == W.MASK_BAND:
            pre, nxt = int(mask.pre_tokens), int(mask.next_tokens)
            i = np.arange(mask.Nq, dtype=np.int64)
            lo = np.maximum(i - pre, 0)
            hi = np.minimum(i + nxt, mask.Nk - 1)
            total += int(np.maximum(hi - lo + 1, 0).sum())
        elif mask.kind == W.MASK_BLOCKSEL:
            sel = mask.sel[b, 0]
            for qb in range(sel.shape[0]):
                r0, r1 = qb * 64, min(qb * 64 + 64, mask.Nq)
                for kb in set(int(x) for x in sel[qb] if x >= 0):
                    c0, c1 = kb * 64, min(kb * 64 + 64, mask.Nk)
                    i = np.arange(r0, r1)
                    total += int(np.clip(np.minimum(i + 1, c1) - c0, 0, None).sum())
        else:  # documents / shared question: the generator's record of the segments
            if mask.docs is None:
                raise ValueError("column-wise mask without a segment record")
            docs = mask.docs[b]
            if mask.name.startswith("shared_question"):
                q_len = docs[0][1]
                total += q_len * (q_len + 1) // 2
                for (s, e) in docs[1:]:
                    L = e - s
                    total += L * q_len + L * (L + 1) // 2
            else:
                total += sum((e - s) * (e - s + 1) // 2 for (s, e) in docs)
    return total


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""
        else:
            self.out = ""

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def oracle_mask(mask):
    """The mask as the oracle takes it (sparse-mode inputs become the oracle's own mode object)."""
    if isinstance(mask, W.SparseModeInput):
        from oracle import sparse_modes as SM
        return SM.SparseMode(**mask.fields())
    return mask


def run_reference(args, prob, pairs, d, Hq):
    """The reference arm: the float64 CPU oracle, each step a bounded sample of the workload."""
    from threadpoolctl import threadpool_info
    heads = list(range(min(args.reference_heads, Hq)))
    flops = 4.0 * d * pairs * len(heads) / (1 if prob.mask.Hm == 1 else Hq)
    omask = oracle_mask(prob.mask)
    times = []
    if args.pass_ == "bwd":
        from oracle import backward as OB
        flops *= 2.5
        dout = bwd_output_gradient(prob)
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        if args.pass_ == "bwd":
            OB.attention_backward(prob.q, prob.k, prob.v, omask, dout, heads=heads)
        else:
            oracle_forward(prob, omask, heads, args.bias, Hq)
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    sec = sum(times) / len(times)
    value = flops / sec / 1e12
    return {
        "metric": BWD_METRIC if args.pass_ == "bwd" else METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": args.workload, "pass": args.pass_, "bias": args.bias,
                   "sample": f"{len(heads)} of {Hq} query heads, all rows"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{len(heads)} of {Hq} query heads, all rows, float64 numpy"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def oracle_forward(prob, omask, heads, bias, Hq):
    """One oracle forward over the sampled heads, with the additive bias when one is named."""
    if bias == "none":
        from oracle import attention as OA
        return OA.attention(prob.q, prob.k, prob.v, omask, heads=heads)
    from oracle import bias as OBias
    kind = {"alibi": OBias.LINEAR, "alibi_sqrt": OBias.SQRT, "alibi_left": OBias.LEFT}[bias]
    return OBias.attention_bias(prob.q, prob.k, prob.v, omask, kind, OBias.alibi_slopes(Hq), heads=heads)


CPU_SAMPLE_S = 15.0  # oracle work per cpu_baseline sample


def timed_sample(run_unit, n_units: int, fixed: int = 0, budget_s: float = CPU_SAMPLE_S):
    """Run run_unit(0), run_unit(1), ... and time them: `fixed` units when it is
    positive, else as many as fit about budget_s seconds (at least one, at most
    n_units). Returns (units run, seconds)."""
    limit = min(fixed, n_units) if fixed > 0 else n_units
    done, total = 0, 0.0
    while done < limit:
        t0 = time.perf_counter()
        run_unit(done)
        total += time.perf_counter() - t0
        done += 1
        if fixed <= 0 and total + total / done > budget_s:
            break
    return done, total


def cpu_baseline(prob, pairs, d, Hq, heads_n, bias="none"):
    from threadpoolctl import threadpool_info
    omask = oracle_mask(prob.mask)
    n, sec = timed_sample(lambda h: oracle_forward(prob, omask, [h], bias, Hq), Hq, heads_n)
    heads = list(range(n))
    flops = 4.0 * d * pairs * len(heads) / (1 if prob.mask.Hm == 1 else Hq)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": flops / sec / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(heads)} of {Hq} query heads, all rows, float64 numpy ({sec:.1f} s)"}


BWD_METRIC = "effective TFLOP/s of the gradient pass (10 d FLOPs per visible pair and head)"


def bwd_output_gradient(prob):
    """Seeded N(0,1) output gradient in bf16, the shape of q."""
    g = torch.Generator(device="cpu")
    g.manual_seed(prob.seed + 29)
    return torch.randn(prob.q.shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def run_backward(args, prob, pairs, rank, world, local):
    """Gradient pass (mfa_bwd: statistics, transposed lists, gradient kernel,
    dq conversion) on a map and forward outputs computed once beforehand."""
    import torch.distributed as dist
    from mask_aware_block_mfa_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    Bsz, Hq, Hkv, N, d = prob.shape
    if prob.q.dtype != torch.bfloat16:
        raise SystemExit("the gradient pass takes bf16 workloads")
    bq = BLOCKS[args.workload][0] if BLOCKS[args.workload][1] == 128 else 64
    flops = 10.0 * d * pairs * (Hq if prob.mask.Hm == 1 else 1)
    sparse = isinstance(prob.mask, W.SparseModeInput)
    dmask = B.SparseModeMask(**prob.mask.fields(), device=dev) if sparse else B.DeviceMask(prob.mask, dev)
    att = B.Attention(dmask, bq, 128, device=dev)
    q, k, v = (t.to(dev) for t in (prob.q, prob.k, prob.v))
    dout = bwd_output_gradient(prob).to(dev)
    att.build()
    out, lse = att(q, k, v)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        att.backward(q, k, v, out, lse, dout, dq, dk, dv)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize(dev)
    if B.device_status(att.tmap, stream) != 0:
        raise RuntimeError("device error word set during warm-up")
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            step()
    stream.wait_stream(cap)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        for e0, e1 in evs:
            flush.fill_(1.0)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        time.sleep(0.2)
    if world > 1:
        dist.barrier()
    if B.device_status(att.tmap, stream) != 0:
        raise RuntimeError("device error word set during the timed steps")
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    total_ms = sum(ms)
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(flops, world, args.steps, total_ms) / 1e12
    achieved = flops / (statistics.mean(ms) * 1e-3) / 1e12
    burst, sustained, src = peaks()

    # End to end: q, k, v, out, lse, dout host -> device, gradients device -> host.
    hin = [t.pin_memory() for t in (prob.q, prob.k, prob.v, out.cpu(), lse.cpu(), dout.cpu())]
    hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]
    dins = [q, k, v, out, lse, dout]
    h2d = sum(t.nbytes for t in hin)
    d2h = sum(t.nbytes for t in hout)
    e2e_ms = []
    for s in range(args.e2e_steps + 1):
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for dst, src_t in zip(dins, hin):
            dst.copy_(src_t, non_blocking=True)
        step()
        for dst, src_t in zip(hout, (dq, dk, dv)):
            dst.copy_(src_t, non_blocking=True)
        z.record(stream)
        torch.cuda.synchronize(dev)
        if s > 0:
            e2e_ms.append(a.elapsed_time(z))
    e2e_value = flops * world / (statistics.mean(e2e_ms) * 1e-3) / 1e12
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    res = {
        "metric": BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "pass": "bwd", "desc": W.WORKLOADS[args.workload], "B": Bsz,
                   "Hq": Hq, "Hkv": Hkv, "N": N, "Nk": prob.Nk, "d": d, "block_q": 64, "block_k": 128,
                   "map_block_q": bq, "seed": prob.seed, "visible_pairs": pairs,
                   "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"replicas x{world}",
                   "launch": "each step replayed as a CUDA graph (the four mfa_bwd kernels)"},
        "frac_of_peak": {"burst": value / burst, "sustained": value / sustained, "peaks": src},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                     "frac": achieved / burst,
                     "traffic": ncu_traffic(args.workload, BWD_NCU_TRAFFIC, BWD_KERNEL_SOURCES),
                     "peak_kind": f"{src} burst bf16 dense; achieved over the whole mfa_bwd call, "
                                  "traffic of its gradient kernel"},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms": statistics.mean(e2e_ms)},
        "gpu_launches": 4 * args.steps,  # statistics, transposed lists, gradient kernel, dq conversion
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and world == 1:
        from threadpoolctl import threadpool_info
        from oracle import backward as OB
        omask, dout = oracle_mask(prob.mask), bwd_output_gradient(prob)
        n, sec = timed_sample(lambda h: OB.attention_backward(prob.q, prob.k, prob.v, omask, dout, heads=[h]),
                              Hq, args.oracle_heads)
        heads = list(range(n))
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        res["cpu_baseline"] = {"value": 10.0 * d * pairs * len(heads) / sec / 1e12, "unit": "TFLOP/s",
                               "cores": threads, "kind": "oracle",
                               "sample": f"{len(heads)} of {Hq} query heads, all rows, float64 numpy ({sec:.1f} s)"}
    print(json.dumps(res), flush=True)


DECODE_METRIC = "GB/s of the selected-key decode (visible selected K/V rows + q + out + lse + lists)"


DECODE_SETS = 6  # selection sets the timed decode steps cycle through


def decode_bytes(q, k, sel):
    """Algorithmic bytes of one decode call: every visible key of every
    deduplicated listed block, K and V, once per (batch, key/value head, row)
    (the G query heads share it), plus q, out, lse and the lists."""
    B_, Hq, Nq, d = q.shape
    Nk = int(k.shape[2])
    keys = 0
    sel3 = sel.reshape(-1, Nq, sel.shape[-1])
    for r in range(sel3.shape[0]):
        for i in range(Nq):
            last = i + Nk - Nq
            for blk in set(int(x) for x in sel3[r, i] if x >= 0):
                keys += max(0, min(64 * blk + 64, last + 1, Nk) - 64 * blk)
    elem = 2
    return keys * d * elem * 2 + 2 * B_ * Hq * Nq * d * elem + B_ * Hq * Nq * 4 + sel.size * 4


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def run_decode(args, rank, world, local):
    """Selected-key decode (mfa_decode and, with several parts per list, its
    combine kernel) on a cache resident in HBM."""
    import torch.distributed as dist
    from threadpoolctl import threadpool_info
    from mask_aware_block_mfa_b200 import binding as B
    q, k, v, sel = W.make_decode_problem(args.workload)
    B_, Hq, Hkv, Nq, Nk, d, sel_k = W.DECODE_SHAPES[args.workload]
    nbytes = decode_bytes(q, k, sel)
    if args.impl == "reference":
        if rank == 0:
            from oracle import decode as OD
            bs = list(range(min(args.reference_heads, B_)))  # a sample of the batch
            frac = len(bs) / B_
            times = []
            for st in range(args.warmup + args.steps):
                t0 = time.perf_counter()
                OD.decode_attention(q[bs], k[bs], v[bs], sel[bs])
                if st >= args.warmup:
                    times.append(time.perf_counter() - t0)
            sec = sum(times) / len(times)
            val = nbytes * frac / sec / 1e9
            threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
            print(json.dumps({
                "metric": DECODE_METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": args.workload, "pass": "decode", "sample": f"{len(bs)} of {B_} sequences"},
                "cpu_baseline": {"value": val, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                 "sample": f"{len(bs)} of {B_} sequences, float64 numpy"},
                "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
                flush=True)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    # The K/V bytes a step reads (~134 MB for decode_sel64k) exceed L2 already;
    # the timed steps also cycle through DECODE_SETS selection sets, so that a
    # step's blocks were last read DECODE_SETS - 1 steps earlier. (A write flush
    # of L2 would leave it full of dirty lines, whose write-back then lands
    # inside the next timed step.)
    sels = W.decode_selection_sets(args.workload, DECODE_SETS)
    nbytes = statistics.mean(decode_bytes(q, k, s) for s in sels)
    seld_all = [torch.from_numpy(s).to(dev) for s in sels]
    seld = seld_all[0]
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:3], dtype=torch.float32, device=dev)
    dec = B.Decode(0)
    stream = torch.cuda.current_stream(dev)

    def step(sd=None):
        dec(qd, kd, vd, seld if sd is None else sd, out, lse)

    for w in range(max(args.warmup, DECODE_SETS)):
        step(seld_all[w % DECODE_SETS])
    if dec.status() != 0:
        raise RuntimeError("device error bits set during warm-up")
    # One CUDA graph holds DECODE_SETS steps (one per selection set), as a
    # serving loop captures its decode calls together; one-step graphs cover
    # a remainder of K.
    cap = torch.cuda.Stream(dev)

    def capture(fn):
        graph = torch.cuda.CUDAGraph()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(graph, stream=cap):
                fn()
        stream.wait_stream(cap)
        return graph

    graphs = [capture(lambda sd=sd: step(sd)) for sd in seld_all]
    graph_all = capture(lambda: [step(sd) for sd in seld_all])
    for w in range(max(args.warmup, 1)):
        graph_all.replay()
    torch.cuda.synchronize(dev)
    # The K steps run back to back between two events, as a serving loop runs
    # them (no flush is needed between them: see DECODE_SETS above).
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        e0.record(stream)
        for _ in range(args.steps // DECODE_SETS):
            graph_all.replay()
        for st in range(args.steps % DECODE_SETS):
            graphs[st].replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        time.sleep(0.2)
    if world > 1:
        dist.barrier()
    if dec.status() != 0:
        raise RuntimeError("device error bits set during the timed steps")
    total_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    value = whole_job_rate(nbytes, world, args.steps, total_ms) / 1e9
    achieved = nbytes / (total_ms / args.steps * 1e-3) / 1e9
    peak, src = hbm_peak()
    # End to end: the cache stays resident (as in serving); each step copies the
    # queries and lists in and out / lse back.
    hq, hsel = q.pin_memory(), torch.from_numpy(sel).pin_memory()
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    e2e_ms = []
    for st in range(args.e2e_steps + 1):
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        qd.copy_(hq, non_blocking=True)
        seld.copy_(hsel, non_blocking=True)
        step()
        ho.copy_(out, non_blocking=True)
        hl.copy_(lse, non_blocking=True)
        z.record(stream)
        torch.cuda.synchronize(dev)
        if st > 0:
            e2e_ms.append(a.elapsed_time(z))
    e2e_value = nbytes * world / (statistics.mean(e2e_ms) * 1e-3) / 1e9
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    n_split = int(dec.ws.numel() > 256)
    res = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "pass": "decode", "desc": W.DECODE_WORKLOADS[args.workload],
                   "B": B_, "Hq": Hq, "Hkv": Hkv, "Nq": Nq, "Nk": Nk, "d": d, "sel_k": sel_k,
                   "algorithmic_bytes": nbytes,
                   "l2": f"inputs larger than L2: no flush; the steps cycle through {DECODE_SETS} seeded selection "
                         "sets, so a step's blocks were last read that many steps earlier",
                   "timing": "the K steps back to back between two CUDA events",
                   "parallelism": f"replicas x{world}",
                   "launch": f"CUDA graphs of {DECODE_SETS} steps (one per selection set), one-step graphs for a "
                             "remainder of K"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": ncu_traffic(args.workload, DEC_NCU_TRAFFIC, DEC_KERNEL_SOURCES),
                     "peak_kind": f"{src} HBM copy bandwidth; achieved over the decode call (decode + combine), "
                                  "traffic of the decode kernel"},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": hq.nbytes + hsel.nbytes,
                "d2h_bytes_per_step": ho.nbytes + hl.nbytes, "ms": statistics.mean(e2e_ms),
                "note": "cache resident in HBM; queries and lists copied in, out and lse copied back"},
        "gpu_launches": (2 if n_split else 1) * args.steps,  # decode kernel (+ combine when the lists are split)
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and world == 1:
        from oracle import decode as OD
        n, sec = timed_sample(lambda b: OD.decode_attention(q[b:b + 1], k[b:b + 1], v[b:b + 1], sel[b:b + 1]), B_,
                              args.oracle_heads)
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        res["cpu_baseline"] = {"value": nbytes * n / B_ / sec / 1e9, "unit": "GB/s", "cores": threads,
                               "kind": "oracle",
                               "sample": f"{n} of {B_} sequences, float64 numpy ({sec:.1f} s)"}
    print(json.dumps(res), flush=True)


def time_target(name: str, dev, stream, flush, steps: int, warmup: int) -> dict:
    """Forward-only and map + forward times of a target workload (CUDA graphs,
    L2 flushed between replays), with its effective TFLOP/s and fraction of
    the measured burst bf16 peak."""
    from mask_aware_block_mfa_b200 import binding as B
    prob = W.make_problem(name)
    _, Hq, _, _, d = prob.shape
    flops = 4.0 * d * visible_pairs(prob.mask) * (Hq if prob.mask.Hm == 1 else 1)
    bq, bk = BLOCKS[name]
    q, k, v = (t.to(dev) for t in (prob.q, prob.k, prob.v))
    att = B.Attention(B.DeviceMask(prob.mask, dev), bq, bk, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    for _ in range(warmup):
        att.build()
        att(q, k, v, out, lse)
    torch.cuda.synchronize(dev)
    g_step, g_fwd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g_step, stream=cap):
            att.build()
            att(q, k, v, out, lse)
        with torch.cuda.graph(g_fwd, stream=cap):
            att(q, k, v, out, lse)
    stream.wait_stream(cap)
    for _ in range(warmup):
        g_step.replay()
        g_fwd.replay()
    times = {}
    for key, graph in (("step", g_step), ("fwd", g_fwd)):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e0, e1 in evs:
            flush.fill_(1.0)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        times[key] = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs)
    if B.device_status(att.tmap, stream) != 0:
        raise RuntimeError(f"device error word set while timing {name}")
    burst, _, src = peaks()
    tf = flops / (times["fwd"] * 1e-3) / 1e12
    return {"fwd_ms": times["fwd"], "fwd_tflops": tf, "frac": tf / burst, "step_ms": times["step"],
            "step_tflops": flops / (times["step"] * 1e-3) / 1e12, "peak": burst, "peaks": src}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=sorted(BLOCKS) + sorted(W.DECODE_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--oracle-heads", type=int, default=0,
                    help="units (query heads; sequences for decode) in the CPU-baseline sample; "
                         "0 = as many as fit about 15 s")
    ap.add_argument("--reference-heads", type=int, default=1, help="query heads per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the forward-only timing of the 8K and 32K document-mask workloads")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--bias", default="none", choices=["none", "alibi", "alibi_sqrt", "alibi_left"],
                    help="additive ALiBi bias in the forward pass (slopes 2^(-8h/Hq))")
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd", "decode"],
                    help="fwd: tile map + forward (the headline); bwd: the gradient pass alone; "
                         "decode: selected-key decode (decode workloads)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.bias != "none" and args.pass_ != "fwd":
        raise SystemExit("--bias applies to the forward pass only")
    if args.pass_ == "decode":
        args.workload = args.workload or "decode_sel64k"
        if args.workload not in W.DECODE_WORKLOADS:
            raise SystemExit("--pass decode takes a decode workload")
        return run_decode(args, rank, world, local)
    args.workload = args.workload or DEFAULT_WORKLOAD
    if args.workload not in BLOCKS:
        raise SystemExit("decode workloads run with --pass decode")

    prob = W.make_problem(args.workload)
    Bsz, Hq, Hkv, N, d = prob.shape
    pairs = visible_pairs(prob.mask)
    flops = 4.0 * d * pairs * (Hq if prob.mask.Hm == 1 else 1)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, prob, pairs, d, Hq)), flush=True)
        return
    if args.pass_ == "bwd":
        return run_backward(args, prob, pairs, rank, world, local)

    import torch.distributed as dist
    from mask_aware_block_mfa_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    bq, bk = BLOCKS[args.workload]
    q, k, v = (t.to(dev) for t in (prob.q, prob.k, prob.v))
    sparse = isinstance(prob.mask, W.SparseModeInput)

    def device_mask(stream=None):
        """Mask arrays host -> device (and, for a sparse mode, its conversion kernel)."""
        if sparse:
            return B.SparseModeMask(**prob.mask.fields(), device=dev, stream=stream)
        return B.DeviceMask(prob.mask, dev)

    att = B.Attention(device_mask(), bq, bk, device=dev)
    bias = None
    if args.bias != "none":
        kind = {"alibi": B.BIAS_ALIBI, "alibi_sqrt": B.BIAS_ALIBI_SQRT, "alibi_left": B.BIAS_ALIBI_LEFT}[args.bias]
        slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / Hq) for h in range(Hq)], dtype=torch.float32, device=dev)
        bias = (kind, slopes)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if sparse:
            att.dmask.convert()
        att.build()
        att(q, k, v, out, lse, bias=bias)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize(dev)
    if B.device_status(att.tmap, stream) != 0:
        raise RuntimeError("device error word set during warm-up")

    # One step (map build + forward) and the forward alone, captured as CUDA
    # graphs so the timed region measures device work, not host launch latency.
    g_step, g_fwd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g_step, stream=cap):
            step()
        with torch.cuda.graph(g_fwd, stream=cap):
            att(q, k, v, out, lse, bias=bias)
    stream.wait_stream(cap)
    for _ in range(args.warmup):
        g_step.replay()
        g_fwd.replay()
    torch.cuda.synchronize(dev)

    def timed(graph):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for e0, e1 in evs:
            flush.fill_(1.0)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        return evs

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        ev_step = timed(g_step)
        ev_fwd = timed(g_fwd)
        torch.cuda.synchronize(dev)
        time.sleep(0.2)
    if world > 1:
        dist.barrier()
    if B.device_status(att.tmap, stream) != 0:
        raise RuntimeError("device error word set during the timed steps")
    step_ms = [e0.elapsed_time(e1) for (e0, e1) in ev_step]
    fwd_ms = [e0.elapsed_time(e1) for (e0, e1) in ev_fwd]
    total_ms = sum(step_ms)
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(flops, world, args.steps, total_ms) / 1e12
    fwd_avg_ms = sum(fwd_ms) / len(fwd_ms)
    achieved = flops / (fwd_avg_ms * 1e-3) / 1e12
    burst, sustained, src = peaks()

    # End to end through the binding: pinned host inputs -> device -> map + forward -> host outputs.
    hq, hk, hv = (t.pin_memory() for t in (prob.q, prob.k, prob.v))
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    mask_fields = ("prefix", "seq_q", "seq_kv") if sparse else ("lts", "lte", "uts", "ute", "sel")
    mask_bytes = sum(getattr(prob.mask, f).nbytes for f in mask_fields if getattr(prob.mask, f) is not None)
    h2d = hq.nbytes + hk.nbytes + hv.nbytes + mask_bytes
    d2h = ho.nbytes + hl.nbytes
    e2e_ms = []
    for s in range(args.e2e_steps + 1):  # the first pass is a warm-up
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        att_e = att
        att_e.dmask = device_mask(stream)
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        att_e.build(stream)
        att_e(q, k, v, out, lse, stream, bias=bias)
        ho.copy_(out, non_blocking=True)
        hl.copy_(lse, non_blocking=True)
        z.record(stream)
        torch.cuda.synchronize(dev)
        if s > 0:
            e2e_ms.append(a.elapsed_time(z))
    e2e_value = flops * world / (statistics.mean(e2e_ms) * 1e-3) / 1e12

    # The target workloads' forward-only figures (the main workload's from the
    # timing above, the other's timed here), on every rank alike.
    targets = {}
    if not args.no_targets and args.bias == "none":
        for name in TARGET_WORKLOADS:
            if name == args.workload:
                burst_t, _, src_t = peaks()
                targets[name] = {"fwd_ms": fwd_avg_ms, "fwd_tflops": achieved, "frac": achieved / burst_t,
                                 "step_ms": ms_per_step, "step_tflops": flops / (ms_per_step * 1e-3) / 1e12,
                                 "peak": burst_t, "peaks": src_t}
            else:
                targets[name] = time_target(name, dev, stream, flush, args.steps, args.warmup)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    res = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "desc": W.WORKLOADS[args.workload], "B": Bsz, "Hq": Hq, "Hkv": Hkv,
                   "N": N, "Nk": prob.Nk, "d": d, "block_q": bq, "block_k": bk, "bias": args.bias, "seed": prob.seed, "visible_pairs": pairs,
                   "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"replicas x{world}",
                   "launch": "each step replayed as a CUDA graph (" + ("sparse-mode conversion + " if sparse else "")
                             + "map build + forward)"},
        "frac_of_peak": {"burst": value / burst, "sustained": value / sustained, "spec_2250": value / 2250.0,
                         "peaks": src},
        "fwd_only": {"ms": fwd_avg_ms, "tflops": achieved},
        "map_ms": ms_per_step - fwd_avg_ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                     "frac": achieved / burst,
                     # counters were taken on the bias-free instantiation only
                     "traffic": ncu_traffic(args.workload) if args.bias == "none" else None,
                     "peak_kind": f"{src} burst bf16 dense"},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms": statistics.mean(e2e_ms)},
        # per step: 2 tile-map kernels + 1 forward kernel (+1 sparse-mode conversion kernel)
        "gpu_launches": (4 if sparse and prob.mask.mode >= 5 else 3) * args.steps,
        "clocks": clk.summary(),
    }
    if targets:
        res["targets"] = targets
    if not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(prob, pairs, d, Hq, args.oracle_heads, args.bias)
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
