"""Seeded synthetic workloads: tensors and compact mask descriptions.

This module only draws random numbers and lays them out as the inputs of the
attention forward pass. It holds none of the method's arithmetic (no mask
expansion, no tile classification, no softmax), so both the CUDA path and the
CPU oracle can take their inputs from it.

The shapes follow the FlashMask author response ("Experiments with FlashInfer",
the A100 set-up paragraph): batch 1, 32 query heads, 8 key/value heads, head
dimension 128, bf16, and causal-document / shared-question masks whose
sub-document lengths are multiples of 64. The band kind follows the Ascend
``sparseMode`` page (sparseMode 0, preTokens / nextTokens). The block-selected
kind follows the selected-key flash attention pull request (a per-query list of
key blocks, with -1 meaning "no entry").

Column-wise bounds. For every key column j the query rows in [LTS[j], LTE[j])
and in [UTS[j], UTE[j]) are masked (half-open, start >= end means empty). A
causal document mask for a document [s, e) gives UT = [0, j) (queries before
the key) and LT = [e, N) (queries in later documents).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch

MASK_COLWISE = 0
MASK_BAND = 1
MASK_BLOCKSEL = 2

SEL_BLOCK = 64


@dataclasses.dataclass
class MaskDesc:
    """A compact mask description for a [B, Hm, Nq, Nk] attention problem."""

    kind: int
    B: int
    Hm: int
    Nq: int
    Nk: int
    lts: Optional[np.ndarray] = None  # int32 [B, Hm, Nk]
    lte: Optional[np.ndarray] = None
    uts: Optional[np.ndarray] = None
    ute: Optional[np.ndarray] = None
    pre_tokens: int = 0
    next_tokens: int = 0
    sel: Optional[np.ndarray] = None  # int32 [B, Hm, ceil(Nq/64), sel_k], -1 = no entry
    sel_block: int = SEL_BLOCK
    # Generation record (not used by any computation).
    docs: Optional[List[List[tuple]]] = None
    name: str = ""

    @property
    def sel_k(self) -> int:
        return 0 if self.sel is None else int(self.sel.shape[-1])


@dataclasses.dataclass
class SparseModeInput:
    """The inputs of an Ascend sparse mode (mode number, tokens, prefix lengths
    or cumulative sequence ends), kept as drawn. The CUDA path turns it into a
    compact description with mfa_mask_from_sparse_mode; the oracle expands the
    same numbers itself."""

    mode: int
    B: int
    Nq: int
    Nk: int
    pre_tokens: int = 0
    next_tokens: int = 0
    prefix: Optional[np.ndarray] = None  # int64 [B]
    seq_q: Optional[np.ndarray] = None   # int64 [n_seq], cumulative query ends
    seq_kv: Optional[np.ndarray] = None  # int64 [n_seq], cumulative key ends
    Hm: int = 1
    name: str = ""

    def fields(self) -> dict:
        return dict(mode=self.mode, B=self.B, Nq=self.Nq, Nk=self.Nk, pre_tokens=self.pre_tokens,
                    next_tokens=self.next_tokens, prefix=self.prefix, seq_q=self.seq_q, seq_kv=self.seq_kv)


@dataclasses.dataclass
class Problem:
    """One attention problem: q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] and its mask
    (a compact description, or the inputs of an Ascend sparse mode)."""

    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    mask: object  # MaskDesc or SparseModeInput
    seed: int

    @property
    def shape(self):
        B, Hq, N, d = self.q.shape
        return B, Hq, int(self.k.shape[1]), N, d

    @property
    def Nk(self) -> int:
        return int(self.k.shape[2])


# ----------------------------------------------------------------------------
# Document lengths
# ----------------------------------------------------------------------------

def split_blocks(rng: np.random.Generator, n_blocks: int, n_parts: int) -> List[int]:
    """Split n_blocks into n_parts positive parts by distinct uniform cut points."""
    if n_parts <= 1:
        return [n_blocks]
    cuts = np.sort(rng.choice(np.arange(1, n_blocks), size=n_parts - 1, replace=False))
    edges = np.concatenate([[0], cuts, [n_blocks]])
    return [int(x) for x in np.diff(edges)]


def doc_lengths_uniform(rng: np.random.Generator, total: int, lo_blocks: int, hi_blocks: int,
                        block: int = 64) -> List[int]:
    """Draw block * U{lo..hi} until the sum reaches ``total``; the last is cut to fit."""
    out: List[int] = []
    s = 0
    while s < total:
        L = block * int(rng.integers(lo_blocks, hi_blocks + 1))
        L = min(L, total - s)
        out.append(L)
        s += L
    return out


def docs_from_lengths(lengths: List[int]) -> List[tuple]:
    docs, s = [], 0
    for L in lengths:
        docs.append((s, s + L))
        s += L
    return docs


# ----------------------------------------------------------------------------
# Column-wise bound layouts (the description a caller hands in)
# ----------------------------------------------------------------------------

def colwise_causal_documents(B: int, N: int, docs_per_batch: List[List[tuple]], name="") -> MaskDesc:
    """Causal document mask: column j of document [s, e) masks rows [0, j) and [e, N)."""
    lts = np.zeros((B, 1, N), np.int32)
    lte = np.zeros((B, 1, N), np.int32)
    uts = np.zeros((B, 1, N), np.int32)
    ute = np.zeros((B, 1, N), np.int32)
    for b in range(B):
        for (s, e) in docs_per_batch[b]:
            j = np.arange(s, e, dtype=np.int32)
            uts[b, 0, s:e] = 0
            ute[b, 0, s:e] = j
            lts[b, 0, s:e] = e
            lte[b, 0, s:e] = N
    return MaskDesc(MASK_COLWISE, B, 1, N, N, lts, lte, uts, ute, docs=docs_per_batch, name=name)


def colwise_shared_question(B: int, N: int, q_len: int, answers_per_batch: List[List[tuple]],
                            name="") -> MaskDesc:
    """Shared-question mask.

    The question [0, q_len) is causal; answer [s, e) sees the whole question and
    itself causally; answers do not see each other. Question column j masks rows
    [0, j); answer column j masks rows [0, j) and [e, N).
    """
    lts = np.full((B, 1, N), N, np.int32)
    lte = np.full((B, 1, N), N, np.int32)
    uts = np.zeros((B, 1, N), np.int32)
    ute = np.tile(np.arange(N, dtype=np.int32), (B, 1, 1)).reshape(B, 1, N)
    for b in range(B):
        for (s, e) in answers_per_batch[b]:
            lts[b, 0, s:e] = e
            lte[b, 0, s:e] = N
    docs = [[(0, q_len)] + list(a) for a in answers_per_batch]
    return MaskDesc(MASK_COLWISE, B, 1, N, N, lts, lte, uts, ute, docs=docs, name=name)


def band(B: int, N: int, pre: int, nxt: int, Hm: int = 1, name="") -> MaskDesc:
    return MaskDesc(MASK_BAND, B, Hm, N, N, pre_tokens=int(pre), next_tokens=int(nxt), name=name)


def blocksel_topk(rng: np.random.Generator, B: int, N: int, topk: int, name="") -> MaskDesc:
    """Per 64-query block qb: keep the top min(topk, qb+1) of uniform scores over kb in [0, qb].

    The list is stored in descending score order and padded with -1. One list is
    shared by every batch element and head (Hm = 1, the same list for each b).
    """
    nqb = (N + SEL_BLOCK - 1) // SEL_BLOCK
    sel = np.full((B, 1, nqb, topk), -1, np.int32)
    one = np.full((nqb, topk), -1, np.int32)
    for qb in range(nqb):
        scores = rng.random(qb + 1)
        keep = np.argsort(-scores, kind="stable")[: min(topk, qb + 1)]
        one[qb, : len(keep)] = keep
    for b in range(B):
        sel[b, 0] = one
    return MaskDesc(MASK_BLOCKSEL, B, 1, N, N, sel=sel, name=name)


def _as_desc_arrays(m: MaskDesc) -> MaskDesc:
    for f in ("lts", "lte", "uts", "ute", "sel"):
        a = getattr(m, f)
        if a is not None:
            setattr(m, f, np.ascontiguousarray(a, dtype=np.int32))
    return m


# ----------------------------------------------------------------------------
# Tensors
# ----------------------------------------------------------------------------

def randn_qkv(seed: int, B: int, Hq: int, Hkv: int, N: int, d: int, dtype=torch.bfloat16,
              Nk: Optional[int] = None):
    Nk = N if Nk is None else Nk
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, Nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, Nk, d), generator=g, dtype=torch.float32)
    return q.to(dtype), k.to(dtype), v.to(dtype)


# ----------------------------------------------------------------------------
# The five named workloads (sizes as stated in the workload list)
# ----------------------------------------------------------------------------

WORKLOADS = {
    "tiny_doc_fp32": "B=1 Hq=Hkv=2 d=64 N=512 fp32; causal document mask, 3 documents",
    "doc8k": "B=1 Hq=32 Hkv=8 d=128 N=8192 bf16; causal document mask, lengths 64*U{4..32}",
    "shared_question8k": "B=1 Hq=32 Hkv=8 d=128 N=8192 bf16; 1024-token question + 4..8 answers",
    "band16k": "B=2 Hq=Hkv=16 d=128 N=16384 bf16; band preTokens=2048 nextTokens=0",
    "band16k_neg": "B=2 Hq=Hkv=16 d=128 N=16384 bf16; band preTokens=4096 nextTokens=-64",
    "doc32k": "B=1 Hq=32 Hkv=8 d=128 N=32768 bf16; causal document mask, 8..32 documents",
    "blocksel32k": "B=1 Hq=32 Hkv=8 d=128 N=32768 bf16; top-16 of 64-key blocks per 64-query block",
    "varlen_prefill16k": "B=1 Hq=32 Hkv=8 d=128 Nk=16384 Nq~8K bf16; sparseMode 7, packed sequences "
                         "of 64*U{8..64} keys whose second halves are the queries (rightDownCausal; the last "
                         "sequence as the band preTokens=its length, nextTokens=0)",
}

SEEDS = {
    "tiny_doc_fp32": 1000,
    "doc8k": 2000,
    "shared_question8k": 3000,
    "band16k": 4000,
    "band16k_neg": 4001,
    "doc32k": 5000,
    "blocksel32k": 5001,
    "varlen_prefill16k": 6000,
}


def make_mask(name: str, seed: Optional[int] = None, N: Optional[int] = None) -> MaskDesc:
    """The mask of a named workload; ``N`` overrides the length for scaled-down tests."""
    seed = SEEDS[name] if seed is None else seed
    rng = np.random.default_rng(seed)
    if name == "tiny_doc_fp32":
        N = 512 if N is None else N
        cuts = np.sort(rng.choice(np.arange(1, N), size=2, replace=False))
        lengths = [int(cuts[0]), int(cuts[1] - cuts[0]), int(N - cuts[1])]
        return colwise_causal_documents(1, N, [docs_from_lengths(lengths)], name)
    if name == "doc8k":
        N = 8192 if N is None else N
        lengths = doc_lengths_uniform(rng, N, 4, 32)
        return colwise_causal_documents(1, N, [docs_from_lengths(lengths)], name)
    if name == "shared_question8k":
        N = 8192 if N is None else N
        q_len = 1024 if N >= 2048 else N // 4 // 64 * 64
        n_ans = int(rng.integers(4, 9))
        parts = split_blocks(rng, (N - q_len) // 64, n_ans)
        answers, s = [], q_len
        for p in parts:
            answers.append((s, s + 64 * p))
            s += 64 * p
        return colwise_shared_question(1, N, q_len, [answers], name)
    if name == "band16k":
        N = 16384 if N is None else N
        return band(2, N, 2048, 0, name=name)
    if name == "band16k_neg":
        N = 16384 if N is None else N
        return band(2, N, 4096, -64, name=name)
    if name == "doc32k":
        N = 32768 if N is None else N
        n_docs = int(rng.integers(8, 33))
        n_docs = min(n_docs, N // 64)
        parts = split_blocks(rng, N // 64, n_docs)
        return colwise_causal_documents(1, N, [docs_from_lengths([64 * p for p in parts])], name)
    if name == "blocksel32k":
        N = 32768 if N is None else N
        return blocksel_topk(rng, 1, N, 16, name)
    if name == "varlen_prefill16k":
        return varlen_prefill(rng, 16384 if N is None else N, name)
    raise KeyError(name)


def varlen_prefill(rng: np.random.Generator, Nk: int, name: str = "") -> SparseModeInput:
    """Packed chunked prefill under sparseMode 7: sequences of 64*U{8..64} keys
    (the last cut to fit Nk); each sequence's queries are its last
    max(64, half rounded down to 64) tokens. The last sequence is the band with
    preTokens = its key length and nextTokens = 0, the page's setting for a
    split rightDownCausal sequence."""
    lk = doc_lengths_uniform(rng, Nk, 8, 64)
    lq = [max(64, (n // 2) // 64 * 64) if n >= 64 else n for n in lk]
    seq_kv = np.cumsum(lk).astype(np.int64)
    seq_q = np.cumsum(lq).astype(np.int64)
    return SparseModeInput(7, 1, int(seq_q[-1]), int(seq_kv[-1]), pre_tokens=int(lk[-1]), next_tokens=0,
                           seq_q=seq_q, seq_kv=seq_kv, name=name)


SHAPES = {
    # name: (B, Hq, Hkv, N, d, dtype)
    "tiny_doc_fp32": (1, 2, 2, 512, 64, torch.float32),
    "doc8k": (1, 32, 8, 8192, 128, torch.bfloat16),
    "shared_question8k": (1, 32, 8, 8192, 128, torch.bfloat16),
    "band16k": (2, 16, 16, 16384, 128, torch.bfloat16),
    "band16k_neg": (2, 16, 16, 16384, 128, torch.bfloat16),
    "doc32k": (1, 32, 8, 32768, 128, torch.bfloat16),
    "blocksel32k": (1, 32, 8, 32768, 128, torch.bfloat16),
    "varlen_prefill16k": (1, 32, 8, 16384, 128, torch.bfloat16),  # N = Nk; Nq from the draw
}


def make_problem(name: str, seed: Optional[int] = None, N: Optional[int] = None,
                 Hq: Optional[int] = None, Hkv: Optional[int] = None) -> Problem:
    """Tensors (seeded N(0,1), on the CPU) and mask of a named workload."""
    seed = SEEDS[name] if seed is None else seed
    B, hq, hkv, n, d, dtype = SHAPES[name]
    N = n if N is None else N
    Hq = hq if Hq is None else Hq
    Hkv = hkv if Hkv is None else Hkv
    mask = make_mask(name, seed, N)
    if isinstance(mask, SparseModeInput):
        q, k, v = randn_qkv(seed + 17, B, Hq, Hkv, mask.Nq, d, dtype, Nk=mask.Nk)
        return Problem(name, q, k, v, mask, seed)
    mask = _as_desc_arrays(mask)
    q, k, v = randn_qkv(seed + 17, B, Hq, Hkv, N, d, dtype)
    return Problem(name, q, k, v, mask, seed)


# ----------------------------------------------------------------------------
# Selected-key decode (a few query rows against a long cache)
# ----------------------------------------------------------------------------

DECODE_WORKLOADS = {
    "decode_sel64k": "B=8 Hq=32 Hkv=8 (GQA 4) d=256 Nq=1 Nk=65536 bf16; per (batch, K/V head) the top 32 of "
                     "uniform scores over the 64-key blocks (2048 selected keys)",
}
DECODE_SHAPES = {  # name: (B, Hq, Hkv, Nq, Nk, d, sel_k)
    "decode_sel64k": (8, 32, 8, 1, 65536, 256, 32),
}
DECODE_SEEDS = {"decode_sel64k": 7000}


def decode_selection(rng: np.random.Generator, B: int, Hkv: int, Nq: int, Nk: int, sel_k: int,
                     pads: int = 0, dups: int = 0) -> np.ndarray:
    """int32 [B, Hkv, Nq, sel_k]: per list the top (sel_k - pads - dups) of
    uniform scores over the 64-key blocks up to the row's position (i + Nk -
    Nq), then `dups` repeated entries and `pads` entries of -1, shuffled."""
    nblk = (Nk + 63) // 64
    out = np.full((B, Hkv, Nq, sel_k), -1, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            for i in range(Nq):
                last = i + Nk - Nq
                avail = last // 64 + 1 if last >= 0 else 0
                avail = min(avail, nblk)
                take = min(sel_k - pads - dups, avail)
                if take <= 0:
                    continue
                picks = np.argsort(rng.random(avail), kind="stable")[:take]
                row = list(picks)
                row += list(rng.choice(picks, size=min(dups, len(picks)), replace=True)) if dups else []
                row += [-1] * (sel_k - len(row))
                out[b, g, i] = rng.permutation(np.asarray(row, dtype=np.int32))
    return out


def make_decode_problem(name: str):
    """q, k, v (seeded N(0,1), bf16, on the CPU) and the selection lists of a decode workload."""
    B, Hq, Hkv, Nq, Nk, d, sel_k = DECODE_SHAPES[name]
    seed = DECODE_SEEDS[name]
    q, k, v = randn_qkv(seed + 17, B, Hq, Hkv, Nq, d, torch.bfloat16, Nk=Nk)
    sel = decode_selection(np.random.default_rng(seed), B, Hkv, Nq, Nk, sel_k)
    return q, k, v, sel


def decode_selection_sets(name: str, count: int) -> list:
    """`count` selection arrays for a decode workload: the workload's own first,
    then lists drawn the same way from further seeds. Timed steps cycle through
    them, so that the blocks a step reads were not read by the step before."""
    B, Hq, Hkv, Nq, Nk, d, sel_k = DECODE_SHAPES[name]
    seed = DECODE_SEEDS[name]
    out = [make_decode_problem(name)[3]]
    for r in range(1, count):
        out.append(decode_selection(np.random.default_rng(seed + 1000 * r), B, Hkv, Nq, Nk, sel_k))
    return out


def random_colwise(rng: np.random.Generator, B: int, Hm: int, Nq: int, Nk: int,
                   p_empty: float = 0.3) -> MaskDesc:
    """Arbitrary column bounds in [0, Nq] (empty intervals included) for stress tests."""
    def interval():
        a = rng.integers(0, Nq + 1, size=(B, Hm, Nk))
        b = rng.integers(0, Nq + 1, size=(B, Hm, Nk))
        s, e = np.minimum(a, b), np.maximum(a, b)
        empty = rng.random((B, Hm, Nk)) < p_empty
        s = np.where(empty, e, s)  # start == end: empty
        return s.astype(np.int32), e.astype(np.int32)
    lts, lte = interval()
    uts, ute = interval()
    return MaskDesc(MASK_COLWISE, B, Hm, Nq, Nk, lts, lte, uts, ute, name="random")


def random_blocksel(rng: np.random.Generator, B: int, Nq: int, Nk: int, sel_k: int,
                    p_pad: float = 0.2) -> MaskDesc:
    """Random selection lists with duplicates, -1 pads and above-diagonal entries."""
    nqb = (Nq + SEL_BLOCK - 1) // SEL_BLOCK
    nkb = (Nk + SEL_BLOCK - 1) // SEL_BLOCK
    sel = rng.integers(0, nkb, size=(B, 1, nqb, sel_k)).astype(np.int32)
    sel[rng.random(sel.shape) < p_pad] = -1
    return MaskDesc(MASK_BLOCKSEL, B, 1, Nq, Nk, sel=sel, name="random_blocksel")
