"""Seeded synthetic inputs for causal self-attention -- shared by the tests,
the benchmark and the smoke check.

This module holds no attention arithmetic: it only draws random tensors and
document layouts.  Both the CUDA path and the CPU oracle consume exactly the
bf16 values produced here (the oracle upcasts them to float64 exactly).

Workloads (head shapes of the GPT configurations the pages print):
  tiny        B=1 H=4  T=64   d=32   -- "Train Your Own LLM from Scratch" (fishgap.com),
                                        section 3: block_size=64, n_layer=4, n_head=4, n_embd=128
  gpt2_small  B=8 H=12 T=1024 d=64   -- same page, section 3: GPTConfig 12 heads, n_embd 768, block 1024
  gpt_400m    B=8 H=16 T=1024 d=64   -- "train-llm-from-scratch" (pomoai.com), core architecture:
                                        n_embed 1024, 16 heads, context 1024
  wide_d128   B=4 H=16 T=2048 d=128  -- a wider-head synthetic shape (no page prints it)
  doc_packed  B=4 H=16 T=2048 d=128  -- BOS-aligned best-fit packing, "How to build an LLM by
                                        hand" (agmtopy.github.io), section 5.5: many documents per row

Recipe: torch.Generator('cpu').manual_seed(seed); fp32 randn for Q, K, V, dO in
that order, each rounded to bf16 (round-to-nearest-even).  Document lengths for
the packed workload come from random.Random(seed): per row, randint(64, 1024)
(inclusive) repeatedly until the row is full; the last document is cut to fit T.
FP8 (e4m3) inputs of a workload: Q, K, V drawn the same way from seed + 100, times 32,
rounded to e4m3 (descale factor 1/32 each).
"""
from __future__ import annotations

import math
import random
from dataclasses import dataclass
from typing import List, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    seed: int
    doc_packed: bool = False

    @property
    def scale(self) -> float:
        """1/sqrt(d) rounded to fp32 -- the value both sides receive."""
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 64, 32, 0),
    "gpt2_small": Workload("gpt2_small", 8, 12, 1024, 64, 1),
    "gpt_400m": Workload("gpt_400m", 8, 16, 1024, 64, 2),
    "wide_d128": Workload("wide_d128", 4, 16, 2048, 128, 3),
    "doc_packed": Workload("doc_packed", 4, 16, 2048, 128, 4, doc_packed=True),
}

DOC_MIN_LEN = 64
DOC_MAX_LEN = 1024


def fp32_scale(d: int) -> float:
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))


def make_qkvdo(B: int, H: int, T: int, d: int, seed: int):
    """Q, K, V, dO as CPU bf16 tensors [B,H,T,d], drawn in that order from one generator."""
    g = torch.Generator("cpu").manual_seed(seed)
    out = []
    for _ in range(4):
        out.append(torch.randn(B, H, T, d, generator=g, dtype=torch.float32).to(torch.bfloat16))
    return tuple(out)


# FP8 (e4m3) inputs: the stored values are FP8_MULT times N(0,1) draws (max |x| ~ 6 * 32 = 192,
# inside e4m3's +-448), so each tensor's descale factor is 1 / FP8_MULT, a power of two.
FP8_MULT = 32.0
FP8_DESCALE = 1.0 / FP8_MULT


def make_qkv_e4m3(B: int, H: int, T: int, d: int, seed: int):
    """Q, K, V as CPU e4m3 codes (uint8 tensors [B,H,T,d]): fp32 randn from one generator, in
    that order, times FP8_MULT, rounded by torch's float8_e4m3fn conversion.  The real values
    are FP8_DESCALE times the codes' values."""
    g = torch.Generator("cpu").manual_seed(seed)
    out = []
    for _ in range(3):
        x = torch.randn(B, H, T, d, generator=g, dtype=torch.float32) * FP8_MULT
        out.append(x.to(torch.float8_e4m3fn).view(torch.uint8))
    return tuple(out)


def make_fp8_workload(w: Workload):
    """(q8, k8, v8, doc_start or None) for a named workload: the workload's shapes and document
    layout, its seed + 100 for the e4m3 draws."""
    q8, k8, v8 = make_qkv_e4m3(w.B, w.H, w.T, w.d, w.seed + 100)
    doc = doc_start_from_lengths(doc_lengths(w.B, w.T, w.seed), w.T) if w.doc_packed else None
    return q8, k8, v8, doc


# FP8 forward workloads (bench.py --workload fp8_<name>): the attention workloads' shapes.
FP8_WORKLOADS = {f"fp8_{name}": w for name, w in WORKLOADS.items()}


def make_decode(B: int, H: int, Tq: int, L: int, d: int, seed: int):
    """KV-cache decode inputs as CPU bf16 tensors: q [B,Tq,H,d], then the K and V caches
    [B,L,H,d], drawn in that order from one generator."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(B, Tq, H, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    kc = torch.randn(B, L, H, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn(B, L, H, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, kc, vc


# KV-cache decode workloads (bench.py --workload decode_8k): one new token per step over a
# cache of L positions, the GPT-2 / 400M head counts with a d = 128 head; the _tq variants
# append 4 or 16 tokens per step (speculative drafts).
DECODE_WORKLOADS = {
    "decode_8k": dict(B=8, H=16, Tq=1, L=8192, d=128, seed=6),
    "decode_8k_tq4": dict(B=8, H=16, Tq=4, L=8192, d=128, seed=6),
    "decode_8k_tq16": dict(B=8, H=16, Tq=16, L=8192, d=128, seed=6),
}


def make_prologue(B: int, H: int, T: int, d: int, seed: int):
    """RoPE + QK-norm inputs as CPU bf16 [B,H,T,d] tensors: q and k (projections, N(0,1)),
    then the incoming gradients dq_out and dk_out (N(0,1)), drawn in that order."""
    g = torch.Generator("cpu").manual_seed(seed)
    return tuple(torch.randn(B, H, T, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
                 for _ in range(4))


# RoPE + QK-norm prologue workloads (bench.py --workload prologue_wide_d128): the Q and K of
# the wide_d128 attention workload.
PROLOGUE_WORKLOADS = {
    "prologue_wide_d128": dict(B=4, H=16, T=2048, d=128, seed=8),
}


def doc_lengths(B: int, T: int, seed: int, lo: int = DOC_MIN_LEN, hi: int = DOC_MAX_LEN) -> List[List[int]]:
    """Per-row document lengths: uniform integers in [lo, hi] until the row holds T tokens."""
    rng = random.Random(seed)
    rows = []
    for _ in range(B):
        lens, total = [], 0
        while total < T:
            n = rng.randint(lo, hi)
            n = min(n, T - total)
            lens.append(n)
            total += n
        rows.append(lens)
    return rows


def doc_start_from_lengths(lengths: List[List[int]], T: int) -> torch.Tensor:
    """int32 [B,T]: entry [b,i] is the first position of the document that holds position i."""
    out = torch.empty(len(lengths), T, dtype=torch.int32)
    for b, lens in enumerate(lengths):
        pos = 0
        for n in lens:
            out[b, pos:pos + n] = pos
            pos += n
        if pos != T:
            raise ValueError(f"row {b}: lengths sum to {pos}, expected {T}")
    return out


def random_doc_start(B: int, T: int, seed: int, lo: int, hi: int) -> torch.Tensor:
    """Document layout with lengths uniform in [lo, hi] (for small edge-case tests)."""
    return doc_start_from_lengths(doc_lengths(B, T, seed, lo, hi), T)


def make_workload(w: Workload):
    """(q, k, v, dout, doc_start or None) for a named workload, all on the CPU."""
    q, k, v, do = make_qkvdo(w.B, w.H, w.T, w.d, w.seed)
    doc = doc_start_from_lengths(doc_lengths(w.B, w.T, w.seed), w.T) if w.doc_packed else None
    return q, k, v, do, doc


def visible_pairs(B: int, H: int, T: int, doc_start: Optional[torch.Tensor] = None) -> int:
    """Number of (query, key) pairs the mask leaves visible -- the unit of the FLOP count.

    Counting only: for each query position i, the visible keys are
    doc_start[i] .. i (or 0 .. i without documents), i.e. i - start + 1 of them.
    """
    if doc_start is None:
        return B * H * T * (T + 1) // 2
    idx = torch.arange(T, dtype=torch.int64)
    per_row = (idx.unsqueeze(0) - doc_start.to(torch.int64) + 1).sum(dim=1)
    return int(per_row.sum().item()) * H
