"""Seeded synthetic workloads: tensors and the four mask boundary vectors.

This module only draws inputs.  It holds none of the attention, tile
classification or localisation arithmetic, imports neither the CUDA binding
nor the oracle, and serves both of them (and the benchmark).

Mask families are the ones listed in "FlashMask-3 targets masked distributed
attention on Hopper GPUs", section "In-depth insight" (document, prefix-LM,
share-question, sliding-window, block-sparse), written in the column-wise
encoding: for key column j, query row i is masked iff
LTS[j] <= i < LTE[j] or UTS[j] <= i < UTE[j].

Recipe (all seeds derive from one config seed s):
  q ~ N(0,1) from torch.Generator(s), k from s+1, v from s+2, dO from s+3,
  drawn in fp32 on the CPU and rounded to bf16; integer draws (document
  lengths, dropped tiles) from numpy.random.default_rng(s+4), inclusive ranges.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    mask: str
    seed: int
    chunks: int = 0  # number of equal query chunks for the localisation check (0 = none)
    description: str = ""


# The five workloads: a tiny causal-document case, 8K causal documents with
# GQA, 32K share-question, 64K prefix-LM + sliding window, 128K causal
# documents with 30 % block-sparse key-column dropout.
CONFIGS: Dict[str, Workload] = {
    "tiny_doc": Workload("tiny_doc", 1, 2, 2, 256, 64, "tiny_doc", 1000,
                         description="3 causal documents, seqlen 256, 2 heads, d64"),
    "doc8k": Workload("doc8k", 1, 32, 8, 8192, 128, "doc8k", 1001,
                      description="causal documents U[256,4096], seqlen 8192, 32q/8kv heads, d128"),
    "sharequestion32k": Workload("sharequestion32k", 1, 16, 16, 32768, 128, "share_question", 1002,
                                 description="8 x (question + 4 answers), seqlen 32768, 16 heads, d128"),
    "prefixwindow64k": Workload("prefixwindow64k", 2, 16, 16, 65536, 128, "prefix_window", 1003,
                                description="2048-token bidirectional prefix + causal 4096 window, "
                                            "seqlen 65536, batch 2, 16 heads, d128"),
    "docblocksparse128k": Workload("docblocksparse128k", 1, 32, 8, 131072, 128, "doc_blocksparse", 1004, chunks=4,
                                   description="causal documents U[1024,32768] + 30% 128-key tile dropout, "
                                               "seqlen 131072, 32q/8kv heads, d128"),
}
CONFIG_ORDER = ["tiny_doc", "doc8k", "sharequestion32k", "prefixwindow64k", "docblocksparse128k"]


# ----------------------------------------------------------------------------
# boundary-vector encodings of the mask families
# ----------------------------------------------------------------------------
def empty_vectors(n: int) -> List[np.ndarray]:
    """All four vectors zero: every interval empty (no masking)."""
    return [np.zeros(n, np.int32) for _ in range(4)]


def causal_vectors(n: int) -> List[np.ndarray]:
    """Causal: key j is hidden from rows i < j (upper interval [0, j))."""
    lts = np.full(n, n, np.int32)
    lte = np.full(n, n, np.int32)
    uts = np.zeros(n, np.int32)
    ute = np.arange(n, dtype=np.int32)
    return [lts, lte, uts, ute]


def doc_lengths_uniform(rng: np.random.Generator, n: int, lo: int, hi: int) -> List[int]:
    """Document lengths uniform in [lo, hi] until n is filled; the last one is truncated."""
    out, total = [], 0
    while total < n:
        L = int(rng.integers(lo, hi, endpoint=True))
        L = min(L, n - total)
        out.append(L)
        total += L
    return out


def causal_document_vectors(lengths: List[int]) -> List[np.ndarray]:
    """Causal documents: key j in document [s, e) is visible to rows j..e-1.

    LTS = e, LTE = n (rows of later documents), UTS = 0, UTE = j (causal).
    """
    n = int(sum(lengths))
    lts = np.empty(n, np.int32)
    s = 0
    for L in lengths:
        lts[s:s + L] = s + L
        s += L
    lte = np.full(n, n, np.int32)
    uts = np.zeros(n, np.int32)
    ute = np.arange(n, dtype=np.int32)
    return [lts, lte, uts, ute]


def share_question_lengths(rng: np.random.Generator, n: int, segments: int = 8, answers: int = 4,
                           q_range=(1024, 4096), a_range=(256, 1024)) -> List[List[int]]:
    """Per segment [question, answer_1..answer_k] lengths, rescaled to sum to n.

    The raw draws are rescaled proportionally (floor) and the remainder goes
    to the very last answer, so that the segments fill exactly n tokens.
    """
    raw = []
    for _ in range(segments):
        seg = [int(rng.integers(q_range[0], q_range[1], endpoint=True))]
        seg += [int(rng.integers(a_range[0], a_range[1], endpoint=True)) for _ in range(answers)]
        raw.append(seg)
    total = sum(sum(s) for s in raw)
    scaled = [[max(1, (x * n) // total) for x in s] for s in raw]
    rem = n - sum(sum(s) for s in scaled)
    scaled[-1][-1] += rem
    assert sum(sum(s) for s in scaled) == n and scaled[-1][-1] > 0
    return scaled


def share_question_vectors(segs: List[List[int]]) -> List[np.ndarray]:
    """Share-question: answers see their question and themselves (causally), not siblings.

    All keys: UTS = 0, UTE = j (causal).  A question key of a segment ending
    at E: LTS = E.  An answer key of an answer ending at ae: LTS = ae (rows of
    later sibling answers and later segments).  LTE = n.
    """
    n = int(sum(sum(s) for s in segs))
    lts = np.empty(n, np.int32)
    pos = 0
    for seg in segs:
        seg_end = pos + sum(seg)
        qlen = seg[0]
        lts[pos:pos + qlen] = seg_end
        p = pos + qlen
        for alen in seg[1:]:
            lts[p:p + alen] = p + alen
            p += alen
        pos = seg_end
    lte = np.full(n, n, np.int32)
    uts = np.zeros(n, np.int32)
    ute = np.arange(n, dtype=np.int32)
    return [lts, lte, uts, ute]


def prefix_window_vectors(n: int, prefix: int, window: int) -> List[np.ndarray]:
    """Bidirectional prefix + causal sliding window.

    Prefix keys (j < prefix): no upper interval (visible to earlier rows).
    Other keys: UTS = 0, UTE = j (causal).  Every key: LTS = min(j + window, n),
    LTE = n (rows at distance >= window no longer see it).
    """
    j = np.arange(n, dtype=np.int64)
    lts = np.minimum(j + window, n).astype(np.int32)
    lte = np.full(n, n, np.int32)
    uts = np.zeros(n, np.int32)
    ute = np.where(j < prefix, 0, j).astype(np.int32)
    return [lts, lte, uts, ute]


def drop_key_tiles(vecs: List[np.ndarray], rng: np.random.Generator, p: float, tile: int = 128) -> List[np.ndarray]:
    """Block-sparse key-column dropout: each `tile`-key block is hidden from all rows with prob p."""
    lts, lte, uts, ute = [x.copy() for x in vecs]
    n = lts.size
    ntiles = -(-n // tile)
    drop = rng.random(ntiles) < p
    for t in np.nonzero(drop)[0]:
        lts[t * tile:(t + 1) * tile] = 0
        lte[t * tile:(t + 1) * tile] = n
    return [lts, lte, uts, ute]


def random_interval_vectors(rng: np.random.Generator, nq: int, nk: int, p_empty: float = 0.2) -> List[np.ndarray]:
    """Unstructured masks for tests: each key gets two random (possibly empty or inverted) intervals."""
    out = []
    for _ in range(2):
        a = rng.integers(-2, nq + 3, size=nk)
        b = rng.integers(-2, nq + 3, size=nk)
        lo, hi = np.minimum(a, b), np.maximum(a, b)
        empty = rng.random(nk) < p_empty
        hi = np.where(empty, lo, hi)
        inverted = rng.random(nk) < 0.05
        lo, hi = np.where(inverted, hi, lo), np.where(inverted, lo, hi)
        out += [lo.astype(np.int32), hi.astype(np.int32)]
    return out


def mask_vectors(w: Workload) -> List[np.ndarray]:
    """The four [B, 1, N] int32 vectors of a workload."""
    rng = np.random.default_rng(w.seed + 4)
    n = w.N
    if w.mask == "tiny_doc":
        cuts = sorted(int(x) for x in rng.choice(np.arange(1, n), size=2, replace=False))
        lengths = [cuts[0], cuts[1] - cuts[0], n - cuts[1]]
        v = causal_document_vectors(lengths)
    elif w.mask == "doc8k":
        v = causal_document_vectors(doc_lengths_uniform(rng, n, 256, 4096))
    elif w.mask == "share_question":
        v = share_question_vectors(share_question_lengths(rng, n))
    elif w.mask == "prefix_window":
        v = prefix_window_vectors(n, 2048, 4096)
    elif w.mask == "doc_blocksparse":
        v = causal_document_vectors(doc_lengths_uniform(rng, n, 1024, 32768))
        v = drop_key_tiles(v, rng, 0.30, 128)
    else:
        raise ValueError(w.mask)
    return [np.repeat(x[None, None, :], w.B, axis=0).astype(np.int32) for x in v]


def randn_bf16(shape, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_inputs(w: Workload, with_grad: bool = True) -> Dict[str, torch.Tensor]:
    """CPU tensors of a workload: q, k, v (and dO) bf16 + the four int32 mask vectors."""
    out = {
        "q": randn_bf16((w.B, w.N, w.Hq, w.d), w.seed),
        "k": randn_bf16((w.B, w.N, w.Hkv, w.d), w.seed + 1),
        "v": randn_bf16((w.B, w.N, w.Hkv, w.d), w.seed + 2),
    }
    if with_grad:
        out["do"] = randn_bf16((w.B, w.N, w.Hq, w.d), w.seed + 3)
    for name, x in zip(("lts", "lte", "uts", "ute"), mask_vectors(w)):
        out[name] = torch.from_numpy(x)
    return out


def sample_rows(w: Workload, n: int, seed: int) -> List[Tuple[int, int, int]]:
    """Seeded (b, h, i) query rows for sampled checks at full size."""
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(0, w.B)), int(rng.integers(0, w.Hq)), int(rng.integers(0, w.N))) for _ in range(n)]


def sample_cols(w: Workload, n: int, seed: int) -> List[Tuple[int, int, int]]:
    """Seeded (b, hkv, j) key columns for sampled checks at full size."""
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(0, w.B)), int(rng.integers(0, w.Hkv)), int(rng.integers(0, w.N))) for _ in range(n)]
