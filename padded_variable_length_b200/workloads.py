"""Seeded synthetic workloads for padded variable-length attention.

This module only draws inputs: sequence lengths, document layouts, element
masks and bf16 Q/K/V/dO tensors.  It holds none of the attention arithmetic
(no bias, no sigmoid, no softmax), so both the CUDA path and the CPU oracle can
take their inputs from it without sharing any of the method.

The workloads stand in for the single-cell RNA-seq batches of "Better Models,
Faster Training: Sigmoid Attention for single-cell Foundation Models"
(section 1, problem statement: cells carry hundreds to thousands of expressed
genes and are padded to the longest cell of the batch) and for the packed-document
masks of "Binary Block Masking for FlashAttention" (section "Applications":
packed fine-tuning).  No dataset is read; shapes, length mixes and mask
structure are reproduced from seeds.

Layout of every activation tensor: ``[B, N, H, d]`` bf16, d contiguous.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

TILE = 128

SIGMOID, SOFTMAX, SOFTMAX1 = 0, 1, 2
EPILOGUE_NAMES = {SIGMOID: "sigmoid", SOFTMAX: "softmax", SOFTMAX1: "softmax1"}


@dataclasses.dataclass
class Workload:
    """One synthetic batch.

    ``counts`` is the per-query-row integer n that the bias b = -log(n) refers
    to: the valid length of the row's sequence, or the length of the row's
    document for packed-document masks.  It is 0 on pad rows.  Turning it into
    a bias is the caller's business (the oracle and the CUDA library each do it
    on their own side).
    """

    name: str
    B: int
    Nq: int
    Nk: int
    H: int
    d: int
    lengths: Optional[np.ndarray]      # int32 [B] for padded batches, else None
    mask: Optional[np.ndarray]         # uint8 [B, Nq, Nk] element mask, else None
    counts: np.ndarray                 # int32 [B, Nq]
    epilogue: int
    backward: bool
    seed: int
    doc_lengths: Optional[list] = None  # per batch row: list of document lengths

    def pairs(self) -> int:
        """Number of unmasked (query, key) pairs, summed over the batch."""
        if self.lengths is not None:
            return int(np.sum(self.lengths.astype(np.int64) ** 2))
        if self.doc_lengths is not None:
            return int(sum(l * (l + 1) // 2 for row in self.doc_lengths for l in row))
        return int(self.mask.astype(np.int64).sum())

    def valid_tokens(self) -> int:
        if self.lengths is not None:
            return int(self.lengths.sum())
        return int(self.B * self.Nq)


def lengths_counts(lengths: np.ndarray, npad: int) -> np.ndarray:
    """Per-row integer n: the sequence's valid length on valid rows, 0 on pad rows."""
    B = lengths.shape[0]
    idx = np.arange(npad)[None, :]
    return np.where(idx < lengths[:, None], lengths[:, None], 0).astype(np.int32).reshape(B, npad)


def padded_workload(name, lengths, H, d, epilogue=SIGMOID, backward=True, seed=0, npad=None):
    lengths = np.asarray(lengths, dtype=np.int32)
    if npad is None:
        npad = int(lengths.max()) if lengths.size else 0
    return Workload(name=name, B=int(lengths.shape[0]), Nq=npad, Nk=npad, H=H, d=d,
                    lengths=lengths, mask=None, counts=lengths_counts(lengths, npad),
                    epilogue=epilogue, backward=backward, seed=seed)


def packed_documents(rng: np.random.Generator, n: int, mean_len: int) -> list:
    """Document lengths ~ Geometric(p = 1/mean_len) (support >= 1), drawn until
    they cover n tokens; the last document is cut to fit."""
    out, total = [], 0
    while total < n:
        l = int(rng.geometric(1.0 / mean_len))
        l = min(l, n - total)
        out.append(l)
        total += l
    return out


def causal_document_mask(doc_lengths: list, n: int) -> tuple:
    """Element mask of one packed row: token i sees token j iff both lie in the
    same document and j <= i.  Returns (mask uint8 [n, n], per-row doc length)."""
    doc_id = np.repeat(np.arange(len(doc_lengths)), doc_lengths)
    dl = np.repeat(np.asarray(doc_lengths, dtype=np.int32), doc_lengths)
    same = doc_id[:, None] == doc_id[None, :]
    causal = np.arange(n)[None, :] <= np.arange(n)[:, None]
    return (same & causal).astype(np.uint8), dl.astype(np.int32)


def masked_workload(name, mask, counts, H, d, epilogue=SIGMOID, backward=True, seed=0,
                    doc_lengths=None):
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    B, Nq, Nk = mask.shape
    return Workload(name=name, B=B, Nq=Nq, Nk=Nk, H=H, d=d, lengths=None, mask=mask,
                    counts=np.asarray(counts, dtype=np.int32).reshape(B, Nq),
                    epilogue=epilogue, backward=backward, seed=seed, doc_lengths=doc_lengths)


# --------------------------------------------------------------------------------------
# The five workloads on which the method is measured.
# --------------------------------------------------------------------------------------

def config(idx: int, seed: Optional[int] = None, epilogue: int = SIGMOID) -> Workload:
    """Workload ``idx`` in 1..5 (default seed 1000 + idx).

    1  tiny: lengths {37, 64, 100, 128} padded to 128, H=2, d=64, forward only.
    2  single-cell: B=32, n = floor(exp(U[ln 200, ln 2049))) clipped to [200, 2048],
       H=8, d=64, forward + backward.
    3  long ragged: B=8, n ~ U{4096..16384}, H=16, d=128, forward + backward.
    4  packed documents: B=4 rows of 8192 tokens, documents ~ Geometric(mean 512),
       causal within a document, H=16, d=128, forward + backward.
    5  as 2 (same seed offset as 2, so same lengths and data) for the epilogue switch.
    """
    if seed is None:
        seed = 1000 + (2 if idx == 5 else idx)
    rng = np.random.default_rng(seed)
    if idx == 1:
        return padded_workload("tiny", [37, 64, 100, 128], H=2, d=64, epilogue=epilogue,
                               backward=False, seed=seed, npad=128)
    if idx in (2, 5):
        n = np.floor(np.exp(rng.uniform(math.log(200), math.log(2049), 32))).astype(np.int64)
        n = np.clip(n, 200, 2048)
        return padded_workload("single_cell" if idx == 2 else "epilogues", n, H=8, d=64,
                               epilogue=epilogue, backward=True, seed=seed)
    if idx == 3:
        n = rng.integers(4096, 16385, 8)
        return padded_workload("long_ragged", n, H=16, d=128, epilogue=epilogue,
                               backward=True, seed=seed)
    if idx == 4:
        N, B = 8192, 4
        masks, counts, docs = [], [], []
        for _ in range(B):
            dls = packed_documents(rng, N, 512)
            m, c = causal_document_mask(dls, N)
            masks.append(m)
            counts.append(c)
            docs.append(dls)
        return masked_workload("packed_docs", np.stack(masks), np.stack(counts), H=16, d=128,
                               epilogue=epilogue, backward=True, seed=seed, doc_lengths=docs)
    raise ValueError(f"no workload {idx}")


def longformer_mask(n: int, radius: int, n_global: int) -> np.ndarray:
    """Longformer-style element mask of one row of n tokens: token i sees token j iff
    |i - j| <= radius (a sliding window) or either of them is one of the first n_global
    tokens (global tokens see everything and are seen by everything)."""
    i = np.arange(n)
    local = np.abs(i[:, None] - i[None, :]) <= radius
    glob = (i[:, None] < n_global) | (i[None, :] < n_global)
    return (local | glob).astype(np.uint8)


def tree_parents(rng: np.random.Generator, nodes: int, max_children: int = 4) -> np.ndarray:
    """A random token tree of `nodes` nodes in breadth-first order: parent[0] = -1 (the root)
    and every later node hangs under an earlier node that has fewer than max_children
    children, picked uniformly -- the shape of the candidate trees that parallel decoding
    verifies in one pass."""
    parent = np.full(nodes, -1, dtype=np.int64)
    children = np.zeros(nodes, dtype=np.int64)
    for k in range(1, nodes):
        open_nodes = np.flatnonzero(children[:k] < max_children)
        pk = int(rng.choice(open_nodes))
        parent[k] = pk
        children[pk] += 1
    return parent


def tree_mask(prefix: int, parent: np.ndarray) -> np.ndarray:
    """Element mask of a causal prefix followed by a token tree: prefix token i sees the
    prefix tokens j <= i; tree node k (token prefix + k) sees the whole prefix and the tree
    nodes on its path to the root (itself included), nothing else."""
    nodes = parent.shape[0]
    n = prefix + nodes
    m = np.zeros((n, n), dtype=np.uint8)
    m[:prefix, :prefix] = np.tril(np.ones((prefix, prefix), dtype=np.uint8))
    m[prefix:, :prefix] = 1
    for k in range(nodes):
        a = k
        while a >= 0:
            m[prefix + k, prefix + a] = 1
            a = int(parent[a])
    return m


def mask_family(kind: str, seed: Optional[int] = None, epilogue: int = SIGMOID, B: int = 4,
                H: int = 16, d: int = 128) -> Workload:
    """The other block-mask families through the element-mask planner ("Binary Block
    Masking", section on applications: tree attention masks, packed fine-tuning, Longformer
    masks); synthetic shapes, the n of b = -log n being each query's number of keys.

    longformer  B rows of N = 8192 tokens, sliding window of radius 256, 32 global tokens
    tree        B rows of N = 4096 tokens: a causal prefix of 3840 and a random token tree of
                256 nodes (at most 4 children per node)
    packed      B rows of N = 8192 tokens of causal documents (the packed-documents workload)
    """
    if kind == "packed":
        return config(4, seed=seed, epilogue=epilogue)
    if seed is None:
        seed = 2000 + {"longformer": 1, "tree": 2}[kind]
    rng = np.random.default_rng(seed)
    masks = []
    for _ in range(B):
        if kind == "longformer":
            masks.append(longformer_mask(8192, 256, 32))
        elif kind == "tree":
            masks.append(tree_mask(3840, tree_parents(rng, 256)))
        else:
            raise ValueError(kind)
    m = np.stack(masks)
    counts = m.sum(axis=2, dtype=np.int64).astype(np.int32)
    return masked_workload(kind, m, counts, H=H, d=d, epilogue=epilogue, backward=True, seed=seed)


CONFIG_IDS = (1, 2, 3, 4, 5)


def tensors(w: Workload, with_grad: Optional[bool] = None) -> dict:
    """bf16 CPU tensors Q, K, V (and dO) ~ N(0, 1), from seed w.seed + 1.

    Pad positions get N(0, 1) values too, so that the kernels' masking is
    exercised rather than hidden by zero padding."""
    if with_grad is None:
        with_grad = w.backward
    g = torch.Generator().manual_seed(w.seed + 1)
    out = {}
    out["q"] = torch.randn(w.B, w.Nq, w.H, w.d, generator=g).to(torch.bfloat16)
    out["k"] = torch.randn(w.B, w.Nk, w.H, w.d, generator=g).to(torch.bfloat16)
    out["v"] = torch.randn(w.B, w.Nk, w.H, w.d, generator=g).to(torch.bfloat16)
    if with_grad:
        out["do"] = torch.randn(w.B, w.Nq, w.H, w.d, generator=g).to(torch.bfloat16)
    return out


def random_mask(rng: np.random.Generator, B: int, Nq: int, Nk: int, density: float,
                empty_rows: int = 0, block_structure: bool = True) -> np.ndarray:
    """An element mask with a mix of empty, full and partial 128x128 blocks, plus a
    few rows that see no key at all (degenerate rows)."""
    m = (rng.random((B, Nq, Nk)) < density)
    if block_structure:
        qt, kt = -(-Nq // TILE), -(-Nk // TILE)
        kind = rng.integers(0, 3, (B, qt, kt))  # 0 empty, 1 full, 2 random
        for b in range(B):
            for i in range(qt):
                for j in range(kt):
                    sl = (b, slice(i * TILE, (i + 1) * TILE), slice(j * TILE, (j + 1) * TILE))
                    if kind[b, i, j] == 0:
                        m[sl] = False
                    elif kind[b, i, j] == 1:
                        m[sl] = True
    for b in range(B):
        if empty_rows:
            rows = rng.choice(Nq, size=min(empty_rows, Nq), replace=False)
            m[b, rows, :] = False
    return m.astype(np.uint8)
