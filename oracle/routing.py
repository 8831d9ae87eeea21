"""Routing bookkeeping: per-expert counts, padded segments, stable permutation.

Test infrastructure only (see the package docstring).

Pages: sitech.ge "Grouped experts instead of a Python loop" (GroupedLinear
gathers the tokens of every expert and takes the per-expert token counts as
``split_sizes``); andresseo.expert "Fragmented Expert Kernels" (uneven counts
must not force a loop).  Readings:

* slot s = t*k + j (token t, its j-th expert) goes to expert topk_idx[t, j];
  a token that picks the same expert twice contributes two slots.
* split_sizes[e] = number of slots routed to e; they sum to T*k.
* expert e owns the padded segment [poffsets[e], poffsets[e] + P_e) of the
  permuted row space, P_e = split_sizes[e] rounded up to ``align`` rows
  (the library uses 128); the first split_sizes[e] rows hold its slots in
  increasing slot order (a stable counting sort), the rest are padding.
* sorted_to_src[row] = slot held by that row, -1 for padding rows;
  src_to_sorted[slot] = its row.
"""
from __future__ import annotations

import numpy as np


def route(topk_idx: np.ndarray, E: int, align: int = 128, capacity: int | None = None):
    topk_idx = np.asarray(topk_idx)
    flat = topk_idx.reshape(-1).astype(np.int64)
    Tk = flat.size
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert index out of range")
    split = np.zeros(E, dtype=np.int64)
    for e in flat:                      # plain histogram
        split[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    poffsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + split[e]
        padded = (split[e] + align - 1) // align * align
        poffsets[e + 1] = poffsets[e] + padded
    if capacity is None:
        capacity = int(poffsets[E])
    sorted_to_src = np.full(capacity, -1, dtype=np.int64)
    src_to_sorted = np.zeros(Tk, dtype=np.int64)
    fill = poffsets[:E].copy()
    for s in range(Tk):                 # stable: slots visited in increasing order
        e = flat[s]
        sorted_to_src[fill[e]] = s
        src_to_sorted[s] = fill[e]
        fill[e] += 1
    return dict(split_sizes=split, offsets=offsets, poffsets=poffsets,
                sorted_to_src=sorted_to_src, src_to_sorted=src_to_sorted)


def capacity_rows(T: int, k: int, E: int, align: int = 128) -> int:
    """Upper bound on the padded row count for any routing: T*k + E*(align-1), rounded to align."""
    n = T * k + E * (align - 1)
    return (n + align - 1) // align * align


def permute_rows(x: np.ndarray, sorted_to_src: np.ndarray, k: int) -> np.ndarray:
    """Row r of the result is x[sorted_to_src[r] // k], or zeros for padding rows."""
    out = np.zeros((sorted_to_src.size,) + x.shape[1:], dtype=x.dtype)
    for r, s in enumerate(sorted_to_src):
        if s >= 0:
            out[r] = x[s // k]
    return out


def permute_probs(topk_prob: np.ndarray, sorted_to_src: np.ndarray) -> np.ndarray:
    """Routing probability of each permuted row (0 for padding rows)."""
    flat = np.asarray(topk_prob).reshape(-1)
    return np.array([flat[s] if s >= 0 else 0.0 for s in sorted_to_src], dtype=np.float32)
