"""Work accounting for the benchmark: valid (query, key) pairs and FLOPs.

A pair (i, j) is valid when key j is visible to query i (same document,
j <= i, and within the window when the window is non-zero; the window counts
the query's own token, as FlintMagiPlan.attention's window parameter states).
The benchmark credits 4 * pairs * D * Hq FLOPs per forward: one multiply-add
per element for S = Q K^T and one for O = P V, counted once per valid pair and
query head; masked or skipped tile elements are not credited.
"""
from __future__ import annotations

import numpy as np


def valid_pairs(cu_seqlens, window: int) -> int:
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    total = 0
    for s, e in zip(cu[:-1], cu[1:]):
        pos = np.arange(int(e) - int(s), dtype=np.int64)  # position of each query in its doc
        seen = pos + 1
        if window > 0:
            seen = np.minimum(seen, window)
        total += int(seen.sum())
    return total


def forward_flops(cu_seqlens, window: int, Hq: int, D: int) -> int:
    return 4 * valid_pairs(cu_seqlens, window) * D * Hq


def row_flops(token_visible_keys: np.ndarray, D: int) -> int:
    """FLOPs credited to a set of (token, head) rows with the given visible-key counts."""
    return int(4 * np.asarray(token_visible_keys, dtype=np.int64).sum() * D)


def visible_keys(cu_seqlens, window: int, tokens: np.ndarray) -> np.ndarray:
    """Number of keys each given token sees."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    tokens = np.asarray(tokens, dtype=np.int64)
    doc = np.searchsorted(cu, tokens, side="right") - 1
    seen = tokens - cu[doc] + 1
    if window > 0:
        seen = np.minimum(seen, window)
    return seen


def algorithmic_bytes(T: int, Hq: int, Hkv: int, D: int, with_lse: bool = True) -> int:
    """Bytes a forward must move at least: Q, K, V read once, O (and LSE) written once."""
    return T * (2 * Hq * D * 2 + 2 * Hkv * D * 2 + (4 * Hq if with_lse else 0))
