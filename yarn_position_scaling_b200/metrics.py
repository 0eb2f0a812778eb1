"""Work accounting for the benchmark: algorithmic FLOPs and bytes of each path.

FLOP convention ("Arch_03_Long_Context", context-length table; "Long Context"
concept page, key math): dense attention for one head costs 4 * T^2 * d
(2 T^2 d for Q K^T and 2 T^2 d for P V).  Only visible (query, key) pairs are
counted, so a causal prefill costs 4 * d * sum_m |visible(m)| per head.

Decode moves the K and V rows of every visible cached key once per KV head:
2 (K and V) * (number of keys) * d * 2 bytes ("LLM context window mechanics",
memory wall: the cache formula; here for one layer).
"""
from __future__ import annotations

import numpy as np


def visible_counts(T: int, causal: bool = True, window: int = 0, n_sink: int = 0) -> np.ndarray:
    """|visible(m)| for every query m in [0, T): keys n <= m (causal) that are within the
    last `window` positions or among the first `n_sink` tokens."""
    m = np.arange(T, dtype=np.int64)
    if not causal:
        return np.full(T, T, dtype=np.int64)
    if window <= 0:
        return m + 1
    in_window = np.minimum(m + 1, window)
    first_in_window = np.maximum(0, m - window + 1)
    return in_window + np.minimum(n_sink, first_in_window)


def visible_pairs(T: int, causal: bool = True, window: int = 0, n_sink: int = 0) -> int:
    return int(visible_counts(T, causal, window, n_sink).sum())


def prefill_flops(B: int, Hq: int, T: int, d: int, causal: bool = True, window: int = 0,
                  n_sink: int = 0) -> float:
    return 4.0 * d * Hq * B * visible_pairs(T, causal, window, n_sink)


def decode_visible_keys(L: int, window: int = 0, n_sink: int = 0) -> int:
    """Keys the new token at position L sees (the cache slots 0..L-1 plus itself)."""
    if window <= 0:
        return L + 1
    return min(L + 1, window) + min(n_sink, max(0, L - window + 1))


def chunk_flops(B: int, Hq: int, d: int, P0: int, Tq: int, window: int = 0,
                n_sink: int = 0) -> float:
    """Causal FLOPs of a chunk of Tq queries at positions P0.. over the cached prefix and the
    chunk itself: 4 d per visible (query, key) pair per head."""
    keys = sum(decode_visible_keys(P0 + i, window, n_sink) for i in range(Tq))
    return 4.0 * d * Hq * B * keys


def decode_kv_bytes(cache_len, Hkv: int, d: int, window: int = 0, n_sink: int = 0,
                    elem_bytes: int = 2) -> float:
    keys = sum(decode_visible_keys(int(L), window, n_sink) for L in cache_len)
    return 2.0 * keys * Hkv * d * elem_bytes


def decode_flops(cache_len, Hq: int, d: int, window: int = 0, n_sink: int = 0) -> float:
    keys = sum(decode_visible_keys(int(L), window, n_sink) for L in cache_len)
    return 4.0 * keys * Hq * d
