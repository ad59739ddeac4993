"""Byte accounting for the KV cache.

"The KV Cache and PagedAttention", section "800 KB a Token": a token leaves
two vectors (its key and its value) behind in each layer, so one token costs
2 x hidden x layers x bytes-per-number (OPT-13B: 2 x 5,120 x 40 x 2 = 819,200
bytes).  Section "What Came After": when groups of heads use common keys and
values, only those common sets count (hidden = kv_heads x head_dim).
"""
from __future__ import annotations

from typing import Iterable


def kv_bytes_per_token(num_kv_heads: int, head_dim: int, num_layers: int, elem_bytes: int) -> int:
    return 2 * num_kv_heads * head_dim * num_layers * elem_bytes


def decode_kv_bytes(context_lens: Iterable[int], num_kv_heads: int, head_dim: int,
                    elem_bytes: int) -> int:
    """K and V bytes that one decode step of one layer must read: every
    stored token of every text, keys and values (unfilled places excluded)."""
    return sum(int(L) for L in context_lens) * kv_bytes_per_token(num_kv_heads, head_dim, 1,
                                                                  elem_bytes)


def tokens_that_fit(cache_bytes: int, num_kv_heads: int, head_dim: int, num_layers: int,
                    elem_bytes: int) -> int:
    return cache_bytes // kv_bytes_per_token(num_kv_heads, head_dim, num_layers, elem_bytes)
