"""Closed-form KV-cache arithmetic from the pages — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use
this module.  Sources are cited by page title and section:
  [Deep Dive]  "vLLM PagedAttention Deep Dive: KV Cache Memory Fragmentation,
               Chunked Prefill & Prefix Caching"
  [Block Mgr]  "PagedAttention: KV cache as virtual memory (block manager &
               fragmentation)"
  [Static]     "PagedAttention: Why Static Batching Wastes Your KV Cache"

Pinned by ``tests/test_oracle_arithmetic.py`` against the values the pages
print (``tests/golden/``).
"""
from __future__ import annotations

__all__ = [
    "kv_bytes_per_token", "blocks_needed", "tail_waste_tokens",
    "contiguous_fit", "paged_fit", "reservation_waste_fraction",
]


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, dtype_bytes: int) -> int:
    """2 (K and V) x layers x kv heads x head_dim x bytes per element.

    [Static] "Why does static KV cache allocation waste so much memory?".
    """
    return 2 * num_layers * num_kv_heads * head_dim * dtype_bytes


def blocks_needed(num_tokens: int, block_size: int) -> int:
    """Physical blocks a sequence of ``num_tokens`` occupies: the ceiling of L / B.

    [Deep Dive] "PagedAttention Mechanism" (30 tokens -> 2 blocks, 50 -> 4).
    """
    if num_tokens < 0 or block_size <= 0:
        raise ValueError("num_tokens >= 0 and block_size > 0 required")
    return (num_tokens + block_size - 1) // block_size


def tail_waste_tokens(num_tokens: int, block_size: int) -> int:
    """Unused slots in a sequence's last block; at most B - 1.

    [Static] "What does PagedAttention actually do differently?".
    """
    return blocks_needed(num_tokens, block_size) * block_size - num_tokens


def contiguous_fit(pool_blocks: int, max_len: int, block_size: int) -> int:
    """Sequences that fit when each one reserves ``max_len`` tokens up front.

    [Block Mgr] "Code": every sequence reserves ceil(MAX_LEN / BLOCK) blocks.
    """
    return pool_blocks // blocks_needed(max_len, block_size)


def paged_fit(lengths, pool_blocks: int, block_size: int, stop_at_first_miss: bool) -> int:
    """Sequences admitted when each takes only ceil(L / BLOCK) blocks.

    [Block Mgr] "Code".  The printed loop skips a sequence that does not fit
    and keeps trying later (shorter) ones; its printed comment gives the count
    of first-come-first-served admission, which stops at the first miss.
    Both readings are offered; the tests pin both.
    """
    used = admitted = 0
    for L in lengths:
        need = blocks_needed(int(L), block_size)
        if used + need <= pool_blocks:
            used += need
            admitted += 1
        elif stop_at_first_miss:
            break
    return admitted


def reservation_waste_fraction(tokens_used: int, tokens_reserved: int) -> float:
    """Share of a contiguous reservation left unused ([Static] "TL;DR")."""
    return (tokens_reserved - tokens_used) / tokens_reserved
