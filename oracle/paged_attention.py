"""CPU oracle for paged attention — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct NumPy fp64 restatement of what the paged
attention path computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  It
shares no code with the CUDA library and the library never calls it.

Sources (web pages; cited by title and section):
  [Deep Dive]  "vLLM PagedAttention Deep Dive: KV Cache Memory Fragmentation,
               Chunked Prefill & Prefix Caching" (locionic.com)
  [Block Mgr]  "PagedAttention: KV cache as virtual memory (block manager &
               fragmentation)" (inference-learning-path)
  [Static]     "PagedAttention: Why Static Batching Wastes Your KV Cache" (dev.to)

What the pages fix: a sequence's KV cache is cut into fixed-size logical
blocks; a per-sequence block table maps logical block -> physical block
([Deep Dive] "Virtual Memory Paging Analogy"); attention looks the blocks up,
gathers K/V from them and runs standard attention ([Deep Dive] "PagedAttention
Mechanism"), and the result is identical to dense attention ([Block Mgr]
"Direct answer" and "Interviewer follow-ups").  So this oracle is dense softmax
attention on the logically contiguous K/V each block table defines.

Readings where the pages are silent (the library takes the same ones):
  * cache layout ``[num_blocks][num_kv_heads][block_size][head_dim]``, K and V
    in separate pools; slot of logical position p = table[p // B] * B + p % B;
    slot -1 means "skip";
  * GQA: q head h reads kv head h // (Hq / Hkv);
  * decode appends the new token first, then attends over L + 1 tokens
    ([Block Mgr] "Deep dive", the lifecycle bullet);
  * a prefill chunk's K/V are written into the cache first; chunk query i of a
    sequence with c prior tokens sees positions 0 .. c + i inclusive
    ([Deep Dive] "Mechanics of Chunked Prefill", step 3);
  * an empty sequence gives an all-zero output row.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(closed forms, library routines on dense tensors, brute force, golden values
from the pages).  None is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "logical_positions_to_slots", "reshape_and_cache", "copy_blocks", "swap_blocks",
    "gather_logical", "attention", "paged_decode", "paged_prefill_chunk",
    "partial_attention", "combine_partials",
]


# ---------------------------------------------------------------------------
# indexing: logical position -> physical slot
# ---------------------------------------------------------------------------

def logical_positions_to_slots(block_tables, seq_ids, positions, block_size):
    """Slot of each (sequence, logical position) through its block table.

    [Deep Dive] "PagedAttention Mechanism": logical block i of a sequence lives
    in physical block ``table[i]``; a token at logical position p is in logical
    block p // B at offset p % B.  The slot encodes (physical block, offset) as
    ``physical * B + offset``.
    """
    bt = np.asarray(block_tables, dtype=np.int64)
    seq_ids = np.asarray(seq_ids, dtype=np.int64)
    positions = np.asarray(positions, dtype=np.int64)
    out = np.empty(positions.shape, dtype=np.int64)
    for t in range(positions.size):
        s, p = int(seq_ids.flat[t]), int(positions.flat[t])
        phys = int(bt[s, p // block_size])
        out.flat[t] = phys * block_size + (p % block_size)
    return out


# ---------------------------------------------------------------------------
# cache writes: bit copies
# ---------------------------------------------------------------------------

def reshape_and_cache(key_cache, value_cache, key, value, slot_mapping, block_size):
    """Write each new token's K and V rows into its slot (bit copy; in place).

    [Block Mgr] "Deep dive" (the lifecycle: decode pops one more block when the
    last one fills) and [Static] "What does PagedAttention actually do
    differently?" (blocks are filled on demand).  Arrays may be any dtype
    (callers pass uint16 views for exact bit copies).  Slot -1 skips a token.
    """
    for t in range(key.shape[0]):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        b, off = slot // block_size, slot % block_size
        key_cache[b, :, off, :] = key[t]
        value_cache[b, :, off, :] = value[t]


def copy_blocks(key_cache, value_cache, block_pairs):
    """Copy-on-write duplication: ``cache[dst] = cache[src]`` for K and V.

    [Static] "How does copy-on-write eliminate duplicate prompt KV cache?":
    on divergence the engine copies just that block and remaps the pointer.
    The copy is a bit copy of the whole physical block (all heads, slots, dims).
    """
    for src, dst in np.asarray(block_pairs, dtype=np.int64).reshape(-1, 2):
        key_cache[dst] = key_cache[src]
        value_cache[dst] = value_cache[src]


def swap_blocks(dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, block_pairs):
    """Swap: ``dst_pool[dst] = src_pool[src]`` for K and V, a bit copy between
    two pools (device and host).

    [Static] "What happens when the GPU runs out of KV blocks?": swapped-out
    blocks are copied to CPU memory and copied back when the sequence resumes.
    """
    for src, dst in np.asarray(block_pairs, dtype=np.int64).reshape(-1, 2):
        dst_key_cache[dst] = src_key_cache[src]
        dst_value_cache[dst] = src_value_cache[src]


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def gather_logical(cache, table_row, length, kv_head, block_size):
    """The logically contiguous ``[length][head_dim]`` rows one block table defines.

    [Deep Dive] "PagedAttention Mechanism", steps 1-2 (look up the physical
    blocks, gather K/V from them).
    """
    p = np.arange(int(length), dtype=np.int64)
    phys = np.asarray(table_row, dtype=np.int64)[p // block_size]
    return np.asarray(cache[phys, kv_head, p % block_size, :], dtype=np.float64)


def attention(q, K, V, scale, visible=None):
    """Standard softmax attention in fp64 for query rows ``q [M][D]``.

    o = softmax(scale * q K^T) V, the softmax taken over the visible keys with
    the row maximum subtracted ([Deep Dive] "PagedAttention Mechanism", step 3:
    standard attention).  ``visible[m]`` is the number of leading keys row m
    may see (causal masks); rows that see no key return zeros.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    M, D = q.shape
    out = np.zeros((M, V.shape[1] if V.ndim == 2 else D), dtype=np.float64)
    for m in range(M):
        n = K.shape[0] if visible is None else int(visible[m])
        if n <= 0:
            continue
        z = scale * (K[:n] @ q[m])
        w = np.exp(z - z.max())
        out[m] = (w @ V[:n]) / w.sum()
    return out


def paged_decode(query, key_cache, value_cache, block_tables, seq_lens, scale, num_kv_heads):
    """One query token per sequence over its paged K/V; fp64 ``[S][Hq][D]``.

    For sequence s and q head h: gather the first ``seq_lens[s]`` logical K/V
    rows of kv head h // G from the block table, then standard attention.
    [Deep Dive] "PagedAttention Mechanism"; output identical to dense per
    [Block Mgr] "Interviewer follow-ups".
    """
    q = np.asarray(query, dtype=np.float64)
    S, Hq, D = q.shape
    B = key_cache.shape[2]
    G = Hq // num_kv_heads
    out = np.zeros((S, Hq, D), dtype=np.float64)
    for s in range(S):
        L = int(seq_lens[s])
        for g in range(num_kv_heads):
            K = gather_logical(key_cache, block_tables[s], L, g, B)
            V = gather_logical(value_cache, block_tables[s], L, g, B)
            heads = slice(g * G, (g + 1) * G)
            out[s, heads] = attention(q[s, heads], K, V, scale)
    return out


def paged_prefill_chunk(query, key_cache, value_cache, block_tables, cu_q_lens, ctx_lens,
                        scale, num_kv_heads, seqs=None, rows=None):
    """Causal chunk attention against the paged context; fp64 ``[total_q][Hq][D]``.

    Sequence s has ``ctx_lens[s]`` prior tokens and a chunk of
    ``cu_q_lens[s+1] - cu_q_lens[s]`` queries whose K/V already sit in the
    cache at positions ``ctx_lens[s]`` onward ([Deep Dive] "Mechanics of
    Chunked Prefill", step 3: each chunk's KV accumulates in paged blocks).
    Chunk query i is at absolute position c + i and sees keys 0 .. c + i.

    ``seqs`` / ``rows`` restrict the work to some sequences / chunk rows (for
    sampled checks at full size); untouched rows stay zero.
    """
    q = np.asarray(query, dtype=np.float64)
    T, Hq, D = q.shape
    B = key_cache.shape[2]
    G = Hq // num_kv_heads
    out = np.zeros((T, Hq, D), dtype=np.float64)
    S = len(ctx_lens)
    for s in (range(S) if seqs is None else seqs):
        q0, q1 = int(cu_q_lens[s]), int(cu_q_lens[s + 1])
        c = int(ctx_lens[s])
        n = q1 - q0
        idx = np.arange(n) if rows is None else np.asarray([i for i in rows if i < n], dtype=np.int64)
        if idx.size == 0:
            continue
        L = c + int(idx.max()) + 1
        for g in range(num_kv_heads):
            K = gather_logical(key_cache, block_tables[s], L, g, B)
            V = gather_logical(value_cache, block_tables[s], L, g, B)
            for h in range(g * G, (g + 1) * G):
                out[q0 + idx, h] = attention(q[q0 + idx, h], K, V, scale, visible=c + idx + 1)
    return out


# ---------------------------------------------------------------------------
# split-KV: partial softmax states and their log-sum-exp combine
# ---------------------------------------------------------------------------

def partial_attention(q, K, V, scale):
    """Unnormalised state of attention over one key range: (m, l, acc).

    m = max_j z_j, l = sum_j exp(z_j - m), acc = sum_j exp(z_j - m) V_j with
    z = scale * K q.  An empty range gives (-inf, 0, 0).

    The pages do not split the key range; this is the standard attention of
    [Deep Dive] "PagedAttention Mechanism" kept unnormalised over one range,
    so that combine_partials can recover it exactly.
    """
    q = np.asarray(q, dtype=np.float64)
    if K.shape[0] == 0:
        return -np.inf, 0.0, np.zeros(V.shape[1], dtype=np.float64)
    z = scale * (np.asarray(K, dtype=np.float64) @ q)
    m = z.max()
    w = np.exp(z - m)
    return m, w.sum(), w @ np.asarray(V, dtype=np.float64)


def combine_partials(states):
    """Combine split-KV partial states into the normalised output.

    With M = max_p m_p: o = sum_p e^(m_p - M) acc_p / sum_p e^(m_p - M) l_p.
    This is exactly softmax attention over the union of the key ranges (the
    rescaling cancels), which the split-KV tests check against the unsplit
    result.  No keys at all gives zeros.  Cited passage: the standard
    attention of [Deep Dive] "PagedAttention Mechanism"; the combine is an
    identity of that softmax, not a step the pages describe.
    """
    ms = np.array([s[0] for s in states], dtype=np.float64)
    if ms.size == 0 or np.all(np.isneginf(ms)):
        return np.zeros_like(states[0][2]) if states else None
    M = ms.max()
    num = sum(np.exp(m - M) * acc for m, l, acc in states if not np.isneginf(m))
    den = sum(np.exp(m - M) * l for m, l, acc in states if not np.isneginf(m))
    return num / den
