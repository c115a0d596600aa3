"""Seeded synthetic inputs for the paged-attention workloads.

This module only draws numbers and lays out a block pool: sequence lengths,
a shuffled assignment of physical blocks to sequences, and N(0,1) query/key/
value data cast to fp16 or bf16.  It holds none of the attention arithmetic,
no slot computation and no kernel logic, so that both the CPU oracle
(``oracle/``) and the CUDA library can be fed from it without sharing code.

Everything is drawn on the CPU from ``torch.Generator('cpu')`` seeded with the
workload's seed, in a fixed order (lengths, physical permutation, data), so the
oracle and the GPU see identical bits.

Workload shapes follow the pages' examples:
  * the "PagedAttention Mechanism" worked block table (a 30-token and a
    50-token sequence, 16-token blocks) of "vLLM PagedAttention Deep Dive";
  * the Llama-2-13B shape (40 layers, 40 KV heads, head_dim 128, fp16) of
    "PagedAttention: Why Static Batching Wastes Your KV Cache", section
    "Why does static KV cache allocation waste so much memory?";
  * the 800-token shared system prompt of the same page, section
    "How does copy-on-write eliminate duplicate prompt KV cache?";
  * chunked prefill of "vLLM PagedAttention Deep Dive", section
    "Mechanics of Chunked Prefill".
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = [
    "PagedDecodeInputs", "PrefillChunkInputs", "WORKLOADS", "make_workload",
    "tiny_decode", "llama2_13b_decode", "llama3_8b_gqa_decode",
    "shared_prefix_cow", "long_context_decode", "chunked_prefill", "random_decode",
    "llama3_8b_gqa_decode_fp8", "NAN_FILL", "FP8_NAN_CODE",
]

NAN_FILL = float("nan")


@dataclasses.dataclass
class PagedDecodeInputs:
    """One batch of decode queries over a paged K/V pool (CPU tensors).

    key_cache / value_cache: ``dtype[num_blocks][num_kv_heads][block_size][head_dim]``.
    block_tables: ``int32[num_seqs][max_blocks_per_seq]``; entries past a
    sequence's allocation hold -1.
    context_lens: tokens already resident before this step.
    new_key / new_value: one appended token per sequence (or None), written at
    logical position ``context_lens[s]`` before attention runs.
    free_blocks: physical blocks referenced by no table (filled with NaN).
    """
    name: str
    seed: int
    dtype: torch.dtype
    block_size: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int
    context_lens: torch.Tensor
    block_tables: torch.Tensor
    key_cache: torch.Tensor
    value_cache: torch.Tensor
    query: torch.Tensor
    new_key: Optional[torch.Tensor]
    new_value: Optional[torch.Tensor]
    free_blocks: torch.Tensor
    scale: float
    # FP8 caches only: the per-cache scale (codes stand for value * scale);
    # None for fp16 / bf16 caches
    kv_scale: Optional[float] = None
    # copy-on-write workload only: the shared physical blocks and, per
    # sequence, a fresh destination block for the diverging block
    shared_blocks: Optional[torch.Tensor] = None
    cow_logical_block: Optional[int] = None
    cow_dst_blocks: Optional[torch.Tensor] = None

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.numel())

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])


@dataclasses.dataclass
class PrefillChunkInputs:
    """Causal prefill chunks of several sequences against their paged prior context.

    query: ``dtype[total_q][num_q_heads][head_dim]`` (chunks packed, ``cu_q_lens``
    gives the offsets).  new_key / new_value: ``dtype[total_q][num_kv_heads][head_dim]``,
    the chunk tokens' own K/V, written to logical positions
    ``ctx_lens[s] .. ctx_lens[s] + q_len[s] - 1`` before attention runs.
    """
    name: str
    seed: int
    dtype: torch.dtype
    block_size: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int
    ctx_lens: torch.Tensor
    cu_q_lens: torch.Tensor
    block_tables: torch.Tensor
    key_cache: torch.Tensor
    value_cache: torch.Tensor
    query: torch.Tensor
    new_key: torch.Tensor
    new_value: torch.Tensor
    free_blocks: torch.Tensor
    scale: float
    num_decode: int = 0  # leading sequences that are decode rows (one query each)

    @property
    def num_seqs(self) -> int:
        return int(self.ctx_lens.numel())

    @property
    def total_q(self) -> int:
        return int(self.query.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _randn(gen: torch.Generator, shape, dtype: torch.dtype, chunk: int = 1 << 24) -> torch.Tensor:
    """N(0,1) in fp32, cast to ``dtype``; drawn in chunks to bound fp32 memory."""
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    n = flat.numel()
    for i in range(0, n, chunk):
        j = min(n, i + chunk)
        flat[i:j] = torch.randn(j - i, generator=gen, dtype=torch.float32).to(dtype)
    return out


def _pool(gen, num_blocks, num_kv_heads, block_size, head_dim, dtype, used_blocks,
          fp8_scale=None):
    shape = (num_blocks, num_kv_heads, block_size, head_dim)
    if fp8_scale is None:
        kc = _randn(gen, shape, dtype)
        vc = _randn(gen, shape, dtype)
    else:
        # FP8 E4M3 codes of N(0,1) / scale, drawn through torch's float8 cast
        kc = _fp8_codes(gen, shape, fp8_scale)
        vc = _fp8_codes(gen, shape, fp8_scale)
    used = torch.zeros(num_blocks, dtype=torch.bool)
    used[used_blocks] = True
    free = torch.nonzero(~used).flatten()
    if fp8_scale is None:
        kc[free] = NAN_FILL
        vc[free] = NAN_FILL
    else:
        kc[free] = FP8_NAN_CODE
        vc[free] = FP8_NAN_CODE
    return kc, vc, free


FP8_NAN_CODE = 0x7F


def _fp8_codes(gen, shape, scale, chunk: int = 1 << 24) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.uint8)
    flat = out.view(-1)
    n = flat.numel()
    for i in range(0, n, chunk):
        j = min(n, i + chunk)
        x = torch.randn(j - i, generator=gen, dtype=torch.float32) / scale
        flat[i:j] = x.to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def _tables_from_counts(perm: torch.Tensor, counts, max_blocks: int, start: int = 0):
    """Hand out physical blocks from ``perm`` in order; pad with -1."""
    bt = torch.full((len(counts), max_blocks), -1, dtype=torch.int32)
    pos = start
    for s, n in enumerate(counts):
        bt[s, :n] = perm[pos:pos + n].to(torch.int32)
        pos += n
    return bt, pos


def _decode_batch(name, seed, gen, lens, *, dtype, block_size, hq, hkv, d, append,
                  pool_factor=1.25, pool_blocks=None, fp8_scale=None):
    lens = [int(x) for x in lens]
    counts = [_ceil_div(L + (1 if append else 0), block_size) for L in lens]
    need = sum(counts)
    num_blocks = pool_blocks if pool_blocks is not None else int(math.ceil(pool_factor * need))
    perm = torch.randperm(num_blocks, generator=gen)
    bt, used = _tables_from_counts(perm, counts, max(1, max(counts)))
    kc, vc, free = _pool(gen, num_blocks, hkv, block_size, d, dtype, perm[:used], fp8_scale)
    q = _randn(gen, (len(lens), hq, d), dtype)
    nk = _randn(gen, (len(lens), hkv, d), dtype) if append else None
    nv = _randn(gen, (len(lens), hkv, d), dtype) if append else None
    return PagedDecodeInputs(
        name=name, seed=seed, dtype=dtype, block_size=block_size, num_q_heads=hq,
        num_kv_heads=hkv, head_dim=d, num_blocks=num_blocks,
        context_lens=torch.tensor(lens, dtype=torch.int32), block_tables=bt,
        key_cache=kc, value_cache=vc, query=q, new_key=nk, new_value=nv,
        free_blocks=free, scale=1.0 / math.sqrt(d), kv_scale=fp8_scale)


def tiny_decode(seed: int = 0) -> PagedDecodeInputs:
    """4 sequences of {30, 50, 17, 64} tokens, 4 q = 4 kv heads, head_dim 64, fp16,
    16-token blocks in a 64-block pool, one appended token per sequence."""
    gen = torch.Generator().manual_seed(seed)
    return _decode_batch("tiny_decode_4x{30,50,17,64}_h4_d64_fp16", seed, gen, [30, 50, 17, 64],
                         dtype=torch.float16, block_size=16, hq=4, hkv=4, d=64, append=True,
                         pool_blocks=64)


def llama2_13b_decode(seed: int = 1, num_seqs: int = 64) -> PagedDecodeInputs:
    """Llama-2-13B-shaped single-layer decode: 40/40 heads, head_dim 128, fp16,
    16-token blocks, lengths uniform in [16, 2048], pool 1.25x the blocks needed."""
    gen = torch.Generator().manual_seed(seed)
    lens = torch.randint(16, 2048 + 1, (num_seqs,), generator=gen).tolist()
    return _decode_batch(f"llama2_13b_decode_{num_seqs}seq_L16-2048_h40_d128_fp16", seed, gen, lens,
                         dtype=torch.float16, block_size=16, hq=40, hkv=40, d=128, append=False)


def llama3_8b_gqa_decode(seed: int = 2, num_seqs: int = 256, block_size: int = 16) -> PagedDecodeInputs:
    """Llama-3-8B-shaped GQA decode: 32 q / 8 kv heads, head_dim 128, bf16,
    lengths uniform in [128, 4096], one appended token per sequence."""
    gen = torch.Generator().manual_seed(seed)
    lens = torch.randint(128, 4096 + 1, (num_seqs,), generator=gen).tolist()
    return _decode_batch(f"llama3_8b_gqa_decode_{num_seqs}seq_L128-4096_h32kv8_d128_bf16_B{block_size}",
                         seed, gen, lens, dtype=torch.bfloat16, block_size=block_size,
                         hq=32, hkv=8, d=128, append=True)


def shared_prefix_cow(seed: int = 3, num_seqs: int = 128) -> PagedDecodeInputs:
    """128 sequences whose tables all start with the same 50 physical blocks
    (an 800-token shared prompt), each followed by a private suffix of 1..512
    tokens.  Each sequence also gets one fresh destination block for the
    copy-on-write of its last shared block (logical block 49)."""
    gen = torch.Generator().manual_seed(seed)
    block_size, hq, hkv, d, dtype = 16, 32, 8, 128, torch.bfloat16
    prefix_blocks = 50
    suffix = torch.randint(1, 512 + 1, (num_seqs,), generator=gen).tolist()
    suffix_counts = [_ceil_div(x, block_size) for x in suffix]
    need = prefix_blocks + sum(suffix_counts) + num_seqs
    num_blocks = int(math.ceil(1.25 * need))
    perm = torch.randperm(num_blocks, generator=gen)
    shared = perm[:prefix_blocks]
    max_blocks = prefix_blocks + max(suffix_counts)
    bt = torch.full((num_seqs, max_blocks), -1, dtype=torch.int32)
    pos = prefix_blocks
    for s, n in enumerate(suffix_counts):
        bt[s, :prefix_blocks] = shared.to(torch.int32)
        bt[s, prefix_blocks:prefix_blocks + n] = perm[pos:pos + n].to(torch.int32)
        pos += n
    dst = perm[pos:pos + num_seqs].clone()
    kc, vc, free = _pool(gen, num_blocks, hkv, block_size, d, dtype, perm[:pos])
    q = _randn(gen, (num_seqs, hq, d), dtype)
    lens = [prefix_blocks * block_size + x for x in suffix]
    return PagedDecodeInputs(
        name=f"shared_prefix_cow_{num_seqs}seq_prefix800_suffix1-512_h32kv8_d128_bf16",
        seed=seed, dtype=dtype, block_size=block_size, num_q_heads=hq, num_kv_heads=hkv,
        head_dim=d, num_blocks=num_blocks, context_lens=torch.tensor(lens, dtype=torch.int32),
        block_tables=bt, key_cache=kc, value_cache=vc, query=q, new_key=None, new_value=None,
        free_blocks=free, scale=1.0 / math.sqrt(d), shared_blocks=shared.clone(),
        cow_logical_block=prefix_blocks - 1, cow_dst_blocks=dst)


def long_context_decode(seed: int = 4, block_size: int = 16, num_seqs: int = 16,
                        context: int = 32768) -> PagedDecodeInputs:
    """16 sequences decoding at a 32768-token context (GQA 32/8, head_dim 128, bf16)."""
    gen = torch.Generator().manual_seed(seed)
    return _decode_batch(f"long_context_decode_{num_seqs}seq_L{context}_h32kv8_d128_bf16_B{block_size}",
                         seed, gen, [context] * num_seqs, dtype=torch.bfloat16,
                         block_size=block_size, hq=32, hkv=8, d=128, append=False)


def chunked_prefill(seed: int = 4, block_size: int = 16, num_seqs: int = 8, ctx: int = 8192,
                    chunk: int = 512, hq: int = 32, hkv: int = 8, d: int = 128,
                    dtype: torch.dtype = torch.bfloat16, ctx_lens=None, q_lens=None,
                    pool_factor: float = 1.25) -> PrefillChunkInputs:
    """Causal prefill chunks (default 8 x 512 tokens) against 8192 prior paged tokens."""
    gen = torch.Generator().manual_seed(seed)
    ctx_lens = [ctx] * num_seqs if ctx_lens is None else [int(x) for x in ctx_lens]
    q_lens = [chunk] * num_seqs if q_lens is None else [int(x) for x in q_lens]
    return _chunk_batch(
        f"chunked_prefill_{len(ctx_lens)}seq_ctx{ctx}_chunk{chunk}_h{hq}kv{hkv}_d{d}_B{block_size}",
        seed, gen, ctx_lens, q_lens, block_size=block_size, hq=hq, hkv=hkv, d=d, dtype=dtype,
        pool_factor=pool_factor)


def mixed_batch(seed: int = 6, block_size: int = 16, num_decode: int = 256, num_prefill: int = 4,
                ctx: int = 8192, chunk: int = 512, hq: int = 32, hkv: int = 8, d: int = 128,
                dtype: torch.dtype = torch.bfloat16, decode_ctx=None, prefill_ctx=None,
                prefill_q=None, pool_factor: float = 1.25) -> PrefillChunkInputs:
    """Ongoing decodes and prompt chunks in one batch: ``num_decode`` decode
    sequences first (one query row each; prior context U[127, 4095], so they
    attend over 128 .. 4096 tokens like the GQA decode batch), then
    ``num_prefill`` chunks of ``chunk`` rows against ``ctx`` prior tokens."""
    gen = torch.Generator().manual_seed(seed)
    if decode_ctx is None:
        decode_ctx = torch.randint(127, 4095 + 1, (num_decode,), generator=gen).tolist()
    decode_ctx = [int(x) for x in decode_ctx]
    prefill_ctx = [ctx] * num_prefill if prefill_ctx is None else [int(x) for x in prefill_ctx]
    prefill_q = [chunk] * len(prefill_ctx) if prefill_q is None else [int(x) for x in prefill_q]
    b = _chunk_batch(
        f"mixed_batch_{len(decode_ctx)}dec_L128-4096_{len(prefill_ctx)}x{chunk}chunk_ctx{ctx}"
        f"_h{hq}kv{hkv}_d{d}_B{block_size}",
        seed, gen, decode_ctx + prefill_ctx, [1] * len(decode_ctx) + prefill_q,
        block_size=block_size, hq=hq, hkv=hkv, d=d, dtype=dtype, pool_factor=pool_factor)
    b.num_decode = len(decode_ctx)
    return b


def _chunk_batch(name, seed, gen, ctx_lens, q_lens, *, block_size, hq, hkv, d, dtype,
                 pool_factor) -> PrefillChunkInputs:
    num_seqs = len(ctx_lens)
    counts = [_ceil_div(c + n, block_size) for c, n in zip(ctx_lens, q_lens)]
    need = sum(counts)
    num_blocks = max(1, int(math.ceil(pool_factor * need)))
    perm = torch.randperm(num_blocks, generator=gen)
    bt, used = _tables_from_counts(perm, counts, max(1, max(counts)))
    kc, vc, free = _pool(gen, num_blocks, hkv, block_size, d, dtype, perm[:used])
    total_q = sum(q_lens)
    q = _randn(gen, (total_q, hq, d), dtype)
    nk = _randn(gen, (total_q, hkv, d), dtype)
    nv = _randn(gen, (total_q, hkv, d), dtype)
    cu = torch.zeros(num_seqs + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(q_lens, dtype=torch.int64), 0).to(torch.int32)
    return PrefillChunkInputs(
        name=name, seed=seed, dtype=dtype, block_size=block_size, num_q_heads=hq, num_kv_heads=hkv,
        head_dim=d, num_blocks=num_blocks, ctx_lens=torch.tensor(ctx_lens, dtype=torch.int32),
        cu_q_lens=cu, block_tables=bt, key_cache=kc, value_cache=vc, query=q, new_key=nk,
        new_value=nv, free_blocks=free, scale=1.0 / math.sqrt(d))


def llama3_8b_gqa_decode_fp8(seed: int = 2, num_seqs: int = 256,
                             block_size: int = 16) -> PagedDecodeInputs:
    """The Llama-3-8B-shaped GQA decode batch with an FP8 (E4M3) K/V pool:
    same lengths and block shuffle as llama3_8b_gqa_decode; the pool holds
    codes of N(0,1) / (1/32), i.e. values N(0,1) under a scale of 1/32; the
    query and the appended token stay bf16."""
    gen = torch.Generator().manual_seed(seed)
    lens = torch.randint(128, 4096 + 1, (num_seqs,), generator=gen).tolist()
    return _decode_batch(f"llama3_8b_gqa_decode_fp8_{num_seqs}seq_L128-4096_h32kv8_d128_e4m3_B{block_size}",
                         seed, gen, lens, dtype=torch.bfloat16, block_size=block_size,
                         hq=32, hkv=8, d=128, append=True, fp8_scale=1.0 / 32)


def random_decode(seed: int, lens, *, dtype=torch.float16, block_size=16, hq=4, hkv=4, d=64,
                  append=True, pool_factor=1.5, fp8_scale=None) -> PagedDecodeInputs:
    """A small decode batch with caller-chosen lengths (for edge cases and sweeps)."""
    gen = torch.Generator().manual_seed(seed)
    return _decode_batch(f"random_decode_s{seed}", seed, gen, lens, dtype=dtype,
                         block_size=block_size, hq=hq, hkv=hkv, d=d, append=append,
                         pool_factor=pool_factor, fp8_scale=fp8_scale)


WORKLOADS = {
    "tiny_decode": tiny_decode,
    "llama2_13b_decode": llama2_13b_decode,
    "llama3_8b_gqa_decode": llama3_8b_gqa_decode,
    "llama3_8b_gqa_decode_fp8": llama3_8b_gqa_decode_fp8,
    "shared_prefix_cow": shared_prefix_cow,
    "long_context_decode": long_context_decode,
    "chunked_prefill": chunked_prefill,
    "mixed_batch": mixed_batch,
}


def make_workload(name: str, **kw):
    return WORKLOADS[name](**kw)
