"""Seeded synthetic inputs (synth/), which the oracle and the library both
read: the same seed gives the same bits, and every workload has the
structure stated for it -- lengths in their ranges, each sequence's blocks
drawn from a shuffled pool with no block shared between sequences (except
the shared prompt of the copy-on-write workload), table entries past a
sequence's allocation -1, every block no table references NaN-filled (so a
kernel that reads one poisons its output), and chunk offsets consistent."""
import dataclasses
import inspect
import math

import pytest
import torch

import synth

SMALL = {
    "tiny_decode": dict(),
    "llama2_13b_decode": dict(num_seqs=6),
    "llama3_8b_gqa_decode": dict(num_seqs=8),
    "llama3_8b_gqa_decode_fp8": dict(num_seqs=8),
    "shared_prefix_cow": dict(num_seqs=6),
    "long_context_decode": dict(num_seqs=2, context=700),
    "chunked_prefill": dict(num_seqs=3, ctx=300, chunk=70),
    "mixed_batch": dict(num_decode=6, num_prefill=2, ctx=300, chunk=70),
}


def _bits(t):
    return t.contiguous().view(torch.uint8) if t.dtype != torch.bool else t


def _fields(x):
    return {f.name: getattr(x, f.name) for f in dataclasses.fields(x)}


def test_every_workload_is_listed():
    assert sorted(SMALL) == sorted(synth.WORKLOADS)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_same_seed_same_bits_other_seed_other_data(name):
    a = synth.make_workload(name, **SMALL[name])
    b = synth.make_workload(name, **SMALL[name])
    for k, v in _fields(a).items():
        w = getattr(b, k)
        if isinstance(v, torch.Tensor):
            assert v.dtype == w.dtype and v.shape == w.shape, k
            assert torch.equal(_bits(v), _bits(w)), k
        else:
            assert v == w or (isinstance(v, float) and math.isnan(v) and math.isnan(w)), k
    c = synth.make_workload(name, seed=a.seed + 100, **SMALL[name])
    assert not torch.equal(_bits(a.query), _bits(c.query))


def _lengths(w):
    """Tokens each table must cover: decode context (+1 when a token is
    appended), or context + chunk rows."""
    if isinstance(w, synth.PrefillChunkInputs):
        q = (w.cu_q_lens[1:] - w.cu_q_lens[:-1]).tolist()
        return [c + n for c, n in zip(w.ctx_lens.tolist(), q)]
    add = 1 if w.new_key is not None else 0
    return [c + add for c in w.context_lens.tolist()]


@pytest.mark.parametrize("name", sorted(SMALL))
def test_pool_and_tables(name):
    w = synth.make_workload(name, **SMALL[name])
    B, nb = w.block_size, w.num_blocks
    bt = w.block_tables
    owners = {}
    for s, L in enumerate(_lengths(w)):
        n = -(-L // B)
        row = bt[s].tolist()
        assert all(0 <= b < nb for b in row[:n]), f"sequence {s}: block id outside the pool"
        assert all(b == -1 for b in row[n:]), f"sequence {s}: entries past its blocks not -1"
        assert len(set(row[:n])) == n, f"sequence {s} lists a block twice"
        for i, b in enumerate(row[:n]):
            owners.setdefault(b, []).append((s, i))
    shared = set(w.shared_blocks.tolist()) if getattr(w, "shared_blocks", None) is not None \
        else set()
    for b, who in owners.items():
        if len(who) > 1:
            assert b in shared, f"block {b} is in several tables: {who[:3]}"
            assert len({i for _, i in who}) == 1  # a shared block has one logical index
    referenced = set(owners)
    free = set(w.free_blocks.tolist())
    assert referenced.isdisjoint(free) and referenced | free == set(range(nb))
    # unreferenced blocks poison any read; referenced ones hold finite data
    fp8 = w.key_cache.dtype == torch.uint8
    for cache in (w.key_cache, w.value_cache):
        idx_free = torch.tensor(sorted(free), dtype=torch.long)
        idx_used = torch.tensor(sorted(referenced), dtype=torch.long)
        if fp8:
            assert bool((cache[idx_free] == synth.FP8_NAN_CODE).all())
            assert not bool(((cache[idx_used] & 0x7F) == 0x7F).any())
        else:
            assert bool(torch.isnan(cache[idx_free]).all())
            assert bool(torch.isfinite(cache[idx_used]).all())
    # blocks are handed out from a shuffle, not in address order
    pairs = [(r[i], r[i + 1]) for r in bt.tolist() for i in range(len(r) - 1) if r[i + 1] >= 0]
    if len(pairs) >= 30:
        assert sum(b == a + 1 for a, b in pairs) < 0.2 * len(pairs)


def test_stated_lengths_and_shapes():
    w = synth.tiny_decode()
    assert w.context_lens.tolist() == [30, 50, 17, 64] and w.num_blocks == 64
    defaults = {n: inspect.signature(f).parameters for n, f in synth.WORKLOADS.items()}
    assert defaults["llama2_13b_decode"]["num_seqs"].default == 64
    assert defaults["llama3_8b_gqa_decode"]["num_seqs"].default == 256
    assert defaults["shared_prefix_cow"]["num_seqs"].default == 128
    w = synth.llama2_13b_decode(num_seqs=16)
    assert (w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim) == (16, 40, 40, 128)
    assert w.dtype == torch.float16 and w.new_key is None
    assert 16 <= int(w.context_lens.min()) and int(w.context_lens.max()) <= 2048
    w = synth.llama3_8b_gqa_decode(num_seqs=16)
    assert (w.num_q_heads, w.num_kv_heads, w.head_dim, w.dtype) == (32, 8, 128, torch.bfloat16)
    assert 128 <= int(w.context_lens.min()) and int(w.context_lens.max()) <= 4096
    assert w.new_key.shape == (16, 8, 128) and w.scale == 1 / math.sqrt(128)
    assert w.num_blocks == math.ceil(1.25 * sum(-(-(L + 1) // 16) for L in w.context_lens.tolist()))
    f = synth.llama3_8b_gqa_decode_fp8(num_seqs=16)
    assert torch.equal(f.context_lens, w.context_lens) and torch.equal(f.block_tables,
                                                                        w.block_tables)
    assert f.key_cache.dtype == torch.uint8 and f.kv_scale == 1 / 32
    w = synth.shared_prefix_cow(num_seqs=6)
    L = w.context_lens.tolist()
    assert all(800 < x <= 800 + 512 for x in L)
    assert bool((w.block_tables[:, :50] == w.shared_blocks.to(torch.int32)).all())
    assert w.cow_logical_block == 49
    dst = w.cow_dst_blocks.tolist()
    assert len(set(dst)) == 6 and set(dst) <= set(w.free_blocks.tolist())
    p = synth.chunked_prefill(num_seqs=3, ctx=300, chunk=70)
    assert p.ctx_lens.tolist() == [300] * 3 and p.cu_q_lens.tolist() == [0, 70, 140, 210]
    assert p.query.shape == (210, 32, 128) and p.num_decode == 0
    m = synth.mixed_batch(num_decode=6, num_prefill=2, ctx=300, chunk=70)
    assert m.num_decode == 6 and m.cu_q_lens.tolist() == [0, 1, 2, 3, 4, 5, 6, 76, 146]
    assert all(127 <= c <= 4095 for c in m.ctx_lens[:6].tolist())
    assert m.ctx_lens[6:].tolist() == [300, 300]
