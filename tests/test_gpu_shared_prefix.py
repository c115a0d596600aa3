"""pa_decode_shared_prefix against pa_decode and the fp64 oracle.

Sequences that share their leading blocks ("PagedAttention: Why Static
Batching Wastes Your KV Cache", "How does copy-on-write eliminate duplicate
prompt KV cache?") have the same K/V for the split-KV partitions inside the
shared prefix; the library computes those partitions once per group of
sequences.  Every query column's arithmetic is pa_decode's, so with the same
partition length the output must be bit-identical to pa_decode, and within
the decode tolerance of the oracle.
"""
import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth
from helpers import TOL, decode_reference, dev, max_err, sample_seqs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def both(w, lens, bt, prefix_blocks, prefix_len, pt):
    kc, vc, q = to_dev(w.key_cache), to_dev(w.value_cache), to_dev(w.query)
    btd, ld = to_dev(bt), to_dev(torch.tensor(lens, dtype=torch.int32))
    a = torch.empty_like(q)
    pa.pa_decode(a, q, kc, vc, btd, ld, max(lens), w.scale, partition_tokens=pt)
    b = torch.full_like(q, float("nan"))
    pa.pa_decode_shared_prefix(b, q, kc, vc, to_dev(prefix_blocks.to(torch.int32)), prefix_len,
                               btd, ld, max(lens), w.scale, partition_tokens=pt)
    torch.cuda.synchronize()
    return a.cpu(), b.cpu()


@pytest.mark.parametrize("pt", [0, 16, 64, 256])
def test_shared_prefix_workload_bit_identical_to_pa_decode(pt):
    # 128 sequences over 49 shared blocks (784 tokens) after the copy-on-write
    # of logical block 49, each with a private suffix of 1..512 tokens
    w = synth.shared_prefix_cow()
    lens = w.context_lens.tolist()
    bt = w.block_tables.clone()
    bt[:, w.cow_logical_block] = w.cow_dst_blocks.to(torch.int32)
    src = w.shared_blocks[w.cow_logical_block].long()
    w.key_cache[w.cow_dst_blocks.long()] = w.key_cache[src].clone()
    w.value_cache[w.cow_dst_blocks.long()] = w.value_cache[src].clone()
    npre = w.cow_logical_block  # 49 blocks still shared by every sequence
    a, b = both(w, lens, bt, w.shared_blocks[:npre], npre * w.block_size, pt)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    w.block_tables = bt
    seqs = sample_seqs(w.num_seqs, 6, seed=pt)
    assert max_err(b[seqs], decode_reference(w, lens, seqs)) <= TOL[w.dtype]


# (q heads, kv heads, dtype, block size): sequences per CTA = 16 / group
SHAPES = [(4, 4, torch.float16, 16), (16, 2, torch.bfloat16, 32), (8, 1, torch.float16, 16)]


@pytest.mark.parametrize("hq,hkv,dtype,B", SHAPES)
def test_shared_leading_blocks_bit_identical(hq, hkv, dtype, B):
    # 21 sequences (not a multiple of the group) share sequence 0's first 4
    # blocks, i.e. two 2-block partitions; lengths from exactly the shared
    # prefix up, with ragged tails
    pt = 2 * B
    lens = [4 * B, 4 * B + 1, 5 * B, 300, 7 * B - 3, 9 * B, 4 * B + 7] * 3
    w = synth.random_decode(90 + hq, lens, dtype=dtype, block_size=B, hq=hq, hkv=hkv, d=128,
                            append=False)
    bt = w.block_tables.clone()
    bt[:, :4] = bt[0, :4]
    w.block_tables = bt
    a, b = both(w, lens, bt, bt[0, :4], 4 * B, pt)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    seqs = sample_seqs(w.num_seqs, 5, seed=hq, must=[0, 1, 20])
    assert max_err(b[seqs], decode_reference(w, lens, seqs)) <= TOL[dtype]


def test_one_partition_sequences_are_written_by_the_prefix_pass():
    # every sequence fits one 64-token partition that lies inside the shared
    # prefix: the shared-prefix pass alone produces the final rows
    B = 16
    lens = [64] * 9
    w = synth.random_decode(77, lens, dtype=torch.bfloat16, block_size=B, hq=8, hkv=2, d=128,
                            append=False)
    bt = w.block_tables.clone()
    bt[:, :4] = bt[0, :4]
    w.block_tables = bt
    a, b = both(w, lens, bt, bt[0, :4], 64, 64)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert max_err(b, decode_reference(w, lens, list(range(9)))) <= TOL[w.dtype]


def test_sequence_shorter_than_the_shared_prefix_is_flagged():
    B = 16
    lens = [64, 64, 40]
    w = synth.random_decode(78, lens, dtype=torch.bfloat16, block_size=B, hq=8, hkv=2, d=128,
                            append=False)
    bt = w.block_tables.clone()
    bt[:2, :4] = bt[0, :4]
    bt[2, :3] = bt[0, :3]
    kc, vc, q = to_dev(w.key_cache), to_dev(w.value_cache), to_dev(w.query)
    out = torch.empty_like(q)
    pa.pa_decode_shared_prefix(out, q, kc, vc, to_dev(bt[0, :4].contiguous()), 64, to_dev(bt),
                               to_dev(torch.tensor(lens, dtype=torch.int32)), 64, w.scale,
                               partition_tokens=64)
    assert pa.pa_get_device_error() & pa.PA_DEVERR_SEQ_RANGE
