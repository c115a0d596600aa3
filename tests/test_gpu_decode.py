"""pa_decode against the fp64 oracle: tiny and full-size workloads, every
compiled shape, split-KV partitions, edge lengths, NaN-poisoned unused slots,
bit-identity under physical block relabelling and across copy-on-write."""
import numpy as np
import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth
from helpers import (TOL, decode_reference, dev, max_err, oracle_append, sample_seqs, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def run_decode(w, lens, partition_tokens=0, kc=None, vc=None, bt=None):
    kc = to_dev(w.key_cache) if kc is None else kc
    vc = to_dev(w.value_cache) if vc is None else vc
    bt = to_dev(w.block_tables) if bt is None else bt
    lens_d = to_dev(torch.as_tensor(lens, dtype=torch.int32))
    out = torch.empty(w.query.shape, dtype=w.dtype, device=dev())
    max_len = max(1, int(max(lens)))
    pa.pa_decode(out, to_dev(w.query), kc, vc, bt, lens_d, max_len, w.scale,
                 partition_tokens=partition_tokens)
    torch.cuda.synchronize()
    return out


def append_on_gpu(w):
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    bt, ctx = to_dev(w.block_tables), to_dev(w.context_lens)
    slots = torch.empty(w.num_seqs, dtype=torch.int64, device=dev())
    pa.pa_slot_mapping(slots, bt, ctx, w.block_size)
    pa.pa_reshape_and_cache(to_dev(w.new_key), to_dev(w.new_value), kc, vc, slots)
    return kc, vc, bt


@pytest.mark.parametrize("partition_tokens", [0, 16, 32, 48, 512])
def test_tiny_decode_with_append(partition_tokens):
    w = synth.tiny_decode()
    kc, vc, bt = append_on_gpu(w)
    lens = (w.context_lens + 1).tolist()
    out = run_decode(w, lens, partition_tokens, kc, vc, bt)
    oracle_append(w)
    ref = decode_reference(w, lens, range(w.num_seqs))
    assert max_err(out, ref) <= TOL[w.dtype]


SHAPES = [  # (dtype, B, Hq, Hkv, D)
    (torch.float16, 16, 4, 4, 64), (torch.bfloat16, 16, 4, 4, 64),
    (torch.float16, 32, 8, 2, 64), (torch.bfloat16, 32, 8, 8, 128),
    (torch.bfloat16, 16, 32, 8, 128), (torch.float16, 16, 16, 2, 128),
    (torch.bfloat16, 32, 32, 4, 128), (torch.bfloat16, 16, 16, 1, 128),
    (torch.float16, 16, 12, 1, 64), (torch.bfloat16, 16, 6, 2, 128),
]


@pytest.mark.parametrize("dtype,B,hq,hkv,D", SHAPES)
@pytest.mark.parametrize("partition_tokens", [0, 64])
def test_shapes_and_edge_lengths(dtype, B, hq, hkv, D, partition_tokens):
    lens = [1, B - 1, B, B + 1, 2 * B + 3, 97, 300, 0, 513]
    w = synth.random_decode(hq * 7 + B + D, lens, dtype=dtype, block_size=B, hq=hq, hkv=hkv,
                            d=D, append=False)
    out = run_decode(w, lens, partition_tokens)
    ref = decode_reference(w, lens, range(len(lens)))
    assert max_err(out, ref) <= TOL[dtype]
    assert torch.count_nonzero(out[lens.index(0)]) == 0  # empty sequence -> zero row


def test_nan_in_tail_slots_and_unused_blocks_is_never_read():
    lens = [5, 16, 17, 40, 100]
    w = synth.random_decode(3, lens, dtype=torch.bfloat16, hq=8, hkv=2, d=128, append=False)
    clean = run_decode(w, lens, 32)
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    B = w.block_size
    for s, L in enumerate(lens):
        last = int(w.block_tables[s, (L - 1) // B])
        if L % B:
            kc[last, :, L % B:] = float("nan")
            vc[last, :, L % B:] = float("nan")
    poisoned = run_decode(w, lens, 32, kc, vc)
    assert torch.equal(clean.view(torch.int16), poisoned.view(torch.int16))
    assert torch.isfinite(poisoned.float()).all()


@pytest.mark.parametrize("partition_tokens", [0, 48])
def test_bit_identical_under_block_relabelling(partition_tokens):
    w = synth.random_decode(21, [1, 33, 64, 200, 777], dtype=torch.bfloat16, hq=16, hkv=4,
                            d=128, append=False)
    lens = w.context_lens.tolist()
    base = run_decode(w, lens, partition_tokens)
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(w.num_blocks, generator=g)  # old block b -> new id perm[b]
    kc2 = torch.empty_like(w.key_cache)
    vc2 = torch.empty_like(w.value_cache)
    kc2[perm] = w.key_cache
    vc2[perm] = w.value_cache
    bt2 = torch.where(w.block_tables >= 0, perm[w.block_tables.clamp(min=0).long()].int(),
                      w.block_tables)
    moved = run_decode(w, lens, partition_tokens, to_dev(kc2), to_dev(vc2), to_dev(bt2))
    assert torch.equal(base.view(torch.int16), moved.view(torch.int16))


def test_llama3_8b_gqa_full_size_sampled():
    w = synth.llama3_8b_gqa_decode()
    kc, vc, bt = append_on_gpu(w)
    lens = (w.context_lens + 1).tolist()
    out = run_decode(w, lens, 0, kc, vc, bt).cpu()
    oracle_append(w)
    seqs = sample_seqs(w.num_seqs, 10, seed=2, must=[int(np.argmax(lens)), int(np.argmin(lens))])
    ref = decode_reference(w, lens, seqs)
    assert max_err(out[seqs], ref) <= TOL[w.dtype]
    assert torch.isfinite(out.float()).all()


def test_llama2_13b_full_size_sampled():
    w = synth.llama2_13b_decode()
    lens = w.context_lens.tolist()
    out = run_decode(w, lens).cpu()
    seqs = sample_seqs(w.num_seqs, 6, seed=1, must=[int(np.argmax(lens))])
    ref = decode_reference(w, lens, seqs)
    assert max_err(out[seqs], ref) <= TOL[w.dtype]


@pytest.mark.parametrize("B", [16, 32])
def test_long_context_split_kv_sampled(B):
    w = synth.long_context_decode(block_size=B)
    lens = w.context_lens.tolist()
    out = run_decode(w, lens).cpu()
    seqs = [0, 11]
    ref = decode_reference(w, lens, seqs)
    assert max_err(out[seqs], ref) <= TOL[w.dtype]


def test_shared_prefix_copy_on_write():
    w = synth.shared_prefix_cow()
    lens = w.context_lens.tolist()
    kc, vc, bt = to_dev(w.key_cache), to_dev(w.value_cache), to_dev(w.block_tables)
    before = run_decode(w, lens, 0, kc, vc, bt)
    src = w.shared_blocks[w.cow_logical_block].repeat(w.num_seqs)
    pairs = to_dev(torch.stack([src, w.cow_dst_blocks], 1).to(torch.int64))
    pa.pa_copy_blocks(kc, vc, pairs)
    bt2 = bt.clone()
    bt2[:, w.cow_logical_block] = to_dev(w.cow_dst_blocks.to(torch.int32))
    after = run_decode(w, lens, 0, kc, vc, bt2)
    # the copy is byte-identical, so the output is too
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))
    seqs = sample_seqs(w.num_seqs, 8, seed=3)
    ref = decode_reference(w, lens, seqs)
    assert max_err(after.cpu()[seqs], ref) <= TOL[w.dtype]


def test_out_of_pool_block_id_is_flagged_not_read():
    w = synth.random_decode(8, [40, 40], dtype=torch.float16, hq=4, hkv=4, d=64, append=False)
    bt = w.block_tables.clone()
    bt[1, 1] = w.num_blocks + 5
    out = run_decode(w, [40, 40], 0, bt=to_dev(bt))
    assert pa.pa_get_device_error() & pa.PA_DEVERR_BLOCK_RANGE
    ref = decode_reference(w, [40, 40], [0])
    assert max_err(out[:1], ref) <= TOL[w.dtype]  # the healthy sequence is unaffected


# The decode ring holds 8 stages of one 16-token block (4 of one 32-token
# block at block size 32); after the first ring positions of an item each
# consumer warp refills the stage it has just consumed with its own next
# position there.  Items of about 1, 7, 8, 9, 15, 16, 17 and 33 blocks of 16
# tokens, one partition per sequence, cover items shorter than the ring,
# exactly the ring, one past it, two rounds and more.
@pytest.mark.parametrize("B", [16, 32])
def test_ring_refill_around_the_ring_depth(B):
    stages = [1, 7, 8, 9, 15, 16, 17, 33]
    lens = [n * 16 - 3 for n in stages] + [n * 16 for n in stages]
    w = synth.random_decode(61 + B, lens, dtype=torch.bfloat16, block_size=B, hq=8, hkv=2,
                            d=128, append=False)
    out = run_decode(w, lens, partition_tokens=1024)  # one partition per sequence
    ref = decode_reference(w, lens, list(range(w.num_seqs)))
    assert max_err(out, ref) <= TOL[w.dtype]
