"""Slot mapping, reshape_and_cache and copy_blocks on the GPU: bit-exact
against the oracle, untouched memory untouched, bad ids flagged."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_397_b200 as pa
import synth
from helpers import dev, int16_view, oracle_append, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.pa_get_device_error()
    yield


@pytest.mark.parametrize("factory", [synth.tiny_decode, synth.llama3_8b_gqa_decode])
def test_decode_append_bit_exact(factory):
    w = factory()
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    bt, ctx = to_dev(w.block_tables), to_dev(w.context_lens)
    slots = torch.empty(w.num_seqs, dtype=torch.int64, device=dev())
    pa.pa_slot_mapping(slots, bt, ctx, w.block_size)
    pa.pa_reshape_and_cache(to_dev(w.new_key), to_dev(w.new_value), kc, vc, slots)
    want_slots = oracle_append(w)  # updates the CPU caches in place
    np.testing.assert_array_equal(slots.cpu().numpy(), want_slots)
    assert torch.equal(kc.view(torch.int16), to_dev(w.key_cache).view(torch.int16))
    assert torch.equal(vc.view(torch.int16), to_dev(w.value_cache).view(torch.int16))
    assert pa.pa_get_device_error() == 0


@pytest.mark.parametrize("B", [16, 32])
def test_prefill_chunk_slots_and_scatter(B):
    p = synth.chunked_prefill(seed=5, block_size=B, hq=8, hkv=2, d=128,
                              ctx_lens=[0, 17, 100, 31], q_lens=[40, 1, 257, 0])
    kc, vc = to_dev(p.key_cache), to_dev(p.value_cache)
    bt, cl, cu = to_dev(p.block_tables), to_dev(p.ctx_lens), to_dev(p.cu_q_lens)
    slots = torch.empty(p.total_q, dtype=torch.int64, device=dev())
    pa.pa_slot_mapping(slots, bt, cl, B, cu_q_lens=cu)
    pa.pa_reshape_and_cache(to_dev(p.new_key), to_dev(p.new_value), kc, vc, slots)
    cuh = p.cu_q_lens.numpy()
    seq_of = np.repeat(np.arange(p.num_seqs), np.diff(cuh))
    pos = np.concatenate([np.arange(c, c + n) for c, n in zip(p.ctx_lens.numpy(), np.diff(cuh))])
    want = oracle.logical_positions_to_slots(p.block_tables.numpy(), seq_of, pos, B)
    np.testing.assert_array_equal(slots.cpu().numpy(), want)
    oracle.reshape_and_cache(int16_view(p.key_cache), int16_view(p.value_cache),
                             int16_view(p.new_key), int16_view(p.new_value), want, B)
    assert torch.equal(kc.cpu().view(torch.int16), p.key_cache.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), p.value_cache.view(torch.int16))
    assert pa.pa_get_device_error() == 0


def test_reshape_skips_negative_and_flags_out_of_range_slots():
    w = synth.tiny_decode()
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    slots = torch.tensor([5, -1, w.num_blocks * w.block_size, 7], dtype=torch.int64,
                         device=dev())
    pa.pa_reshape_and_cache(to_dev(w.new_key), to_dev(w.new_value), kc, vc, slots)
    assert pa.pa_get_device_error() & pa.PA_DEVERR_SLOT_RANGE
    oracle.reshape_and_cache(int16_view(w.key_cache), int16_view(w.value_cache),
                             int16_view(w.new_key), int16_view(w.new_value), [5, -1, -1, 7],
                             w.block_size)
    assert torch.equal(kc.cpu().view(torch.int16), w.key_cache.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), w.value_cache.view(torch.int16))


def test_copy_blocks_shared_prefix_bit_exact():
    w = synth.shared_prefix_cow()
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    src = w.shared_blocks[w.cow_logical_block].repeat(w.num_seqs)
    pairs = torch.stack([src, w.cow_dst_blocks], 1).to(torch.int64)
    pa.pa_copy_blocks(kc, vc, to_dev(pairs))
    oracle.copy_blocks(int16_view(w.key_cache), int16_view(w.value_cache), pairs.numpy())
    assert torch.equal(kc.cpu().view(torch.int16), w.key_cache.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), w.value_cache.view(torch.int16))
    assert pa.pa_get_device_error() == 0


def test_copy_blocks_flags_bad_ids():
    w = synth.tiny_decode()
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    k0 = kc.clone()
    pairs = torch.tensor([[0, w.num_blocks], [-3, 1]], dtype=torch.int64, device=dev())
    pa.pa_copy_blocks(kc, vc, pairs)
    assert pa.pa_get_device_error() & pa.PA_DEVERR_BLOCK_RANGE
    assert torch.equal(kc.view(torch.int16), k0.view(torch.int16))


def test_slot_mapping_flags_positions_past_the_table():
    w = synth.tiny_decode()
    bt = to_dev(w.block_tables)
    ctx = to_dev(torch.tensor([0, 1, w.block_tables.shape[1] * w.block_size, 3],
                              dtype=torch.int32))
    slots = torch.empty(4, dtype=torch.int64, device=dev())
    pa.pa_slot_mapping(slots, bt, ctx, w.block_size)
    assert pa.pa_get_device_error() & pa.PA_DEVERR_SEQ_RANGE
    assert int(slots[2]) == -1


@pytest.mark.parametrize("factory", [synth.tiny_decode, synth.llama3_8b_gqa_decode])
def test_fused_append_matches_slot_mapping_plus_scatter(factory):
    w = factory()
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    slots = torch.full((w.num_seqs,), -7, dtype=torch.int64, device=dev())
    pa.pa_append(to_dev(w.new_key), to_dev(w.new_value), kc, vc, to_dev(w.block_tables),
                 to_dev(w.context_lens), slot_mapping=slots)
    want = oracle_append(w)
    np.testing.assert_array_equal(slots.cpu().numpy(), want)
    assert torch.equal(kc.cpu().view(torch.int16), w.key_cache.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), w.value_cache.view(torch.int16))
    assert pa.pa_get_device_error() == 0


def test_fused_append_of_prefill_chunks():
    p = synth.chunked_prefill(seed=5, block_size=32, hq=8, hkv=2, d=128,
                              ctx_lens=[0, 17, 100, 31], q_lens=[40, 1, 257, 0])
    kc, vc = to_dev(p.key_cache), to_dev(p.value_cache)
    pa.pa_append(to_dev(p.new_key), to_dev(p.new_value), kc, vc, to_dev(p.block_tables),
                 to_dev(p.ctx_lens), cu_q_lens=to_dev(p.cu_q_lens))
    cuh = p.cu_q_lens.numpy()
    seq_of = np.repeat(np.arange(p.num_seqs), np.diff(cuh))
    pos = np.concatenate([np.arange(c, c + n) for c, n in zip(p.ctx_lens.numpy(), np.diff(cuh))])
    want = oracle.logical_positions_to_slots(p.block_tables.numpy(), seq_of, pos, 32)
    oracle.reshape_and_cache(int16_view(p.key_cache), int16_view(p.value_cache),
                             int16_view(p.new_key), int16_view(p.new_value), want, 32)
    assert torch.equal(kc.cpu().view(torch.int16), p.key_cache.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), p.value_cache.view(torch.int16))
    assert pa.pa_get_device_error() == 0


def test_fused_append_flags_positions_past_the_table():
    w = synth.tiny_decode()
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    ctx = w.context_lens.clone()
    ctx[1] = w.block_tables.shape[1] * w.block_size
    slots = torch.zeros(w.num_seqs, dtype=torch.int64, device=dev())
    pa.pa_append(to_dev(w.new_key), to_dev(w.new_value), kc, vc, to_dev(w.block_tables),
                 to_dev(ctx), slot_mapping=slots)
    assert pa.pa_get_device_error() & pa.PA_DEVERR_SEQ_RANGE
    assert int(slots[1]) == -1
