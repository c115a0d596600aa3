"""pa_append_decode: one decode step (append of each sequence's new token,
then decode over the grown sequence) in one launch.  Output and cache bytes
must equal pa_append followed by pa_decode bit for bit, the slots the
oracle's slot arithmetic gives, and the fp64 oracle within tolerance."""
import numpy as np
import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth
from helpers import TOL, decode_reference, dev, max_err, oracle_append, sample_seqs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def two_calls(w, partition_tokens):
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    bt, ctx = to_dev(w.block_tables), to_dev(w.context_lens)
    q = to_dev(w.query)
    out = torch.empty_like(q)
    pa.pa_append(to_dev(w.new_key), to_dev(w.new_value), kc, vc, bt, ctx)
    pa.pa_decode(out, q, kc, vc, bt, ctx + 1, int(w.context_lens.max()) + 1, w.scale,
                 partition_tokens=partition_tokens)
    torch.cuda.synchronize()
    return out, kc, vc


def fused(w, partition_tokens):
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    bt, ctx = to_dev(w.block_tables), to_dev(w.context_lens)
    q = to_dev(w.query)
    out = torch.empty_like(q)
    slots = torch.full((w.num_seqs,), -7, dtype=torch.int64, device=dev())
    pa.pa_append_decode(out, q, to_dev(w.new_key), to_dev(w.new_value), kc, vc, bt, ctx,
                        int(w.context_lens.max()), w.scale, slot_mapping=slots,
                        partition_tokens=partition_tokens)
    torch.cuda.synchronize()
    return out, kc, vc, slots


def bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t


@pytest.mark.parametrize("dtype,B,hq,hkv,D", [
    (torch.bfloat16, 16, 32, 8, 128), (torch.float16, 32, 8, 8, 128),
    (torch.bfloat16, 16, 16, 1, 128), (torch.float16, 16, 12, 4, 64),
    (torch.bfloat16, 32, 4, 2, 64)])
@pytest.mark.parametrize("partition_tokens", [0, 32, 64])
def test_fused_step_is_bitwise_append_then_decode(dtype, B, hq, hkv, D, partition_tokens):
    # lengths on both sides of block and partition edges (the new token may
    # open a new block, end a partition or start a new one)
    lens = [1, B - 1, B, B + 1, 63, 64, 65, 200, 777]
    w = synth.random_decode(60 + B + hq, lens, dtype=dtype, block_size=B, hq=hq, hkv=hkv, d=D)
    a_out, a_k, a_v, slots = fused(w, partition_tokens)
    b_out, b_k, b_v = two_calls(w, partition_tokens)
    assert torch.equal(bits(a_out), bits(b_out))
    assert torch.equal(bits(a_k), bits(b_k)) and torch.equal(bits(a_v), bits(b_v))
    np.testing.assert_array_equal(slots.cpu().numpy(), oracle_append(w))


def test_fused_step_full_size_matches_oracle():
    w = synth.llama3_8b_gqa_decode()
    out, _, _, slots = fused(w, 0)
    want_slots = oracle_append(w)  # also writes the new tokens into the CPU caches
    np.testing.assert_array_equal(slots.cpu().numpy(), want_slots)
    lens = (w.context_lens + 1).tolist()
    seqs = sample_seqs(w.num_seqs, 6, seed=3, must=[int(np.argmax(lens))])
    ref = decode_reference(w, lens, seqs)
    assert max_err(out[seqs].cpu(), ref) <= TOL[w.dtype]


def test_fused_step_flags_context_past_the_table_and_writes_nothing():
    w = synth.random_decode(71, [20, 40], dtype=torch.bfloat16, hq=8, hkv=2, d=128)
    width = w.block_tables.shape[1]
    ctx = w.context_lens.clone()
    ctx[1] = width * w.block_size  # the new token would need a block past the table
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    k0 = kc.clone()
    q = to_dev(w.query)
    out = torch.empty_like(q)
    slots = torch.zeros(2, dtype=torch.int64, device=dev())
    pa.pa_append_decode(out, q, to_dev(w.new_key), to_dev(w.new_value), kc, vc,
                        to_dev(w.block_tables), to_dev(ctx), width * w.block_size - 1, w.scale,
                        slot_mapping=slots)
    assert pa.pa_get_device_error() & pa.PA_DEVERR_SEQ_RANGE
    assert int(slots[1]) == -1
    # sequence 0 got its token; nothing else in the pool changed
    b0 = int(w.block_tables[0, int(w.context_lens[0]) // w.block_size])
    off = int(w.context_lens[0]) % w.block_size
    changed = (kc.view(torch.int16) != k0.view(torch.int16)).nonzero()
    assert all(int(r[0]) == b0 and int(r[2]) == off for r in changed)
