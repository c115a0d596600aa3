"""FP8 (E4M3) KV cache on the GPU: the cache write is bit-exact against the
oracle's fp32-division / nearest-even / saturating quantizer, and decode over
FP8 caches matches the oracle's decode of the dequantized values."""
import numpy as np
import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth
from helpers import TOL, dev, max_err, sample_seqs, to_dev
from oracle import fp8 as ofp8

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def fp8_reference(w, lens, seqs):
    """Oracle decode over the FP8 pool for the chosen sequences (sub-pool)."""
    B = w.block_size
    used = sorted({int(b) for s in seqs for b in w.block_tables[s, :-(-int(lens[s]) // B)]})
    remap = {b: i for i, b in enumerate(used)}
    idx = torch.tensor(used)
    kc = w.key_cache.index_select(0, idx).numpy()
    vc = w.value_cache.index_select(0, idx).numpy()
    bt = np.full((len(seqs), w.block_tables.shape[1]), -1, dtype=np.int64)
    for r, s in enumerate(seqs):
        n = -(-int(lens[s]) // B)
        bt[r, :n] = [remap[int(b)] for b in w.block_tables[s, :n]]
    q = w.query[list(seqs)].double().numpy()
    return ofp8.paged_decode_fp8(q, kc, vc, bt, [int(lens[s]) for s in seqs], w.scale,
                                 w.kv_scale, w.kv_scale, w.num_kv_heads)


def run(w, lens, partition_tokens=0, kc=None, vc=None, bt=None):
    kc = to_dev(w.key_cache) if kc is None else kc
    vc = to_dev(w.value_cache) if vc is None else vc
    bt = to_dev(w.block_tables) if bt is None else bt
    out = torch.empty(w.query.shape, dtype=w.dtype, device=dev())
    pa.pa_decode_fp8(out, to_dev(w.query), kc, vc, bt,
                     to_dev(torch.as_tensor(lens, dtype=torch.int32)), max(1, max(lens)), w.scale,
                     w.kv_scale, w.kv_scale, partition_tokens=partition_tokens)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_fp8_cache_write_bit_exact(dtype):
    g = torch.Generator().manual_seed(5)
    T, hkv, D, B, nb = 300, 4, 128, 16, 40
    key = (torch.randn(T, hkv, D, generator=g) * 4).to(dtype)
    value = (torch.randn(T, hkv, D, generator=g) * 0.01).to(dtype)  # subnormal codes
    key[0, 0, :8] = torch.tensor([500., -1e4, 463.9, 464., 0., -0., 1.0625, 1.1875]).to(dtype)
    slots = torch.randperm(nb * B, generator=g)[:T].to(torch.int64)
    slots[7] = -1
    kc = torch.full((nb, hkv, B, D), 0x55, dtype=torch.uint8)
    vc = kc.clone()
    ks, vs = 0.75, 0.03125
    kd, vd = to_dev(kc), to_dev(vc)
    pa.pa_reshape_and_cache_fp8(to_dev(key), to_dev(value), kd, vd, to_dev(slots), ks, vs)
    kh, vh = kc.numpy().copy(), vc.numpy().copy()
    for t in range(T):
        s = int(slots[t])
        if s < 0:
            continue
        kh[s // B, :, s % B, :] = ofp8.quantize(key[t].float().numpy(), ks)
        vh[s // B, :, s % B, :] = ofp8.quantize(value[t].float().numpy(), vs)
    np.testing.assert_array_equal(kd.cpu().numpy(), kh)
    np.testing.assert_array_equal(vd.cpu().numpy(), vh)


SHAPES = [(torch.bfloat16, 16, 32, 8), (torch.float16, 16, 8, 8), (torch.bfloat16, 32, 16, 2),
          (torch.bfloat16, 16, 16, 1), (torch.float16, 32, 12, 1)]


@pytest.mark.parametrize("dtype,B,hq,hkv", SHAPES)
@pytest.mark.parametrize("partition_tokens", [0, 48, 64])
def test_fp8_decode_matches_oracle(dtype, B, hq, hkv, partition_tokens):
    lens = [1, B - 1, B, B + 1, 77, 300, 0, 1030]
    w = synth.random_decode(11 + hq + B, lens, dtype=dtype, block_size=B, hq=hq, hkv=hkv, d=128,
                            append=False, fp8_scale=1.0 / 32)
    out = run(w, lens, partition_tokens)
    ref = fp8_reference(w, lens, range(len(lens)))
    assert max_err(out, ref) <= TOL[dtype]
    assert torch.count_nonzero(out[lens.index(0)]) == 0


def test_fp8_nan_codes_past_the_end_are_never_read():
    lens = [5, 16, 17, 40, 100]
    w = synth.random_decode(3, lens, dtype=torch.bfloat16, hq=8, hkv=2, d=128, append=False,
                            fp8_scale=1.0 / 32)
    clean = run(w, lens, 32)
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    for s, L in enumerate(lens):
        last = int(w.block_tables[s, (L - 1) // 16])
        if L % 16:
            kc[last, :, L % 16:] = synth.FP8_NAN_CODE
            vc[last, :, L % 16:] = synth.FP8_NAN_CODE
    poisoned = run(w, lens, 32, kc, vc)
    assert torch.equal(clean.view(torch.int16), poisoned.view(torch.int16))


def test_fp8_bit_identical_under_block_relabelling():
    w = synth.random_decode(21, [1, 33, 64, 200, 777], dtype=torch.bfloat16, hq=16, hkv=4, d=128,
                            append=False, fp8_scale=1.0 / 32)
    lens = w.context_lens.tolist()
    base = run(w, lens, 48)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(99))
    kc2 = torch.empty_like(w.key_cache)
    vc2 = torch.empty_like(w.value_cache)
    kc2[perm] = w.key_cache
    vc2[perm] = w.value_cache
    bt2 = torch.where(w.block_tables >= 0, perm[w.block_tables.clamp(min=0).long()].int(),
                      w.block_tables)
    moved = run(w, lens, 48, to_dev(kc2), to_dev(vc2), to_dev(bt2))
    assert torch.equal(base.view(torch.int16), moved.view(torch.int16))


def test_fp8_full_size_gqa_decode_with_append_sampled():
    w = synth.llama3_8b_gqa_decode_fp8()
    kc, vc, bt = to_dev(w.key_cache), to_dev(w.value_cache), to_dev(w.block_tables)
    slots = torch.empty(w.num_seqs, dtype=torch.int64, device=dev())
    pa.pa_slot_mapping(slots, bt, to_dev(w.context_lens), w.block_size)
    pa.pa_reshape_and_cache_fp8(to_dev(w.new_key), to_dev(w.new_value), kc, vc, slots,
                                w.kv_scale, w.kv_scale)
    lens = (w.context_lens + 1).tolist()
    out = run(w, lens, 0, kc, vc, bt).cpu()
    # the oracle's own append: slots through the tables, codes by its quantizer
    B = w.block_size
    for s in range(w.num_seqs):
        p_ = int(w.context_lens[s])
        phys = int(w.block_tables[s, p_ // B])
        w.key_cache[phys, :, p_ % B] = torch.from_numpy(
            ofp8.quantize(w.new_key[s].float().numpy(), w.kv_scale))
        w.value_cache[phys, :, p_ % B] = torch.from_numpy(
            ofp8.quantize(w.new_value[s].float().numpy(), w.kv_scale))
    assert torch.equal(kc.cpu(), w.key_cache) and torch.equal(vc.cpu(), w.value_cache)
    seqs = sample_seqs(w.num_seqs, 10, seed=2, must=[int(np.argmax(lens))])
    assert max_err(out[seqs], fp8_reference(w, lens, seqs)) <= TOL[w.dtype]


def test_copy_blocks_on_fp8_caches():
    w = synth.random_decode(4, [40, 50], dtype=torch.bfloat16, hq=8, hkv=2, d=128, append=False,
                            fp8_scale=1.0 / 32)
    kc, vc = to_dev(w.key_cache), to_dev(w.value_cache)
    src = w.block_tables[0, :3].long()
    dst = w.free_blocks[:3].long()
    pa.pa_copy_blocks(kc, vc, to_dev(torch.stack([src, dst], 1)))
    want_k, want_v = w.key_cache.clone(), w.value_cache.clone()
    want_k[dst] = w.key_cache[src]
    want_v[dst] = w.value_cache[src]
    assert torch.equal(kc.cpu(), want_k) and torch.equal(vc.cpu(), want_v)


# (dtype, block size, q heads, kv heads): packed kv-head pairs (16-token
# blocks, G <= 4), unpacked 16-token blocks (G = 16), 32-token blocks
FUSED_SHAPES = [(torch.bfloat16, 16, 32, 8), (torch.float16, 16, 16, 1), (torch.bfloat16, 32, 16, 4)]


@pytest.mark.parametrize("dtype,B,hq,hkv", FUSED_SHAPES)
@pytest.mark.parametrize("partition_tokens", [0, 64])
def test_fused_append_decode_fp8_matches_three_calls(dtype, B, hq, hkv, partition_tokens):
    # One launch (pa_append_decode_fp8) against slot mapping + FP8 scatter +
    # FP8 decode: same cache bytes, same slots, same output bit for bit; and
    # the output against the oracle's FP8 decode of the appended pool.
    w = synth.random_decode(61 + B + hq, [0, 15, 16, 31, 100, 700], dtype=dtype, block_size=B,
                            hq=hq, hkv=hkv, d=128, append=True, fp8_scale=1.0 / 16)
    ctx = w.context_lens
    lens = (ctx + 1).tolist()
    q, nk, nv = to_dev(w.query), to_dev(w.new_key), to_dev(w.new_value)
    bt, cd = to_dev(w.block_tables), to_dev(ctx)
    mc = int(ctx.max())
    # three calls
    kc_a, vc_a = to_dev(w.key_cache), to_dev(w.value_cache)
    slots_a = torch.empty(w.num_seqs, dtype=torch.int64, device=dev())
    pa.pa_slot_mapping(slots_a, bt, cd, B)
    pa.pa_reshape_and_cache_fp8(nk, nv, kc_a, vc_a, slots_a, w.kv_scale, w.kv_scale)
    out_a = torch.empty_like(q)
    pa.pa_decode_fp8(out_a, q, kc_a, vc_a, bt, to_dev(torch.tensor(lens, dtype=torch.int32)),
                     mc + 1, w.scale, w.kv_scale, w.kv_scale, partition_tokens=partition_tokens)
    # one launch
    kc_b, vc_b = to_dev(w.key_cache), to_dev(w.value_cache)
    slots_b = torch.full((w.num_seqs,), -7, dtype=torch.int64, device=dev())
    out_b = torch.empty_like(q)
    pa.pa_append_decode_fp8(out_b, q, nk, nv, kc_b, vc_b, bt, cd, mc, w.scale, w.kv_scale,
                            w.kv_scale, slot_mapping=slots_b, partition_tokens=partition_tokens)
    torch.cuda.synchronize()
    assert torch.equal(slots_a, slots_b)
    assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    # oracle: the appended pool decoded in fp64
    w.key_cache, w.value_cache = kc_b.cpu(), vc_b.cpu()
    ref = fp8_reference(w, lens, list(range(w.num_seqs)))
    assert max_err(out_b.cpu(), ref) <= TOL[dtype]


# The FP8 ring holds 8 stages (at block size 16 a stage is one block of two
# packed KV heads, at 32 one block of one head); after the first 8 positions of
# an item each consumer warp refills the stage it has just consumed.  Items of
# about 1, 7, 8, 9, 15, 16, 17 and 33 blocks of 16 tokens, one partition per
# sequence, cover items shorter than the ring, exactly the ring, one past it,
# two rounds and more.
@pytest.mark.parametrize("B", [16, 32])
def test_fp8_ring_refill_around_the_ring_depth(B):
    stages = [1, 7, 8, 9, 15, 16, 17, 33]
    lens = [n * 16 - 3 for n in stages] + [n * 16 for n in stages]
    w = synth.random_decode(71 + B, lens, dtype=torch.bfloat16, block_size=B, hq=8, hkv=2,
                            d=128, append=False, fp8_scale=1.0 / 32)
    out = run(w, lens, partition_tokens=1024)  # one partition per sequence
    ref = fp8_reference(w, lens, list(range(w.num_seqs)))
    assert max_err(out, ref) <= TOL[w.dtype]
