"""pa_mixed_attention: decode rows and prefill chunks in one launch.

Against the fp64 oracle (the chunk rule of "vLLM PagedAttention Deep Dive",
"Mechanics of Chunked Prefill", which covers a decode row as a one-row
chunk), bit-identical to running pa_decode and pa_prefill_chunk (without the
key-range split of its last wave) separately on the two halves of the batch, bit-identical under relabelling of physical
blocks, and at the full mixed workload (256 decode rows + 4 x 512-row chunks
over 8192 cached tokens) on sampled rows against the oracle and on every row
against the two calls."""
import numpy as np
import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth
from helpers import TOL, chunk_reference, dev, max_err, oracle_scatter_chunks, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.pa_get_device_error()
    yield
    assert pa.pa_get_device_error() == 0


def _max_q(p):
    q = np.diff(p.cu_q_lens.numpy())[p.num_decode:]
    return int(q.max()) if q.size else 0


def gpu_inputs(p):
    """Device copies with every query row's own K/V appended (pa_append)."""
    d = dict(kc=to_dev(p.key_cache), vc=to_dev(p.value_cache), bt=to_dev(p.block_tables),
             cl=to_dev(p.ctx_lens), cu=to_dev(p.cu_q_lens), q=to_dev(p.query))
    pa.pa_append(to_dev(p.new_key), to_dev(p.new_value), d["kc"], d["vc"], d["bt"], d["cl"],
                 cu_q_lens=d["cu"])
    return d


def run_mixed(p, d, partition_tokens=0):
    out = torch.full(p.query.shape, float("nan"), dtype=p.dtype, device=dev())
    pa.pa_mixed_attention(out, d["q"], d["kc"], d["vc"], d["bt"], d["cu"], d["cl"], p.num_decode,
                          _max_q(p), int(p.ctx_lens.max()), p.scale,
                          partition_tokens=partition_tokens)
    torch.cuda.synchronize()
    return out


def run_separately(p, d, partition_tokens=0):
    """pa_decode on the decode rows, pa_prefill_chunk on the chunks."""
    out = torch.full(p.query.shape, float("nan"), dtype=p.dtype, device=dev())
    nd, max_ctx = p.num_decode, int(p.ctx_lens.max())
    if nd:
        pa.pa_decode(out[:nd], d["q"][:nd], d["kc"], d["vc"], d["bt"][:nd].contiguous(),
                     (d["cl"][:nd] + 1).contiguous(), max_ctx + 1, p.scale,
                     partition_tokens=partition_tokens)
    if nd < p.num_seqs:
        r0 = int(p.cu_q_lens[nd])
        cu = (d["cu"][nd:] - r0).contiguous()
        pa.pa_prefill_chunk(out[r0:], d["q"][r0:].contiguous(), d["kc"], d["vc"],
                            d["bt"][nd:].contiguous(), cu, d["cl"][nd:].contiguous(),
                            max(1, _max_q(p)), max_ctx, p.scale, split_tail=False)
    torch.cuda.synchronize()
    return out


def small_batch(seed, B, dtype, hq, hkv, decode_ctx=(0, 1, 15, 16, 17, 100, 500, 1000),
                prefill_ctx=(0, 17, 300, 40), prefill_q=(40, 1, 257, 0)):
    return synth.mixed_batch(seed=seed, block_size=B, hq=hq, hkv=hkv, d=128, dtype=dtype,
                             decode_ctx=list(decode_ctx), prefill_ctx=list(prefill_ctx),
                             prefill_q=list(prefill_q))


@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("hq,hkv", [(8, 2), (16, 1)])
@pytest.mark.parametrize("partition_tokens", [0, 64])
def test_mixed_matches_oracle(B, dtype, hq, hkv, partition_tokens):
    p = small_batch(30 + B + hq, B, dtype, hq, hkv)
    d = gpu_inputs(p)
    out = run_mixed(p, d, partition_tokens).cpu()
    oracle_scatter_chunks(p)
    ref, _ = chunk_reference(p)
    assert max_err(out, ref) <= TOL[dtype]


@pytest.mark.parametrize("decode_ctx,prefill_ctx,prefill_q", [
    ((0, 1, 15, 16, 17, 100, 500, 1000), (0, 17, 300, 40), (40, 1, 257, 0)),
    ((3, 700, 2000), (), ()),                        # decode rows only
    ((), (0, 129, 1000), (600, 128, 3)),             # prefill chunks only
    ((63,), (5,), (1,)),                             # a one-row chunk after a decode row
])
def test_mixed_is_bitwise_the_two_calls(decode_ctx, prefill_ctx, prefill_q):
    p = small_batch(41, 16, torch.bfloat16, 8, 2, decode_ctx, prefill_ctx, prefill_q)
    d = gpu_inputs(p)
    for pt in (32, 256):  # the same explicit partition length for both
        a = run_mixed(p, d, pt)
        b = run_separately(p, d, pt)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("num_decode,prefill_ctx,prefill_q", [
    (256, (8192,) * 4, (512,) * 4),   # the full mixed workload: every row compared
    (6, (0, 900, 3000), (512, 300, 600)),  # more tiles than the leading share, few decode items
    (300, (100,), (1,)),               # decode CTAs beyond the early share, one tile
])
def test_mixed_launch_order_is_bitwise_the_two_calls(num_decode, prefill_ctx, prefill_q):
    # Grid order: a leading share of prefill tiles, decode CTAs started beside
    # them, the remaining tiles, then the rest of the decode CTAs (all in CTA
    # pairs).  Every row must still equal the separate calls bit for bit.
    p = synth.mixed_batch(seed=71, num_decode=num_decode, prefill_ctx=list(prefill_ctx),
                          prefill_q=list(prefill_q))
    d = gpu_inputs(p)
    a = run_mixed(p, d, 1024)
    b = run_separately(p, d, 1024)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_mixed_odd_tile_count():
    # 5 query heads over one KV head: an odd number of prefill tiles, so the
    # last CTA pair holds one tile and one spare slot
    p = small_batch(83, 16, torch.bfloat16, 5, 1, decode_ctx=(7, 300, 2500), prefill_ctx=(40,),
                    prefill_q=(200,))
    d = gpu_inputs(p)
    a = run_mixed(p, d, 256)
    b = run_separately(p, d, 256)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    oracle_scatter_chunks(p)
    ref, _ = chunk_reference(p)
    assert max_err(a.cpu(), ref) <= TOL[p.dtype]


def test_mixed_bit_identical_under_block_relabelling():
    p = small_batch(52, 16, torch.bfloat16, 8, 2)
    out_a = run_mixed(p, gpu_inputs(p)).cpu()
    # move every block to a new physical id; tables follow
    perm = torch.randperm(p.num_blocks, generator=torch.Generator().manual_seed(9))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(p.num_blocks)
    p.key_cache = p.key_cache[inv].contiguous()
    p.value_cache = p.value_cache[inv].contiguous()
    bt = p.block_tables.clone()
    bt[bt >= 0] = perm[bt[bt >= 0].long()].to(bt.dtype)
    p.block_tables = bt
    out_b = run_mixed(p, gpu_inputs(p)).cpu()
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


def test_mixed_full_size_sampled_rows():
    p = synth.mixed_batch()  # 256 decode rows + 4 chunks of 512 rows over 8192 tokens, bf16
    d = gpu_inputs(p)
    out = run_mixed(p, d).cpu()
    assert torch.isfinite(out.float()).all()
    oracle_scatter_chunks(p)
    rng = np.random.default_rng(0)
    dec = sorted(set(rng.choice(p.num_decode, 6, replace=False).tolist()) | {0, p.num_decode - 1})
    ref, sub_cu = chunk_reference(p, seqs=dec)
    assert max_err(out[dec], ref) <= TOL[p.dtype]
    cu = p.cu_q_lens.numpy()
    rows = [0, 1, 127, 128, 255, 256, 383, 511]
    for s in (p.num_decode, p.num_seqs - 1):
        ref, sub_cu = chunk_reference(p, seqs=[s], rows=rows)
        got = out[torch.as_tensor(cu[s] + np.asarray(rows))]
        assert max_err(got, ref[rows]) <= TOL[p.dtype]


def test_mixed_flags_a_decode_sequence_with_several_rows():
    # sequence 1 is declared a decode row but owns two query rows
    p = synth.mixed_batch(seed=8, num_decode=0, hq=8, hkv=2, prefill_ctx=[10, 20, 30],
                          prefill_q=[1, 2, 1])
    d = gpu_inputs(p)
    out = torch.zeros(p.query.shape, dtype=p.dtype, device=dev())
    pa.pa_mixed_attention(out, d["q"], d["kc"], d["vc"], d["bt"], d["cu"], d["cl"], 2, 1, 30,
                          p.scale)
    assert pa.pa_get_device_error() & pa.PA_DEVERR_SEQ_RANGE
