"""pa_prefill_chunk (tcgen05) against the fp64 oracle: ragged chunks and
contexts across several 128-row / 128-key tiles, both block sizes, both
16-bit types and head_dim 128 and 64, NaN in unused slots, the full-size
8 x 512-token chunk workload on sampled rows, and bit-identical output under a
relabelling of the physical blocks, with and without the key-range split of
the last wave."""
import dataclasses

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


def run_prefill(p, split_tail=True):
    """Slot mapping + scatter of the chunk K/V, then the chunk attention (GPU);
    with split_tail the units of the last wave are split along the key range."""
    kc, vc = to_dev(p.key_cache), to_dev(p.value_cache)
    bt, cl, cu = to_dev(p.block_tables), to_dev(p.ctx_lens), to_dev(p.cu_q_lens)
    slots = torch.empty(p.total_q, dtype=torch.int64, device=dev())
    pa.pa_slot_mapping(slots, bt, cl, p.block_size, cu_q_lens=cu)
    pa.pa_reshape_and_cache(to_dev(p.new_key), to_dev(p.new_value), kc, vc, slots)
    out = torch.full(p.query.shape, float("nan"), dtype=p.dtype, device=dev())
    qlens = np.diff(p.cu_q_lens.numpy())
    pa.pa_prefill_chunk(out, to_dev(p.query), kc, vc, bt, cu, cl, int(qlens.max()),
                        int(p.ctx_lens.max()), p.scale, split_tail=split_tail)
    torch.cuda.synchronize()
    return out.cpu()


oracle_scatter = oracle_scatter_chunks
reference = chunk_reference


@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
@pytest.mark.parametrize("split_tail", [True, False])
def test_ragged_chunks_match_oracle(B, dtype, hq, hkv, split_tail):
    # 2 tiles x hq x 5 sequences = 40 or 80 units: with 4 heads the 40 units
    # are split three ways along the key range, some parts empty (short keys)
    ctx = [0, 5, 40, 200, 129]
    qn = [1, 130, 7, 300, 256]
    p = synth.chunked_prefill(seed=B + hq, block_size=B, hq=hq, hkv=hkv, d=128, dtype=dtype,
                              ctx_lens=ctx, q_lens=qn)
    out = run_prefill(p, split_tail)
    oracle_scatter(p)
    ref, _ = reference(p)
    assert max_err(out, ref) <= TOL[dtype]


@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("split_tail", [True, False])
def test_head_dim_64_matches_oracle(B, dtype, split_tail):
    # the same ragged batch at head_dim 64 (one 64-column half per row, 8-stage
    # ring, PV products N = 64): 2 tiles x 8 heads x 5 sequences = 80 units
    ctx = [0, 5, 40, 200, 129]
    qn = [1, 130, 7, 300, 256]
    p = synth.chunked_prefill(seed=B + 64, block_size=B, hq=8, hkv=2, d=64, dtype=dtype,
                              ctx_lens=ctx, q_lens=qn)
    out = run_prefill(p, split_tail)
    oracle_scatter(p)
    ref, _ = reference(p)
    assert torch.isfinite(out.float()).all()
    assert max_err(out, ref) <= TOL[dtype]


def test_head_dim_64_long_context_split_tail():
    # one sequence over 8192 + 512 keys at head_dim 64: 16 units, each split
    # four ways, so the partial rows (D / 4 float4 per row) and their combine
    # run at head_dim 64 too
    p = synth.chunked_prefill(seed=13, block_size=16, num_seqs=1, hq=8, hkv=2, d=64)
    a = run_prefill(p, split_tail=True)
    b = run_prefill(p, split_tail=False)
    oracle_scatter(p)
    rows = [0, 1, 127, 128, 255, 256, 300, 511]
    ref, _ = reference(p, rows=rows)
    assert max_err(a[rows], ref[rows]) <= TOL[p.dtype]
    assert max_err(b[rows], ref[rows]) <= TOL[p.dtype]


def test_nan_in_unused_slots_does_not_leak():
    p = synth.chunked_prefill(seed=7, block_size=16, hq=8, hkv=2, d=128, ctx_lens=[3, 50],
                              q_lens=[20, 77])
    B = p.block_size
    lens = (p.ctx_lens + torch.diff(p.cu_q_lens)).tolist()
    for s, L in enumerate(lens):  # poison the tail of each sequence's last block
        last = int(p.block_tables[s, (L - 1) // B])
        if L % B:
            p.key_cache[last, :, L % B:] = float("nan")
            p.value_cache[last, :, L % B:] = float("nan")
    out = run_prefill(p)
    oracle_scatter(p)
    ref, _ = reference(p)
    assert max_err(out, ref) <= TOL[p.dtype]


@pytest.mark.parametrize("B", [16, 32])
def test_full_size_chunked_prefill_sampled_rows(B):
    p = synth.chunked_prefill(block_size=B)
    out = run_prefill(p)
    oracle_scatter(p)
    rows = [0, 1, 63, 127, 128, 200, 255, 256, 383, 384, 510, 511]
    seqs = [0, 5, 7]  # 512 units on 148 SMs: the last 68 (sequence 7 and two heads of 6) split
    ref, sub_cu = reference(p, seqs=seqs, rows=rows)
    cu = p.cu_q_lens.numpy()
    got = torch.cat([out[cu[s] + np.array(rows)] for s in seqs])
    want = np.concatenate([ref[sub_cu[i] + np.array(rows)] for i in range(len(seqs))])
    assert max_err(got, want) <= TOL[p.dtype]
    assert torch.isfinite(out.float()).all()


def test_split_tail_long_context_matches_oracle():
    # one sequence, 2 tiles x 8 heads = 16 units, each split four ways over
    # 8192 + 512 keys (17 key tiles per part on average)
    p = synth.chunked_prefill(seed=11, block_size=16, num_seqs=1, hq=8, hkv=2)
    a = run_prefill(p, split_tail=True)
    b = run_prefill(p, split_tail=False)
    oracle_scatter(p)
    rows = [0, 1, 127, 128, 255, 256, 300, 511]
    ref, _ = reference(p, rows=rows)
    assert max_err(a[rows], ref[rows]) <= TOL[p.dtype]
    assert max_err(b[rows], ref[rows]) <= TOL[p.dtype]
    # the two differ only in fp32 rounding order
    assert (a.float() - b.float()).abs().max().item() <= TOL[p.dtype]


def test_split_tail_is_deterministic():
    # 1 sequence x 2 tiles x 8 heads = 16 units, split 4 ways: whichever part
    # finishes last combines in part order, so repeated runs agree bit for bit
    p = synth.chunked_prefill(seed=12, block_size=32, num_seqs=1, hq=8, hkv=2)
    runs = [run_prefill(p, split_tail=True) for _ in range(3)]
    for r in runs[1:]:
        assert torch.equal(r.view(torch.int16), runs[0].view(torch.int16))


def _relabelled(p, seed):
    """The same chunk batch with every physical block moved to a new id
    (block b -> perm[b]); the tables follow, so the logical K/V are unchanged."""
    perm = torch.randperm(p.num_blocks, generator=torch.Generator().manual_seed(seed))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(p.num_blocks)
    bt = p.block_tables.clone()
    bt[bt >= 0] = perm[bt[bt >= 0].long()].to(bt.dtype)
    return dataclasses.replace(p, key_cache=p.key_cache[inv].contiguous(),
                               value_cache=p.value_cache[inv].contiguous(), block_tables=bt)


# Work units = 256-row tiles x query heads x sequences; on 148 SMs the units of
# the last wave are cut along the key range into k parts: 16 units -> k = 4,
# 40 units -> k = 3, 64 units -> k = 2 (k minimises ceil(units * k / 148) / k).
RELABEL_CASES = {
    "split4": dict(hq=4, hkv=2, ctx_lens=[700, 3], q_lens=[300, 257]),
    "split3": dict(hq=4, hkv=4, ctx_lens=[0, 5, 40, 900, 129], q_lens=[1, 130, 7, 300, 256]),
    "split2": dict(hq=8, hkv=2, ctx_lens=[1000, 17, 260, 64], q_lens=[511, 300, 2, 129]),
}


@pytest.mark.parametrize("case", sorted(RELABEL_CASES))
@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("d", [128, 64])
def test_prefill_bit_identical_under_block_relabelling(case, B, dtype, d):
    # The result may depend only on logical positions, never on where the
    # blocks sit in the pool ("vLLM PagedAttention Deep Dive", "PagedAttention
    # Mechanism"): with and without the key-range split of the last wave.
    p = synth.chunked_prefill(seed=31 + B, block_size=B, dtype=dtype, d=d,
                              **RELABEL_CASES[case])
    moved = _relabelled(p, seed=5 + B)
    for split_tail in (True, False):
        a = run_prefill(p, split_tail)
        b = run_prefill(moved, split_tail)
        assert torch.isfinite(a.float()).all()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), (case, split_tail)
    oracle_scatter(p)
    ref, _ = reference(p)
    assert max_err(a, ref) <= TOL[dtype]
