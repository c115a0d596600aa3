"""pa_prefill_chunk (tcgen05) against the fp64 oracle: ragged chunks and
contexts across several 128-row / 128-key tiles, both block sizes and both
16-bit types, NaN in unused slots, and the full-size 8 x 512-token chunk
workload on sampled rows."""
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


def run_prefill(p):
    """Slot mapping + scatter of the chunk K/V, then the chunk attention (GPU)."""
    kc, vc = to_dev(p.key_cache), to_dev(p.value_cache)
    bt, cl, cu = to_dev(p.block_tables), to_dev(p.ctx_lens), to_dev(p.cu_q_lens)
    slots = torch.empty(p.total_q, dtype=torch.int64, device=dev())
    pa.pa_slot_mapping(slots, bt, cl, p.block_size, cu_q_lens=cu)
    pa.pa_reshape_and_cache(to_dev(p.new_key), to_dev(p.new_value), kc, vc, slots)
    out = torch.full(p.query.shape, float("nan"), dtype=p.dtype, device=dev())
    qlens = np.diff(p.cu_q_lens.numpy())
    pa.pa_prefill_chunk(out, to_dev(p.query), kc, vc, bt, cu, cl, int(qlens.max()),
                        int(p.ctx_lens.max()), p.scale)
    torch.cuda.synchronize()
    return out.cpu()


oracle_scatter = oracle_scatter_chunks
reference = chunk_reference


@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_ragged_chunks_match_oracle(B, dtype, hq, hkv):
    ctx = [0, 5, 40, 200, 129]
    qn = [1, 130, 7, 300, 256]
    p = synth.chunked_prefill(seed=B + hq, block_size=B, hq=hq, hkv=hkv, d=128, dtype=dtype,
                              ctx_lens=ctx, q_lens=qn)
    out = run_prefill(p)
    oracle_scatter(p)
    ref, _ = reference(p)
    assert max_err(out, ref) <= TOL[dtype]


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
    seqs = [0, 5]
    ref, sub_cu = reference(p, seqs=seqs, rows=rows)
    cu = p.cu_q_lens.numpy()
    got = torch.cat([out[cu[s] + np.array(rows)] for s in seqs])
    want = np.concatenate([ref[sub_cu[i] + np.array(rows)] for i in range(len(seqs))])
    assert max_err(got, want) <= TOL[p.dtype]
    assert torch.isfinite(out.float()).all()
