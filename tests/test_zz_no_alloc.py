"""pa_decode_static_workspace: decode for callers that cannot allocate device memory.

Some callers of this library may not call cudaMalloc — a plugin inside an
inference runtime that owns and budgets every byte of device memory, or a
serving loop that must not allocate after start-up.  This entry point keeps
pa_decode's split-KV scratch in the library's own per-device array instead of
a caller workspace.

The test calls it through the C ABI (ctypes) twice in a row, on two different
batches whose partial results have different shapes (sequence count,
partitions per sequence, hence the row stride inside the shared array), so a
reduce that read partials left over from the first call would be caught.
Each result must equal pa_decode with a caller-provided workspace and the same
partition length bit for bit (the same kernels run on the same inputs), and
must match the fp64 oracle within the decode tolerance.  A request needing more
scratch than the array holds must be refused up front.

The file is named to be collected last, so a run that stops at the first
failure has already run every other test; it passes alone in a fresh process
as well.
"""
import ctypes

import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth
from helpers import TOL, decode_reference, dev, max_err, to_dev

pytestmark = pytest.mark.gpu


def _c_call(out, q, kc, vc, bt, lens, max_len, scale, partition_tokens):
    nb, hkv, bs, d = (int(x) for x in kc.shape)
    return pa.lib().pa_decode_static_workspace(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(q.data_ptr()),
        ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
        ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(lens.data_ptr()), int(q.shape[0]),
        int(q.shape[1]), hkv, d, bs, nb, int(bt.shape[1]), int(max_len), int(partition_tokens),
        float(scale), pa.PA_BF16 if kc.dtype == torch.bfloat16 else pa.PA_F16,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


# Two batches in a row: 8 sequences x 17 partitions of 256 tokens, then 5
# sequences x 16 partitions of 128 tokens (a different partial-row layout).
CALLS = [
    dict(seed=42, lens=[1, 16, 17, 300, 1000, 2049, 3000, 4097], pt=256),
    dict(seed=43, lens=[2000, 50, 1, 700, 1500], pt=128),
]


def test_static_workspace_matches_pa_decode_on_two_calls():
    pa.pa_get_device_error()
    parts_seen = set()
    for c in CALLS:
        lens, pt = c["lens"], c["pt"]
        w = synth.random_decode(c["seed"], lens, dtype=torch.bfloat16, block_size=16, hq=32,
                                hkv=8, d=128, append=False)
        need = pa.pa_decode_workspace_size(w.num_seqs, 32, 8, 128, 16, max(lens), pt)
        assert 0 < need <= pa.PA_STATIC_WORKSPACE_BYTES
        parts_seen.add((w.num_seqs, -(-max(lens) // pt)))
        kc, vc, bt = to_dev(w.key_cache), to_dev(w.value_cache), to_dev(w.block_tables)
        ld = to_dev(torch.tensor(lens, dtype=torch.int32))
        q = to_dev(w.query)
        want = torch.empty_like(q)
        pa.pa_decode(want, q, kc, vc, bt, ld, max(lens), w.scale, partition_tokens=pt)
        got = torch.full_like(q, float("nan"))
        st = _c_call(got, q, kc, vc, bt, ld, max(lens), w.scale, pt)
        assert st == pa.PA_OK, pa.pa_status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
        ref = decode_reference(w, lens, list(range(w.num_seqs)))
        assert max_err(got.cpu(), ref) <= TOL[w.dtype]
    assert len(parts_seen) == 2  # the two calls really lay the scratch out differently
    assert pa.pa_get_device_error() == 0


def test_static_workspace_refuses_oversized_requests():
    # 4096 sequences x 32 heads x 128 partitions of scratch is far beyond the array
    need = pa.pa_decode_workspace_size(4096, 32, 8, 128, 16, 32768, 256)
    assert need > pa.PA_STATIC_WORKSPACE_BYTES
    q = torch.empty(4096, 32, 128, dtype=torch.bfloat16, device=dev())
    kc = torch.empty(8, 8, 16, 128, dtype=torch.bfloat16, device=dev())
    bt = torch.zeros(4096, 2048, dtype=torch.int32, device=dev())
    ld = torch.zeros(4096, dtype=torch.int32, device=dev())
    st = _c_call(torch.empty_like(q), q, kc, kc, bt, ld, 32768, 0.1, 256)
    assert st == pa.PA_ERR_WORKSPACE
