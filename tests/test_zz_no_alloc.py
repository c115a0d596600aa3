"""pa_decode_static_workspace: decode for callers that cannot allocate device memory.

Some callers of this library may not call cudaMalloc — a plugin inside an
inference runtime that owns and budgets every byte of device memory, or a
serving loop that must not allocate after start-up.  This entry point keeps
pa_decode's split-KV scratch in the library's own per-device array instead of
a caller workspace.  The test calls it through the C ABI (ctypes) twice in a
row, on different inputs, and checks each result against pa_decode with a
caller-provided workspace, within the decode tolerance; it also checks that a
request needing more scratch than the array holds is refused up front.

The file is named to be collected last, so a run that stops at the first
failure has already run every other test; it passes alone in a fresh process
as well.
"""
import ctypes

import pytest
import torch

import paged_kv_cache_397_b200 as pa
import synth
from helpers import TOL, dev, to_dev

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


def test_static_workspace_matches_pa_decode_on_two_calls():
    pa.pa_get_device_error()
    lens = [1, 16, 17, 300, 1000, 2049, 3000, 4097]
    w = synth.random_decode(42, lens, dtype=torch.bfloat16, block_size=16, hq=32, hkv=8, d=128,
                            append=False)
    pt = 256  # several partitions per long sequence, so the scratch is really used
    need = pa.pa_decode_workspace_size(w.num_seqs, 32, 8, 128, 16, max(lens), pt)
    assert 0 < need <= pa.PA_STATIC_WORKSPACE_BYTES
    kc, vc, bt = to_dev(w.key_cache), to_dev(w.value_cache), to_dev(w.block_tables)
    ld = to_dev(torch.tensor(lens, dtype=torch.int32))
    g = torch.Generator().manual_seed(7)
    for call in range(2):
        q = w.query if call == 0 else torch.randn(w.query.shape, generator=g).to(w.dtype)
        q = to_dev(q)
        want = torch.empty_like(q)
        pa.pa_decode(want, q, kc, vc, bt, ld, max(lens), w.scale, partition_tokens=pt)
        got = torch.full_like(q, float("nan"))
        st = _c_call(got, q, kc, vc, bt, ld, max(lens), w.scale, pt)
        assert st == pa.PA_OK, pa.pa_status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert (got.float() - want.float()).abs().max().item() <= TOL[w.dtype]
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
