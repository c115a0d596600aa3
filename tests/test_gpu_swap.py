"""pa_swap_blocks: swap blocks out to pinned host memory and back in to other
device blocks; bit-exact against the oracle's pool-to-pool copy, and decode
over the swapped-in blocks is bit-identical to decode before the swap."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_397_b200 as pa
import synth
from helpers import dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fp8", [False, True])
def test_swap_out_and_in_round_trip(fp8):
    pa.pa_get_device_error()
    lens = [40, 100, 17, 333]
    w = synth.random_decode(6, lens, dtype=torch.bfloat16, hq=8, hkv=2, d=128, append=False,
                            pool_factor=3.0, fp8_scale=(1 / 32) if fp8 else None)
    kc, vc, bt = to_dev(w.key_cache), to_dev(w.value_cache), to_dev(w.block_tables)
    ld = to_dev(torch.tensor(lens, dtype=torch.int32))

    def decode(table):
        out = torch.empty(w.query.shape, dtype=w.dtype, device=dev())
        if fp8:
            pa.pa_decode_fp8(out, to_dev(w.query), kc, vc, table, ld, max(lens), w.scale,
                             w.kv_scale, w.kv_scale)
        else:
            pa.pa_decode(out, to_dev(w.query), kc, vc, table, ld, max(lens), w.scale)
        torch.cuda.synchronize()
        return out

    before = decode(bt)
    # swap out sequence 3's blocks to a pinned host pool
    n3 = -(-lens[3] // 16)
    src = w.block_tables[3, :n3].long()
    host_k = torch.zeros((n3 + 2,) + tuple(w.key_cache.shape[1:]), dtype=w.key_cache.dtype,
                         pin_memory=True)
    host_v = torch.zeros_like(host_k).pin_memory()
    out_pairs = torch.stack([src, torch.arange(n3) + 2], 1)
    pa.pa_swap_blocks(host_k, host_v, kc, vc, to_dev(out_pairs))
    torch.cuda.synchronize()
    hk = np.zeros_like(host_k.view(torch.uint8).numpy())
    hv = np.zeros_like(hk)
    oracle.swap_blocks(hk, hv, w.key_cache.view(torch.uint8).numpy(),
                       w.value_cache.view(torch.uint8).numpy(), out_pairs.numpy())
    np.testing.assert_array_equal(host_k.view(torch.uint8).numpy(), hk)
    np.testing.assert_array_equal(host_v.view(torch.uint8).numpy(), hv)
    # the device blocks are reused by someone else (poisoned), then swap back
    # in to free blocks and remap the table
    kc[src.to(dev())] = 0x7F if fp8 else float("nan")
    vc[src.to(dev())] = 0x7F if fp8 else float("nan")
    dst = w.free_blocks[:n3].long()
    in_pairs = torch.stack([torch.arange(n3) + 2, dst], 1)
    pa.pa_swap_blocks(kc, vc, host_k, host_v, to_dev(in_pairs))
    bt2 = bt.clone()
    bt2[3, :n3] = dst.to(dev()).int()
    after = decode(bt2)
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))
    assert pa.pa_get_device_error() == 0
