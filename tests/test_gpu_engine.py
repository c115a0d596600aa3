"""End to end on the GPU, driven by the host block manager: prompts that
share prefixes (prefix-cache hits), forks (parallel sampling), decode steps
that append through copy-on-write, and after every step pa_decode over the
paged cache compared with plain dense attention computed straight from each
sequence's token list — no block table on the reference side.  K/V of a
token are a fixed function of its token id, so shared prefixes really are
byte-identical ("PagedAttention: KV cache as virtual memory", "Deep dive":
KV is byte-identical so outputs are unchanged)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_397_b200 as pa
from helpers import TOL, dev

pytestmark = pytest.mark.gpu

VOCAB, HQ, HKV, D, B = 4096, 8, 2, 128, 16


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_block_manager_drives_decode_with_sharing_and_cow(dtype):
    pa.pa_get_device_error()
    g = torch.Generator().manual_seed(17)
    ktab = torch.randn(VOCAB, HKV, D, generator=g).to(dtype)   # K/V of each token id
    vtab = torch.randn(VOCAB, HKV, D, generator=g).to(dtype)
    kt_d, vt_d = ktab.to(dev()), vtab.to(dev())
    rng = np.random.default_rng(17)
    nb = 400
    bm = pa.BlockManager(nb, B)
    kc = torch.zeros(nb, HKV, B, D, dtype=dtype, device=dev())
    vc = torch.zeros_like(kc)
    seqs = {}  # id -> token list

    def write(sid, start, toks):
        slots = torch.from_numpy(bm.slots(sid, start, len(toks))).to(dev())
        t = torch.as_tensor(np.asarray(toks), dtype=torch.long, device=dev())
        pa.pa_reshape_and_cache(kt_d[t].contiguous(), vt_d[t].contiguous(), kc, vc, slots)

    prefixes = [rng.integers(0, VOCAB, n).tolist() for n in (40, 64, 100)]
    sid = 0
    for fam in range(3):
        for k in range(3):
            toks = prefixes[fam] + rng.integers(0, VOCAB, int(rng.integers(1, 30))).tolist()
            cached = bm.add_sequence(sid, toks)
            assert cached == ((len(prefixes[fam]) // B) * B if k > 0 else 0)
            write(sid, cached, toks[cached:])   # hit tokens are already in the cache
            seqs[sid] = toks
            sid += 1
    for parent in (0, 4, 8):                    # parallel samples share everything
        bm.fork(parent, sid)
        seqs[sid] = list(seqs[parent])
        sid += 1

    for step in range(12):
        ids = sorted(seqs)
        new = {s: int(rng.integers(0, VOCAB)) for s in ids}
        for s in ids:
            bm.append(s, [new[s]])
        pairs = bm.take_copies()
        if len(pairs):
            pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).to(dev()))
        for s in ids:
            write(s, len(seqs[s]), [new[s]])
            seqs[s].append(new[s])
        width = max(len(bm.block_table(s)) for s in ids)
        bt = torch.from_numpy(np.stack([bm.block_table(s, width) for s in ids])).to(dev())
        lens = torch.tensor([len(seqs[s]) for s in ids], dtype=torch.int32, device=dev())
        q = torch.randn(len(ids), HQ, D, generator=g).to(dtype)
        out = torch.empty(len(ids), HQ, D, dtype=dtype, device=dev())
        pa.pa_decode(out, q.to(dev()), kc, vc, bt, lens, int(lens.max()), D ** -0.5,
                     partition_tokens=32)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        for r, s in enumerate(ids):
            t = np.asarray(seqs[s])
            K = ktab[t].double().numpy()        # dense, straight from the token list
            V = vtab[t].double().numpy()
            for h in range(HQ):
                want = oracle.attention(q[r, h].double().numpy()[None], K[:, h // (HQ // HKV)],
                                        V[:, h // (HQ // HKV)], D ** -0.5)[0]
                assert np.abs(got[r, h] - want).max() <= TOL[dtype]
    assert pa.pa_get_device_error() == 0
    for s in list(seqs):
        bm.free(s)
    assert bm.num_free_blocks == nb
