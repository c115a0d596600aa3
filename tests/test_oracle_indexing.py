"""Pins the oracle's slot indexing and its bit-copy cache writes."""
import numpy as np
import torch

import oracle
import synth


def _golden_tables(golden):
    rows = golden("block_table_example.txt")
    B = int(rows[0][1])
    seqs = [(int(t), [int(x) for x in tab.split(",")]) for t, _n, tab in rows[1:]]
    width = max(len(t) for _, t in seqs)
    bt = np.full((len(seqs), width), -1, dtype=np.int64)
    for s, (_, tab) in enumerate(seqs):
        bt[s, :len(tab)] = tab
    return B, seqs, bt


def test_slots_of_the_worked_example(golden):
    B, seqs, bt = _golden_tables(golden)
    for s, (tokens, tab) in enumerate(seqs):
        pos = np.arange(tokens)
        slots = oracle.logical_positions_to_slots(bt, np.full(tokens, s), pos, B)
        # the i-th token sits in the (i // 16)-th listed physical block
        for p in range(tokens):
            assert slots[p] // B == tab[p // B]
            assert slots[p] % B == p % B
        # distinct slots, all inside the listed blocks
        assert len(set(slots.tolist())) == tokens
    # spot values: seq 0 token 17 -> block 25, offset 1; seq 1 token 49 -> block 18, offset 1
    assert oracle.logical_positions_to_slots(bt, [0], [17], B)[0] == 25 * 16 + 1
    assert oracle.logical_positions_to_slots(bt, [1], [49], B)[0] == 18 * 16 + 1
    assert oracle.logical_positions_to_slots(bt, [1], [0], B)[0] == 3 * 16


def test_write_then_gather_round_trip():
    # a pool of token ids: writing token t through its slot and gathering the
    # sequence back through its table returns 0..L-1 in order
    rng = np.random.default_rng(0)
    for B in (16, 32):
        lens = [1, B - 1, B, B + 1, 3 * B + 5]
        nblk = sum(-(-L // B) for L in lens) + 4
        perm = rng.permutation(nblk)
        bt = np.full((len(lens), 8), -1, dtype=np.int64)
        pos = 0
        for s, L in enumerate(lens):
            n = -(-L // B)
            bt[s, :n] = perm[pos:pos + n]
            pos += n
        kc = np.full((nblk, 1, B, 1), -7.0)
        vc = np.full((nblk, 1, B, 1), -7.0)
        for s, L in enumerate(lens):
            ids = np.arange(L, dtype=np.float64)
            slots = oracle.logical_positions_to_slots(bt, np.full(L, s), np.arange(L), B)
            oracle.reshape_and_cache(kc, vc, ids.reshape(L, 1, 1), -ids.reshape(L, 1, 1), slots, B)
            k = oracle.gather_logical(kc, bt[s], L, 0, B)[:, 0]
            v = oracle.gather_logical(vc, bt[s], L, 0, B)[:, 0]
            np.testing.assert_array_equal(k, ids)
            np.testing.assert_array_equal(v, -ids)


def test_reshape_and_cache_bits_and_skip():
    w = synth.tiny_decode()
    kc = w.key_cache.view(torch.int16).numpy().copy()
    vc = w.value_cache.view(torch.int16).numpy().copy()
    k0, v0 = kc.copy(), vc.copy()
    nk = w.new_key.view(torch.int16).numpy()
    nv = w.new_value.view(torch.int16).numpy()
    B = w.block_size
    slots = oracle.logical_positions_to_slots(w.block_tables.numpy(), np.arange(w.num_seqs),
                                              w.context_lens.numpy(), B)
    slots[2] = -1  # skipped token
    oracle.reshape_and_cache(kc, vc, nk, nv, slots, B)
    touched = np.zeros(kc.shape, dtype=bool)
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        b, off = slot // B, slot % B
        np.testing.assert_array_equal(kc[b, :, off, :], nk[t])
        np.testing.assert_array_equal(vc[b, :, off, :], nv[t])
        touched[b, :, off, :] = True
    np.testing.assert_array_equal(kc[~touched], k0[~touched])
    np.testing.assert_array_equal(vc[~touched], v0[~touched])


def test_copy_blocks_bits():
    w = synth.tiny_decode()
    kc = w.key_cache.view(torch.int16).numpy().copy()
    vc = w.value_cache.view(torch.int16).numpy().copy()
    k0, v0 = kc.copy(), vc.copy()
    src = w.block_tables[0, :2].numpy().astype(np.int64)
    dst = w.free_blocks[:2].numpy().astype(np.int64)
    oracle.copy_blocks(kc, vc, np.stack([src, dst], 1))
    for s_, d_ in zip(src, dst):
        np.testing.assert_array_equal(kc[d_], k0[s_])
        np.testing.assert_array_equal(vc[d_], v0[s_])
    others = np.setdiff1d(np.arange(kc.shape[0]), dst)
    np.testing.assert_array_equal(kc[others], k0[others])
    np.testing.assert_array_equal(vc[others], v0[others])


def test_swap_blocks_copies_between_pools_only_the_listed_blocks():
    rng = np.random.default_rng(8)
    dev_k = rng.integers(-5000, 5000, (10, 2, 16, 8)).astype(np.int16)
    dev_v = rng.integers(-5000, 5000, (10, 2, 16, 8)).astype(np.int16)
    host_k = np.zeros((4, 2, 16, 8), np.int16)
    host_v = np.zeros((4, 2, 16, 8), np.int16)
    pairs = np.array([[7, 0], [2, 3], [9, 1]])
    oracle.swap_blocks(host_k, host_v, dev_k, dev_v, pairs)      # swap out
    for s, d in pairs:
        np.testing.assert_array_equal(host_k[d], dev_k[s])
        np.testing.assert_array_equal(host_v[d], dev_v[s])
    assert not host_k[2].any() and not host_v[2].any()
    back_k, back_v = np.zeros_like(dev_k), np.zeros_like(dev_v)
    oracle.swap_blocks(back_k, back_v, host_k, host_v, pairs[:, ::-1])  # swap back in
    for s, _ in pairs:
        np.testing.assert_array_equal(back_k[s], dev_k[s])
        np.testing.assert_array_equal(back_v[s], dev_v[s])
