"""Pins the oracle's attention against things other than itself.

* paged == dense: torch's scaled_dot_product_attention (fp64, CPU) on the dense
  K/V, the pages' claim that paging leaves the output unchanged
  ("PagedAttention: KV cache as virtual memory", "Interviewer follow-ups");
* closed forms: uniform keys and q = 0 give mean(V), one key gives V[0], one
  dominant key gives its value;
* brute force with scalar Python loops on tiny inputs;
* invariance under relabelling physical blocks;
* split-KV log-sum-exp combine equals the unsplit result.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth


def _contiguous_pool(K, V, B):
    """Dense [L][Hkv][D] -> pool [nblk][Hkv][B][D] with the identity table (reshape only)."""
    L, H, D = K.shape
    nblk = -(-L // B)
    pad = nblk * B - L
    Kp = np.concatenate([K, np.full((pad, H, D), np.nan)], 0)
    Vp = np.concatenate([V, np.full((pad, H, D), np.nan)], 0)
    kc = Kp.reshape(nblk, B, H, D).transpose(0, 2, 1, 3).copy()
    vc = Vp.reshape(nblk, B, H, D).transpose(0, 2, 1, 3).copy()
    return kc, vc, np.arange(nblk)


def _sdpa(q, K, V, scale, mask=None):
    # q [Hq][M][D], K/V [Hkv][L][D] in fp64 -> [Hq][M][D]
    qt = torch.from_numpy(q)[None]
    kt = torch.from_numpy(K)[None]
    vt = torch.from_numpy(V)[None]
    m = None if mask is None else torch.from_numpy(mask)
    out = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale,
                                         enable_gqa=qt.shape[1] != kt.shape[1])
    return out[0].numpy()


@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (32, 8)])
@pytest.mark.parametrize("L", [1, 15, 16, 17, 100])
def test_decode_equals_dense_sdpa(B, hq, hkv, L):
    rng = np.random.default_rng(L * 131 + B + hq)
    D = 16
    K = rng.standard_normal((L, hkv, D))
    V = rng.standard_normal((L, hkv, D))
    q = rng.standard_normal((1, hq, D))
    kc, vc, table = _contiguous_pool(K, V, B)
    scale = 1 / math.sqrt(D)
    got = oracle.paged_decode(q, kc, vc, table[None], [L], scale, hkv)[0]
    want = _sdpa(q[0][:, None, :], K.transpose(1, 0, 2), V.transpose(1, 0, 2), scale)[:, 0, :]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_decode_gqa_grouping_is_contiguous():
    # q heads 0..3 share kv head 0, 4..7 share kv head 1 (not interleaved)
    rng = np.random.default_rng(5)
    L, D = 9, 8
    K = rng.standard_normal((L, 2, D))
    V = rng.standard_normal((L, 2, D))
    V[:, 1] += 100.0  # kv head 1 values are far from kv head 0's
    q = rng.standard_normal((1, 8, D))
    kc, vc, table = _contiguous_pool(K, V, 16)
    out = oracle.paged_decode(q, kc, vc, table[None], [L], 0.3, 2)[0]
    assert np.all(out[:4] < 50) and np.all(out[4:] > 50)


def test_uniform_keys_give_mean_of_values():
    rng = np.random.default_rng(1)
    L, D = 37, 8
    K = np.repeat(rng.standard_normal((1, 1, D)), L, 0)
    V = rng.standard_normal((L, 1, D))
    kc, vc, table = _contiguous_pool(K, V, 16)
    q = rng.standard_normal((1, 1, D)) * 10
    out = oracle.paged_decode(q, kc, vc, table[None], [L], 0.5, 1)[0, 0]
    np.testing.assert_allclose(out, V[:, 0].mean(0), atol=1e-12)


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(2)
    L, D = 50, 8
    K = rng.standard_normal((L, 1, D)) * 5
    V = rng.standard_normal((L, 1, D))
    kc, vc, table = _contiguous_pool(K, V, 16)
    out = oracle.paged_decode(np.zeros((1, 1, D)), kc, vc, table[None], [L], 1.0, 1)[0, 0]
    np.testing.assert_allclose(out, V[:, 0].mean(0), atol=1e-12)


def test_single_key_returns_its_value():
    rng = np.random.default_rng(3)
    D = 8
    K = rng.standard_normal((1, 1, D))
    V = rng.standard_normal((1, 1, D))
    kc, vc, table = _contiguous_pool(K, V, 16)
    out = oracle.paged_decode(rng.standard_normal((1, 1, D)), kc, vc, table[None], [1], 0.7, 1)[0, 0]
    np.testing.assert_array_equal(out, V[0, 0])


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(4)
    L, D, j = 40, 16, 23
    q = rng.standard_normal(D)
    K = rng.standard_normal((L, 1, D)) * 0.1
    K[j, 0] = 50 * q / np.linalg.norm(q)
    V = rng.standard_normal((L, 1, D))
    kc, vc, table = _contiguous_pool(K, V, 16)
    out = oracle.paged_decode(q[None, None], kc, vc, table[None], [L], 1.0, 1)[0, 0]
    np.testing.assert_allclose(out, V[j, 0], atol=1e-9)


def test_empty_sequence_gives_zeros():
    w = synth.tiny_decode()
    lens = w.context_lens.numpy().copy()
    lens[1] = 0
    kc = w.key_cache.double().numpy()
    vc = w.value_cache.double().numpy()
    out = oracle.paged_decode(w.query.double().numpy(), kc, vc, w.block_tables.numpy(), lens,
                              w.scale, w.num_kv_heads)
    assert np.all(out[1] == 0)
    assert np.all(np.isfinite(out))


def _brute_decode(q, kc, vc, bt, lens, scale, hkv, B):
    S, Hq, D = len(q), len(q[0]), len(q[0][0])
    G = Hq // hkv
    out = [[[0.0] * D for _ in range(Hq)] for _ in range(S)]
    for s in range(S):
        for h in range(Hq):
            g = h // G
            z = []
            for p in range(lens[s]):
                blk = bt[s][p // B]
                z.append(scale * sum(q[s][h][d] * kc[blk][g][p % B][d] for d in range(D)))
            if not z:
                continue
            mx = max(z)
            w = [math.exp(x - mx) for x in z]
            tot = sum(w)
            for d in range(D):
                acc = 0.0
                for p in range(lens[s]):
                    blk = bt[s][p // B]
                    acc += w[p] * vc[blk][g][p % B][d]
                out[s][h][d] = acc / tot
    return out


@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("G", [1, 2, 4])
def test_decode_brute_force_grid(B, G):
    # every length 1..40: one and two partial blocks, exact block boundaries
    hkv = 2
    lens = list(range(1, 41))
    w = synth.random_decode(100 + B + G, lens, dtype=torch.float16, block_size=B,
                            hq=hkv * G, hkv=hkv, d=4, append=False)
    kc = w.key_cache.double().numpy()
    vc = w.value_cache.double().numpy()
    q = w.query.double().numpy()
    bt = w.block_tables.numpy()
    got = oracle.paged_decode(q, kc, vc, bt, lens, 0.5, hkv)
    want = _brute_decode(q.tolist(), kc.tolist(), vc.tolist(), bt.tolist(), lens, 0.5, hkv, B)
    np.testing.assert_allclose(got, np.array(want), rtol=0, atol=1e-12)


def test_tiny_workload_brute_force():
    w = synth.tiny_decode()
    kc = w.key_cache.double().numpy()
    vc = w.value_cache.double().numpy()
    q = w.query.double().numpy()
    bt = w.block_tables.numpy()
    lens = w.context_lens.tolist()  # before the append: all slots are initialised
    got = oracle.paged_decode(q, kc, vc, bt, lens, w.scale, w.num_kv_heads)
    want = _brute_decode(q.tolist(), kc.tolist(), vc.tolist(), bt.tolist(), lens, w.scale,
                         w.num_kv_heads, w.block_size)
    np.testing.assert_allclose(got, np.array(want), rtol=0, atol=1e-12)
    assert np.all(np.isfinite(got))


def test_decode_invariant_under_physical_relabelling():
    w = synth.random_decode(7, [5, 33, 64, 1, 90], hq=8, hkv=2, d=16, append=False)
    kc = w.key_cache.double().numpy()
    vc = w.value_cache.double().numpy()
    q = w.query.double().numpy()
    bt = w.block_tables.numpy()
    base = oracle.paged_decode(q, kc, vc, bt, w.context_lens.numpy(), w.scale, 2)
    rng = np.random.default_rng(11)
    perm = rng.permutation(w.num_blocks)  # physical b -> perm[b]
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1)
    moved = oracle.paged_decode(q, kc2, vc2, bt2, w.context_lens.numpy(), w.scale, 2)
    np.testing.assert_array_equal(base, moved)


@pytest.mark.parametrize("B", [16, 32])
def test_prefill_chunk_equals_masked_sdpa(B):
    rng = np.random.default_rng(B)
    hq, hkv, D = 4, 2, 16
    ctx, n = [0, 5, 40], [7, 16, 33]
    w = synth.chunked_prefill(seed=9, block_size=B, hq=hq, hkv=hkv, d=D, ctx_lens=ctx, q_lens=n,
                              dtype=torch.float16)
    kc = w.key_cache.double().numpy()
    vc = w.value_cache.double().numpy()
    q = w.query.double().numpy()
    bt = w.block_tables.numpy()
    cu = w.cu_q_lens.numpy()
    got = oracle.paged_prefill_chunk(q, kc, vc, bt, cu, ctx, w.scale, hkv)
    for s in range(len(ctx)):
        L = ctx[s] + n[s]
        # dense K/V of the sequence, read by block table row (blocks are whole tensors)
        nblk = -(-L // B)
        K = np.concatenate([kc[bt[s, i]] for i in range(nblk)], axis=1)[:, :L]  # [Hkv][L][D]
        V = np.concatenate([vc[bt[s, i]] for i in range(nblk)], axis=1)[:, :L]
        mask = np.arange(L)[None, :] <= (ctx[s] + np.arange(n[s]))[:, None]
        want = _sdpa(q[cu[s]:cu[s + 1]].transpose(1, 0, 2), K, V, w.scale, mask)
        np.testing.assert_allclose(got[cu[s]:cu[s + 1]], want.transpose(1, 0, 2), atol=1e-12, rtol=0)
    del rng


def test_mixed_batch_rows_equal_masked_sdpa():
    # decode rows (one query, ctx + 1 keys) and prefill chunks in one batch:
    # the chunk rule covers both ("Mechanics of Chunked Prefill")
    B, hq, hkv, D = 16, 4, 2, 16
    w = synth.mixed_batch(seed=12, block_size=B, hq=hq, hkv=hkv, d=D, dtype=torch.float16,
                          decode_ctx=[0, 15, 16, 40], prefill_ctx=[5, 0, 33], prefill_q=[20, 1, 0])
    assert w.num_decode == 4 and w.cu_q_lens.tolist()[:5] == [0, 1, 2, 3, 4]
    kc = w.key_cache.double().numpy()
    vc = w.value_cache.double().numpy()
    q = w.query.double().numpy()
    bt = w.block_tables.numpy()
    cu = w.cu_q_lens.numpy()
    ctx = w.ctx_lens.numpy()
    got = oracle.paged_prefill_chunk(q, kc, vc, bt, cu, ctx, w.scale, hkv)
    for s in range(w.num_seqs):
        n = int(cu[s + 1] - cu[s])
        if n == 0:
            continue
        L = int(ctx[s]) + n
        nblk = -(-L // B)
        K = np.concatenate([kc[bt[s, i]] for i in range(nblk)], axis=1)[:, :L]
        V = np.concatenate([vc[bt[s, i]] for i in range(nblk)], axis=1)[:, :L]
        mask = np.arange(L)[None, :] <= (ctx[s] + np.arange(n))[:, None]
        want = _sdpa(q[cu[s]:cu[s + 1]].transpose(1, 0, 2), K, V, w.scale, mask)
        np.testing.assert_allclose(got[cu[s]:cu[s + 1]], want.transpose(1, 0, 2), atol=1e-12,
                                   rtol=0)


def test_prefill_row_equals_decode_at_that_length():
    w = synth.chunked_prefill(seed=3, block_size=16, hq=4, hkv=2, d=16, ctx_lens=[21, 0],
                              q_lens=[9, 4], dtype=torch.float16)
    kc = w.key_cache.double().numpy()
    vc = w.value_cache.double().numpy()
    q = w.query.double().numpy()
    bt = w.block_tables.numpy()
    cu = w.cu_q_lens.numpy()
    pre = oracle.paged_prefill_chunk(q, kc, vc, bt, cu, [21, 0], w.scale, 2)
    for s, (c, n) in enumerate([(21, 9), (0, 4)]):
        for i in range(n):
            dec = oracle.paged_decode(q[cu[s] + i][None], kc, vc, bt[s][None], [c + i + 1], w.scale, 2)
            np.testing.assert_array_equal(pre[cu[s] + i], dec[0])
    # the sampled-row path matches the full computation
    part = oracle.paged_prefill_chunk(q, kc, vc, bt, cu, [21, 0], w.scale, 2, seqs=[0], rows=[0, 8])
    np.testing.assert_array_equal(part[[0, 8]], pre[[0, 8]])


@pytest.mark.parametrize("cuts", [[], [1], [16, 17], [3, 50, 51, 99], [0, 0, 100]])
def test_split_kv_combine_equals_unsplit(cuts):
    rng = np.random.default_rng(len(cuts))
    L, D = 100, 16
    K = rng.standard_normal((L, D)) * 2
    V = rng.standard_normal((L, D))
    q = rng.standard_normal(D)
    bounds = [0] + cuts + [L]
    states = [oracle.partial_attention(q, K[a:b], V[a:b], 0.4) for a, b in zip(bounds[:-1], bounds[1:])]
    got = oracle.combine_partials(states)
    want = oracle.attention(q[None], K, V, 0.4)[0]
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)


@pytest.mark.parametrize("parts", [2, 3, 4])
def test_causal_chunk_rows_from_key_range_parts(parts):
    # A chunk row split along the key range into equal runs of 128-key tiles
    # (the last wave's split of the prefill kernel): each part keeps only the
    # keys the row may see, a part with none contributes (-inf, 0, 0), and the
    # parts' combine equals the row's causal attention.
    w = synth.chunked_prefill(seed=21 + parts, block_size=16, hq=2, hkv=1, d=16,
                              ctx_lens=[300], q_lens=[90], dtype=torch.float16)
    kc = w.key_cache.double().numpy()
    vc = w.value_cache.double().numpy()
    q = w.query.double().numpy()
    bt = w.block_tables.numpy()
    c, n = 300, 90
    whole = oracle.paged_prefill_chunk(q, kc, vc, bt, w.cu_q_lens.numpy(), [c], w.scale, 1)
    L = c + n
    K = oracle.gather_logical(kc, bt[0], L, 0, 16)
    V = oracle.gather_logical(vc, bt[0], L, 0, 16)
    ntiles = -(-L // 128)
    for i in (0, 1, 45, 89):
        for h in range(2):
            states = []
            for part in range(parts):
                a = part * ntiles // parts * 128
                b = min((part + 1) * ntiles // parts * 128, c + i + 1)  # causal limit
                states.append(oracle.partial_attention(q[i, h], K[a:max(a, b)], V[a:max(a, b)],
                                                       w.scale))
            np.testing.assert_allclose(oracle.combine_partials(states), whole[i, h], atol=1e-12,
                                       rtol=0)


def test_split_kv_partial_state_definition():
    rng = np.random.default_rng(9)
    K = rng.standard_normal((5, 4))
    V = rng.standard_normal((5, 4))
    q = rng.standard_normal(4)
    m, l, acc = oracle.partial_attention(q, K, V, 1.0)
    z = [float(K[j] @ q) for j in range(5)]
    assert m == max(z)
    assert l == pytest.approx(sum(math.exp(x - max(z)) for x in z), abs=1e-14)
    # one-state combine is acc / l
    np.testing.assert_allclose(oracle.combine_partials([(m, l, acc)]), acc / l, atol=1e-15)
    m0, l0, a0 = oracle.partial_attention(q, K[:0], V[:0], 1.0)
    assert np.isneginf(m0) and l0 == 0 and not np.any(a0)
