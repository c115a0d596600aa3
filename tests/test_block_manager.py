"""Host block manager (C++ in libpa.so): allocation order, the pages'
fragmentation arithmetic on live allocation, prefix sharing of full blocks,
eviction order, copy-on-write after fork, out-of-memory behaviour and the
pool invariants under random churn.  CPU only (host code)."""
import numpy as np
import pytest

import oracle
import paged_kv_cache_397_b200 as pa
from paged_kv_cache_397_b200 import _build


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    pa.lib()


def toks(n, base=0):
    return np.arange(base, base + n, dtype=np.int32)


def test_fresh_pool_hands_out_blocks_in_order():
    bm = pa.BlockManager(10, 16)
    assert bm.num_free_blocks == 10
    bm.add_sequence(1, toks(30))
    np.testing.assert_array_equal(bm.block_table(1), [0, 1])
    bm.add_sequence(2, toks(50, 1000))
    np.testing.assert_array_equal(bm.block_table(2), [2, 3, 4, 5])
    assert bm.num_free_blocks == 4
    # slots follow the table, as the oracle's indexing says
    for s in (1, 2):
        n = bm.num_tokens(s)
        want = oracle.logical_positions_to_slots(bm.block_table(s)[None], np.zeros(n, int),
                                                 np.arange(n), 16)
        np.testing.assert_array_equal(bm.slots(s, 0, n), want)


def test_fragmentation_fit_on_live_allocation(golden):
    g = {r[0]: r[1] for r in golden("fragmentation_fit.txt")}
    B, pool, max_len = int(g["block"]), int(g["pool"]), int(g["max_len"])
    lens = [int(x) for x in g["lens"].split(",")]
    # paged: admit first come first served until the pool refuses
    bm = pa.BlockManager(pool, B, enable_prefix_caching=False)
    admitted = 0
    for i, L in enumerate(lens):
        try:
            bm.add_sequence(i, toks(L, 10_000 * i))
        except pa.PAError as e:
            assert e.status == pa.PA_ERR_OUT_OF_RANGE
            break
        admitted += 1
    assert admitted == int(g["paged_first_come_first_served"])
    # contiguous: every sequence reserves max_len tokens up front
    bm = pa.BlockManager(pool, B, enable_prefix_caching=False)
    reserved = 0
    for i in range(len(lens)):
        try:
            bm.add_sequence(i, toks(max_len, 10_000 * i))
        except pa.PAError:
            break
        reserved += 1
    assert reserved == int(g["contiguous"])


def test_full_prefix_blocks_are_shared_partial_ones_are_not():
    bm = pa.BlockManager(64, 16)
    prefix = toks(56)                      # 3 full blocks + 8 tokens
    a = np.concatenate([prefix, toks(10, 500)])
    b = np.concatenate([prefix, toks(20, 900)])
    assert bm.add_sequence(1, a) == 0
    assert bm.add_sequence(2, b) == 48     # the three full blocks hit
    ta, tb = bm.block_table(1), bm.block_table(2)
    np.testing.assert_array_equal(ta[:3], tb[:3])
    assert ta[3] != tb[3]                  # the partial fourth block is private
    for blk in ta[:3]:
        assert bm.ref_count(blk) == 2
    assert bm.ref_count(ta[3]) == 1 and bm.ref_count(tb[3]) == 1
    # a different first block breaks the chain even if later blocks match
    c = np.concatenate([toks(16, 7000), prefix[16:]])
    assert bm.add_sequence(3, c) == 0


def test_freed_cached_blocks_are_revived_then_evicted_lru():
    bm = pa.BlockManager(8, 16)
    bm.add_sequence(1, toks(64))           # blocks 0..3, all full and cached
    bm.free(1)                             # free queue: 4 5 6 7 3 2 1 0
    assert bm.num_free_blocks == 8
    assert bm.add_sequence(2, toks(64)) == 64   # all four revived from the free queue
    np.testing.assert_array_equal(bm.block_table(2), [0, 1, 2, 3])
    assert bm.num_free_blocks == 4
    bm.free(2)                             # free queue: 4 5 6 7 3 2 1 0
    # other content takes the six least recently freed blocks: 4 5 6 7 3 2,
    # evicting the keys of blocks 3 and 2
    bm.add_sequence(3, toks(96, 9000))
    np.testing.assert_array_equal(bm.block_table(3), [4, 5, 6, 7, 3, 2])
    assert bm.num_free_blocks == 2
    # the 64-token prompt again: blocks 0 and 1 still hit, the third misses;
    # it needs two fresh blocks but only 0 and 1 are free -> refused, unchanged
    with pytest.raises(pa.PAError):
        bm.add_sequence(4, toks(64))
    assert bm.num_free_blocks == 2
    bm.free(3)                             # free queue: 1 0 2 3 7 6 5 4
    assert bm.add_sequence(4, toks(64)) == 32
    np.testing.assert_array_equal(bm.block_table(4), [0, 1, 2, 3])
    assert bm.num_free_blocks == 4


def test_add_is_all_or_nothing_when_the_pool_is_short():
    bm = pa.BlockManager(4, 16)
    bm.add_sequence(1, toks(40))           # 3 blocks
    before = (bm.num_free_blocks, list(bm.block_table(1)))
    with pytest.raises(pa.PAError) as e:
        bm.add_sequence(2, toks(40, 100))
    assert e.value.status == pa.PA_ERR_OUT_OF_RANGE
    assert (bm.num_free_blocks, list(bm.block_table(1))) == before
    assert bm.num_tokens(2) == -1
    bm.append(1, toks(8, 50))              # fills block 3 exactly (48 tokens)
    with pytest.raises(pa.PAError):
        bm.append(1, toks(20, 60))         # needs two more blocks
    assert bm.num_tokens(1) == 48


def test_append_takes_a_block_exactly_when_the_last_fills():
    bm = pa.BlockManager(16, 16)
    bm.add_sequence(1, toks(15))
    assert len(bm.block_table(1)) == 1
    bm.append(1, toks(1, 99))              # 16 tokens: still one block
    assert len(bm.block_table(1)) == 1
    bm.append(1, toks(1, 100))             # 17th token opens block 2
    assert len(bm.block_table(1)) == 2
    for L in range(18, 60):
        bm.append(1, toks(1, L))
        assert len(bm.block_table(1)) == oracle.blocks_needed(L, 16)
        waste = len(bm.block_table(1)) * 16 - L
        assert 0 <= waste <= 15


def test_fork_then_diverge_copies_only_the_shared_partial_block():
    bm = pa.BlockManager(32, 16)
    bm.add_sequence(1, toks(40))           # blocks 0, 1 full, 2 partial
    bm.fork(1, 2)
    t1 = bm.block_table(1)
    assert all(bm.ref_count(b) == 2 for b in t1)
    bm.append(2, toks(1, 777))             # child writes into the shared partial block
    copies = bm.take_copies()
    assert copies.shape == (1, 2) and copies[0, 0] == t1[2]
    t2 = bm.block_table(2)
    np.testing.assert_array_equal(t2[:2], t1[:2])
    assert t2[2] == copies[0, 1] and t2[2] != t1[2]
    assert bm.ref_count(t1[2]) == 1 and bm.ref_count(t2[2]) == 1
    bm.append(1, toks(1, 888))             # the parent now owns its block alone
    assert bm.take_copies().shape == (0, 2)
    np.testing.assert_array_equal(bm.block_table(1), t1)
    # appending past a full shared block needs no copy
    bm.fork(1, 3)
    bm.append(3, toks(7, 1000))            # 41 + 7 = 48: fills block 2 (shared) -> copy
    assert bm.take_copies().shape == (1, 2)
    bm.free(1)
    bm.free(2)
    bm.free(3)
    assert bm.num_free_blocks == 32


def test_random_churn_keeps_the_pool_consistent():
    rng = np.random.default_rng(0)
    bm = pa.BlockManager(200, 16)
    live = {}
    next_id = 0
    prefixes = [toks(int(rng.integers(16, 120)), 100_000 * k) for k in range(5)]
    for step in range(3000):
        op = rng.random()
        try:
            if op < 0.3 or not live:
                pre = prefixes[rng.integers(0, 5)]
                tail = toks(int(rng.integers(0, 40)), 1_000_000 + step * 50)
                bm.add_sequence(next_id, np.concatenate([pre, tail]))
                live[next_id] = True
                next_id += 1
            elif op < 0.7:
                sid = list(live)[rng.integers(0, len(live))]
                bm.append(sid, toks(int(rng.integers(1, 20)), 5_000_000 + step * 20))
            elif op < 0.8:
                sid = list(live)[rng.integers(0, len(live))]
                bm.fork(sid, next_id)
                live[next_id] = True
                next_id += 1
            else:
                sid = list(live)[rng.integers(0, len(live))]
                bm.free(sid)
                del live[sid]
        except pa.PAError as e:
            assert e.status == pa.PA_ERR_OUT_OF_RANGE
        bm.take_copies()
        if step % 100 == 0:
            refs = np.zeros(200, int)
            for sid in live:
                t = bm.block_table(sid)
                assert len(t) == oracle.blocks_needed(bm.num_tokens(sid), 16)
                for b in t:
                    refs[b] += 1
            for b in range(200):
                assert bm.ref_count(b) == refs[b]
            assert bm.num_free_blocks == int((refs == 0).sum())


@pytest.mark.parametrize("seed,B", [(1, 16), (2, 32), (3, 16)])
def test_simulated_pool_reads_back_every_sequence(seed, B):
    # The kernels' view of the manager: every token is written through the
    # slots it hands out, copy-on-write pairs are applied before the writes of
    # the step that needs them, and reading a sequence through its block table
    # must give back exactly its tokens -- prefix hits, revived free blocks,
    # forks and copy-on-write included ("PagedAttention: KV cache as virtual
    # memory", "Deep dive").
    rng = np.random.default_rng(seed)
    nb = 160
    bm = pa.BlockManager(nb, B)
    pool = np.full((nb, B), -1, dtype=np.int64)  # token id held by each slot
    seqs = {}
    next_id = 0
    prefixes = [toks(int(rng.integers(B, 6 * B)), 10_000 * k) for k in range(4)]

    def write(sid, start, tokens):
        if len(tokens) == 0:
            return
        for slot, t in zip(bm.slots(sid, start, len(tokens)), tokens):
            pool[slot // B, slot % B] = t

    def apply_copies():
        for src, dst in bm.take_copies():
            pool[dst] = pool[src]

    for step in range(1500):
        op = rng.random()
        try:
            if op < 0.3 or not seqs:
                pre = prefixes[rng.integers(0, len(prefixes))]
                cut = int(rng.integers(0, len(pre) + 1))
                tail = toks(int(rng.integers(0, 2 * B)), 1_000_000 + 100 * step)
                prompt = np.concatenate([pre[:cut], tail])
                if len(prompt) == 0:
                    continue
                cached = bm.add_sequence(next_id, prompt)
                apply_copies()
                write(next_id, cached, prompt[cached:])
                seqs[next_id] = list(prompt)
                next_id += 1
            elif op < 0.7:
                sid = list(seqs)[rng.integers(0, len(seqs))]
                new = toks(int(rng.integers(1, B + 3)), 5_000_000 + 100 * step)
                bm.append(sid, new)
                apply_copies()
                write(sid, len(seqs[sid]), new)
                seqs[sid] += list(new)
            elif op < 0.82:
                sid = list(seqs)[rng.integers(0, len(seqs))]
                bm.fork(sid, next_id)
                seqs[next_id] = list(seqs[sid])
                next_id += 1
            else:
                sid = list(seqs)[rng.integers(0, len(seqs))]
                bm.free(sid)
                del seqs[sid]
        except pa.PAError as e:
            assert e.status == pa.PA_ERR_OUT_OF_RANGE  # pool exhausted; state unchanged
        for sid, want in seqs.items():
            table = bm.block_table(sid)
            got = [pool[table[p // B], p % B] for p in range(len(want))]
            assert got == want, f"sequence {sid} reads back wrong tokens at step {step}"
    for sid in list(seqs):
        bm.free(sid)
    assert bm.num_free_blocks == nb


def test_c_abi_error_returns_leave_the_manager_unchanged():
    # every documented error of the pa_bm_* calls, through the raw C ABI
    import ctypes
    L = pa.lib()
    _p = ctypes.c_void_p
    assert L.pa_bm_create(2**27, 32, 1, ctypes.byref(_p())) == pa.PA_ERR_INVALID_ARG  # > INT32_MAX tokens
    assert L.pa_bm_create(0, 16, 1, ctypes.byref(_p())) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_create(4, 16, 1, None) == pa.PA_ERR_INVALID_ARG

    bm = pa.BlockManager(4, 16)
    h = bm._h
    bm.add_sequence(1, toks(20))
    bm.fork(1, 2)
    before = (bm.num_free_blocks, list(bm.block_table(1)), bm.ref_count(0), bm.ref_count(1))

    def ptr(a):
        return a.ctypes.data_as(_p)

    small = toks(16)
    cached = ctypes.c_int(-5)
    assert L.pa_bm_add_sequence(h, 1, ptr(small), 16, ctypes.byref(cached)) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_add_sequence(h, 3, ptr(small), -1, None) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_add_sequence(h, 3, None, 1, None) == pa.PA_ERR_INVALID_ARG
    big = toks(5 * 16)  # needs more blocks than the pool has
    assert L.pa_bm_add_sequence(h, 3, ptr(big), big.size, None) == pa.PA_ERR_OUT_OF_RANGE
    # a count whose block total overflows int is refused before any token is read
    assert L.pa_bm_add_sequence(h, 3, ptr(small), 2**31 - 1, None) == pa.PA_ERR_OUT_OF_RANGE
    assert cached.value == -5 and bm.num_tokens(3) == -1

    assert L.pa_bm_append(h, 9, ptr(small), 1) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_append(h, 1, ptr(small), -1) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_append(h, 1, None, 1) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_append(h, 1, ptr(small), 2**31 - 1) == pa.PA_ERR_OUT_OF_RANGE
    assert bm.num_tokens(1) == 20

    assert L.pa_bm_fork(h, 9, 5) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_fork(h, 1, 2) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_free(h, 9) == pa.PA_ERR_INVALID_ARG

    n = ctypes.c_int(0)
    out = np.full(1, 77, dtype=np.int32)
    assert L.pa_bm_block_table(h, 1, ptr(out), 1, ctypes.byref(n)) == pa.PA_ERR_WORKSPACE
    assert n.value == 2 and out[0] == 77
    assert L.pa_bm_block_table(h, 9, ptr(out), 1, None) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_block_table(h, 1, None, 2, None) == pa.PA_ERR_INVALID_ARG

    slots = np.full(16, -9, dtype=np.int64)
    # past the tokens held but inside the last block: allowed
    assert L.pa_bm_slots(h, 1, 20, 12, ptr(slots)) == pa.PA_OK
    assert list(slots[:12]) == list(range(20, 32)) and slots[12] == -9  # table [0, 1]
    slots[:] = -9
    assert L.pa_bm_slots(h, 1, 25, 8, ptr(slots)) == pa.PA_ERR_OUT_OF_RANGE  # past block 2
    assert np.all(slots == -9)
    assert L.pa_bm_slots(h, 1, 2**31 - 2, 5, ptr(slots)) == pa.PA_ERR_OUT_OF_RANGE  # no overflow
    assert L.pa_bm_slots(h, 1, -1, 1, ptr(slots)) == pa.PA_ERR_INVALID_ARG
    assert L.pa_bm_slots(h, 9, 0, 1, ptr(slots)) == pa.PA_ERR_INVALID_ARG

    bm.append(2, toks(1, 500))  # copy-on-write of the shared partial block: one pair pending
    pairs = np.zeros((1, 2), dtype=np.int64)
    assert L.pa_bm_take_copies(h, ptr(pairs), 0) == -1  # too small: nothing taken
    assert L.pa_bm_take_copies(h, None, 1) == -1
    assert L.pa_bm_take_copies(h, ptr(pairs), 1) == 1 and list(pairs[0]) == [1, 2]

    assert bm.ref_count(-1) == -1 and bm.ref_count(4) == -1 and bm.num_tokens(9) == -1
    assert L.pa_bm_num_free_blocks(None) == -1
    # sequence 1 saw only refused calls
    assert list(bm.block_table(1)) == before[1] and bm.num_tokens(1) == 20
    assert bm.ref_count(0) == 2 and bm.ref_count(1) == 1 and bm.num_free_blocks == 1
