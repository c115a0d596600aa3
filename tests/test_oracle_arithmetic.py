"""Pins the oracle's closed-form KV arithmetic to the numbers the pages print."""
import itertools

import pytest

from oracle import arithmetic as ar


def _kv(golden):
    return {r[0]: r[1] for r in golden("kv_bytes_llama2_13b.txt")}


def test_kv_bytes_per_token_llama2_13b(golden):
    g = _kv(golden)
    got = ar.kv_bytes_per_token(int(g["num_layers"]), int(g["num_kv_heads"]),
                                int(g["head_dim"]), int(g["dtype_bytes"]))
    assert got == int(g["kv_bytes_per_token"])
    # "about 0.8 MB per token" holds in decimal megabytes
    assert abs(got / 1e6 - float(g["approx_mb_per_token"])) < 0.05


def test_kv_bytes_per_sequence(golden):
    g = _kv(golden)
    per_seq = int(g["sequence_tokens"]) * int(g["kv_bytes_per_token"])
    assert per_seq == 1_677_721_600
    approx = float(g["approx_gb_per_sequence"])
    # "about 1.6 GB": 1.68 GB decimal, 1.5625 GiB binary; both round to it
    assert abs(per_seq / 1e9 - approx) < 0.1
    assert abs(per_seq / 2**30 - approx) < 0.1


def test_kv_bytes_is_linear_in_each_factor():
    base = ar.kv_bytes_per_token(3, 5, 7, 2)
    assert base == 2 * 3 * 5 * 7 * 2
    assert ar.kv_bytes_per_token(6, 5, 7, 2) == 2 * base
    assert ar.kv_bytes_per_token(3, 10, 7, 2) == 2 * base
    assert ar.kv_bytes_per_token(3, 5, 14, 2) == 2 * base
    assert ar.kv_bytes_per_token(3, 5, 7, 1) * 2 == base


def test_block_table_example_counts(golden):
    rows = golden("block_table_example.txt")
    B = int(rows[0][1])
    for tokens, blocks, _table in rows[1:]:
        assert ar.blocks_needed(int(tokens), B) == int(blocks)


def test_blocks_needed_brute_force():
    # smallest n with n * B >= L, by search
    for B in (1, 8, 16, 32, 64):
        for L in range(0, 300):
            n = 0
            while n * B < L:
                n += 1
            assert ar.blocks_needed(L, B) == n


def test_tail_waste_bound_exhaustive(golden):
    g = _kv(golden)
    assert 16 - 1 == int(g["max_tail_waste_at_16"])
    for B in (8, 16, 32, 64):
        worst = 0
        for L in range(1, 10_001):
            w = ar.tail_waste_tokens(L, B)
            assert 0 <= w <= B - 1
            worst = max(worst, w)
        assert worst == B - 1


def test_reservation_waste(golden):
    g = _kv(golden)
    frac = ar.reservation_waste_fraction(int(g["reply_tokens"]), int(g["reserved_tokens"]))
    assert frac == pytest.approx(2018 / 2048)
    assert int(frac * 100) == int(g["approx_waste_percent"])


def test_fragmentation_fit(golden):
    g = {r[0]: r[1] for r in golden("fragmentation_fit.txt")}
    B, pool, max_len = int(g["block"]), int(g["pool"]), int(g["max_len"])
    lens = [int(x) for x in g["lens"].split(",")]
    assert ar.contiguous_fit(pool, max_len, B) == int(g["contiguous"])
    assert ar.paged_fit(lens, pool, B, stop_at_first_miss=True) == int(g["paged_first_come_first_served"])
    assert ar.paged_fit(lens, pool, B, stop_at_first_miss=False) == int(g["paged_skip_and_continue"])


def test_paged_fit_brute_force_small():
    # skip-and-continue greedy equals a direct simulation over every prefix order
    for pool in range(0, 12):
        for lens in itertools.product([1, 5, 16, 17, 33], repeat=3):
            used, n = 0, 0
            for L in lens:
                need = -(-L // 16)
                if used + need <= pool:
                    used, n = used + need, n + 1
            assert ar.paged_fit(lens, pool, 16, False) == n
            first = 0
            used = 0
            for L in lens:
                need = -(-L // 16)
                if used + need > pool:
                    break
                used, first = used + need, first + 1
            assert ar.paged_fit(lens, pool, 16, True) == first


def test_contiguous_fit_brute_force():
    # each admitted sequence takes whole blocks for max_len tokens up front;
    # admit until the next reservation no longer fits in what is left
    for B in (1, 4, 16):
        for max_len in range(1, 40):
            need = -(-max_len // B)
            for pool in range(0, 30):
                free = pool
                n = 0
                while need <= free:
                    free -= need
                    n += 1
                assert ar.contiguous_fit(pool, max_len, B) == n
