"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of an oracle function (on the CPU),
swaps it in for the real one, and checks that the pin written for that part
of the oracle now fails: a scale applied twice, an off-by-one block index, an
interleaved GQA grouping, an exclusive causal mask, a split-KV combine
without the log-sum-exp rescale, a slot built from the wrong quotient, K and
V swapped in the scatter, ties rounded away from the even E4M3 code, a KV
byte count without the K/V factor, a floor where the pages take a ceiling,
a block copy in the wrong direction, a swap of one pool only, admission that
never skips, FP8 quantisation dividing in fp64, an off-by-one tail waste, a
contiguous reservation counted in tokens rather than whole blocks, the waste
share inverted, an E4M3 exponent bias of 8, a subnormal step of 2^-10, V
dequantised with the K scale, a partial state already normalised, a chunk
whose rows ignore the cached context, overflow to NaN instead of saturation,
and a skipped slot (-1) written to the last block.
The real functions pass the same pins (they run in the rest of the suite)."""
import numpy as np
import pytest

import oracle
import oracle.arithmetic as oa
import oracle.fp8 as of
import oracle.paged_attention as opa
import test_oracle_arithmetic as t_arith
import test_oracle_attention as t_attn
import test_oracle_fp8 as t_fp8
import test_oracle_indexing as t_idx
from conftest import read_golden


def _swap(monkeypatch, module, name, fn):
    monkeypatch.setattr(module, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)


def _fails(pin, *args):
    with pytest.raises(AssertionError):
        pin(*args)


def test_scale_applied_twice_is_caught(monkeypatch):
    def attention(q, K, V, scale, visible=None):
        q, K, V = (np.asarray(a, dtype=np.float64) for a in (q, K, V))
        out = np.zeros((q.shape[0], V.shape[1]))
        for m in range(q.shape[0]):
            n = K.shape[0] if visible is None else int(visible[m])
            if n > 0:
                z = scale * scale * (K[:n] @ q[m])  # planted mistake
                w = np.exp(z - z.max())
                out[m] = (w @ V[:n]) / w.sum()
        return out
    _swap(monkeypatch, opa, "attention", attention)
    _fails(t_attn.test_decode_equals_dense_sdpa, 16, 8, 2, 100)


def test_off_by_one_block_index_is_caught(monkeypatch):
    def gather_logical(cache, table_row, length, kv_head, block_size):
        p = np.arange(int(length))
        phys = np.asarray(table_row)[(p + 1) // block_size]  # planted mistake
        return np.asarray(cache[phys, kv_head, p % block_size, :], dtype=np.float64)
    _swap(monkeypatch, opa, "gather_logical", gather_logical)
    _fails(t_attn.test_decode_equals_dense_sdpa, 16, 4, 4, 17)


def test_interleaved_gqa_grouping_is_caught(monkeypatch):
    def paged_decode(query, key_cache, value_cache, block_tables, seq_lens, scale, num_kv_heads):
        q = np.asarray(query, dtype=np.float64)
        S, Hq, D = q.shape
        B = key_cache.shape[2]
        out = np.zeros((S, Hq, D))
        for s in range(S):
            for h in range(Hq):
                g = h % num_kv_heads  # planted mistake (contiguous groups: h // G)
                K = opa.gather_logical(key_cache, block_tables[s], seq_lens[s], g, B)
                V = opa.gather_logical(value_cache, block_tables[s], seq_lens[s], g, B)
                out[s, h] = opa.attention(q[s, h][None], K, V, scale)[0]
        return out
    _swap(monkeypatch, opa, "paged_decode", paged_decode)
    _fails(t_attn.test_decode_gqa_grouping_is_contiguous)


def _chunk_with_visible(visible_of):
    """paged_prefill_chunk with the keys row i may see given by visible_of(c, i)."""
    def paged_prefill_chunk(query, key_cache, value_cache, block_tables, cu_q_lens, ctx_lens,
                            scale, num_kv_heads, seqs=None, rows=None):
        q = np.asarray(query, dtype=np.float64)
        T, Hq, D = q.shape
        B = key_cache.shape[2]
        G = Hq // num_kv_heads
        out = np.zeros((T, Hq, D))
        for s in range(len(ctx_lens)):
            q0, q1, c = int(cu_q_lens[s]), int(cu_q_lens[s + 1]), int(ctx_lens[s])
            idx = np.arange(q1 - q0)
            if idx.size == 0:
                continue
            L = c + idx.size
            for g in range(num_kv_heads):
                K = opa.gather_logical(key_cache, block_tables[s], L, g, B)
                V = opa.gather_logical(value_cache, block_tables[s], L, g, B)
                for h in range(g * G, (g + 1) * G):
                    out[q0 + idx, h] = opa.attention(q[q0 + idx, h], K, V, scale,
                                                     visible=visible_of(c, idx))
        return out
    return paged_prefill_chunk


def test_exclusive_causal_mask_is_caught(monkeypatch):
    # planted mistake: row i does not see itself
    _swap(monkeypatch, opa, "paged_prefill_chunk", _chunk_with_visible(lambda c, i: c + i))
    _fails(t_attn.test_prefill_chunk_equals_masked_sdpa, 16)


def test_chunk_that_ignores_the_context_is_caught(monkeypatch):
    # planted mistake: row i is placed at position i, not after the c cached tokens
    _swap(monkeypatch, opa, "paged_prefill_chunk", _chunk_with_visible(lambda c, i: i + 1))
    _fails(t_attn.test_prefill_chunk_equals_masked_sdpa, 16)


def test_combine_without_rescale_is_caught(monkeypatch):
    def combine_partials(states):
        num = sum(acc for m, l, acc in states if not np.isneginf(m))  # planted mistake
        den = sum(l for m, l, acc in states if not np.isneginf(m))
        return num / den
    _swap(monkeypatch, opa, "combine_partials", combine_partials)
    _fails(t_attn.test_split_kv_combine_equals_unsplit, [16, 17])


def test_slot_offset_from_the_wrong_quotient_is_caught(monkeypatch):
    def logical_positions_to_slots(block_tables, seq_ids, positions, block_size):
        bt = np.asarray(block_tables, dtype=np.int64)
        s = np.asarray(seq_ids, dtype=np.int64).reshape(-1)
        p = np.asarray(positions, dtype=np.int64).reshape(-1)
        return bt[s, p // block_size] * block_size + p // block_size  # planted mistake
    _swap(monkeypatch, opa, "logical_positions_to_slots", logical_positions_to_slots)
    _fails(t_idx.test_slots_of_the_worked_example, read_golden)


def test_key_value_swap_in_the_scatter_is_caught(monkeypatch):
    def reshape_and_cache(key_cache, value_cache, key, value, slot_mapping, block_size):
        for t, slot in enumerate(np.asarray(slot_mapping).reshape(-1)):
            if slot >= 0:
                key_cache[slot // block_size, :, slot % block_size, :] = value[t]  # planted
                value_cache[slot // block_size, :, slot % block_size, :] = key[t]
    _swap(monkeypatch, opa, "reshape_and_cache", reshape_and_cache)
    _fails(t_idx.test_reshape_and_cache_bits_and_skip)


def test_ties_away_from_even_are_caught(monkeypatch):
    values = of._POS_VALUES

    def e4m3_encode(x):
        x = np.asarray(x, dtype=np.float64)
        mag = np.minimum(np.abs(np.nan_to_num(x)), values[0x7E])
        hi = np.minimum(np.searchsorted(values, mag, side="left"), 0x7E)
        lo = np.maximum(np.where(values[hi] > mag, hi - 1, hi), 0)
        pick_hi = (values[hi] - mag) <= (mag - values[lo])  # planted mistake: ties go up
        code = np.where(pick_hi, hi, lo).astype(np.uint8)
        code = np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)
        return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)
    _swap(monkeypatch, of, "e4m3_encode", e4m3_encode)
    _fails(t_fp8.test_ties_go_to_the_even_code)


def test_kv_bytes_without_the_kv_factor_is_caught(monkeypatch):
    def kv_bytes_per_token(num_layers, num_kv_heads, head_dim, dtype_bytes):
        return num_layers * num_kv_heads * head_dim * dtype_bytes  # planted mistake
    _swap(monkeypatch, oa, "kv_bytes_per_token", kv_bytes_per_token)
    _fails(t_arith.test_kv_bytes_per_token_llama2_13b, read_golden)


def test_floor_instead_of_ceiling_is_caught(monkeypatch):
    def blocks_needed(num_tokens, block_size):
        return num_tokens // block_size  # planted mistake
    _swap(monkeypatch, oa, "blocks_needed", blocks_needed)
    _fails(t_arith.test_block_table_example_counts, read_golden)


def test_copy_in_the_wrong_direction_is_caught(monkeypatch):
    def copy_blocks(key_cache, value_cache, block_pairs):
        for src, dst in np.asarray(block_pairs, dtype=np.int64).reshape(-1, 2):
            key_cache[src] = key_cache[dst]  # planted mistake: dst -> src
            value_cache[src] = value_cache[dst]
    _swap(monkeypatch, opa, "copy_blocks", copy_blocks)
    _fails(t_idx.test_copy_blocks_bits)


def test_swap_of_one_pool_only_is_caught(monkeypatch):
    def swap_blocks(dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, block_pairs):
        for src, dst in np.asarray(block_pairs, dtype=np.int64).reshape(-1, 2):
            dst_key_cache[dst] = src_key_cache[src]  # planted mistake: V not swapped
    _swap(monkeypatch, opa, "swap_blocks", swap_blocks)
    _fails(t_idx.test_swap_blocks_copies_between_pools_only_the_listed_blocks)


def test_admission_that_never_skips_is_caught(monkeypatch):
    def paged_fit(lengths, pool_blocks, block_size, stop_at_first_miss):
        used = admitted = 0
        for L in lengths:
            need = oa.blocks_needed(int(L), block_size)
            if used + need > pool_blocks:
                break  # planted mistake: both readings stop at the first miss
            used += need
            admitted += 1
        return admitted
    _swap(monkeypatch, oa, "paged_fit", paged_fit)
    _fails(t_arith.test_fragmentation_fit, read_golden)


def test_quantize_in_double_precision_is_caught(monkeypatch):
    def quantize(x, scale):
        q = np.asarray(x, dtype=np.float64) / float(scale)  # planted mistake: fp64 division
        return of.e4m3_encode(q)
    _swap(monkeypatch, of, "quantize", quantize)
    _fails(t_fp8.test_quantize_divides_in_fp32_at_ties)


def test_tail_waste_off_by_one_is_caught(monkeypatch):
    def tail_waste_tokens(num_tokens, block_size):
        return oa.blocks_needed(num_tokens, block_size) * block_size - num_tokens + 1  # planted
    _swap(monkeypatch, oa, "tail_waste_tokens", tail_waste_tokens)
    _fails(t_arith.test_tail_waste_bound_exhaustive, read_golden)


def test_contiguous_fit_in_tokens_is_caught(monkeypatch):
    def contiguous_fit(pool_blocks, max_len, block_size):
        return pool_blocks * block_size // max_len  # planted mistake: reservation not whole blocks
    _swap(monkeypatch, oa, "contiguous_fit", contiguous_fit)
    _fails(t_arith.test_contiguous_fit_brute_force)


def test_inverted_waste_share_is_caught(monkeypatch):
    def reservation_waste_fraction(tokens_used, tokens_reserved):
        return tokens_used / tokens_reserved  # planted mistake: the used share
    _swap(monkeypatch, oa, "reservation_waste_fraction", reservation_waste_fraction)
    _fails(t_arith.test_reservation_waste, read_golden)


@pytest.mark.parametrize("bias,sub_exp", [(8, -6), (7, -7)])
def test_wrong_e4m3_code_values_are_caught(monkeypatch, bias, sub_exp):
    def e4m3_value(code):
        code = int(code) & 0xFF
        s = -1.0 if code & 0x80 else 1.0
        e, m = (code >> 3) & 0xF, code & 0x7
        if e == 0xF and m == 0x7:
            return float("nan")
        if e == 0:
            return s * (m / 8.0) * 2.0 ** sub_exp  # planted mistake when sub_exp != -6
        return s * (1.0 + m / 8.0) * 2.0 ** (e - bias)  # planted mistake when bias != 7
    table = np.array([e4m3_value(c) for c in range(256)])
    _swap(monkeypatch, of, "e4m3_value", e4m3_value)
    monkeypatch.setattr(of, "E4M3_TABLE", table)
    monkeypatch.setattr(of, "_POS_VALUES", table[:0x7F])
    _fails(t_fp8.test_code_values_closed_forms)


def test_values_dequantised_with_the_key_scale_are_caught(monkeypatch):
    def paged_decode_fp8(query, key_codes, value_codes, block_tables, seq_lens, scale, k_scale,
                         v_scale, num_kv_heads):
        kc = of.E4M3_TABLE[np.asarray(key_codes, dtype=np.uint8)] * float(np.float32(k_scale))
        vc = of.E4M3_TABLE[np.asarray(value_codes, dtype=np.uint8)] * float(np.float32(k_scale))
        return opa.paged_decode(query, kc, vc, block_tables, seq_lens, scale, num_kv_heads)
    _swap(monkeypatch, of, "paged_decode_fp8", paged_decode_fp8)
    _fails(t_fp8.test_fp8_decode_is_decode_of_the_dequantized_cache)


def test_normalised_partial_state_is_caught(monkeypatch):
    def partial_attention(q, K, V, scale):
        q = np.asarray(q, dtype=np.float64)
        if K.shape[0] == 0:
            return -np.inf, 0.0, np.zeros(V.shape[1])
        z = scale * (np.asarray(K, dtype=np.float64) @ q)
        w = np.exp(z - z.max())
        return z.max(), w.sum(), (w @ np.asarray(V, dtype=np.float64)) / w.sum()  # planted
    _swap(monkeypatch, opa, "partial_attention", partial_attention)
    _fails(t_attn.test_split_kv_combine_equals_unsplit, [16, 17])


def test_overflow_to_nan_is_caught(monkeypatch):
    real = of.e4m3_encode

    def e4m3_encode(x):
        x = np.asarray(x, dtype=np.float64)
        code = real(x)
        # planted mistake: magnitudes above 448 become NaN instead of saturating
        return np.where(np.abs(x) > 448.0, (code & 0x80) | 0x7F, code).astype(np.uint8)
    _swap(monkeypatch, of, "e4m3_encode", e4m3_encode)
    _fails(t_fp8.test_saturation_and_nan)


def test_skipped_slot_written_is_caught(monkeypatch):
    def reshape_and_cache(key_cache, value_cache, key, value, slot_mapping, block_size):
        for t, slot in enumerate(np.asarray(slot_mapping).reshape(-1)):
            slot = int(slot)  # planted mistake: -1 is not skipped (lands in the last block)
            key_cache[slot // block_size, :, slot % block_size, :] = key[t]
            value_cache[slot // block_size, :, slot % block_size, :] = value[t]
    _swap(monkeypatch, opa, "reshape_and_cache", reshape_and_cache)
    _fails(t_idx.test_reshape_and_cache_bits_and_skip)
