"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

Every mutant is applied with monkeypatch, so the oracle itself is untouched
once the test ends.
"""
import numpy as np
import pytest

import oracle.paged_attention as pa
import oracle.quant as oq
import test_oracle_attention as pins
import test_oracle_quant as qpins
from conftest import read_golden


def _fails(check):
    with pytest.raises(AssertionError):
        check()


def test_interleaved_gqa_mapping_is_caught(monkeypatch):
    monkeypatch.setattr(pa, "kv_head_of", lambda h, n_q, n_kv: h % n_kv)
    _fails(pins.check_contiguous_equals_sdpa)
    _fails(lambda: pins.test_gqa_mapping_example(read_golden))


def test_dropped_scale_is_caught(monkeypatch):
    real = pa.attention_one_sequence
    monkeypatch.setattr(pa, "attention_one_sequence", lambda q, K, V, sm_scale, **kw: real(q, K, V, 1.0, **kw))
    _fails(pins.check_against_brute)


def test_missing_length_truncation_is_caught(monkeypatch):
    def whole_blocks(cache, block_row, length, block_size):
        n_blocks = -(-length // block_size)
        return np.concatenate([cache[int(block_row[j])] for j in range(n_blocks)], axis=0) if n_blocks else cache[:0, 0]

    monkeypatch.setattr(pa, "gather_sequence", whole_blocks)
    _fails(pins.check_against_brute)


def test_wrong_row_order_is_caught(monkeypatch):
    real = pa.gather_sequence

    def reversed_rows(cache, block_row, length, block_size):
        n_blocks = -(-length // block_size)
        blocks = [cache[int(block_row[j])][::-1] for j in range(n_blocks)]
        return np.concatenate(blocks, axis=0)[:length] if blocks else real(cache, block_row, length, block_size)

    monkeypatch.setattr(pa, "gather_sequence", reversed_rows)
    _fails(pins.check_against_brute)


def test_swapped_key_value_is_caught(monkeypatch):
    real = pa.attention_one_sequence
    monkeypatch.setattr(pa, "attention_one_sequence", lambda q, K, V, s, **kw: real(q, V, K, s, **kw))
    _fails(pins.check_against_brute)


def test_unnormalised_softmax_is_caught(monkeypatch):
    real = pa.attention_one_sequence

    def unnormalised(q, K, V, sm_scale, **kw):
        out, lse = real(q, K, V, sm_scale)
        return out * np.exp(lse - lse.max())[:, None], lse

    monkeypatch.setattr(pa, "attention_one_sequence", unnormalised)
    _fails(pins.check_against_brute)


def test_wrong_largest_code_is_caught(monkeypatch):
    real = oq.absmax_quantize
    monkeypatch.setattr(qpins, "absmax_quantize", lambda v, bits, ft=np.float64: real(v, bits + 1, ft))
    _fails(lambda: qpins.test_absmax_4bit_worked_example_float64(read_golden))


def test_truncating_rounding_is_caught(monkeypatch):
    monkeypatch.setattr(oq.np, "rint", np.trunc)
    _fails(lambda: qpins.test_absmax_4bit_worked_example_float64(read_golden))


def test_int8_scale_of_wrong_head_is_caught(monkeypatch):
    real = pa.dequantize_rows

    def head0_scale(rows, cache_dtype, row_scales=None, head_scales=None):
        if cache_dtype == "int8":
            row_scales = np.repeat(np.asarray(row_scales)[:, :1], rows.shape[1], axis=1)
        return real(rows, cache_dtype, row_scales, head_scales)

    monkeypatch.setattr(pa, "dequantize_rows", head0_scale)
    _fails(lambda: pins.test_quantized_decode_is_attention_over_dequantized_rows("int8"))


def test_copy_direction_swapped_is_caught(monkeypatch):
    import numpy as np

    import oracle.block_ops as bo
    import test_oracle_block_ops as bpins

    real = bo.copy_blocks
    monkeypatch.setattr(bpins, "copy_blocks", lambda pools, pairs: real(pools, np.asarray(pairs)[:, ::-1]))
    _fails(bpins.test_copy_on_write_divergence)


def test_swap_ignoring_destination_slot_is_caught(monkeypatch):
    import numpy as np

    import oracle.block_ops as bo
    import test_oracle_block_ops as bpins

    real = bo.swap_blocks
    monkeypatch.setattr(bpins, "swap_blocks",
                        lambda s, d, pairs: real(s, d, np.stack([np.asarray(pairs)[:, 0]] * 2, axis=1)))
    _fails(lambda: bpins.test_offload_example(read_golden))


def test_window_off_by_one_is_caught(monkeypatch):
    import numpy as np

    def shifted(length, window=0, sinks=0):
        pos = np.arange(length)
        if window <= 0:
            return pos
        return pos[(pos > length - window) | (pos < sinks)]

    import test_oracle_window as wpins

    monkeypatch.setattr(pa, "attended_positions", shifted)
    _fails(lambda: wpins.test_sliding_window_example(read_golden))


def test_quest_score_without_min_is_caught(monkeypatch):
    import numpy as np

    import oracle.quest as oq
    import test_oracle_quest as qpins

    def max_only(q, mins, maxs):
        q = np.asarray(q, dtype=np.float64)
        n_q, n_kv = q.shape[0], mins.shape[1]
        return np.stack([(q[h] * maxs[:, h // (n_q // n_kv), :]).sum(axis=1) for h in range(n_q)])

    monkeypatch.setattr(oq, "page_scores", max_only)
    _fails(qpins.check_upper_bound)


def test_quest_selecting_lowest_scores_is_caught(monkeypatch):
    import numpy as np

    import oracle.quest as oq
    import test_oracle_quest as qpins

    monkeypatch.setattr(oq, "select_pages", lambda s, k: np.sort(np.argsort(np.asarray(s))[: min(k, len(s))]))
    _fails(lambda: qpins.test_quest_worked_example(read_golden))


def test_swapped_int4_nibbles_are_caught(monkeypatch):
    import test_oracle_formats as fpins

    def swapped(codes):
        c = np.asarray(codes, dtype=np.int64)
        nib = (c & 0xF).astype(np.uint8)
        return (nib[..., 1::2] | (nib[..., 0::2] << 4)).astype(np.uint8)

    monkeypatch.setattr(oq, "pack_int4", swapped)
    monkeypatch.setattr(pa, "pack_int4", swapped)
    _fails(fpins.test_int4_nibble_order)
    _fails(fpins.test_int4_cache_decode_is_attention_over_restored_values)


def test_e5m2_wrong_bias_is_caught(monkeypatch):
    import test_oracle_formats as fpins

    t = oq.e5m2_value_table() * 2.0  # bias 14 instead of 15
    monkeypatch.setattr(oq, "e5m2_value_table", lambda: t)
    _fails(fpins.test_e5m2_table_closed_forms)
    _fails(fpins.test_e5m2_table_matches_torch_float8)


def test_kivi_keys_grouped_per_token_are_caught(monkeypatch):
    import oracle.kivi as ok
    import test_oracle_kivi as kpins

    def per_token(k_rows, v_rows, bits=ok.KIVI_BITS):
        k_rows = np.asarray(k_rows, np.float32)
        kc, ksc, vc, vsc = real(k_rows, v_rows, bits)
        for t in range(k_rows.shape[0]):
            for h in range(k_rows.shape[1]):
                codes, scale, _ = oq.absmax_quantize(k_rows[t, h], bits, np.float32)
                kc[t, h] = codes
                ksc[h] = scale  # the last token's scale stands for the block
        return kc, ksc, vc, vsc

    real = ok.kivi_quantize_block
    monkeypatch.setattr(ok, "kivi_quantize_block", per_token)
    _fails(kpins.test_two_bit_codes_closed_form)
    _fails(kpins.test_key_groups_are_channels)


def test_kivi_at_four_bits_is_caught(monkeypatch):
    import oracle.kivi as ok
    import test_oracle_kivi as kpins

    real = ok.kivi_quantize_block
    monkeypatch.setattr(ok, "kivi_quantize_block", lambda k, v, bits=4: real(k, v, 4))
    _fails(kpins.test_two_bit_codes_closed_form)
    _fails(kpins.test_round_trip_bounds)


def test_kivi_residual_dropped_is_caught(monkeypatch):
    import oracle.kivi as ok
    import test_oracle_kivi as kpins

    real = ok.kivi_decode
    monkeypatch.setattr(ok, "kivi_decode", lambda q, b, rk, rv, s: real(q, b, rk[:0], rv[:0], s))
    _fails(kpins.test_decode_is_attention_over_restored_rows)
