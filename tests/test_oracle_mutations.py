"""Plants plausible mistakes in the oracle (on the CPU) and checks that at
least one of its pins fails for each, so the pins are not vacuous."""
import math

import numpy as np
import pytest

import oracle as O
import tests.test_oracle_pins as P

_orig_rows = O.attention_rows
_orig_merge = O.merge


def _rows_natural_log(q, k, v, scale, key_counts=None):
    o, l = _orig_rows(q, k, v, scale, key_counts)
    return o, l * math.log(2.0)                    # LSE left in natural units


def _rows_no_scale(q, k, v, scale, key_counts=None):
    return _orig_rows(q, k, v, 1.0, key_counts)


def _rows_scale_twice(q, k, v, scale, key_counts=None):
    return _orig_rows(q, k, v, scale * scale, key_counts)


def _rows_transposed_v(q, k, v, scale, key_counts=None):
    o, l = _orig_rows(q, k, v, scale, key_counts)
    return o[:, ::-1].copy(), l                    # channel order reversed


def _rows_drop_last_key(q, k, v, scale, key_counts=None):
    if key_counts is not None:
        return _orig_rows(q, k, v, scale, key_counts)
    if k.shape[0] > 1:
        return _orig_rows(q, k[:-1], v[:-1], scale)
    return _orig_rows(q, k, v, scale)


_orig_counts = O.causal_key_counts


_orig_quant = O.quantize_int8_blocks


def _quant_scale_128(x_rows, block=128):
    codes, scales = _orig_quant(x_rows, block)
    x32 = np.asarray(x_rows, dtype=np.float32)
    out = codes.copy()
    for b in range(len(scales)):
        blk = x32[b * block:(b + 1) * block]
        s = np.float32(np.abs(blk).max() / np.float32(128.0)) if blk.size and np.abs(blk).max() > 0 else np.float32(1)
        out[b * block:(b + 1) * block] = np.clip(np.rint(blk / s), -127, 127).astype(np.int8)
        scales[b] = s
    return out, scales


def _causal_counts_top_left(n_q, n_k):
    return [min(i + 1, n_k) for i in range(n_q)]   # top-left instead of bottom-right alignment


def _causal_counts_off_by_one(n_q, n_k):
    return [max(c - 1, 0) for c in _orig_counts(n_q, n_k)]   # the diagonal key excluded


def _merge_natural(o_parts, lse_parts):
    op, lp = O.to_f64(o_parts), O.to_f64(lse_parts)
    M = lp.max(axis=0)
    w = np.exp(lp - M[None])                       # e instead of 2
    W = w.sum(axis=0)
    return (w[..., None] * op).sum(0) / W[..., None], M + np.log2(W)


def _shift_wrong_sign(q_rows, mu, scale):
    return -scale * (np.asarray(q_rows) @ np.asarray(mu)) / math.log(2.0)


_orig_bounds = O.split_bounds
_orig_auto = O.auto_num_splits
_orig_sched = O.varlen_schedule


def _bounds_align_32(n, num_splits):
    if n <= 0:
        return _orig_bounds(n, num_splits)
    C = -(-(-(-n // num_splits)) // 32) * 32          # chunk rounded to 32 keys instead of 64
    return [min(s * C, n) for s in range(num_splits + 1)]


def _auto_one_row_group(B, Hkv, Hq, Lq, n, num_sms, D=128):
    return _orig_auto(B, Hkv, Hkv, 1, n, num_sms, D)   # G * Lq rows ignored: one row group per kv head


def _sched_shortest_first(cu_seqlens_q, cu_seqlens_k, H, rows_per_cta=O.PREFILL_ROWS_PER_CTA):
    order, offsets, items = _orig_sched(cu_seqlens_q, cu_seqlens_k, H, rows_per_cta)
    return order[::-1], offsets, items                 # sequences taken shortest first


def _hnd_ignores_layout(x, layout):
    return x                                           # NHD read as if it were HND


def _kv_mean_as_sum(k_rows):
    return np.asarray(k_rows, dtype=np.float64).sum(axis=0)   # column sum, not mean


PIN_TESTS = [
    lambda g: [P.test_brute_force_tiny(s) for s in range(6)],
    lambda g: [P.test_against_torch_float64(s) for s in range(3)],
    lambda g: P.test_closed_forms(),
    lambda g: P.test_randn_lse_near_log2_kv_len(g),
    lambda g: P.test_per16_store_error_magnitude(g),
    lambda g: P.test_smooth_k_invariance(),
    lambda g: [P.test_merge_of_splits_equals_full(s) for s in range(4)],
    lambda g: P.test_merge_special_cases(),
    lambda g: P.test_chunked_merge_equals_full_with_smoothing(),
    lambda g: P.test_causal_key_counts_hand_values(),
    lambda g: [P.test_causal_against_torch_sdpa_float64(sq, sk) for sq, sk in [(7, 7), (5, 9), (9, 5)]],
    lambda g: P.test_causal_decode_and_varlen_reduce_to_dense(),
    lambda g: P.test_int8_quantizer_properties(),
    lambda g: P.test_int8_attention_is_exact_for_representable_inputs(),
    lambda g: P.test_int8_smoothing_is_what_makes_int8_keys_accurate(),
    lambda g: P.test_nhd_matches_hnd(),
    lambda g: P.test_gqa_head_mapping(),
    lambda g: P.test_varlen_equals_dense_per_sequence(),
    lambda g: P.test_lse_layout_adapters(),
    lambda g: P.test_decode_equals_dense_and_kv_len(),
    lambda g: P.test_split_bounds_partition(),
    lambda g: P.test_split_plan_hand_values(),
    lambda g: P.test_varlen_schedule_config4(),
    lambda g: P.test_smooth_k_uncorrected_error_magnitude(g),
    lambda g: P.test_smoothed_rows_with_stored_k_prime_against_torch_float64(),
]


def _some_pin_fails(golden_dir):
    for t in PIN_TESTS:
        try:
            t(golden_dir)
        except (AssertionError, ValueError, IndexError):
            return True
    return False


@pytest.mark.parametrize("name,attr,fn", [
    ("natural log", "attention_rows", _rows_natural_log),
    ("scale dropped", "attention_rows", _rows_no_scale),
    ("scale squared", "attention_rows", _rows_scale_twice),
    ("value channels permuted", "attention_rows", _rows_transposed_v),
    ("last key dropped", "attention_rows", _rows_drop_last_key),
    ("merge weights in base e", "merge", _merge_natural),
    ("smoothing shift sign", "smooth_shift", _shift_wrong_sign),
    ("causal mask aligned top-left", "causal_key_counts", _causal_counts_top_left),
    ("causal mask misses the diagonal", "causal_key_counts", _causal_counts_off_by_one),
    ("int8 scale amax / 128", "quantize_int8_blocks", _quant_scale_128),
    ("split chunk aligned to 32 keys", "split_bounds", _bounds_align_32),
    ("split plan ignores the query row groups", "auto_num_splits", _auto_one_row_group),
    ("varlen work order shortest first", "varlen_schedule", _sched_shortest_first),
    ("NHD read as HND", "_hnd", _hnd_ignores_layout),
    ("smoothing mean is a sum", "kv_mean", _kv_mean_as_sum),
])
def test_planted_mistake_is_caught(monkeypatch, golden_dir, name, attr, fn):
    monkeypatch.setattr(O, attr, fn)
    assert _some_pin_fails(golden_dir), f"no pin caught: {name}"


def test_unmutated_oracle_passes_all(golden_dir):
    assert not _some_pin_fails(golden_dir)
