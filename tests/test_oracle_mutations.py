"""Plant a plausible mistake in the oracle (on the CPU) and check that one of
the pins catches it -- evidence that the pins have teeth."""

import numpy as np
import pytest

import tests.test_oracle_pins as pins
from oracle import attention, fp8_e4m3, kv_size, paging


def test_gqa_mapping_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(attention, "kv_head_of", lambda h, hq, hkv: h % hkv)
    with pytest.raises(AssertionError):
        pins.test_attention_matches_sdpa_on_contiguous(4, 16, 2, 128, 16, [511, 512, 513, 40])


def test_offset_mistake_is_caught(monkeypatch):
    orig = paging.locate
    monkeypatch.setattr(paging, "locate", lambda bt, pos, bs: orig(bt, pos + 1, bs) if pos % bs == bs - 1 and (pos + 1) // bs < len(bt) else orig(bt, pos, bs))
    with pytest.raises(AssertionError):
        pins.test_locate({"table": [7, 3, 9, 2, 12], "pos": 47, "physical": 9, "offset": 15, "cite": ""})


def test_missing_max_subtraction_is_caught(monkeypatch):
    def naive(x):
        e = np.exp(x)
        return e / np.sum(e)
    monkeypatch.setattr(attention, "softmax_weights", naive)
    with np.errstate(all="ignore"), pytest.raises(AssertionError):
        pins.test_attention_large_scores_stable()


def test_unnormalised_weights_are_caught(monkeypatch):
    monkeypatch.setattr(attention, "softmax_weights", lambda x: np.exp(x - np.max(x)))
    with pytest.raises(AssertionError):
        pins.test_attention_matches_sdpa_on_contiguous(2, 8, 2, 64, 16, [15, 16])


def test_ties_away_from_zero_is_caught(monkeypatch):
    table = fp8_e4m3.VALUES[:0x7F]

    def away(x):
        x = np.asarray(x, dtype=np.float32)
        a = np.minimum(np.abs(x.astype(np.float64)), 448.0)
        hi = np.minimum(np.searchsorted(table, a), 0x7E)
        lo = np.maximum(hi - 1, 0)
        mid = (table[lo] + table[hi]) / 2
        code = np.where(a >= mid, hi, lo)
        return (code | (np.signbit(x).astype(np.int64) << 7)).astype(np.uint8)
    monkeypatch.setattr(fp8_e4m3, "encode", away)
    with pytest.raises(AssertionError):
        pins.test_fp8_midpoints_round_to_even_and_saturate()


def test_dropped_factor_two_is_caught(monkeypatch):
    monkeypatch.setattr(kv_size, "kv_cache_bytes", lambda L, H, D, S, B, b: L * H * D * S * B * b)
    case = {"args": [32, 32, 128, 2048, 4, 2], "expect_bytes": 4294967296, "printed": "", "cite": ""}
    with pytest.raises(AssertionError):
        pins.test_kv_size_worked_values(case)
