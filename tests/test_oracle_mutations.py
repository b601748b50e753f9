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


# ---------------------------------------------------------------- later oracles

import tests.test_oracle_block_manager as bm_pins
import tests.test_oracle_prefill as pf_pins
import tests.test_oracle_prefix_sharing as ps_pins
from oracle import block_manager, prefix_sharing


def _prefill_off_by_one(query, key_cache, value_cache, block_tables, seq_lens, query_start, scale,
                        q_dtype="f16", kv_dtype="f16", k_scale=1.0, v_scale=1.0, rows=None):
    """The causal mask one key short (keys < p instead of <= p, but at least one)."""
    from oracle import dtypes
    T, Hq, D = query.shape
    Hkv = key_cache.shape[2]
    q = dtypes.to_f64(query, q_dtype)
    out = np.full((T, Hq, D), np.nan)
    for s in range(len(seq_lens)):
        a, b, n = int(query_start[s]), int(query_start[s + 1]), int(seq_lens[s])
        K = attention._kv_f64(key_cache, block_tables[s], n, kv_dtype, k_scale)
        V = attention._kv_f64(value_cache, block_tables[s], n, kv_dtype, v_scale)
        for t in range(a, b):
            p = n - (b - a) + (t - a)
            for h in range(Hq):
                g = attention.kv_head_of(h, Hq, Hkv)
                x = float(scale) * (K[:max(p, 1), g, :] @ q[t, h])
                out[t, h] = attention.softmax_weights(x) @ V[:max(p, 1), g, :]
    return out


def test_prefill_causal_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(attention, "prefill_attention", _prefill_off_by_one)
    with pytest.raises(AssertionError):
        pf_pins.test_whole_prompt_equals_causal_sdpa()


def test_free_list_taken_from_the_front_is_caught(monkeypatch):
    def allocate_front(self):
        if not self.free_blocks and not self._evict_one_cached():
            raise block_manager.OutOfBlocks("none")
        blk = self.free_blocks.pop(0)
        self.ref_counts[blk] = 1
        return blk
    monkeypatch.setattr(block_manager.BlockManager, "allocate", allocate_front)
    with pytest.raises(AssertionError):
        bm_pins.test_free_list_pops_the_end()


def test_write_into_a_shared_block_without_copy_is_caught(monkeypatch):
    def append_no_cow(self, sid, n):
        table = self._seq(sid)
        slots = []
        for _ in range(n):
            pos = self.lens[sid]
            lb, off = divmod(pos, self.block_size)
            if lb == len(table):
                table.append(self.allocate())
            slots.append(table[lb] * self.block_size + off)
            self.lens[sid] = pos + 1
        return slots, []
    monkeypatch.setattr(block_manager.BlockManager, "append_tokens", append_no_cow)
    with pytest.raises(AssertionError):
        bm_pins.test_fork_then_write_copies_the_shared_partial_block()


def test_partial_block_counted_as_shared_is_caught(monkeypatch):
    def common_with_partial(rows, lens, block_size=16):
        rows = [list(r) for r in rows]
        if not rows:
            return 0
        full = min(-(-int(n) // block_size) for n in lens)  # rounds up: a partly filled block counts
        b = 0
        while b < full and all(r[b] == rows[0][b] for r in rows):
            b += 1
        return b
    monkeypatch.setattr(prefix_sharing, "common_prefix_blocks", common_with_partial)
    with pytest.raises(AssertionError):
        ps_pins.test_fork_shares_every_whole_block()
