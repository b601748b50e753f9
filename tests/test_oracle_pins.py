"""Pins for the CPU oracle: worked values printed on the pages, closed forms,
invariants, and library routines on special cases.  CPU only."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention, cache_write, dtypes, fp8_e4m3, kv_size, paging

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return json.load(f)


# ----------------------------------------------------------------- KV size
@pytest.mark.parametrize("case", _golden("kv_size_worked_values.json")["cases"], ids=lambda c: c["printed"])
def test_kv_size_worked_values(case):
    got = kv_size.kv_cache_bytes(*case["args"])
    assert got == case["expect_bytes"], case["cite"]
    if "printed_equals_half" in case:
        # the page's printed figure is the single-tensor (K-only) size
        assert got // 2 == case["printed_equals_half"]


def test_kv_size_gqa_and_fp8_ratios():
    # page "5.KV Cache 管理 & PagedAttention", Q1.1: GQA replaces num_heads by
    # num_kv_heads (LLaMA-2 70B: 64 -> 8) ; Q1.3: FP8 halves the FP16 size.
    mha = kv_size.kv_cache_bytes(80, 64, 128, 8192, 1, 2)
    gqa = kv_size.kv_cache_bytes(80, 8, 128, 8192, 1, 2)
    assert mha == 8 * gqa
    assert gqa == 2684354560  # 2.5 GiB for one 8k-token sequence of the GQA 70B shape
    assert kv_size.kv_cache_bytes(80, 8, 128, 8192, 1, 1) * 2 == gqa


# ----------------------------------------------------------------- paging
PG = _golden("paging_worked_examples.json")


@pytest.mark.parametrize("case", PG["blocks_needed"], ids=lambda c: str(c["tokens"]))
def test_blocks_needed(case):
    assert paging.blocks_needed(case["tokens"], 16) == case["blocks"], case["cite"]


@pytest.mark.parametrize("case", PG["last_block_fill"], ids=lambda c: str(c["tokens"]))
def test_last_block_fill(case):
    n = case["tokens"]
    nb = paging.blocks_needed(n, 16)
    assert n - (nb - 1) * 16 == case["used_in_last"], case["cite"]


@pytest.mark.parametrize("case", PG["locate"], ids=lambda c: str(c["pos"]))
def test_locate(case):
    phys, off = paging.locate(case["table"], case["pos"], 16)
    assert (phys, off) == (case["physical"], case["offset"]), case["cite"]
    assert paging.slot_of(case["table"], case["pos"], 16) == case["physical"] * 16 + case["offset"]


def test_read_range_roundtrip_any_block_size():
    """Scatter a contiguous sequence into random physical blocks, read any
    [start, end) back: it must equal the contiguous slice."""
    rng = np.random.default_rng(0)
    for bs in (1, 3, 8, 16, 32):
        n = 97
        nb = paging.blocks_needed(n, bs)
        pool = nb + 7
        table = rng.permutation(pool)[:nb]
        seq = rng.standard_normal((n, 2, 5)).astype(np.float16)
        cache = rng.standard_normal((pool, bs, 2, 5)).astype(np.float16)
        for pos in range(n):
            b, o = paging.locate(table, pos, bs)
            cache[b, o] = seq[pos]
        for start, end in [(0, n), (0, 1), (bs - 1, bs + 1), (5, 60), (n - 1, n), (3, 3)]:
            np.testing.assert_array_equal(paging.read_range(cache, table, start, end), seq[start:end])


# ----------------------------------------------------------------- formats
def test_fp8_spec_values():
    for c in _golden("fp8_e4m3_spec_values.json")["codes"]:
        v = fp8_e4m3.code_value(c["code"])
        if c["value"] == "nan":
            assert math.isnan(v), c["what"]
        else:
            assert v == c["value"] and math.copysign(1, v) == math.copysign(1, c["value"]), c["what"]


def test_fp8_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = fp8_e4m3.decode(codes.numpy())
    np.testing.assert_array_equal(np.isnan(ref), np.isnan(ours))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ref[ok], ours[ok])


def test_fp8_encode_matches_torch_in_range():
    """torch's float -> float8_e4m3fn cast rounds to nearest-even inside the
    finite range; ours must agree bit for bit there."""
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(50000) * 100).astype(np.float32),
        (rng.standard_normal(50000) * 1e-3).astype(np.float32),
        rng.uniform(-448, 448, 50000).astype(np.float32),
    ])
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(fp8_e4m3.encode(x), ref)


def test_fp8_midpoints_round_to_even_and_saturate():
    vals = fp8_e4m3.VALUES[:0x7F]
    for c in range(0x7E):
        mid = np.float32((vals[c] + vals[c + 1]) / 2)
        assert float(mid) == (vals[c] + vals[c + 1]) / 2  # exact in fp32
        got = int(fp8_e4m3.encode(np.array([mid]))[0])
        assert got == (c if c % 2 == 0 else c + 1), (c, float(mid))
        assert int(fp8_e4m3.encode(np.array([-mid]))[0]) == got | 0x80
    big = np.array([448.0, 449.0, 464.0, 480.0, 1e6, np.inf, -500.0, -np.inf], dtype=np.float32)
    np.testing.assert_array_equal(fp8_e4m3.encode(big), [0x7E] * 6 + [0xFE] * 2)
    assert fp8_e4m3.encode(np.array([np.nan], dtype=np.float32))[0] == 0x7F
    # round trip of every finite code
    finite = [c for c in range(256) if not math.isnan(fp8_e4m3.code_value(c))]
    back = fp8_e4m3.encode(fp8_e4m3.decode(np.array(finite, dtype=np.uint8)).astype(np.float32))
    np.testing.assert_array_equal(back, finite)


def test_bf16_decode_matches_torch():
    bits = torch.arange(0, 65536, 7, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    ours = dtypes.bf16_bits_to_f64(bits.numpy().view(np.uint16))
    np.testing.assert_array_equal(np.isnan(ref), np.isnan(ours))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ref[ok], ours[ok])


# ----------------------------------------------------------------- attention
def _paged_case(rng, S, Hq, Hkv, D, bs, lens, pool_extra=5, q_dtype=np.float16):
    """Contiguous per-sequence K/V drawn first, then scattered into a random pool."""
    nbs = [paging.blocks_needed(n, bs) for n in lens]
    pool = sum(nbs) + pool_extra
    perm = rng.permutation(pool)
    mb = max(max(nbs), 1)
    tables = -np.ones((S, mb), dtype=np.int64)
    kc = rng.standard_normal((pool, bs, Hkv, D)).astype(np.float16)
    vc = rng.standard_normal((pool, bs, Hkv, D)).astype(np.float16)
    Ks, Vs, used = [], [], 0
    for s, n in enumerate(lens):
        tables[s, :nbs[s]] = perm[used:used + nbs[s]]
        used += nbs[s]
        K = rng.standard_normal((n, Hkv, D)).astype(np.float16)
        V = rng.standard_normal((n, Hkv, D)).astype(np.float16)
        for pos in range(n):
            b, o = paging.locate(tables[s], pos, bs)
            kc[b, o] = K[pos]
            vc[b, o] = V[pos]
        Ks.append(K)
        Vs.append(V)
    q = rng.standard_normal((S, Hq, D)).astype(q_dtype)
    return q, kc, vc, tables, np.array(lens), Ks, Vs


def _sdpa_contiguous(q, Ks, Vs, Hq, scale):
    """torch SDPA on contiguous K/V, KV heads repeated for GQA (page "5.KV Cache
    管理 & PagedAttention", Q7 repeat_interleave)."""
    outs = []
    for s in range(q.shape[0]):
        K = torch.from_numpy(Ks[s].astype(np.float64)).permute(1, 0, 2)  # [Hkv, n, D]
        V = torch.from_numpy(Vs[s].astype(np.float64)).permute(1, 0, 2)
        G = Hq // K.shape[0]
        K = K.repeat_interleave(G, dim=0)
        V = V.repeat_interleave(G, dim=0)
        qs = torch.from_numpy(q[s].astype(np.float64)).unsqueeze(1)  # [Hq, 1, D]
        o = torch.nn.functional.scaled_dot_product_attention(qs, K, V, scale=scale)
        outs.append(o.squeeze(1).numpy())
    return np.stack(outs)


CASES = [
    # S, Hq, Hkv, D, bs, lens
    (3, 4, 4, 64, 16, [1, 17, 100]),
    (2, 8, 2, 64, 16, [15, 16]),
    (2, 8, 1, 32, 8, [33, 9]),
    (4, 16, 2, 128, 16, [511, 512, 513, 40]),
    (2, 6, 3, 16, 4, [7, 22]),
    (1, 8, 8, 128, 32, [95]),
]


@pytest.mark.parametrize("S,Hq,Hkv,D,bs,lens", CASES)
def test_attention_matches_sdpa_on_contiguous(S, Hq, Hkv, D, bs, lens):
    rng = np.random.default_rng(S * 100 + Hq + D)
    q, kc, vc, bt, sl, Ks, Vs = _paged_case(rng, S, Hq, Hkv, D, bs, lens)
    scale = 1.0 / math.sqrt(D)
    ours = attention.decode_attention(q, kc, vc, bt, sl, scale)
    ref = _sdpa_contiguous(q, Ks, Vs, Hq, scale)
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-12)


def test_attention_matches_padded_batch_formulation():
    """Page "5.KV Cache 管理 & PagedAttention", Q4 decode_step: pad every
    sequence's history to max_len, fill padded scores with -inf, softmax,
    multiply by V -- done here with torch ops in fp64."""
    rng = np.random.default_rng(7)
    S, Hq, Hkv, D, bs, lens = 3, 4, 4, 32, 16, [5, 40, 23]
    q, kc, vc, bt, sl, Ks, Vs = _paged_case(rng, S, Hq, Hkv, D, bs, lens)
    L = max(lens)
    pk = torch.zeros(S, Hkv, L, D, dtype=torch.float64)
    pv = torch.zeros_like(pk)
    mask = torch.zeros(S, L, dtype=torch.bool)
    for s, n in enumerate(lens):
        pk[s, :, :n] = torch.from_numpy(Ks[s].astype(np.float64)).permute(1, 0, 2)
        pv[s, :, :n] = torch.from_numpy(Vs[s].astype(np.float64)).permute(1, 0, 2)
        mask[s, :n] = True
    qt = torch.from_numpy(q.astype(np.float64)).unsqueeze(2)  # [S, H, 1, D]
    scores = torch.matmul(qt, pk.transpose(-2, -1)) / math.sqrt(D)
    scores = scores.masked_fill(~mask[:, None, None, :], float("-inf"))
    ref = torch.matmul(torch.softmax(scores, dim=-1), pv).squeeze(2).numpy()
    ours = attention.decode_attention(q, kc, vc, bt, sl, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-12)


def test_attention_large_scores_stable():
    """Scores of order 1e3 overflow exp() unless the max is subtracted first."""
    rng = np.random.default_rng(8)
    q, kc, vc, bt, sl, Ks, Vs = _paged_case(rng, 2, 4, 2, 64, 16, [30, 70])
    ours = attention.decode_attention(q, kc, vc, bt, sl, 100.0)
    ref = _sdpa_contiguous(q, Ks, Vs, 4, 100.0)
    assert np.all(np.isfinite(ours))
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-10)


def test_block_permutation_invariance_bit_identical():
    rng = np.random.default_rng(9)
    q, kc, vc, bt, sl, _, _ = _paged_case(rng, 3, 8, 2, 64, 16, [50, 1, 77])
    base = attention.decode_attention(q, kc, vc, bt, sl, 0.125)
    perm = rng.permutation(kc.shape[0])          # new position of each old block
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1)
    out2 = attention.decode_attention(q, kc2, vc2, bt2, sl, 0.125)
    np.testing.assert_array_equal(base, out2)


def test_unused_slots_and_blocks_do_not_matter():
    rng = np.random.default_rng(10)
    q, kc, vc, bt, sl, _, _ = _paged_case(rng, 3, 4, 4, 64, 16, [17, 31, 48])
    base = attention.decode_attention(q, kc, vc, bt, sl, 0.125)
    used = set()
    kc2, vc2 = kc.copy(), vc.copy()
    for s, n in enumerate(sl):
        nb = paging.blocks_needed(n, 16)
        used.update(bt[s, :nb].tolist())
        tail = n - (nb - 1) * 16
        kc2[bt[s, nb - 1], tail:] = np.nan
        vc2[bt[s, nb - 1], tail:] = np.inf
    for b in range(kc.shape[0]):
        if b not in used:
            kc2[b] = np.nan
            vc2[b] = np.nan
    out = attention.decode_attention(q, kc2, vc2, bt, sl, 0.125)
    np.testing.assert_array_equal(base, out)


def test_closed_forms():
    rng = np.random.default_rng(11)
    D, bs = 16, 4
    # length 1: the output is exactly the single value row
    q, kc, vc, bt, sl, Ks, Vs = _paged_case(rng, 1, 2, 1, D, bs, [1])
    out = attention.decode_attention(q, kc, vc, bt, sl, 0.3)
    np.testing.assert_array_equal(out[0, 0], Vs[0][0, 0].astype(np.float64))
    np.testing.assert_array_equal(out[0, 1], Vs[0][0, 0].astype(np.float64))
    # all keys equal (or q = 0): uniform weights, output = mean of V
    n = 13
    q, kc, vc, bt, sl, Ks, Vs = _paged_case(rng, 1, 1, 1, D, bs, [n])
    for pos in range(n):
        b, o = paging.locate(bt[0], pos, bs)
        kc[b, o] = kc[bt[0, 0], 0]
    out = attention.decode_attention(q, kc, vc, bt, sl, 0.7)
    np.testing.assert_allclose(out[0, 0], Vs[0][:, 0].astype(np.float64).mean(0), rtol=0, atol=1e-14)
    q0 = np.zeros_like(q)
    q, kc, vc, bt, sl, Ks, Vs = _paged_case(rng, 1, 1, 1, D, bs, [n])
    out = attention.decode_attention(q0, kc, vc, bt, sl, 0.7)
    np.testing.assert_allclose(out[0, 0], Vs[0][:, 0].astype(np.float64).mean(0), rtol=0, atol=1e-14)
    # identical value rows: output = that row, whatever the scores
    for pos in range(n):
        b, o = paging.locate(bt[0], pos, bs)
        vc[b, o] = vc[bt[0, 0], 0]
    out = attention.decode_attention(q, kc, vc, bt, sl, 0.7)
    np.testing.assert_allclose(out[0, 0], vc[bt[0, 0], 0, 0].astype(np.float64), rtol=0, atol=1e-14)
    # two tokens: weights are the logistic function of the score difference
    q, kc, vc, bt, sl, Ks, Vs = _paged_case(rng, 1, 1, 1, D, bs, [2])
    K = Ks[0][:, 0].astype(np.float64)
    V = Vs[0][:, 0].astype(np.float64)
    qq = q[0, 0].astype(np.float64)
    d = 0.5 * (qq @ K[0] - qq @ K[1])
    w0 = 1.0 / (1.0 + math.exp(-d))
    out = attention.decode_attention(q, kc, vc, bt, sl, 0.5)
    np.testing.assert_allclose(out[0, 0], w0 * V[0] + (1 - w0) * V[1], rtol=0, atol=1e-14)


def test_zero_length_sequence_gives_zeros():
    rng = np.random.default_rng(12)
    q, kc, vc, bt, sl, _, _ = _paged_case(rng, 2, 2, 2, 16, 4, [5, 3])
    sl = np.array([5, 0])
    out = attention.decode_attention(q, kc, vc, bt, sl, 0.25)
    assert np.all(out[1] == 0)


@pytest.mark.parametrize("part", [1, 5, 16, 32, 64, 1000])
def test_split_merge_equals_unsplit(part):
    rng = np.random.default_rng(13)
    n, D = 200, 32
    x = rng.standard_normal(n) * 3
    V = rng.standard_normal((n, D))
    direct = attention.softmax_weights(x) @ V
    parts = [attention.partition_summary(x, V, a, min(n, a + part)) for a in range(0, n, part)]
    parts.append(attention.partition_summary(x, V, n, n))  # an empty partition
    np.testing.assert_allclose(attention.merge_partitions(parts), direct, rtol=0, atol=1e-13)


def test_gqa_equals_mha_on_repeated_heads():
    """G-fold GQA == MHA on K/V whose heads are explicitly repeated (Q7)."""
    rng = np.random.default_rng(14)
    q, kc, vc, bt, sl, _, _ = _paged_case(rng, 2, 8, 2, 32, 16, [20, 45])
    gqa = attention.decode_attention(q, kc, vc, bt, sl, 0.2)
    mha = attention.decode_attention(q, np.repeat(kc, 4, axis=2), np.repeat(vc, 4, axis=2), bt, sl, 0.2)
    np.testing.assert_array_equal(gqa, mha)


def test_fp8_cache_dequantisation_matches_torch_cast():
    """fp8 cache: the oracle's value is SDPA on torch-decoded codes x scale."""
    rng = np.random.default_rng(15)
    S, Hq, Hkv, D, bs = 2, 8, 2, 64, 16
    lens = [37, 64]
    q, kc, vc, bt, sl, _, _ = _paged_case(rng, S, Hq, Hkv, D, bs, lens)
    ks, vs = 0.011, 0.013
    kc8 = torch.from_numpy(kc.astype(np.float32) / np.float32(ks)).to(torch.float8_e4m3fn)
    vc8 = torch.from_numpy(vc.astype(np.float32) / np.float32(vs)).to(torch.float8_e4m3fn)
    ours = attention.decode_attention(q, kc8.view(torch.uint8).numpy(), vc8.view(torch.uint8).numpy(),
                                      bt, sl, 0.125, kv_dtype="fp8_e4m3", k_scale=ks, v_scale=vs)
    Ks, Vs = [], []
    kd = kc8.to(torch.float64).numpy() * ks
    vd = vc8.to(torch.float64).numpy() * vs
    for s, n in enumerate(lens):
        Ks.append(np.stack([kd[bt[s, p // bs], p % bs] for p in range(n)]))
        Vs.append(np.stack([vd[bt[s, p // bs], p % bs] for p in range(n)]))
    ref = _sdpa_contiguous(q, Ks, Vs, Hq, 0.125)
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-12)


def test_bf16_query_and_cache():
    rng = np.random.default_rng(16)
    S, Hq, Hkv, D, bs = 2, 4, 2, 32, 16
    q, kc, vc, bt, sl, Ks, Vs = _paged_case(rng, S, Hq, Hkv, D, bs, [20, 9])
    to_bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
    qb, kb, vb = to_bf(q), to_bf(kc), to_bf(vc)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    ours = attention.decode_attention(bits(qb), bits(kb), bits(vb), bt, sl, 0.17, q_dtype="bf16", kv_dtype="bf16")
    kd, vd = kb.double().numpy(), vb.double().numpy()
    Ks = [np.stack([kd[bt[s, p // bs], p % bs] for p in range(n)]) for s, n in enumerate(sl)]
    Vs = [np.stack([vd[bt[s, p // bs], p % bs] for p in range(n)]) for s, n in enumerate(sl)]
    ref = _sdpa_contiguous(qb.double().numpy(), Ks, Vs, Hq, 0.17)
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-12)


# ----------------------------------------------------------------- cache write
def test_cache_write_slots_and_untouched_bytes():
    rng = np.random.default_rng(17)
    NB, bs, Hkv, D, T = 10, 16, 2, 8, 6
    kc = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float16)
    vc = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float16)
    k0, v0 = kc.copy(), vc.copy()
    key = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    val = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    slots = np.array([0, 17, -1, 159, 40, -5])
    cache_write.reshape_and_cache(key, val, kc, vc, slots)
    touched = np.zeros((NB, bs), dtype=bool)
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        touched[sl // bs, sl % bs] = True
        np.testing.assert_array_equal(kc[sl // bs, sl % bs].view(np.uint16), key[t].view(np.uint16))
        np.testing.assert_array_equal(vc[sl // bs, sl % bs].view(np.uint16), val[t].view(np.uint16))
    np.testing.assert_array_equal(kc[~touched].view(np.uint16), k0[~touched].view(np.uint16))
    np.testing.assert_array_equal(vc[~touched].view(np.uint16), v0[~touched].view(np.uint16))


def test_append_rule_round_trip():
    """Page "5.KV Cache 管理 & PagedAttention", Q12: appending tokens one at a
    time at (block_table[len // bs], len % bs) and reading the sequence back
    (Q11) returns the tokens in order."""
    rng = np.random.default_rng(18)
    bs, Hkv, D = 16, 2, 8
    free = list(rng.permutation(20))
    table, n = [], 0
    kc = np.zeros((20, bs, Hkv, D), dtype=np.float16)
    vc = np.zeros_like(kc)
    toks = rng.standard_normal((70, Hkv, D)).astype(np.float16)
    for t in range(70):
        if n % bs == 0:
            table.append(free.pop())
        slot = paging.slot_of(table, n, bs)
        cache_write.reshape_and_cache(toks[t:t + 1], toks[t:t + 1], kc, vc, [slot])
        n += 1
    np.testing.assert_array_equal(paging.gather_sequence(kc, table, n), toks)
    assert len(table) == paging.blocks_needed(70, bs)


def test_cache_write_fp8_matches_torch_cast():
    rng = np.random.default_rng(19)
    NB, bs, Hkv, D, T = 6, 16, 2, 64, 5
    key = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    val = (rng.standard_normal((T, Hkv, D)) * 3).astype(np.float16)
    ks, vs = np.float32(0.00873), np.float32(0.031)
    kc = np.zeros((NB, bs, Hkv, D), dtype=np.uint8)
    vc = np.zeros_like(kc)
    slots = np.array([3, 50, 51, 95, 0])
    cache_write.reshape_and_cache(key, val, kc, vc, slots, src_dtype="f16", cache_dtype="fp8_e4m3",
                                  k_scale=float(ks), v_scale=float(vs))
    for t, sl in enumerate(slots):
        kref = (torch.from_numpy(key[t].astype(np.float32)) / torch.tensor(ks)).to(torch.float8_e4m3fn)
        vref = (torch.from_numpy(val[t].astype(np.float32)) / torch.tensor(vs)).to(torch.float8_e4m3fn)
        np.testing.assert_array_equal(kc[sl // bs, sl % bs], kref.view(torch.uint8).numpy())
        np.testing.assert_array_equal(vc[sl // bs, sl % bs], vref.view(torch.uint8).numpy())
