"""Decode attention over a paged KV cache, in fp64, straight from its definition.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

Definition (page "5.KV Cache 管理 & PagedAttention", Q4 decode_step, step 4:
scores = q K^T scaled, masked past each sequence's length, softmax, times V;
page "KV Cache 优化与内存管理深度解析", attention formula
softmax(Q K^T / sqrt(d)) V).  For sequence s and query head h:

    g      = h // (num_heads // num_kv_heads)      grouped-query mapping:
             each KV head is repeated num_heads/num_kv_heads times along the
             head axis (Q7 broadcast_kv_for_gqa, repeat_interleave)
    K_s    = the seq_len_s cached keys of s, re-assembled in token order
             through its block table (Q11 read_kv_range), head g
    V_s    = the same for values
    x_j    = scale * sum_d q[s, h, d] * K_s[j, d]
    out    = sum_j softmax(x)_j * V_s[j, :],
             softmax(x)_j = exp(x_j - max_i x_i) / sum_i exp(x_i - max_i x_i)

computed as two explicit passes (max, then exp and sum) over the whole
sequence.  Only tokens j < seq_len_s take part: slots past the end of the last
block and block-table entries past the last block are never read.  For an
fp8 cache the stored codes are decoded and multiplied by the per-tensor scale
(k_scale for keys, v_scale for values) before any arithmetic.  A sequence of
length 0 yields a zero output row.

Split-KV (``partition_summary`` / ``merge_partitions``) is not on the pages;
it is the log-sum-exp merge of per-partition softmax summaries that the GPU
path uses for long contexts, written here as its plain definition so that the
tests can pin "merge of any partitioning == unsplit".
"""

from __future__ import annotations

import numpy as np

from . import dtypes, paging


def _kv_f64(cache: np.ndarray, block_table, seq_len: int, kv_dtype: str, kv_scale: float) -> np.ndarray:
    raw = paging.gather_sequence(cache, block_table, seq_len)
    vals = dtypes.to_f64(raw, kv_dtype)
    if kv_dtype == dtypes.FP8:
        vals = vals * float(kv_scale)
    return vals  # [seq_len, num_kv_heads, head_dim]


def kv_head_of(h: int, num_heads: int, num_kv_heads: int) -> int:
    """KV head read by query head h: K/V heads repeated num_heads/num_kv_heads
    times along the head axis (repeat_interleave), so h -> h // group."""
    return h // (num_heads // num_kv_heads)


def softmax_weights(x: np.ndarray) -> np.ndarray:
    """softmax of a 1-D score vector: max pass, then exp and sum."""
    m = np.max(x)
    e = np.exp(x - m)
    return e / np.sum(e)


def decode_attention(query, key_cache, value_cache, block_tables, seq_lens, scale,
                     q_dtype="f16", kv_dtype="f16", k_scale=1.0, v_scale=1.0,
                     pairs=None) -> np.ndarray:
    """fp64 decode attention.

    query        [S, Hq, D] raw storage of ``q_dtype``
    key_cache    [NB, block_size, Hkv, D] raw storage of ``kv_dtype``
    value_cache  same shape as key_cache
    block_tables [S, max_blocks_per_seq] int, -1 past each sequence's blocks
    seq_lens     [S] int
    pairs        optional iterable of (s, h): compute only those rows (others
                 stay NaN) -- used to check sampled outputs of large inputs.
    Returns [S, Hq, D] fp64.
    """
    S, Hq, D = query.shape
    Hkv = key_cache.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    q = dtypes.to_f64(query, q_dtype)
    out = np.full((S, Hq, D), np.nan)
    wanted = {}
    if pairs is None:
        for s in range(S):
            wanted[s] = list(range(Hq))
    else:
        for s, h in pairs:
            wanted.setdefault(int(s), []).append(int(h))
    for s, heads in wanted.items():
        n = int(seq_lens[s])
        if n == 0:
            out[s, heads] = 0.0
            continue
        K = _kv_f64(key_cache, block_tables[s], n, kv_dtype, k_scale)
        V = _kv_f64(value_cache, block_tables[s], n, kv_dtype, v_scale)
        for h in heads:
            g = kv_head_of(h, Hq, Hkv)
            x = float(scale) * (K[:, g, :] @ q[s, h])
            w = softmax_weights(x)
            out[s, h] = w @ V[:, g, :]
    return out


def partition_summary(x: np.ndarray, V: np.ndarray, start: int, end: int):
    """Softmax summary of scores x[start:end] against values V[start:end].

    Returns (o_p, m_p, l_p): m_p = max of the scores, l_p = sum of
    exp(x - m_p), o_p = sum of exp(x - m_p) * V / l_p.  An empty range gives
    (0, -inf, 0).
    """
    if end <= start:
        return np.zeros(V.shape[1]), -np.inf, 0.0
    xs = x[start:end]
    m = np.max(xs)
    e = np.exp(xs - m)
    l = np.sum(e)
    return (e @ V[start:end]) / l, m, l


def merge_partitions(parts) -> np.ndarray:
    """Log-sum-exp merge: M = max m_p, w_p = l_p exp(m_p - M), out = sum w_p o_p / sum w_p."""
    ms = [m for (_, m, l) in parts if l > 0]
    M = max(ms)
    num = 0.0
    den = 0.0
    for o, m, l in parts:
        if l == 0:
            continue
        w = l * np.exp(m - M)
        num = num + w * o
        den = den + w
    return num / den


def prefill_attention(query, key_cache, value_cache, block_tables, seq_lens, query_start, scale,
                      q_dtype="f16", kv_dtype="f16", k_scale=1.0, v_scale=1.0, rows=None) -> np.ndarray:
    """fp64 multi-query (prefill / chunked prefill) attention over the paged cache.

    Page "5.KV Cache 管理 & PagedAttention", Q6 ``MHAWithCache`` prefill branch:
    every query position attends causally (the ``torch.tril`` mask) to the
    keys at its own and earlier positions; Q3.3 / Q19: the keys are the
    sequence's cached K/V, read block by block through its table.  Sequence s
    has seq_lens[s] cached tokens (this chunk's K/V already written) and the
    query rows query_start[s] .. query_start[s+1]-1, which are its last
    q_len = query_start[s+1] - query_start[s] positions: row i of the chunk is
    position p = seq_lens[s] - q_len + i and sees keys 0..p.

    query        [T, Hq, D] raw storage of ``q_dtype`` (T = query_start[-1])
    rows         optional iterable of (t, h): compute only those (others NaN)
    Returns [T, Hq, D] fp64.
    """
    T, Hq, D = query.shape
    Hkv = key_cache.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    q = dtypes.to_f64(query, q_dtype)
    out = np.full((T, Hq, D), np.nan)
    wanted = None
    if rows is not None:
        wanted = {}
        for t, h in rows:
            wanted.setdefault(int(t), []).append(int(h))
    for s in range(len(seq_lens)):
        a, b = int(query_start[s]), int(query_start[s + 1])
        n = int(seq_lens[s])
        if b <= a:
            continue
        if b - a > n:
            raise ValueError("more query rows than cached tokens")
        K = _kv_f64(key_cache, block_tables[s], n, kv_dtype, k_scale)
        V = _kv_f64(value_cache, block_tables[s], n, kv_dtype, v_scale)
        for t in range(a, b):
            heads = range(Hq) if wanted is None else wanted.get(t, [])
            p = n - (b - a) + (t - a)  # this row's position
            for h in heads:
                g = kv_head_of(h, Hq, Hkv)
                x = float(scale) * (K[:p + 1, g, :] @ q[t, h])
                w = softmax_weights(x)
                out[t, h] = w @ V[:p + 1, g, :]
    return out
