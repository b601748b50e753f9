"""Pins for the oracle's multi-query (prefill / chunked prefill) attention:
a library routine on the contiguous K/V (torch's causal SDPA in fp64), the
decode special case, the chunking invariant and a closed form.  CPU only."""

import numpy as np
import torch

from oracle import attention, paging


def _case(rng, lens, Hq=4, Hkv=2, D=16, bs=16, pool=None):
    nblk = [-(-n // bs) for n in lens]
    pool = pool or sum(nblk) + 3
    perm = rng.permutation(pool)
    tables, k = [], 0
    for nb in nblk:
        tables.append(list(perm[k:k + nb]) + [-1] * (max(nblk) - nb))
        k += nb
    kc = rng.standard_normal((pool, bs, Hkv, D)).astype(np.float16)
    vc = rng.standard_normal((pool, bs, Hkv, D)).astype(np.float16)
    return kc, vc, np.array(tables), np.array(lens)


def test_whole_prompt_equals_causal_sdpa():
    """q_len = len: torch scaled_dot_product_attention(is_causal=True) in fp64
    on the contiguous K/V (GQA by repeating the KV heads), per sequence."""
    rng = np.random.default_rng(3)
    lens = [37, 16, 5]
    Hq, Hkv, D = 4, 2, 16
    kc, vc, bt, sl = _case(rng, lens, Hq, Hkv, D)
    qs = np.concatenate([[0], np.cumsum(lens)])
    q = rng.standard_normal((qs[-1], Hq, D)).astype(np.float16)
    out = attention.prefill_attention(q, kc, vc, bt, sl, qs, 0.25)
    for s, n in enumerate(lens):
        K = paging.gather_sequence(kc, bt[s], n).astype(np.float64)   # [n, Hkv, D]
        V = paging.gather_sequence(vc, bt[s], n).astype(np.float64)
        Kr = torch.from_numpy(K).repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
        Vr = torch.from_numpy(V).repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
        Q = torch.from_numpy(q[qs[s]:qs[s + 1]].astype(np.float64)).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, Kr, Vr, is_causal=True, scale=0.25)
        np.testing.assert_allclose(out[qs[s]:qs[s + 1]], ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_one_query_row_is_decode():
    rng = np.random.default_rng(4)
    lens = [40, 17, 1]
    kc, vc, bt, sl = _case(rng, lens)
    q = rng.standard_normal((3, 4, 16)).astype(np.float16)
    out = attention.prefill_attention(q, kc, vc, bt, sl, np.arange(4), 0.3)
    ref = attention.decode_attention(q, kc, vc, bt, sl, 0.3)
    np.testing.assert_array_equal(out, ref)


def test_chunks_equal_the_whole_prompt():
    """A prompt processed in two chunks (the first chunk's call sees only its
    own tokens cached) gives the rows of the one-shot prefill."""
    rng = np.random.default_rng(5)
    n, c = 45, 20
    kc, vc, bt, _ = _case(rng, [n])
    q = rng.standard_normal((n, 4, 16)).astype(np.float16)
    whole = attention.prefill_attention(q, kc, vc, bt, np.array([n]), np.array([0, n]), 0.25)
    first = attention.prefill_attention(q[:c], kc, vc, bt, np.array([c]), np.array([0, c]), 0.25)
    second = attention.prefill_attention(q[c:], kc, vc, bt, np.array([n]), np.array([0, n - c]), 0.25)
    np.testing.assert_array_equal(first, whole[:c])
    np.testing.assert_array_equal(second, whole[c:])


def test_first_position_sees_only_itself():
    rng = np.random.default_rng(6)
    kc, vc, bt, _ = _case(rng, [30])
    q = rng.standard_normal((30, 4, 16)).astype(np.float16)
    out = attention.prefill_attention(q, kc, vc, bt, np.array([30]), np.array([0, 30]), 0.25)
    v0 = vc[bt[0][0], 0].astype(np.float64)  # [Hkv, D]
    np.testing.assert_array_equal(out[0], np.repeat(v0, 2, axis=0))
