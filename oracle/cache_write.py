"""The per-step cache write ("reshape_and_cache"): scatter new K/V into slots.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

Page "5.KV Cache 管理 & PagedAttention", Q12 append_token: a new token at
position len is written to physical block block_table[len // block_size] at
offset len % block_size.  Batched over tokens, the caller passes each token's
flat slot = physical_block * block_size + offset directly ("slot_mapping");
a negative slot means "do not write this token".

For 16-bit caches the bytes of key[t, h, :] are copied unchanged.  For an
fp8 E4M3 cache each element is converted to fp32 (exact), divided by the
per-tensor scale in IEEE fp32 (correctly rounded), and encoded with
``fp8_e4m3.encode`` (nearest, ties to even, saturating at +-448).
"""

from __future__ import annotations

import numpy as np

from . import dtypes, fp8_e4m3


def quantize(x_raw: np.ndarray, x_dtype: str, scale: float) -> np.ndarray:
    """16-bit storage -> E4M3 codes of x / scale (division in fp32)."""
    x32 = dtypes.to_f32(x_raw, x_dtype)
    q = x32 / np.float32(scale)  # numpy float32 / float32: IEEE binary32 division
    return fp8_e4m3.encode(q.astype(np.float32))


def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping,
                      src_dtype="f16", cache_dtype="f16", k_scale=1.0, v_scale=1.0) -> None:
    """In place: for every token t with slot >= 0 and every KV head,
    key_cache[slot // bs, slot % bs] = key[t] (value likewise).

    key, value            [T, Hkv, D] raw 16-bit storage of ``src_dtype``
    key_cache, value_cache [NB, bs, Hkv, D] raw storage of ``cache_dtype``
    slot_mapping          [T] int
    """
    bs = key_cache.shape[1]
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        blk, off = slot // bs, slot % bs
        if cache_dtype == dtypes.FP8:
            key_cache[blk, off] = quantize(key[t], src_dtype, k_scale)
            value_cache[blk, off] = quantize(value[t], src_dtype, v_scale)
        else:
            if cache_dtype != src_dtype:
                raise ValueError("16-bit caches store the source format unchanged")
            key_cache[blk, off] = key[t]
            value_cache[blk, off] = value[t]
