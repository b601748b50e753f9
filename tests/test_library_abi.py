"""The C-ABI library: builds, loads, exports every declared symbol, and its
host-side validation answers without a GPU.  CPU only (no compute calls)."""

import ctypes
import os

import pytest

from paged_kv_cache_463_b200 import binding as b
from paged_kv_cache_463_b200 import build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return b.load_library()


def test_exports_every_declared_symbol(lib):
    declared = b.header_functions()
    assert len(declared) >= 11
    for name in declared:
        assert hasattr(lib, name), name
    # and the binding types exactly the declared set
    assert {"paged_attn_create", "paged_attn_destroy", "reshape_and_cache", "paged_attention_decode"} <= set(declared)


def test_status_strings(lib):
    for st in (b.PA_OK, b.PA_ERR_INVALID_ARG, b.PA_ERR_UNSUPPORTED, b.PA_ERR_CUDA, b.PA_ERR_DEVICE_CHECK,
               b.PA_ERR_NO_MEMORY):
        s = lib.paged_attn_status_string(st).decode()
        assert s and s != "unknown status"
    assert lib.paged_attn_status_string(12345).decode() == "unknown status"


def _create(lib, **kw):
    base = dict(num_heads=32, num_kv_heads=8, head_dim=128, block_size=16, num_blocks=64, q_dtype=0, kv_dtype=0,
                max_num_seqs=4, max_blocks_per_seq=8, partition_tokens=-1, device=0, flags=0)
    base.update(kw)
    cfg = b.PaConfig(*[base[n] for n, _ in b.PaConfig._fields_])
    ctx = ctypes.c_void_p()
    st = lib.paged_attn_create(ctypes.byref(cfg), ctypes.byref(ctx))
    return st, ctx


@pytest.mark.parametrize("kw,expect", [
    (dict(num_kv_heads=5), b.PA_ERR_INVALID_ARG),         # Hq % Hkv != 0
    (dict(num_heads=0), b.PA_ERR_INVALID_ARG),
    (dict(num_blocks=0), b.PA_ERR_INVALID_ARG),
    (dict(max_num_seqs=0), b.PA_ERR_INVALID_ARG),
    (dict(flags=2), b.PA_ERR_INVALID_ARG),              # unknown flag bit
    (dict(partition_tokens=100), b.PA_ERR_INVALID_ARG),   # not a block multiple
    (dict(partition_tokens=-2), b.PA_ERR_INVALID_ARG),
    (dict(block_size=32), b.PA_ERR_UNSUPPORTED),
    (dict(head_dim=96), b.PA_ERR_UNSUPPORTED),
    (dict(kv_dtype=2, head_dim=64), b.PA_ERR_UNSUPPORTED),  # fp8 needs 128-byte rows
    (dict(kv_dtype=2, q_dtype=1), b.PA_ERR_UNSUPPORTED),    # fp8 pairs with fp16 queries
    (dict(kv_dtype=1, q_dtype=0), b.PA_ERR_UNSUPPORTED),    # 16-bit cache == query type
    (dict(q_dtype=7), b.PA_ERR_INVALID_ARG),
])
def test_create_validation(lib, kw, expect):
    st, ctx = _create(lib, **kw)
    assert st == expect
    assert not ctx.value


def test_null_arguments(lib):
    assert lib.paged_attn_create(None, None) == b.PA_ERR_INVALID_ARG
    ctx = ctypes.c_void_p()
    assert lib.paged_attn_create(None, ctypes.byref(ctx)) == b.PA_ERR_INVALID_ARG
    assert lib.paged_attn_destroy(None) == b.PA_ERR_INVALID_ARG
    assert lib.paged_attention_decode(None, *([None] * 5), 1, None, 1, 1, 1.0, 1.0, 1.0, None) == b.PA_ERR_INVALID_ARG
    assert lib.reshape_and_cache(None, None, None, 8, 8, None, None, None, 1, 1.0, 1.0, None) == b.PA_ERR_INVALID_ARG
    assert lib.paged_attn_get_error(None, None) == b.PA_ERR_INVALID_ARG


def test_library_is_in_tree():
    assert os.path.dirname(b.DEFAULT_LIB).startswith(os.path.dirname(os.path.abspath(b.__file__)))
