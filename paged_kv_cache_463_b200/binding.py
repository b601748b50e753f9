"""ctypes binding of ``libpaged_attn.so`` (include/paged_attn.h).

Argument marshalling only: torch tensors are passed as device pointers plus
sizes, the stream is torch's current stream unless one is given, and every
step of the computation runs in the library's kernels.  There is no fallback:
if the library is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
DEFAULT_LIB = os.path.join(_PKG, "lib", "libpaged_attn.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "paged_attn.h")
HEADERS = [HEADER, os.path.join(os.path.dirname(_PKG), "include", "block_manager.h")]

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_UNSUPPORTED = -2
PA_ERR_CUDA = -3
PA_ERR_DEVICE_CHECK = -4
PA_ERR_NO_MEMORY = -5
PA_ERR_SCRATCH_TOO_SMALL = -6
PA_ERR_OUT_OF_BLOCKS = -7
PA_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
PA_CHECK_BAD_BLOCK, PA_CHECK_BAD_SLOT, PA_CHECK_SEQ_TOO_LONG, PA_CHECK_WAIT_TIMEOUT = 1, 2, 4, 8
PA_CHECK_BAD_PREFIX = 16
PA_FLAG_SHARED_PREFIX = 1
PA_PARTITION_NONE, PA_PARTITION_AUTO = 0, -1
DTYPE_CODES = {"f16": 0, "bf16": 1, "fp8_e4m3": 2}
TORCH_OF = {"f16": torch.float16, "bf16": torch.bfloat16, "fp8_e4m3": torch.float8_e4m3fn}


class PaConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "num_heads", "num_kv_heads", "head_dim", "block_size", "num_blocks", "q_dtype", "kv_dtype",
        "max_num_seqs", "max_blocks_per_seq", "partition_tokens", "device", "flags")]


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(what)
        self.status = status


_LIBS: dict[str, ctypes.CDLL] = {}
_P = ctypes.c_void_p


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load (once) and type the library; raises if it is not built."""
    path = os.path.abspath(path or DEFAULT_LIB)
    if path in _LIBS:
        return _LIBS[path]
    if not os.path.exists(path):
        raise PagedAttnError(PA_ERR_CUDA, f"{path} not built: run `python -m paged_kv_cache_463_b200.build`")
    lib = ctypes.CDLL(path)
    i, i64, f = ctypes.c_int, ctypes.c_int64, ctypes.c_float
    sig = {
        "paged_attn_create": (i, [ctypes.POINTER(PaConfig), ctypes.POINTER(_P)]),
        "paged_attn_destroy": (i, [_P]),
        "reshape_and_cache": (i, [_P, _P, _P, i64, i64, _P, _P, _P, i, f, f, _P]),
        "paged_attention_decode": (i, [_P, _P, _P, _P, _P, _P, i, _P, i, i, f, f, f, _P]),
        "paged_attention_decode_shared_prefix": (i, [_P, _P, _P, _P, _P, _P, i, _P, i, i, _P, _P, i, i, i, f, f, f,
                                                     _P]),
        "paged_attention_prefill": (i, [_P, _P, _P, _P, _P, _P, i, _P, _P, i, i, i, i, f, f, f, _P]),
        "paged_attn_get_error": (i, [_P, _P]),
        "paged_attn_test_wait_timeout": (i, [_P, ctypes.c_longlong]),
        "paged_attn_last_check_bits": (i, [_P]),
        "paged_attn_status_string": (ctypes.c_char_p, [i]),
        "paged_attn_last_error": (ctypes.c_char_p, [_P]),
        "paged_attn_set_partition_tokens": (i, [_P, i]),
        "paged_attn_get_partition_tokens": (i, [_P, ctypes.POINTER(i)]),
        "paged_gather_kv": (i, [_P, _P, _P, _P, _P, _P, i, _P]),
        "paged_copy_blocks": (i, [_P, _P, _P, i64, _P, _P, i64, _P, i, _P]),
        "paged_attention_decode_noalloc": (i, [_P, _P, _P, _P, _P, i, _P, i, i, i, i, i, i, i, i, i, i, f, f, f,
                                               _P, _P]),
        # block manager (include/block_manager.h)
        "pa_bm_create": (i, [i, i, ctypes.POINTER(_P)]),
        "pa_bm_destroy": (i, [_P]),
        "pa_bm_num_free": (i, [_P, _P]),
        "pa_bm_ref_count": (i, [_P, i, _P]),
        "pa_bm_cached_blocks": (i, [_P, _P]),
        "pa_bm_add_sequence": (i, [_P, i64]),
        "pa_bm_free_sequence": (i, [_P, i64]),
        "pa_bm_ensure_capacity": (i, [_P, i64, i64]),
        "pa_bm_append_tokens": (i, [_P, i64, i, _P, _P, _P, _P]),
        "pa_bm_append_batch": (i, [_P, _P, i, _P, _P, _P, _P]),
        "pa_bm_fork": (i, [_P, i64, i64]),
        "pa_bm_seq_len": (i, [_P, i64, _P]),
        "pa_bm_block_table": (i, [_P, i64, _P, i, _P]),
        "pa_bm_build_batch": (i, [_P, _P, i, _P, i, _P]),
        "pa_bm_evict_lru_sequence": (i, [_P, i64, i, _P]),
        "pa_bm_allocate_with_prefix": (i, [_P, i64, _P, i, _P, _P, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIBS[path] = lib
    return lib


def header_functions(header: str | None = None) -> list[str]:
    """Names of the functions the headers under include/ declare (or one header)."""
    if header is None:
        return sorted(set(n for h in HEADERS for n in header_functions(h)))
    text = open(header, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w ]*?\**\s*\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)))


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def paged_attention_decode_noalloc(out, query, key_cache, value_cache, block_tables, seq_lens, max_seq_len: int,
                                   scale: float, *, num_kv_heads: int, q_dtype: str, kv_dtype: str,
                                   partition_tokens: int = 0, k_scale=1.0, v_scale=1.0, check_bits=None,
                                   stream=None, lib_path: str | None = None) -> None:
    """Decode without a context and without any device allocation by the
    library: for callers that cannot allocate (e.g. while capturing a CUDA
    graph, or under a host-owned memory pool).  Split-KV partials go to the
    library's fixed 16 MiB per-GPU array; calls that overlap on one GPU race on
    it.  Arguments as in ``PagedAttention.paged_attention_decode``; the cache
    shape is taken from the tensors."""
    lib = load_library(lib_path)
    num_blocks, block_size, hkv, head_dim = key_cache.shape
    if hkv != num_kv_heads:
        raise PagedAttnError(PA_ERR_INVALID_ARG, "key_cache head count differs from num_kv_heads")
    st = lib.paged_attention_decode_noalloc(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables), block_tables.stride(0),
        _ptr(seq_lens), query.shape[0], int(max_seq_len), query.shape[1], num_kv_heads, head_dim, block_size,
        num_blocks, DTYPE_CODES[q_dtype], DTYPE_CODES[kv_dtype], int(partition_tokens), float(scale),
        float(k_scale), float(v_scale), _ptr(check_bits), _stream_ptr(stream))
    if st != PA_OK:
        raise PagedAttnError(st, f"paged_attention_decode_noalloc: {lib.paged_attn_status_string(st).decode()}")


class PagedAttention:
    """One attention layer's paged-cache shape bound to a library context."""

    def __init__(self, num_heads: int, num_kv_heads: int, head_dim: int, num_blocks: int, *, block_size: int = 16,
                 q_dtype: str = "f16", kv_dtype: str = "f16", max_num_seqs: int, max_blocks_per_seq: int,
                 partition_tokens: int = PA_PARTITION_AUTO, device: int | None = None, lib_path: str | None = None,
                 shared_prefix: bool = False):
        self.lib = load_library(lib_path)
        if device is None:
            device = torch.cuda.current_device() if torch.cuda.is_available() else 0
        self.cfg = PaConfig(num_heads, num_kv_heads, head_dim, block_size, num_blocks, DTYPE_CODES[q_dtype],
                            DTYPE_CODES[kv_dtype], max_num_seqs, max_blocks_per_seq, partition_tokens, device,
                            PA_FLAG_SHARED_PREFIX if shared_prefix else 0)
        self.q_dtype, self.kv_dtype = q_dtype, kv_dtype
        self.device = device
        ctx = _P()
        st = self.lib.paged_attn_create(ctypes.byref(self.cfg), ctypes.byref(ctx))
        if st != PA_OK:
            raise PagedAttnError(st, f"paged_attn_create: {self.lib.paged_attn_status_string(st).decode()}")
        self.ctx = ctx

    # -- helpers
    def _check(self, st: int, what: str) -> None:
        if st != PA_OK:
            msg = self.lib.paged_attn_last_error(self.ctx).decode()
            raise PagedAttnError(st, f"{what}: {self.lib.paged_attn_status_string(st).decode()} {msg}".strip())

    def close(self) -> None:
        if getattr(self, "ctx", None):
            self.lib.paged_attn_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- the C ABI, one method per entry point
    def reshape_and_cache(self, key, value, key_cache, value_cache, slot_mapping, k_scale=1.0, v_scale=1.0,
                          stream=None) -> None:
        st = self.lib.reshape_and_cache(self.ctx, _ptr(key), _ptr(value), key.stride(0), value.stride(0),
                                        _ptr(key_cache), _ptr(value_cache), _ptr(slot_mapping), key.shape[0],
                                        float(k_scale), float(v_scale), _stream_ptr(stream))
        self._check(st, "reshape_and_cache")

    def paged_attention_decode(self, out, query, key_cache, value_cache, block_tables, seq_lens, max_seq_len: int,
                               scale: float, k_scale=1.0, v_scale=1.0, stream=None) -> None:
        st = self.lib.paged_attention_decode(self.ctx, _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
                                             _ptr(block_tables), block_tables.stride(0), _ptr(seq_lens),
                                             query.shape[0], int(max_seq_len), float(scale), float(k_scale),
                                             float(v_scale), _stream_ptr(stream))
        self._check(st, "paged_attention_decode")

    def paged_attention_decode_shared_prefix(self, out, query, key_cache, value_cache, block_tables, seq_lens,
                                             max_seq_len: int, group_start, group_prefix_len, max_group_size: int,
                                             max_prefix_len: int, scale: float, k_scale=1.0, v_scale=1.0,
                                             stream=None) -> None:
        """Decode with groups of sequences sharing prefix blocks: group g is
        sequences [group_start[g], group_start[g+1]) sharing group_prefix_len[g]
        tokens (device int32 tensors).  Needs ``shared_prefix=True`` at construction."""
        st = self.lib.paged_attention_decode_shared_prefix(
            self.ctx, _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
            block_tables.stride(0), _ptr(seq_lens), query.shape[0], int(max_seq_len), _ptr(group_start),
            _ptr(group_prefix_len), group_prefix_len.shape[0], int(max_group_size), int(max_prefix_len),
            float(scale), float(k_scale), float(v_scale), _stream_ptr(stream))
        self._check(st, "paged_attention_decode_shared_prefix")

    def paged_attention_prefill(self, out, query, key_cache, value_cache, block_tables, seq_lens, query_start,
                                max_query_len: int, max_seq_len: int, scale: float, k_scale=1.0, v_scale=1.0,
                                stream=None) -> None:
        """Causal multi-query attention: the rows query[query_start[s]:query_start[s+1]]
        are sequence s's last positions (device int32 tensors for the index arrays)."""
        st = self.lib.paged_attention_prefill(self.ctx, _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
                                              _ptr(block_tables), block_tables.stride(0), _ptr(seq_lens),
                                              _ptr(query_start), query_start.shape[0] - 1, query.shape[0],
                                              int(max_query_len), int(max_seq_len), float(scale), float(k_scale),
                                              float(v_scale), _stream_ptr(stream))
        self._check(st, "paged_attention_prefill")

    def paged_gather_kv(self, k_out, v_out, key_cache, value_cache, block_table_row, seq_len: int,
                        stream=None) -> None:
        st = self.lib.paged_gather_kv(self.ctx, _ptr(k_out), _ptr(v_out), _ptr(key_cache), _ptr(value_cache),
                                      _ptr(block_table_row), int(seq_len), _stream_ptr(stream))
        self._check(st, "paged_gather_kv")

    def paged_copy_blocks(self, dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, block_pairs,
                          stream=None) -> None:
        """dst[pairs[i, 1]] = src[pairs[i, 0]] for whole blocks (copy-on-write, swap).
        The caches may be device tensors or pinned host tensors."""
        st = self.lib.paged_copy_blocks(self.ctx, _ptr(dst_key_cache), _ptr(dst_value_cache),
                                        dst_key_cache.shape[0], _ptr(src_key_cache), _ptr(src_value_cache),
                                        src_key_cache.shape[0], _ptr(block_pairs), block_pairs.shape[0],
                                        _stream_ptr(stream))
        self._check(st, "paged_copy_blocks")

    def get_error(self, stream=None) -> int:
        """Synchronise and return (then clear) the device check bits."""
        st = self.lib.paged_attn_get_error(self.ctx, _stream_ptr(stream))
        if st == PA_ERR_DEVICE_CHECK:
            return self.lib.paged_attn_last_check_bits(self.ctx)
        self._check(st, "paged_attn_get_error")
        return 0

    def test_wait_timeout(self, wait_limit_cycles: int) -> None:
        """Failure-path test hook: the next decode call's waits are bounded by
        ``wait_limit_cycles`` and its consumers wait on a barrier nothing
        completes, so the call must take the timeout exit (one-shot)."""
        self._check(self.lib.paged_attn_test_wait_timeout(self.ctx, int(wait_limit_cycles)),
                    "paged_attn_test_wait_timeout")

    def set_partition_tokens(self, n: int) -> None:
        self._check(self.lib.paged_attn_set_partition_tokens(self.ctx, int(n)), "paged_attn_set_partition_tokens")

    def get_partition_tokens(self) -> int:
        """The partition setting: tokens, PA_PARTITION_NONE or PA_PARTITION_AUTO."""
        v = ctypes.c_int(0)
        self._check(self.lib.paged_attn_get_partition_tokens(self.ctx, ctypes.byref(v)),
                    "paged_attn_get_partition_tokens")
        return v.value

    # -- conveniences (allocation of outputs only)
    def decode(self, query, key_cache, value_cache, block_tables, seq_lens, max_seq_len, scale, k_scale=1.0,
               v_scale=1.0, stream=None) -> torch.Tensor:
        out = torch.empty_like(query)
        self.paged_attention_decode(out, query, key_cache, value_cache, block_tables, seq_lens, max_seq_len, scale,
                                    k_scale, v_scale, stream)
        return out

    def new_cache(self) -> torch.Tensor:
        c = self.cfg
        return torch.empty((c.num_blocks, c.block_size, c.num_kv_heads, c.head_dim), dtype=TORCH_OF[self.kv_dtype],
                           device=f"cuda:{self.device}")


class BlockManager:
    """Host block manager of the library (include/block_manager.h): argument
    marshalling only; failures raise PagedAttnError with the status code."""

    def __init__(self, num_blocks: int, block_size: int = 16, lib_path: str | None = None):
        self.lib = load_library(lib_path)
        h = _P()
        self._check(self.lib.pa_bm_create(int(num_blocks), int(block_size), ctypes.byref(h)), "pa_bm_create")
        self.h = h
        self.block_size = block_size

    def _check(self, st: int, what: str) -> None:
        if st != PA_OK:
            raise PagedAttnError(st, f"{what}: {self.lib.paged_attn_status_string(st).decode()}")

    def close(self) -> None:
        if getattr(self, "h", None):
            self.lib.pa_bm_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _int_out(self, fn, *args) -> int:
        v = ctypes.c_int(0)
        self._check(fn(self.h, *args, ctypes.byref(v)), fn.__name__)
        return v.value

    def num_free(self) -> int:
        return self._int_out(self.lib.pa_bm_num_free)

    def ref_count(self, block: int) -> int:
        return self._int_out(self.lib.pa_bm_ref_count, int(block))

    def cached_blocks(self) -> int:
        return self._int_out(self.lib.pa_bm_cached_blocks)

    def add_sequence(self, sid: int) -> None:
        self._check(self.lib.pa_bm_add_sequence(self.h, int(sid)), "pa_bm_add_sequence")

    def free_sequence(self, sid: int) -> None:
        self._check(self.lib.pa_bm_free_sequence(self.h, int(sid)), "pa_bm_free_sequence")

    def ensure_capacity(self, sid: int, required_tokens: int) -> None:
        self._check(self.lib.pa_bm_ensure_capacity(self.h, int(sid), int(required_tokens)), "pa_bm_ensure_capacity")

    def append_tokens(self, sid: int, n: int):
        """Returns (status, slots, copy pairs) for the positions appended
        (all n on PA_OK, fewer on PA_ERR_OUT_OF_BLOCKS); other failures raise."""
        slots = (ctypes.c_int64 * max(1, n))()
        pairs = (ctypes.c_int64 * max(2, 2 * n))()
        nc, na = ctypes.c_int(0), ctypes.c_int(0)
        st = self.lib.pa_bm_append_tokens(self.h, int(sid), int(n), slots, pairs, ctypes.byref(nc), ctypes.byref(na))
        if st not in (PA_OK, PA_ERR_OUT_OF_BLOCKS):
            self._check(st, "pa_bm_append_tokens")
        return st, list(slots[:na.value]), [(pairs[2 * k], pairs[2 * k + 1]) for k in range(nc.value)]

    def append_batch(self, sids):
        """One position for each sequence in ``sids``: returns (status, slots
        as an int64 tensor, copy pairs as an int64 [k, 2] tensor); only the
        sequences served before a PA_ERR_OUT_OF_BLOCKS are in the slots."""
        n = len(sids)
        ids = torch.as_tensor(sids, dtype=torch.int64)
        slots = torch.empty((max(1, n),), dtype=torch.int64)
        pairs = torch.empty((max(1, n), 2), dtype=torch.int64)
        nc, na = ctypes.c_int(0), ctypes.c_int(0)
        st = self.lib.pa_bm_append_batch(self.h, ids.data_ptr() if n else None, n, slots.data_ptr(),
                                         pairs.data_ptr(), ctypes.byref(nc), ctypes.byref(na))
        if st not in (PA_OK, PA_ERR_OUT_OF_BLOCKS):
            self._check(st, "pa_bm_append_batch")
        return st, slots[:na.value], pairs[:nc.value]

    def fork(self, parent: int, child: int) -> None:
        self._check(self.lib.pa_bm_fork(self.h, int(parent), int(child)), "pa_bm_fork")

    def seq_len(self, sid: int) -> int:
        v = ctypes.c_int64(0)
        self._check(self.lib.pa_bm_seq_len(self.h, int(sid), ctypes.byref(v)), "pa_bm_seq_len")
        return v.value

    def block_table(self, sid: int) -> list[int]:
        n = ctypes.c_int(0)
        self._check(self.lib.pa_bm_block_table(self.h, int(sid), None, 0, ctypes.byref(n)), "pa_bm_block_table")
        buf = (ctypes.c_int32 * max(1, n.value))()
        self._check(self.lib.pa_bm_block_table(self.h, int(sid), buf, n.value, ctypes.byref(n)), "pa_bm_block_table")
        return list(buf[:n.value])

    def build_batch(self, sids, bt_stride: int):
        """int32 tables [n, bt_stride] (-1 padded) and lengths [n], as torch CPU tensors."""
        n = len(sids)
        ids = (ctypes.c_int64 * max(1, n))(*[int(x) for x in sids])
        tables = torch.empty((n, bt_stride), dtype=torch.int32)
        lens = torch.empty((n,), dtype=torch.int32)
        self._check(self.lib.pa_bm_build_batch(self.h, ids, n, tables.data_ptr() if n else None, int(bt_stride),
                                               lens.data_ptr() if n else None), "pa_bm_build_batch")
        return tables, lens

    def evict_lru_sequence(self, exclude: int | None = None) -> int:
        v = ctypes.c_int64(0)
        self._check(self.lib.pa_bm_evict_lru_sequence(self.h, int(exclude or 0), 0 if exclude is None else 1,
                                                      ctypes.byref(v)), "pa_bm_evict_lru_sequence")
        return v.value

    def allocate_with_prefix(self, sid: int, tokens):
        """Returns (matched tokens, slots of the positions from the match on)."""
        n = len(tokens)
        toks = (ctypes.c_int32 * max(1, n))(*[int(t) for t in tokens])
        slots = (ctypes.c_int64 * max(1, n))()
        m, ns = ctypes.c_int(0), ctypes.c_int(0)
        self._check(self.lib.pa_bm_allocate_with_prefix(self.h, int(sid), toks, n, ctypes.byref(m), slots,
                                                        ctypes.byref(ns)), "pa_bm_allocate_with_prefix")
        return m.value, list(slots[:ns.value])
