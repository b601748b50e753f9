"""The allocation-free decode entry point, for callers that cannot allocate
device memory (a stream being captured into a CUDA graph, a host that owns
every allocation through its own pool).  It must give the same result as the
context-based entry point, call after call, although every call reuses the
same fixed scratch array; and it must refuse a split that does not fit.

Kept in a file that pytest collects last, so that a run stopping at the first
failure has already run every other test."""

import pytest
import torch

from paged_kv_cache_463_b200 import binding as b
from paged_kv_cache_463_b200 import workloads as wl
from tests.helpers import TOL

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_463_b200 import build
    build.build()
    torch.cuda.init()


def _reference_and_noalloc(spec, lens, partition):
    w = wl.make_workload(spec, DEV, seq_lens=lens)
    pa = b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks, q_dtype=spec.q_dtype,
                          kv_dtype=spec.kv_dtype, max_num_seqs=len(lens), max_blocks_per_seq=w.block_tables.shape[1],
                          partition_tokens=partition)
    ref = pa.decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.max_seq_len, w.scale)
    assert pa.get_error() == 0
    out = torch.full_like(w.query, float("nan"))
    bits = torch.zeros(1, dtype=torch.int32, device=DEV)
    b.paged_attention_decode_noalloc(out, w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens,
                                     w.max_seq_len, w.scale, num_kv_heads=spec.num_kv_heads, q_dtype=spec.q_dtype,
                                     kv_dtype=spec.kv_dtype, partition_tokens=partition, check_bits=bits)
    torch.cuda.synchronize()
    assert int(bits.item()) == 0
    pa.close()
    return ref, out


def test_noalloc_matches_context_entry_point_two_calls_in_a_row():
    # call 1: long sequences split into 16 partitions of 512 tokens (grouped-query, bf16)
    spec1 = wl.scaled(wl.SPEC_BY_NAME["long-context-split-kv"], num_seqs=4)
    ref1, out1 = _reference_and_noalloc(spec1, [8192, 8000, 4097, 1], 512)
    # call 2 right after: other shapes and lengths (MHA, fp16), 1024-token partitions,
    # reading scratch that call 1 left behind
    spec2 = wl.scaled(wl.SPEC_BY_NAME["llama2-7b-mha"], num_seqs=6, pool_blocks=None)
    ref2, out2 = _reference_and_noalloc(spec2, [2048, 1500, 3000, 17, 1024, 4096], 1024)
    for ref, out, dt in ((ref1, out1, spec1.q_dtype), (ref2, out2, spec2.q_dtype)):
        assert torch.isfinite(out.float()).all()
        assert (out.float() - ref.float()).abs().max().item() <= TOL[dt]


def test_noalloc_refuses_a_split_larger_than_its_scratch():
    spec = wl.scaled(wl.SPEC_BY_NAME["gqa-70b-like"], num_seqs=128, seq_len_min=4096, seq_len_max=4096)
    w = wl.make_workload(spec, DEV)
    need = 128 * spec.num_heads * (4096 // 256) * (spec.head_dim + 2) * 4
    assert need > b.PA_NOALLOC_SCRATCH_BYTES
    out = torch.zeros_like(w.query)
    with pytest.raises(b.PagedAttnError) as e:
        b.paged_attention_decode_noalloc(out, w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens,
                                         w.max_seq_len, w.scale, num_kv_heads=spec.num_kv_heads,
                                         q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype, partition_tokens=256)
    assert e.value.status == b.PA_ERR_SCRATCH_TOO_SMALL
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0  # nothing was launched
