"""The allocation-free decode entry point, for callers that cannot allocate
device memory: hosts that hand out every byte of device memory from their own
pool and forbid outside allocations, or serving loops that must not risk an
allocation failure (or the allocator's implicit synchronisation) in the middle
of a step.

It runs the same decode kernel with the same explicit partition as the
context-based entry point, so its output must be bit-identical to that
entry point's, call after call, although every call reuses the same fixed
scratch array; it must also match the fp64 oracle, refuse a split that does
not fit, and order its one-time set-up correctly when its very first call is
made on a non-blocking stream.

Kept in a file that pytest collects last, so that a run stopping at the first
failure has already run every other test."""

import os
import subprocess
import sys
import textwrap

import pytest
import torch

from oracle import attention, cache_write
from paged_kv_cache_463_b200 import binding as b
from paged_kv_cache_463_b200 import workloads as wl
from tests.helpers import TOL, assert_out_close, raw

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_463_b200 import build
    build.build()
    torch.cuda.init()


def _caches(w):
    """Device caches and the oracle's host copies (fp8: the oracle's own encoding)."""
    sp = w.spec
    if sp.kv_dtype == "fp8_e4m3":
        kh = cache_write.quantize(raw(w.key_src), sp.q_dtype, w.k_scale)
        vh = cache_write.quantize(raw(w.value_src), sp.q_dtype, w.v_scale)
        return (torch.from_numpy(kh).to(DEV).view(torch.float8_e4m3fn),
                torch.from_numpy(vh).to(DEV).view(torch.float8_e4m3fn), kh, vh)
    return w.key_cache, w.value_cache, raw(w.key_cache), raw(w.value_cache)


def _reference_and_noalloc(spec, lens, partition, use_check_bits=True):
    """The context entry point's output and the allocation-free one's, on the
    same inputs and the same explicit partition."""
    w = wl.make_workload(spec, DEV, seq_lens=lens)
    kc, vc, kh, vh = _caches(w)
    pa = b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks, q_dtype=spec.q_dtype,
                          kv_dtype=spec.kv_dtype, max_num_seqs=len(lens), max_blocks_per_seq=w.block_tables.shape[1],
                          partition_tokens=partition)
    ref = pa.decode(w.query, kc, vc, w.block_tables, w.seq_lens, w.max_seq_len, w.scale, w.k_scale, w.v_scale)
    assert pa.get_error() == 0
    out = torch.full_like(w.query, float("nan"))
    bits = torch.zeros(1, dtype=torch.int32, device=DEV) if use_check_bits else None
    b.paged_attention_decode_noalloc(out, w.query, kc, vc, w.block_tables, w.seq_lens, w.max_seq_len, w.scale,
                                     num_kv_heads=spec.num_kv_heads, q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype,
                                     partition_tokens=partition, k_scale=w.k_scale, v_scale=w.v_scale,
                                     check_bits=bits)
    torch.cuda.synchronize()
    if bits is not None:
        assert int(bits.item()) == 0
    pa.close()
    return w, kh, vh, ref, out


def _oracle(w, kh, vh):
    sp = w.spec
    return attention.decode_attention(raw(w.query), kh, vh, raw(w.block_tables), raw(w.seq_lens), w.scale,
                                      q_dtype=sp.q_dtype, kv_dtype=sp.kv_dtype, k_scale=w.k_scale,
                                      v_scale=w.v_scale)


def test_noalloc_matches_context_entry_point_two_calls_in_a_row():
    # call 1: long sequences split into 16 partitions of 512 tokens (grouped-query, bf16)
    spec1 = wl.scaled(wl.SPEC_BY_NAME["long-context-split-kv"], num_seqs=4)
    w1, kh1, vh1, ref1, out1 = _reference_and_noalloc(spec1, [8192, 8000, 4097, 1], 512)
    # call 2 right after: other shapes and lengths (MHA, fp16), 1024-token partitions,
    # on the scratch call 1 left behind
    spec2 = wl.scaled(wl.SPEC_BY_NAME["llama2-7b-mha"], num_seqs=6, pool_blocks=None)
    w2, kh2, vh2, ref2, out2 = _reference_and_noalloc(spec2, [2048, 1500, 3000, 17, 1024, 4096], 1024)
    # same kernel, same partition: bit for bit the context entry point's output
    assert torch.equal(out1, ref1)
    assert torch.equal(out2, ref2)
    # and the oracle's, within the decode tolerance
    assert_out_close(out1, _oracle(w1, kh1, vh1), TOL[spec1.q_dtype], spec1.q_dtype, "call 1")
    assert_out_close(out2, _oracle(w2, kh2, vh2), TOL[spec2.q_dtype], spec2.q_dtype, "call 2")


def test_noalloc_fp8_split_and_no_check_word():
    # fp8 cache with a split (partials through the array), check bits to the array's own word
    base = wl.SPEC_BY_NAME["shared-prefix-fp8"]
    spec = wl.scaled(base, num_seqs=5, prefix_groups=0, pool_blocks=None)
    w, kh, vh, ref, out = _reference_and_noalloc(spec, [1500, 700, 33, 1024, 2048], 512, use_check_bits=False)
    assert torch.equal(out, ref)
    assert_out_close(out, _oracle(w, kh, vh), TOL["fp8_e4m3"], spec.q_dtype, "fp8 split")
    # and one without a split (no partials), again without a check word
    w, kh, vh, ref, out = _reference_and_noalloc(spec, [1500, 700, 33, 1024, 2048], 0, use_check_bits=False)
    assert torch.equal(out, ref)


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


FIRST_CALL_ON_NONBLOCKING_STREAM = textwrap.dedent("""
    import sys, torch
    sys.path.insert(0, {root!r})
    from paged_kv_cache_463_b200 import binding as b
    from paged_kv_cache_463_b200 import workloads as wl
    spec = wl.scaled(wl.SPEC_BY_NAME["long-context-split-kv"], num_seqs=3)
    w = wl.make_workload(spec, "cuda:0", seq_lens=[6000, 3000, 513])
    torch.cuda.synchronize()
    s = torch.cuda.Stream(device="cuda:0")          # cudaStreamNonBlocking
    outs = []
    for _ in range(2):                              # the first call does the one-time set-up
        out = torch.full_like(w.query, float("nan"))
        bits = torch.zeros(1, dtype=torch.int32, device="cuda:0")
        s.wait_stream(torch.cuda.current_stream())
        b.paged_attention_decode_noalloc(out, w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens,
                                         w.max_seq_len, w.scale, num_kv_heads=spec.num_kv_heads,
                                         q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype, partition_tokens=512,
                                         check_bits=bits, stream=s)
        s.synchronize()
        assert int(bits.item()) == 0, int(bits.item())
        outs.append(out)
    pa = b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks, q_dtype=spec.q_dtype,
                          kv_dtype=spec.kv_dtype, max_num_seqs=3, max_blocks_per_seq=w.block_tables.shape[1],
                          partition_tokens=512)
    ref = pa.decode(w.query, w.key_cache, w.value_cache, w.block_tables, w.seq_lens, w.max_seq_len, w.scale)
    assert pa.get_error() == 0
    assert torch.equal(outs[0], ref) and torch.equal(outs[1], ref)
    print("ok")
""")


def test_noalloc_first_call_on_a_nonblocking_stream():
    """A fresh process whose very first allocation-free call runs on a
    non-blocking stream: the one-time clearing of the array's counters is
    ordered before that call's kernels, so both calls are exact."""
    r = subprocess.run([sys.executable, "-c", FIRST_CALL_ON_NONBLOCKING_STREAM.format(root=ROOT)],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]
