"""Failure detection on the GPU without any GPU fault.

Every pipeline wait in the decode kernel is bounded; a wait that runs out
sets PA_CHECK_WAIT_TIMEOUT, and the CTA waits (bounded) for the copies it
still has in flight before it exits, so the context stays usable.  The
library's test hook makes one decode call's consumer warps wait on a barrier
that nothing completes, with a short limit (about a millisecond), so that
every CTA of that call takes the timeout exit.  The call must report the bit,
and the very next normal call on the same context must match the oracle.
Nothing here traps, asserts, reads a bad address or spins without bound."""

import numpy as np
import pytest
import torch

from oracle import attention, cache_write
from paged_kv_cache_463_b200 import binding as b
from paged_kv_cache_463_b200 import workloads as wl
from tests.helpers import TOL, assert_out_close, raw

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LIMIT = 2_000_000  # cycles: about 1 ms at the B200's clocks


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_463_b200 import build
    build.build()
    torch.cuda.init()


def _caches(w):
    sp = w.spec
    if sp.kv_dtype == "fp8_e4m3":
        kh = cache_write.quantize(raw(w.key_src), sp.q_dtype, w.k_scale)
        vh = cache_write.quantize(raw(w.value_src), sp.q_dtype, w.v_scale)
        return (torch.from_numpy(kh).to(DEV).view(torch.float8_e4m3fn),
                torch.from_numpy(vh).to(DEV).view(torch.float8_e4m3fn), kh, vh)
    return w.key_cache, w.value_cache, raw(w.key_cache), raw(w.value_cache)


def _oracle(w, kh, vh):
    sp = w.spec
    return attention.decode_attention(raw(w.query), kh, vh, raw(w.block_tables), raw(w.seq_lens), w.scale,
                                      q_dtype=sp.q_dtype, kv_dtype=sp.kv_dtype, k_scale=w.k_scale,
                                      v_scale=w.v_scale)


def _tol(sp):
    return TOL[sp.kv_dtype] if sp.kv_dtype == "fp8_e4m3" else TOL[sp.q_dtype]


CASES = {
    # uniform lengths: ticket hand-out, one partition per sequence
    "mha-f16-tickets": (wl.scaled(wl.SPEC_BY_NAME["llama2-7b-mha"], num_seqs=4, pool_blocks=None), b.PA_PARTITION_AUTO),
    # varying lengths: stream-K ranges and the merge kernel
    "gqa-bf16-streamk": (wl.scaled(wl.SPEC_BY_NAME["gqa-70b-like"], num_seqs=6), b.PA_PARTITION_AUTO),
    # an explicit split: partials and the merge kernel
    "long-bf16-split": (wl.scaled(wl.SPEC_BY_NAME["long-context-split-kv"], num_seqs=1, seq_len_min=5000,
                                  seq_len_max=5000), 512),
    # fp8 cache: the two-tile consumer step
    "fp8": (wl.scaled(wl.SPEC_BY_NAME["shared-prefix-fp8"], num_seqs=6, prefix_groups=0, pool_blocks=None),
            b.PA_PARTITION_AUTO),
}


@pytest.mark.parametrize("name", list(CASES))
def test_wait_that_runs_out_is_reported_and_the_next_call_is_exact(name):
    spec, part = CASES[name]
    w = wl.make_workload(spec, DEV)
    kc, vc, kh, vh = _caches(w)
    pa = b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks,
                          q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype, max_num_seqs=spec.num_seqs,
                          max_blocks_per_seq=w.block_tables.shape[1], partition_tokens=part)
    ref = _oracle(w, kh, vh)
    # the failing call: every CTA gives up after ~LIMIT cycles
    pa.test_wait_timeout(LIMIT)
    pa.decode(w.query, kc, vc, w.block_tables, w.seq_lens, w.max_seq_len, w.scale, w.k_scale, w.v_scale)
    bits = pa.get_error()
    assert bits & b.PA_CHECK_WAIT_TIMEOUT, f"expected the timeout bit, got {bits}"
    # the hook is one-shot: the next calls run normally and are exact
    for _ in range(2):
        out = pa.decode(w.query, kc, vc, w.block_tables, w.seq_lens, w.max_seq_len, w.scale, w.k_scale,
                        w.v_scale)
        assert pa.get_error() == 0
        assert_out_close(out, ref, _tol(spec), spec.q_dtype, name)
    pa.close()


def test_shared_prefix_call_reports_a_wait_that_runs_out_and_recovers():
    base = wl.SPEC_BY_NAME["shared-prefix-fp8"]
    spec = wl.scaled(base, num_seqs=8, prefix_groups=2, prefix_tokens=256, pool_blocks=None)
    w = wl.make_workload(spec, DEV)
    kc, vc, kh, vh = _caches(w)
    pa = b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks,
                          q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype, max_num_seqs=spec.num_seqs,
                          max_blocks_per_seq=w.block_tables.shape[1], shared_prefix=True)
    sizes = (w.group_start[1:] - w.group_start[:-1]).cpu()
    mg, mp = int(sizes.max().item()), int(w.group_prefix_len.max().item())
    ref = _oracle(w, kh, vh)
    out = torch.empty_like(w.query)

    def call():
        pa.paged_attention_decode_shared_prefix(out, w.query, kc, vc, w.block_tables, w.seq_lens, w.max_seq_len,
                                                w.group_start, w.group_prefix_len, mg, mp, w.scale, w.k_scale,
                                                w.v_scale)

    pa.test_wait_timeout(LIMIT)
    call()
    assert pa.get_error() & b.PA_CHECK_WAIT_TIMEOUT
    call()
    assert pa.get_error() == 0
    assert_out_close(out, ref, _tol(spec), spec.q_dtype, "shared-prefix after a timeout")
    pa.close()


def test_hook_arguments_are_checked():
    spec = wl.SPEC_BY_NAME["tiny"]
    pa = b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, 64, max_num_seqs=4,
                          max_blocks_per_seq=8)
    for bad in (0, 999, 10 ** 12):
        with pytest.raises(b.PagedAttnError) as e:
            pa.test_wait_timeout(bad)
        assert e.value.status == b.PA_ERR_INVALID_ARG
    pa.close()
