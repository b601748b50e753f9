"""The decode step (cache write + paged decode, with the merge kernel as a
programmatic dependent launch) captured once into a CUDA graph and replayed
with new inputs written in place: every replay equals the eager calls
bit for bit, and the oracle."""

import numpy as np
import pytest
import torch

from oracle import attention
from paged_kv_cache_463_b200 import binding as b
from paged_kv_cache_463_b200 import workloads as wl
from tests.helpers import TOL, assert_out_close, raw

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_463_b200 import build
    build.build()
    torch.cuda.init()


@pytest.mark.parametrize("name", ["gqa-70b-like", "long-context-split-kv"])
def test_graph_replay_matches_eager(name):
    spec = wl.scaled(wl.SPEC_BY_NAME[name], num_seqs=6, pool_blocks=None)
    w = wl.make_workload(spec, DEV)
    pa = b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks, q_dtype=spec.q_dtype,
                          kv_dtype=spec.kv_dtype, max_num_seqs=spec.num_seqs,
                          max_blocks_per_seq=w.block_tables.shape[1])
    kc, vc = w.key_cache, w.value_cache
    ml = w.max_seq_len
    q = w.query.clone()
    out = torch.empty_like(q)
    s = torch.cuda.Stream()

    def step(stream):
        pa.reshape_and_cache(w.new_key, w.new_value, kc, vc, w.slot_mapping, stream=stream)
        pa.paged_attention_decode(out, q, kc, vc, w.block_tables, w.seq_lens, ml, w.scale, stream=stream)

    with torch.cuda.stream(s):
        step(s)  # first call outside the capture (tensor maps encoded, workspace touched)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    torch.cuda.synchronize()
    gen = torch.Generator(device=DEV).manual_seed(3)
    for _ in range(3):
        q.copy_(torch.randn(q.shape, generator=gen, device=DEV).to(q.dtype))
        g.replay()
        torch.cuda.synchronize()
        got = out.clone()
        with torch.cuda.stream(s):
            step(s)
        torch.cuda.synchronize()
        assert pa.get_error() == 0
        assert torch.equal(got, out)
        ref = attention.decode_attention(raw(q), raw(kc), raw(vc), raw(w.block_tables), raw(w.seq_lens), w.scale,
                                         q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype)
        assert_out_close(got, ref, TOL[spec.q_dtype], spec.q_dtype, f"{name} graph replay")


def test_fp8_decode_is_deterministic():
    """fp8 decode (two tiles per step by block position) over 64 sequences of
    the shared-prefix workload: repeated eager calls and a graph replay give
    the same bits, and the oracle's result on the dequantised cache."""
    from oracle import cache_write
    spec = wl.scaled(wl.SPEC_BY_NAME["shared-prefix-fp8"], num_seqs=64, prefix_groups=2, pool_blocks=None)
    w = wl.make_workload(spec, DEV)
    kh = cache_write.quantize(raw(w.key_src), spec.q_dtype, w.k_scale)
    vh = cache_write.quantize(raw(w.value_src), spec.q_dtype, w.v_scale)
    kc = torch.from_numpy(kh).to(DEV).view(torch.float8_e4m3fn)
    vc = torch.from_numpy(vh).to(DEV).view(torch.float8_e4m3fn)
    pa = b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks, q_dtype=spec.q_dtype,
                          kv_dtype=spec.kv_dtype, max_num_seqs=spec.num_seqs,
                          max_blocks_per_seq=w.block_tables.shape[1])
    out = torch.empty_like(w.query)
    s = torch.cuda.Stream()
    ml = w.max_seq_len  # (a host read: not inside the capture)

    def call():
        pa.paged_attention_decode(out, w.query, kc, vc, w.block_tables, w.seq_lens, ml, w.scale,
                                  w.k_scale, w.v_scale, stream=s)

    with torch.cuda.stream(s):
        call()
    torch.cuda.synchronize()
    first = out.clone()
    for _ in range(4):
        with torch.cuda.stream(s):
            call()
        torch.cuda.synchronize()
        assert torch.equal(out, first)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert pa.get_error() == 0
    assert torch.equal(out, first)
    ref = attention.decode_attention(raw(w.query), kh, vh, raw(w.block_tables), raw(w.seq_lens), w.scale,
                                     q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype, k_scale=w.k_scale,
                                     v_scale=w.v_scale)
    assert_out_close(first, ref, TOL["fp8_e4m3"], spec.q_dtype, "fp8 decode")
