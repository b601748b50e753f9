"""A serving loop driven entirely through the library's public calls, against
the oracle step by step: the native block manager places every token (prefix
cache for prompts that share their first blocks, a fork for parallel
sampling, copy-on-write on the first write into a shared block), the device
calls do the rest (paged_copy_blocks for the copy pairs, reshape_and_cache for
the slots, paged_attention_decode and its shared-prefix form for the batch
tables).  The oracle runs the same steps with its own block manager, block
copy, cache write and attention.  Caches must stay bit-identical; outputs
within the decode tolerance."""

import numpy as np
import pytest
import torch

from oracle import attention, block_copy, cache_write
from oracle.block_manager import BlockManager as OracleBM
from paged_kv_cache_463_b200 import binding as b
from tests.helpers import TOL, assert_out_close, raw

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_463_b200 import build
    build.build()
    torch.cuda.init()


@pytest.mark.parametrize("kv_dtype", ["f16", "fp8_e4m3"])
def test_serving_loop(kv_dtype):
    torch.manual_seed(11)
    NB, BS, H, HKV, D = 96, 16, 8, 2, 128
    q_dtype = "f16"
    fp8 = kv_dtype == "fp8_e4m3"
    k_scale = v_scale = 0.02 if fp8 else 1.0
    pa = b.PagedAttention(H, HKV, D, NB, q_dtype=q_dtype, kv_dtype=kv_dtype, max_num_seqs=8, max_blocks_per_seq=16,
                          shared_prefix=True)
    bm = b.BlockManager(NB, BS)
    obm = OracleBM(NB, BS)
    kc = pa.new_cache().zero_()
    vc = pa.new_cache().zero_()
    okc, ovc = raw(kc), raw(vc)
    scale = 1.0 / np.sqrt(D)

    def write(slots, n):
        """n new tokens' K/V (random) to the given slots, on both sides."""
        k = torch.randn((n, HKV, D), device=DEV).half()
        v = torch.randn((n, HKV, D), device=DEV).half()
        sl = torch.tensor(slots, dtype=torch.int64, device=DEV)
        pa.reshape_and_cache(k, v, kc, vc, sl, k_scale, v_scale)
        cache_write.reshape_and_cache(raw(k), raw(v), okc, ovc, np.array(slots), src_dtype=q_dtype, cache_dtype=kv_dtype,
                                      k_scale=k_scale, v_scale=v_scale)

    def cow(pairs):
        if not pairs:
            return
        t = torch.tensor(pairs, dtype=torch.int64, device=DEV)
        pa.paged_copy_blocks(kc, vc, kc, vc, t)
        block_copy.copy_blocks(okc, ovc, okc, ovc, pairs)

    # prompts: two share their first 48 tokens (3 whole blocks), one does not
    base = list(range(1000, 1048))
    prompts = {0: base + [1, 2, 3, 4, 5], 1: base + [7] * 20, 2: list(range(2000, 2030))}
    for sid, toks in prompts.items():
        m, slots = bm.allocate_with_prefix(sid, toks)
        om, oslots = obm.allocate_with_prefix(sid, toks)
        assert (m, slots) == (om, oslots)
        write(slots, len(slots))                 # prefill writes only the unmatched positions
    assert bm.block_table(1)[:3] == bm.block_table(0)[:3]
    # parallel sampling: sequence 3 forks from sequence 0 (shares its partly filled last block)
    bm.fork(0, 3)
    obm.fork(0, 3)
    live = [0, 1, 2, 3]
    for step in range(6):
        for sid in live:
            st, slots, pairs = bm.append_tokens(sid, 1)
            oslots, opairs = obm.append_tokens(sid, 1)
            assert st == b.PA_OK and slots == oslots and pairs == [tuple(x) for x in opairs]
            cow(pairs)
            write(slots, 1)
        tables, lens = bm.build_batch(live, 16)
        otables, olens = obm.build_batch(live, 16)
        assert tables.tolist() == otables and lens.tolist() == olens
        np.testing.assert_array_equal(raw(kc), okc)
        np.testing.assert_array_equal(raw(vc), ovc)
        q = torch.randn((len(live), H, D), device=DEV).half()
        bt, sl = tables.to(DEV), lens.to(DEV)
        out = pa.decode(q, kc, vc, bt, sl, int(lens.max()), scale, k_scale, v_scale)
        assert pa.get_error() == 0
        ref = attention.decode_attention(raw(q), okc, ovc, np.array(otables), np.array(olens), scale,
                                         q_dtype=q_dtype, kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale)
        tol = TOL[kv_dtype] if fp8 else TOL[q_dtype]
        assert_out_close(out, ref, tol, q_dtype, f"step {step}")
        # the same batch as shared-prefix groups: 0, its fork 3 and 1 share the
        # prompt's three whole blocks (prefix cache); the rest decode alone
        order = [0, 3, 1] + [s for s in live if s not in (0, 1, 3)]
        tables2, lens2 = bm.build_batch(order, 16)
        t0, t3, t1 = bm.block_table(0), bm.block_table(3), bm.block_table(1)
        common = 0
        while common < min(len(t0), len(t3), len(t1)) and t0[common] == t3[common] == t1[common]:
            common += 1
        full = min(common, int(lens2[:3].min()) // BS)
        assert full == 3
        gs = torch.tensor([0, 3] + list(range(4, len(order) + 1)), dtype=torch.int32, device=DEV)
        pl = torch.tensor([full * BS] + [0] * (len(order) - 3), dtype=torch.int32, device=DEV)
        q2 = q[[live.index(s) for s in order]]
        out2 = torch.empty_like(q2)
        pa.paged_attention_decode_shared_prefix(out2, q2, kc, vc, tables2.to(DEV), lens2.to(DEV), int(lens2.max()),
                                                gs, pl, 3, full * BS, scale, k_scale, v_scale)
        assert pa.get_error() == 0
        ref2 = ref[[live.index(s) for s in order]]
        assert_out_close(out2, ref2, tol, q_dtype, f"shared-prefix step {step}")
        if step == 2:  # a sequence finishes; its blocks (not the shared ones) go back to the pool
            bm.free_sequence(2)
            obm.free_sequence(2)
            live.remove(2)
            assert bm.num_free() == obm.num_free()
