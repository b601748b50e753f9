"""GPU parity of shared-prefix decode (paged_attention_decode_shared_prefix)
against the fp64 CPU oracle.

Sequences forked from one prompt share its physical blocks (page "5.KV Cache
管理 & PagedAttention", Q18); the library reads each shared block once per
group and combines that pass with a decode of each private suffix.  The result
is plain decode attention over every member's whole sequence, so the oracle is
``attention.decode_attention`` on the same tables; tolerances as for decode
(2e-3 fp16, 8e-3 bf16, 2e-3 fp8 against the oracle on the dequantised cache).
"""

import numpy as np
import pytest
import torch

from oracle import attention, cache_write, prefix_sharing
from paged_kv_cache_463_b200 import binding as b
from paged_kv_cache_463_b200 import workloads as wl
from tests.helpers import TOL, assert_out_close, compact_sequences, raw

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_463_b200 import build
    build.build()
    torch.cuda.init()


def _ctx(spec, num_blocks, max_blocks, num_seqs=None, partition=b.PA_PARTITION_AUTO, shared=True):
    return b.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, num_blocks,
                            block_size=spec.block_size, q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype,
                            max_num_seqs=num_seqs or spec.num_seqs, max_blocks_per_seq=max_blocks,
                            partition_tokens=partition, shared_prefix=shared)


def _caches(w):
    """Device caches and the oracle's host copies (fp8: the oracle's own encoding)."""
    sp = w.spec
    if sp.kv_dtype == "fp8_e4m3":
        kh = cache_write.quantize(raw(w.key_src), sp.q_dtype, w.k_scale)
        vh = cache_write.quantize(raw(w.value_src), sp.q_dtype, w.v_scale)
        return (torch.from_numpy(kh).to(DEV).view(torch.float8_e4m3fn),
                torch.from_numpy(vh).to(DEV).view(torch.float8_e4m3fn), kh, vh)
    return w.key_cache, w.value_cache, raw(w.key_cache), raw(w.value_cache)


def _tol(sp):
    return TOL[sp.kv_dtype] if sp.kv_dtype == "fp8_e4m3" else TOL[sp.q_dtype]


def _shared(pa, w, kc, vc, group_start=None, prefix_len=None, max_group_size=None, max_prefix_len=None):
    gs = w.group_start if group_start is None else group_start
    pl = w.group_prefix_len if prefix_len is None else prefix_len
    sizes = (gs[1:] - gs[:-1]).cpu()
    mg = int(sizes.max().item()) if max_group_size is None else max_group_size
    mp = int(pl.max().item()) if max_prefix_len is None else max_prefix_len
    out = torch.empty_like(w.query)
    pa.paged_attention_decode_shared_prefix(out, w.query, kc, vc, w.block_tables, w.seq_lens, w.max_seq_len,
                                            gs, pl, mg, mp, w.scale, w.k_scale, w.v_scale)
    return out, pa.get_error()


def _oracle(w, kh, vh):
    sp = w.spec
    return attention.decode_attention(raw(w.query), kh, vh, raw(w.block_tables), raw(w.seq_lens), w.scale,
                                      q_dtype=sp.q_dtype, kv_dtype=sp.kv_dtype, k_scale=w.k_scale,
                                      v_scale=w.v_scale)


def _spec(q_dtype, kv_dtype, head_dim, group, prefix_tokens, num_seqs=12, groups=3, suffix=(0, 40), Hkv=2):
    base = wl.SPEC_BY_NAME["shared-prefix-fp8"]
    return wl.scaled(base, num_seqs=num_seqs, prefix_groups=groups, prefix_tokens=prefix_tokens,
                     seq_len_min=suffix[0], seq_len_max=suffix[1], num_heads=Hkv * group, num_kv_heads=Hkv,
                     head_dim=head_dim, q_dtype=q_dtype, kv_dtype=kv_dtype, pool_blocks=None,
                     seed=base.seed + 31 * group + head_dim + prefix_tokens)


DTYPES = [("f16", "f16"), ("bf16", "bf16"), ("f16", "fp8_e4m3")]


@pytest.mark.parametrize("q_dtype,kv_dtype", DTYPES)
@pytest.mark.parametrize("head_dim", [64, 128, 256])
@pytest.mark.parametrize("group", [1, 4, 8, 16])
def test_small_groups(q_dtype, kv_dtype, head_dim, group):
    """Three groups sharing a 4-block prefix, suffixes of 0..40 tokens (empty
    and ragged last blocks): every output element against the oracle."""
    if kv_dtype == "fp8_e4m3" and head_dim == 64:
        pytest.skip("fp8 caches need 128-byte rows (head_dim >= 128)")
    sp = _spec(q_dtype, kv_dtype, head_dim, group, 64)
    w = wl.make_workload(sp, DEV)
    kc, vc, kh, vh = _caches(w)
    pa = _ctx(sp, w.num_blocks, w.block_tables.shape[1])
    out, bits = _shared(pa, w, kc, vc)
    assert bits == 0
    assert_out_close(out, _oracle(w, kh, vh), _tol(sp), q_dtype, f"{q_dtype}/{kv_dtype} D{head_dim} G{group}")


@pytest.mark.parametrize("q_dtype,kv_dtype", DTYPES)
@pytest.mark.parametrize("partition", [b.PA_PARTITION_AUTO, b.PA_PARTITION_NONE, 512])
def test_long_prefix_many_rows(q_dtype, kv_dtype, partition):
    """A 65-block prefix (three 32-block chunks, the last one ragged) shared
    by 20 members x 8 query heads (160 rows: three row blocks), a second group
    of one member, and suffixes up to 700 tokens (several partitions)."""
    sp = _spec(q_dtype, kv_dtype, 128, 8, 65 * 16, num_seqs=21, groups=1, suffix=(0, 700))
    w = wl.make_workload(sp, DEV)
    # all 21 share the prefix; declare them as a group of 20 and a group of one
    gs = torch.tensor([0, 20, 21], dtype=torch.int32, device=DEV)
    t = w.block_tables.cpu().tolist()
    assert prefix_sharing.common_prefix_blocks(t, w.seq_lens.cpu().tolist()) == 65
    kc, vc, kh, vh = _caches(w)
    pa = _ctx(sp, w.num_blocks, w.block_tables.shape[1], partition=partition)
    out, bits = _shared(pa, w, kc, vc, group_start=gs,
                        prefix_len=torch.full((gs.numel() - 1,), 65 * 16, dtype=torch.int32, device=DEV))
    assert bits == 0
    assert_out_close(out, _oracle(w, kh, vh), _tol(sp), q_dtype, f"partition={partition}")


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f16", "f16"), ("f16", "fp8_e4m3")])
def test_many_sequences(q_dtype, kv_dtype):
    """520 sequences in 10 groups (the decode kernel's work hand-out reads the
    lengths and suffix offsets 256 sequences at a time; the merge folds two
    heads per thread): every output element against the oracle."""
    sp = _spec(q_dtype, kv_dtype, 128, 4, 64, num_seqs=520, groups=10, suffix=(0, 100))
    w = wl.make_workload(sp, DEV)
    kc, vc, kh, vh = _caches(w)
    pa = _ctx(sp, w.num_blocks, w.block_tables.shape[1])
    out, bits = _shared(pa, w, kc, vc)
    assert bits == 0
    assert_out_close(out, _oracle(w, kh, vh), _tol(sp), q_dtype, f"520 seqs {q_dtype}/{kv_dtype}")


def test_ungrouped_sequences_and_zero_prefix():
    """Sequences before the first group and after the last share nothing, and
    a group may declare a zero-length prefix: all are decoded in full."""
    sp = _spec("f16", "f16", 128, 4, 128, num_seqs=12, groups=3)
    w = wl.make_workload(sp, DEV)
    kc, vc, kh, vh = _caches(w)
    pa = _ctx(sp, w.num_blocks, w.block_tables.shape[1])
    ref = _oracle(w, kh, vh)
    # groups as generated are [0,4) [4,8) [8,12); declare [1,4) (128) and [4,8) (0)
    gs = torch.tensor([1, 4, 8], dtype=torch.int32, device=DEV)
    pl = torch.tensor([128, 0], dtype=torch.int32, device=DEV)
    out, bits = _shared(pa, w, kc, vc, group_start=gs, prefix_len=pl)
    assert bits == 0
    assert_out_close(out, ref, _tol(sp), "f16", "ungrouped")
    # a shorter shared run than the physical one is still a valid prefix
    pl = torch.tensor([64, 32], dtype=torch.int32, device=DEV)
    out, bits = _shared(pa, w, kc, vc, group_start=gs, prefix_len=pl)
    assert bits == 0
    assert_out_close(out, ref, _tol(sp), "f16", "shorter prefix")


def _bad_case(kind):
    sp = _spec("f16", "f16", 128, 4, 128, num_seqs=12, groups=3, suffix=(5, 40))
    w = wl.make_workload(sp, DEV)
    gs, pl = w.group_start.clone(), w.group_prefix_len.clone()
    kw = {}
    if kind == "not_block_multiple":
        pl[1] = 120
    elif kind == "longer_than_member":
        w.seq_lens[5] = 100  # member 5 of group 1 now ends inside the 128-token prefix
    elif kind == "tables_differ":
        bt = w.block_tables.clone()
        spare = int(bt[0, 0].item())  # another valid block (group 0's first prefix block)
        bt[6, 3] = spare
        w.block_tables = bt
    elif kind == "group_too_large":
        kw["max_group_size"] = 3
    elif kind == "prefix_over_bound":
        kw["max_prefix_len"] = 64
    return sp, w, gs, pl, kw


@pytest.mark.parametrize("kind", ["not_block_multiple", "longer_than_member", "tables_differ", "group_too_large",
                                  "prefix_over_bound"])
def test_unusable_group_is_flagged_and_decoded_in_full(kind):
    """A group whose description breaks a rule sets PA_CHECK_BAD_PREFIX; its
    members are then decoded without sharing and the output stays exact."""
    sp, w, gs, pl, kw = _bad_case(kind)
    kc, vc, kh, vh = _caches(w)
    pa = _ctx(sp, w.num_blocks, w.block_tables.shape[1])
    out, bits = _shared(pa, w, kc, vc, group_start=gs, prefix_len=pl, **kw)
    assert bits == b.PA_CHECK_BAD_PREFIX
    assert_out_close(out, _oracle(w, kh, vh), _tol(sp), "f16", kind)


def test_alternating_with_plain_decode():
    """Shared-prefix and plain decode calls on one context, back to back,
    with uniform suffixes (the ticket hand-out) and varying ones (stream-K)."""
    for suffix in ((200, 200), (1, 300)):
        sp = _spec("bf16", "bf16", 128, 8, 256, num_seqs=24, groups=4, suffix=suffix)
        w = wl.make_workload(sp, DEV)
        kc, vc, kh, vh = _caches(w)
        pa = _ctx(sp, w.num_blocks, w.block_tables.shape[1])
        ref = _oracle(w, kh, vh)
        for _ in range(2):
            out, bits = _shared(pa, w, kc, vc)
            assert bits == 0
            assert_out_close(out, ref, _tol(sp), "bf16", f"shared {suffix}")
            plain = pa.decode(w.query, kc, vc, w.block_tables, w.seq_lens, w.max_seq_len, w.scale)
            assert pa.get_error() == 0
            assert_out_close(plain, ref, _tol(sp), "bf16", f"plain {suffix}")


def test_full_size_sampled():
    """The 256-sequence fp8 workload (8 groups of 32 sharing 1024 tokens) in
    the bench's launch configuration: sampled rows against the oracle, and
    every row against plain decode of the same cache."""
    spec = wl.SPEC_BY_NAME["shared-prefix-fp8"]
    w = wl.make_workload(spec, DEV)
    pa = _ctx(spec, w.num_blocks, w.block_tables.shape[1])
    NB, bs, Hkv, D = w.key_src.shape
    kc = torch.empty((NB, bs, Hkv, D), dtype=torch.float8_e4m3fn, device=DEV)
    vc = torch.empty_like(kc)
    slots = torch.arange(NB * bs, dtype=torch.int64, device=DEV)
    pa.reshape_and_cache(w.key_src.view(NB * bs, Hkv, D), w.value_src.view(NB * bs, Hkv, D), kc, vc, slots,
                         w.k_scale, w.v_scale)
    out, bits = _shared(pa, w, kc, vc)
    assert bits == 0
    plain = pa.decode(w.query, kc, vc, w.block_tables, w.seq_lens, w.max_seq_len, w.scale, w.k_scale, w.v_scale)
    assert pa.get_error() == 0
    assert_out_close(out, plain.double().cpu().numpy(), 2 * TOL["fp8_e4m3"], "f16", "vs plain decode")
    rng = np.random.default_rng(spec.seed)
    seqs = sorted(set([0, 31, 32, 255] + rng.choice(256, size=4, replace=False).tolist()))
    heads = [0, 3, 4, 31]
    khc, vhc, bt, lens, uniq = compact_sequences(kc, vc, w.block_tables, w.seq_lens, seqs)
    idx = uniq.to(DEV)
    okh = cache_write.quantize(raw(w.key_src.index_select(0, idx)), spec.q_dtype, w.k_scale)
    ovh = cache_write.quantize(raw(w.value_src.index_select(0, idx)), spec.q_dtype, w.v_scale)
    np.testing.assert_array_equal(khc, okh)
    np.testing.assert_array_equal(vhc, ovh)
    pairs = [(i, h) for i in range(len(seqs)) for h in heads]
    ref = attention.decode_attention(raw(w.query)[seqs], okh, ovh, bt, lens, w.scale, q_dtype=spec.q_dtype,
                                     kv_dtype=spec.kv_dtype, k_scale=w.k_scale, v_scale=w.v_scale, pairs=pairs)
    assert_out_close(out[seqs], ref, TOL["fp8_e4m3"], "f16", "sampled")


def test_host_validation():
    sp = _spec("f16", "f16", 128, 4, 64)
    w = wl.make_workload(sp, DEV)
    kc, vc, _, _ = _caches(w)
    plain_ctx = _ctx(sp, w.num_blocks, w.block_tables.shape[1], shared=False)
    with pytest.raises(b.PagedAttnError) as e:
        _shared(plain_ctx, w, kc, vc)
    assert e.value.status == b.PA_ERR_UNSUPPORTED
    pa = _ctx(sp, w.num_blocks, w.block_tables.shape[1])
    for kw in (dict(max_group_size=0), dict(max_group_size=13), dict(max_prefix_len=-1),
               dict(max_prefix_len=w.max_seq_len + 1)):
        with pytest.raises(b.PagedAttnError) as e:
            _shared(pa, w, kc, vc, **kw)
        assert e.value.status == b.PA_ERR_INVALID_ARG, kw
    with pytest.raises(b.PagedAttnError) as e:  # no groups
        _shared(pa, w, kc, vc, group_start=w.group_start[:1], prefix_len=w.group_prefix_len[:0],
                max_group_size=1, max_prefix_len=0)
    assert e.value.status == b.PA_ERR_INVALID_ARG
