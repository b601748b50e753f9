"""The seeded input generator: block tables, lengths and slots are what the
workload recipe says, checked against the oracle's paging functions. CPU only."""

import math

import numpy as np
import pytest
import torch

from oracle import paging
from paged_kv_cache_463_b200 import workloads as wl


@pytest.mark.parametrize("spec", wl.SPECS, ids=lambda s: s.name)
def test_layout_full_size(spec):
    lay = wl.build_layout(spec)
    bs = spec.block_size
    bt = lay.block_tables.numpy()
    assert len(lay.seq_lens) == spec.num_seqs
    lo, hi = spec.prefix_tokens + spec.seq_len_min, spec.prefix_tokens + spec.seq_len_max
    assert all(lo <= n <= hi for n in lay.seq_lens)
    owners = {}
    for s, n in enumerate(lay.seq_lens):
        nb = paging.blocks_needed(n, bs)
        row = bt[s]
        assert np.all(row[:nb] >= 0) and np.all(row[:nb] < lay.num_blocks)
        assert np.all(row[nb:] == -1)
        assert lay.slot_mapping[s] == paging.slot_of(row, n - 1, bs)
        for j, b in enumerate(row[:nb].tolist()):
            owners.setdefault(b, []).append((s, j))
    for b, users in owners.items():
        assert lay.ref_counts[b] == len(users)
        if len(users) > 1:  # only shared-prefix blocks are shared, at the same logical index
            assert spec.prefix_groups > 0
            assert len({j for _, j in users}) == 1 and users[0][1] < spec.prefix_tokens // bs


def test_layout_specific_shapes():
    c1 = wl.build_layout(wl.SPEC_BY_NAME["llama2-7b-mha"])
    assert c1.num_blocks == 12288 and c1.block_tables.shape == (64, 128)
    assert all(n == 2048 for n in c1.seq_lens)
    assert sum(1 for c in c1.ref_counts if c) == 8192
    c2 = wl.build_layout(wl.SPEC_BY_NAME["gqa-70b-like"])
    assert any(n % 16 for n in c2.seq_lens)            # partially filled last blocks
    assert c2.block_tables.shape[1] == 256
    c3 = wl.build_layout(wl.SPEC_BY_NAME["long-context-split-kv"])
    assert c3.block_tables.shape == (8, 2048) and c3.num_blocks == math.ceil(1.25 * 16384)
    c4 = wl.build_layout(wl.SPEC_BY_NAME["shared-prefix-fp8"])
    shared = [c for c in c4.ref_counts if c > 1]
    assert len(shared) == 8 * 64 and all(c == 32 for c in shared)
    # tables are non-contiguous: consecutive logical blocks rarely adjacent physically
    bt = c1.block_tables.numpy()
    assert np.mean(np.diff(bt, axis=1) == 1) < 0.01


def test_small_workload_tensors_and_fp8_scale():
    spec = wl.scaled(wl.SPEC_BY_NAME["shared-prefix-fp8"], num_seqs=8, prefix_groups=2, prefix_tokens=64,
                     seq_len_min=16, seq_len_max=40)
    w = wl.make_workload(spec, "cpu")
    assert w.key_cache is None and w.key_src.dtype == torch.float16
    amax = max(w.key_src.abs().max().item(), w.new_key.abs().max().item())
    assert w.k_scale == pytest.approx(amax / 448.0, rel=1e-6)
    w2 = wl.make_workload(spec, "cpu")
    assert torch.equal(w.query, w2.query) and torch.equal(w.key_src, w2.key_src)  # seeded


def test_edge_lengths_override():
    spec = wl.scaled(wl.SPEC_BY_NAME["tiny"], pool_blocks=None)
    lens = [1, 15, 16, 17, 0]
    lay = wl.build_layout(spec, seq_lens=lens)
    assert lay.seq_lens == lens and lay.slot_mapping[-1] == -1
