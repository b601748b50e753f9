"""GPU block copies (copy-on-write inside the device cache, swap to and from a
pinned host cache) against the oracle: bit-exact."""

import numpy as np
import pytest
import torch

from oracle import block_copy
from paged_kv_cache_463_b200 import binding as b
from tests.helpers import raw

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_463_b200 import build
    build.build()
    torch.cuda.init()


def _ctx(kv_dtype, nb, hkv=8, d=128):
    q = "f16" if kv_dtype in ("f16", "fp8_e4m3") else "bf16"
    return b.PagedAttention(hkv * 4, hkv, d, nb, q_dtype=q, kv_dtype=kv_dtype, max_num_seqs=4, max_blocks_per_seq=8)


def _rand_cache(nb, hkv, d, kv_dtype, device, seed):
    g = torch.Generator(device=device).manual_seed(seed)
    if kv_dtype == "fp8_e4m3":
        x = torch.randint(0, 256, (nb, 16, hkv, d), generator=g, device=device, dtype=torch.int32).to(torch.uint8)
        return x.view(torch.float8_e4m3fn)
    dt = torch.float16 if kv_dtype == "f16" else torch.bfloat16
    return torch.randn((nb, 16, hkv, d), generator=g, device=device).to(dt)


@pytest.mark.parametrize("kv_dtype", ["f16", "bf16", "fp8_e4m3"])
def test_copy_on_write_in_device_cache(kv_dtype):
    nb = 300
    pa = _ctx(kv_dtype, nb)
    kc = _rand_cache(nb, 8, 128, kv_dtype, DEV, 1)
    vc = _rand_cache(nb, 8, 128, kv_dtype, DEV, 2)
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(3))
    pairs = torch.stack([perm[:100], perm[100:200]], dim=1).to(torch.int64)  # disjoint src / dst
    kh, vh = raw(kc).copy(), raw(vc).copy()
    pa.paged_copy_blocks(kc, vc, kc, vc, pairs.to(DEV))
    assert pa.get_error() == 0
    block_copy.copy_blocks(kh, vh, kh, vh, pairs.numpy())
    np.testing.assert_array_equal(raw(kc), kh)
    np.testing.assert_array_equal(raw(vc), vh)


def test_swap_out_and_in_through_pinned_host_memory():
    nb, host_nb = 256, 64
    pa = _ctx("f16", nb)
    kc = _rand_cache(nb, 8, 128, "f16", DEV, 4)
    vc = _rand_cache(nb, 8, 128, "f16", DEV, 5)
    hk = torch.zeros((host_nb, 16, 8, 128), dtype=torch.float16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    seq_blocks = torch.tensor([7, 91, 3, 250, 128, 17], dtype=torch.int64)
    out_pairs = torch.stack([seq_blocks, torch.arange(6) + 10], 1).contiguous()
    kh0, vh0 = raw(kc).copy(), raw(vc).copy()
    pa.paged_copy_blocks(hk, hv, kc, vc, out_pairs.to(DEV))           # swap out: GPU -> pinned host
    assert pa.get_error() == 0
    ohk, ohv = np.zeros_like(raw(hk)), np.zeros_like(raw(hv))
    block_copy.copy_blocks(kh0, vh0, ohk, ohv, out_pairs.numpy())
    np.testing.assert_array_equal(raw(hk), ohk)
    np.testing.assert_array_equal(raw(hv), ohv)
    new_blocks = torch.tensor([200, 4, 66, 99, 150, 31], dtype=torch.int64)
    in_pairs = torch.stack([torch.arange(6) + 10, new_blocks], 1).contiguous().pin_memory()  # pairs in host memory
    pa.paged_copy_blocks(kc, vc, hk, hv, in_pairs)                    # swap in: pinned host -> GPU
    assert pa.get_error() == 0
    block_copy.copy_blocks(ohk, ohv, kh0, vh0, in_pairs.numpy())
    np.testing.assert_array_equal(raw(kc), kh0)
    np.testing.assert_array_equal(raw(vc), vh0)
    np.testing.assert_array_equal(raw(kc)[new_blocks.numpy()], raw(kc)[seq_blocks.numpy()])


def test_copy_blocks_out_of_range_pairs_flagged_and_skipped():
    nb = 32
    pa = _ctx("f16", nb)
    kc = _rand_cache(nb, 8, 128, "f16", DEV, 6)
    vc = _rand_cache(nb, 8, 128, "f16", DEV, 7)
    k0 = raw(kc).copy()
    pairs = torch.tensor([[-1, 2], [1, nb], [nb + 5, 0], [3, 4]], dtype=torch.int64, device=DEV)
    pa.paged_copy_blocks(kc, vc, kc, vc, pairs)
    assert pa.get_error() & b.PA_CHECK_BAD_BLOCK
    expect = k0.copy()
    expect[4] = k0[3]
    np.testing.assert_array_equal(raw(kc), expect)
