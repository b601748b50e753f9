"""Seeded synthetic inputs for the paged decode path.

This module only builds inputs: random queries and caches, block tables drawn
from a shuffled free list, sequence lengths, and the slot each sequence's
newest token is written to.  It holds none of the attention arithmetic and
none of the cache-write arithmetic, and it serves both the CUDA path and the
CPU oracle (which import nothing from each other).

Recipe (every tensor is seeded; seed = 1000 + workload index):

* values: float32 N(0, 1) cast to the storage type (fp16 / bf16).  For an fp8
  cache the workload carries the 16-bit pre-quantisation pools plus one
  per-tensor scale per cache, scale = amax(|x|) / 448 in fp32 (448 is the
  largest finite E4M3 magnitude); quantising them is left to the caller (the
  cache-write kernel on the GPU, the oracle's codec on the CPU);
* block tables: physical blocks are handed out by a reference-counting free
  list allocator whose free list is a seeded permutation of the pool (page
  "5.KV Cache 管理 & PagedAttention", Q9.1 BlockAllocator / Q9.4
  RefCountBlockAllocator), so tables are non-contiguous; unused table entries
  are -1 (Q8.3); a shared prefix is allocated once per group and its blocks'
  reference count raised once per extra sequence (Q9.4, Q18 fork);
* lengths: uniform integers, inclusive bounds; the length includes the token
  appended by this step's cache write, whose slot is returned in
  ``slot_mapping``;
* the rest of the pool (unused blocks, the tail of each last block) holds
  N(0, 1) values too, i.e. data that must not influence the result.
"""

from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field

import torch

TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "fp8_e4m3": torch.float8_e4m3fn}
FP8_MAX_FINITE = 448.0


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    q_dtype: str
    kv_dtype: str
    seq_len_min: int          # for shared-prefix workloads: private suffix bounds
    seq_len_max: int
    seed: int
    pool_blocks: int | None = None   # None: 1.25 x the blocks the tables need
    prefix_groups: int = 0
    prefix_tokens: int = 0
    max_blocks_per_seq: int | None = None  # None: enough for the longest possible sequence
    description: str = ""

    @property
    def group_size(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def max_seq_len_bound(self) -> int:
        return self.prefix_tokens + self.seq_len_max


SPECS = [
    WorkloadSpec("tiny", 4, 4, 4, 64, 16, "f16", "f16", 1, 100, seed=1000, pool_blocks=64,
                 description="4 seqs, 4 heads MHA, head_dim 64, lengths U[1,100], 64-block pool permuted"),
    WorkloadSpec("llama2-7b-mha", 64, 32, 32, 128, 16, "f16", "f16", 2048, 2048, seed=1001,
                 pool_blocks=12288,
                 description="LLaMA-2-7B layer shape: 64 seqs x 2048 tokens, 32 heads MHA, head_dim 128, "
                             "fp16, blocks shuffled across a 12288-block pool"),
    WorkloadSpec("gqa-70b-like", 128, 64, 8, 128, 16, "bf16", "bf16", 512, 4096, seed=1002,
                 description="128 seqs, lengths U[512,4096], 64 q / 8 kv heads, head_dim 128, bf16"),
    WorkloadSpec("long-context-split-kv", 8, 32, 8, 128, 16, "bf16", "bf16", 32768, 32768, seed=1003,
                 description="8 seqs x 32768 tokens, 32 q / 8 kv heads, head_dim 128, bf16"),
    WorkloadSpec("shared-prefix-fp8", 256, 32, 8, 128, 16, "f16", "fp8_e4m3", 16, 1024, seed=1004,
                 prefix_groups=8, prefix_tokens=1024,
                 description="256 seqs in 8 groups of 32 sharing a 1024-token prefix + private suffix "
                             "U[16,1024], 32 q / 8 kv heads, head_dim 128, fp8-E4M3 cache, fp16 q/out"),
]
SPEC_BY_NAME = {s.name: s for s in SPECS}


def scaled(spec: WorkloadSpec, **overrides) -> WorkloadSpec:
    """A copy of ``spec`` with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(spec, **overrides)


class RefCountAllocator:
    """Free-list block allocator with reference counts (page "5.KV Cache 管理 &
    PagedAttention", Q9.1 / Q9.4): allocate pops the end of the free list and
    sets the count to 1; incref/decref adjust it; a block whose count reaches 0
    goes back on the free list."""

    def __init__(self, free_order: list[int]):
        self.total = len(free_order)
        self.free_blocks = list(free_order)
        self.ref_counts = [0] * self.total

    def allocate(self) -> int:
        if not self.free_blocks:
            raise MemoryError(f"free list empty: pool of {self.total} blocks exhausted")
        blk = self.free_blocks.pop()
        self.ref_counts[blk] = 1
        return blk

    def incref(self, blk: int) -> None:
        self.ref_counts[blk] += 1

    def decref(self, blk: int) -> None:
        self.ref_counts[blk] -= 1
        if self.ref_counts[blk] == 0:
            self.free_blocks.append(blk)


@dataclass
class Workload:
    spec: WorkloadSpec
    seq_lens: torch.Tensor          # [S] int32
    block_tables: torch.Tensor      # [S, max_blocks_per_seq] int32, -1 padded
    slot_mapping: torch.Tensor      # [S] int64: slot of each sequence's newest token
    query: torch.Tensor             # [S, Hq, D] q dtype
    new_key: torch.Tensor           # [S, Hkv, D] q dtype: this step's K
    new_value: torch.Tensor         # [S, Hkv, D]
    key_cache: torch.Tensor | None  # [NB, bs, Hkv, D] kv dtype (16-bit caches)
    value_cache: torch.Tensor | None
    key_src: torch.Tensor | None = None    # fp8 caches: 16-bit pre-quantisation pools
    value_src: torch.Tensor | None = None
    k_scale: float = 1.0
    v_scale: float = 1.0
    scale: float = 1.0
    ref_counts: list[int] = field(default_factory=list)
    num_blocks: int = 0
    group_start: torch.Tensor | None = None       # [G + 1] int32: group g = sequences [start[g], start[g+1])
    group_prefix_len: torch.Tensor | None = None  # [G] int32: tokens the group's sequences share

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max().item()) if self.seq_lens.numel() else 0


def _draw_lengths(spec: WorkloadSpec, gen: torch.Generator) -> list[int]:
    lens = torch.randint(spec.seq_len_min, spec.seq_len_max + 1, (spec.num_seqs,), generator=gen)
    return [spec.prefix_tokens + int(x) for x in lens.tolist()]


def _randn_pool(shape, dtype, gen, device, chunk_rows=1024) -> torch.Tensor:
    """N(0,1) fp32 draws cast to ``dtype``, drawn in chunks along dim 0."""
    out = torch.empty(shape, dtype=dtype, device=device)
    for i in range(0, shape[0], chunk_rows):
        j = min(shape[0], i + chunk_rows)
        out[i:j] = torch.randn((j - i,) + tuple(shape[1:]), generator=gen, device=device,
                               dtype=torch.float32).to(dtype)
    return out


@dataclass
class Layout:
    """Lengths, block tables and slots of a workload (no tensors of values)."""
    seq_lens: list[int]
    block_tables: torch.Tensor      # [S, max_blocks_per_seq] int32, -1 padded
    slot_mapping: list[int]
    ref_counts: list[int]
    num_blocks: int
    group_start: list[int] = field(default_factory=list)  # prefix groups: [G + 1] sequence ranges
    group_prefix_len: list[int] = field(default_factory=list)  # [G] shared tokens (whole blocks)


def build_layout(spec: WorkloadSpec, seq_lens: list[int] | None = None) -> Layout:
    """Seeded lengths and block tables of ``spec`` (host only, cheap).

    ``seq_lens`` overrides the drawn lengths (edge-case sweeps); for
    shared-prefix specs it must include the prefix.
    """
    hgen = torch.Generator().manual_seed(spec.seed)
    bs = spec.block_size
    lens = _draw_lengths(spec, hgen) if seq_lens is None else [int(x) for x in seq_lens]
    S = len(lens)
    if spec.max_blocks_per_seq is not None:
        mb = spec.max_blocks_per_seq
    else:
        mb = max(1, math.ceil(max(spec.max_seq_len_bound, max(lens) if lens else 0) / bs))

    groups = spec.prefix_groups if spec.prefix_groups else 0
    prefix_blocks = spec.prefix_tokens // bs if groups else 0
    needed = sum(math.ceil(n / bs) for n in lens)
    if groups:
        needed = groups * prefix_blocks + sum(math.ceil(n / bs) - prefix_blocks for n in lens)
    pool = spec.pool_blocks if spec.pool_blocks is not None else max(1, math.ceil(1.25 * needed))
    if needed > pool:
        raise MemoryError(f"workload needs {needed} blocks, pool has {pool}")

    alloc = RefCountAllocator(torch.randperm(pool, generator=hgen).tolist())
    tables = torch.full((S, mb), -1, dtype=torch.int32)
    group_prefix: dict[int, list[int]] = {}
    slots = []
    for s, n in enumerate(lens):
        nblk = math.ceil(n / bs)
        if nblk > mb:
            raise ValueError(f"sequence {s} needs {nblk} blocks > max_blocks_per_seq {mb}")
        row = []
        if groups:
            grp = s * groups // S
            if grp not in group_prefix:
                group_prefix[grp] = [alloc.allocate() for _ in range(prefix_blocks)]
            else:
                for b in group_prefix[grp]:
                    alloc.incref(b)
            row.extend(group_prefix[grp])
        while len(row) < nblk:
            row.append(alloc.allocate())
        if nblk:
            tables[s, :nblk] = torch.tensor(row, dtype=torch.int32)
        last = n - 1
        slots.append(row[last // bs] * bs + last % bs if n > 0 else -1)
    group_start, group_prefix_len = [], []
    if groups:
        group_start = [0] + [next((s for s in range(S) if s * groups // S > g), S) for g in range(groups)]
        group_prefix_len = [prefix_blocks * bs] * groups
    return Layout(lens, tables, slots, alloc.ref_counts, pool, group_start, group_prefix_len)


def make_workload(spec: WorkloadSpec, device="cpu", seq_lens: list[int] | None = None) -> Workload:
    """Build the seeded inputs of ``spec`` on ``device`` (see ``build_layout``)."""
    device = torch.device(device)
    lay = build_layout(spec, seq_lens)
    S, pool, bs = len(lay.seq_lens), lay.num_blocks, spec.block_size
    dgen = torch.Generator(device=device).manual_seed(spec.seed)
    qdt = TORCH_DTYPES[spec.q_dtype]
    H, Hkv, D = spec.num_heads, spec.num_kv_heads, spec.head_dim
    query = torch.randn((S, H, D), generator=dgen, device=device, dtype=torch.float32).to(qdt)
    new_key = torch.randn((S, Hkv, D), generator=dgen, device=device, dtype=torch.float32).to(qdt)
    new_value = torch.randn((S, Hkv, D), generator=dgen, device=device, dtype=torch.float32).to(qdt)
    shape = (pool, bs, Hkv, D)
    w = Workload(spec=spec, seq_lens=torch.tensor(lay.seq_lens, dtype=torch.int32).to(device),
                 block_tables=lay.block_tables.to(device),
                 slot_mapping=torch.tensor(lay.slot_mapping, dtype=torch.int64).to(device),
                 query=query, new_key=new_key, new_value=new_value,
                 key_cache=None, value_cache=None, scale=1.0 / math.sqrt(D),
                 ref_counts=lay.ref_counts, num_blocks=pool)
    if lay.group_start:
        w.group_start = torch.tensor(lay.group_start, dtype=torch.int32).to(device)
        w.group_prefix_len = torch.tensor(lay.group_prefix_len, dtype=torch.int32).to(device)
    if spec.kv_dtype == "fp8_e4m3":
        w.key_src = _randn_pool(shape, qdt, dgen, device)
        w.value_src = _randn_pool(shape, qdt, dgen, device)
        # the step's new tokens are part of the tensors the scale is taken over
        kmax = max(w.key_src.abs().max().float().item(), new_key.abs().max().float().item())
        vmax = max(w.value_src.abs().max().float().item(), new_value.abs().max().float().item())
        w.k_scale = float(torch.tensor(kmax, dtype=torch.float32) / torch.tensor(FP8_MAX_FINITE))
        w.v_scale = float(torch.tensor(vmax, dtype=torch.float32) / torch.tensor(FP8_MAX_FINITE))
    else:
        kvdt = TORCH_DTYPES[spec.kv_dtype]
        w.key_cache = _randn_pool(shape, kvdt, dgen, device)
        w.value_cache = _randn_pool(shape, kvdt, dgen, device)
    return w


def kv_read_bytes(seq_lens, num_kv_heads: int, head_dim: int, kv_bytes: int) -> int:
    """Bytes of K and V a decode call must read: sum_s len_s * Hkv * D * 2 * kv_bytes."""
    total = int(torch.as_tensor(seq_lens).to(torch.int64).sum().item())
    return total * num_kv_heads * head_dim * 2 * kv_bytes


def decode_bytes(w: Workload) -> int:
    """Algorithmic bytes of one decode call: K/V reads plus q read and out write."""
    sp = w.spec
    kvb = 1 if sp.kv_dtype == "fp8_e4m3" else 2
    qb = 2
    S = int(w.seq_lens.numel())
    return kv_read_bytes(w.seq_lens.cpu(), sp.num_kv_heads, sp.head_dim, kvb) + S * sp.num_heads * sp.head_dim * 2 * qb


def shared_decode_bytes(w: Workload) -> int:
    """Algorithmic bytes of one decode call that reads every shared prefix
    block once per group: the groups' prefixes, every sequence's private
    suffix, plus q read and out write."""
    sp = w.spec
    if w.group_start is None:
        return decode_bytes(w)
    kvb = 1 if sp.kv_dtype == "fp8_e4m3" else 2
    per_token = sp.num_kv_heads * sp.head_dim * 2 * kvb
    starts = w.group_start.cpu().tolist()
    plen = w.group_prefix_len.cpu().tolist()
    lens = w.seq_lens.cpu().tolist()
    skip = [0] * len(lens)
    for g, n in enumerate(plen):
        for s in range(starts[g], starts[g + 1]):
            skip[s] = n
    tokens = sum(plen) + sum(max(0, n - k) for n, k in zip(lens, skip))
    S = len(lens)
    return tokens * per_token + S * sp.num_heads * sp.head_dim * 2 * 2
