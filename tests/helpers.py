"""Shared test plumbing: moving tensors to the oracle's raw numpy formats,
extracting sampled sequences of a large cache, and the output comparison.
Contains no attention arithmetic."""

from __future__ import annotations

import numpy as np
import torch

# Output tolerances (max abs error vs the fp64 oracle) by output / cache type.
TOL = {"f16": 2e-3, "bf16": 8e-3, "fp8_e4m3": 2e-3}


def raw(t: torch.Tensor) -> np.ndarray:
    """torch tensor -> numpy raw storage in the oracle's conventions."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float16:
        return t.numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.float8_e4m3fn, torch.uint8):
        return t.view(torch.uint8).numpy()
    if t.dtype in (torch.int32, torch.int64):
        return t.numpy()
    raise TypeError(t.dtype)


def half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Half a unit in the last place of |x| in the output format (its own rounding)."""
    mant = {"f16": 10, "bf16": 7}[dtype]
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -14)))
    return 0.5 * 2.0 ** (e - mant)


def assert_out_close(got: torch.Tensor, ref: np.ndarray, tol: float, out_dtype: str, where="") -> float:
    """Element-wise |got - ref| <= tol, widened only by the output format's own
    rounding where |ref| is so large that one half-ulp exceeds tol / 2."""
    g = got.detach().float().cpu().double().numpy()
    mask = ~np.isnan(ref)
    assert np.all(np.isfinite(g[mask])), f"non-finite output {where}"
    err = np.abs(g - ref)[mask]
    allow = tol + np.where(half_ulp(ref, out_dtype) > tol / 2, half_ulp(ref, out_dtype), 0.0)[mask]
    worst = float(err.max()) if err.size else 0.0
    assert np.all(err <= allow), f"max abs err {worst:.3e} > tol {tol} {where}"
    return worst


def compact_sequences(key_cache: torch.Tensor, value_cache: torch.Tensor, block_tables: torch.Tensor,
                      seq_lens: torch.Tensor, seqs: list[int]):
    """Copy only the blocks of the chosen sequences to the host: returns a
    compact pool (raw numpy), tables renumbered into it (-1 elsewhere), lengths."""
    bs = key_cache.shape[1]
    lens = seq_lens.cpu().tolist()
    bt = block_tables.cpu()
    rows, ids = [], []
    for s in seqs:
        nb = -(-lens[s] // bs)
        ids.append(bt[s, :nb].to(torch.int64))
    uniq = torch.unique(torch.cat(ids)) if ids else torch.zeros(0, dtype=torch.int64)
    remap = {int(b): i for i, b in enumerate(uniq.tolist())}
    idx = uniq.to(key_cache.device)
    kc = raw(key_cache.index_select(0, idx))
    vc = raw(value_cache.index_select(0, idx))
    mb = max((len(x) for x in ids), default=1)
    tables = -np.ones((len(seqs), max(mb, 1)), dtype=np.int64)
    for r, x in enumerate(ids):
        tables[r, :len(x)] = [remap[int(b)] for b in x.tolist()]
        rows.append(lens[seqs[r]])
    return kc, vc, tables, np.array(rows), uniq
