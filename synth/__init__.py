"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module only draws random numbers and lays out a paged KV pool; it holds
none of the zigzag method's arithmetic (no block sizes, no rank assignment, no
attention).  Both the tests and the benchmark call it so that the oracle and
the CUDA path see byte-identical inputs.

Recipe (all seeded):
  * sequence lengths for varlen batches: numpy ``default_rng(seed).integers``;
  * Q, K, V: one generator, drawn in the order Q, K, V, each ``[T, H, D]`` in
    natural token order, standard normal times ``scale``; bf16 tensors are the
    fp32 draw rounded to nearest-even;
  * pool pages: a seeded permutation of the pool's pages, handed out to the
    sequences in order, each sequence starting on a page boundary;
  * growing scores (optional): key row at position t of its sequence scaled by
    ``1 + per_tile * t / 128``, so that attention scores grow along the
    sequence (drives the kernel's redo of tiles whose row sum leaves range).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

_DTYPES = {"fp32": torch.float32, "bf16": torch.bfloat16}


def varlen_lengths(n: int, lo: int, hi: int, seed: int = 0) -> list[int]:
    """``n`` lengths uniform in ``[lo, hi]`` (both ends included)."""
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lo, hi + 1, n)]


def normal(shape, seed: int, scale: float = 1.0, dtype: str = "bf16",
           device: str = "cpu", generator=None) -> torch.Tensor:
    """Standard normal times ``scale``, drawn in fp32 then cast to ``dtype``.

    On the CPU the draw comes from numpy's PCG64; on a CUDA device from torch's
    Philox generator (so large tensors never cross the PCIe bus).  Either way
    the same seed gives the same tensor on every run.
    """
    if str(device).startswith("cuda"):
        g = generator
        if g is None:
            g = torch.Generator(device=device)
            g.manual_seed(seed)
        x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    else:
        rng = generator if generator is not None else np.random.default_rng(seed)
        x = torch.from_numpy(rng.standard_normal(tuple(shape), dtype=np.float32))
    if scale != 1.0:
        x.mul_(scale)
    return x.to(_DTYPES[dtype])


def qkv(total_tokens: int, h_q: int, h_kv: int, d: int, seed: int, scale: float,
        dtype: str = "bf16", device: str = "cpu"):
    """Q ``[T,h_q,d]``, K and V ``[T,h_kv,d]`` from one seeded stream, in that order."""
    if str(device).startswith("cuda"):
        g = torch.Generator(device=device)
        g.manual_seed(seed)
    else:
        g = np.random.default_rng(seed)
    q = normal((total_tokens, h_q, d), seed, scale, dtype, device, g)
    k = normal((total_tokens, h_kv, d), seed, scale, dtype, device, g)
    v = normal((total_tokens, h_kv, d), seed, scale, dtype, device, g)
    return q, k, v


def key_ramp(k: torch.Tensor, seq_lens, per_tile: float) -> torch.Tensor:
    """``k`` ``[T, H, D]`` (natural order, sequences back to back) with the row at
    position t of its sequence scaled by ``1 + per_tile * t / 128`` (in fp32,
    then cast back to ``k``'s dtype)."""
    pos = torch.cat([torch.arange(n, dtype=torch.float32) for n in seq_lens]).to(k.device)
    f = (1.0 + per_tile * pos / 128.0).view(-1, 1, 1)
    return (k.float() * f).to(k.dtype)


@dataclass
class PagedPool:
    page_size: int
    num_pages: int
    page_table: np.ndarray      # [bs, max_pages] int32, unused entries -1
    out_cache_loc: np.ndarray   # [T] int64, pool slot of every natural token

    @property
    def num_slots(self) -> int:
        return self.num_pages * self.page_size

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])


def paged_pool(lengths, page_size: int, seed: int | None, spare_pages: int = 0) -> PagedPool:
    """Lay the sequences out in a pool of ``page_size``-token pages.

    Sequence ``s`` takes ``ceil(L_s / page_size)`` pages; which physical pages
    it gets comes from a seeded permutation (``seed=None`` keeps them in
    order).  Slot of token ``t`` of sequence ``s`` is
    ``page_table[s][t // page_size] * page_size + t % page_size``.
    """
    need = [max(1, math.ceil(int(L) / page_size)) for L in lengths]
    num_pages = sum(need) + spare_pages
    order = (np.arange(num_pages) if seed is None
             else np.random.default_rng(seed).permutation(num_pages))
    max_pages = max(need)
    table = np.full((len(lengths), max_pages), -1, dtype=np.int32)
    loc = []
    cursor = 0
    for s, L in enumerate(lengths):
        pages = order[cursor:cursor + need[s]]
        cursor += need[s]
        table[s, :need[s]] = pages
        t = np.arange(int(L))
        loc.append(pages[t // page_size].astype(np.int64) * page_size + t % page_size)
    return PagedPool(page_size, num_pages, table, np.concatenate(loc).astype(np.int64))
