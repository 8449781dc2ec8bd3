"""Prefill of one long prompt over G ranks: the prompt's query rows are split zig-zag, every rank holds the
whole prompt's pools and runs the usual three calls on its own rows.

Causal rows grow in cost with their position, so the rows are cut into 2G equal chunks and rank r takes
chunks r and 2G-1-r: every rank then scores about the same number of (row, key) pairs.  Each chunk of rows
is expressed as a sequence of the batch: the prompt truncated after the chunk's last row, whose last
rows are the chunk (the batch convention: a sequence's query rows are its last tokens), reading the prompt's
block table.  The pools are filled once before the prefill: each rank writes the pages of its own tokens and
one all-gather of pages gives every rank the whole prompt (`allgather_pages`, torch.distributed: NCCL over
NVLink on GPUs).  After that no rank exchanges anything.
"""
from __future__ import annotations

import copy

import numpy as np
import torch


def zigzag_chunks(n_rows: int, world: int):
    """For each rank, its two row ranges [(lo, hi), (lo, hi)] (query-row indices of the prompt): the rows
    cut into 2*world chunks of sizes differing by at most one, rank r taking chunks r and 2*world-1-r."""
    bounds = [(c * n_rows) // (2 * world) for c in range(2 * world + 1)]
    return [[(bounds[r], bounds[r + 1]), (bounds[2 * world - 1 - r], bounds[2 * world - r])] for r in range(world)]


def local_prefill_workload(wl, rank: int, world: int):
    """The rank's batch for a one-prompt prefill workload `wl` (one sequence, its last T tokens the query
    rows): one sequence per chunk, each the prompt truncated after the chunk, with the chunk's rows and the
    prompt's block table.  Returns (workload, rows): rows are the prompt's query-row indices in the local
    batch's row order."""
    if wl.num_seqs != 1:
        raise ValueError("zig-zag prefill takes one prompt (one sequence)")
    T = wl.total_q
    p0 = int(wl.seq_lens[0]) - T                          # position of query row 0
    chunks = [c for c in zigzag_chunks(T, world)[rank] if c[1] > c[0]]
    rows = np.concatenate([np.arange(lo, hi) for lo, hi in chunks]).astype(np.int64)
    loc = copy.copy(wl)
    loc.seq_lens = np.array([p0 + hi for _, hi in chunks], dtype=np.int32)
    loc.q_lens = np.array([hi - lo for lo, hi in chunks], dtype=np.int32)
    loc.cu_q = np.concatenate([[0], np.cumsum(loc.q_lens)]).astype(np.int32)
    loc.block_table = np.repeat(wl.block_table[:1], len(chunks), axis=0)
    for name in ("q", "qI", "w"):
        a = getattr(wl, name)
        if a is not None:
            setattr(loc, name, np.ascontiguousarray(a[rows]))
    return loc, rows


def pages_of_rank(n_pages: int, rank: int, world: int):
    """The contiguous page range [lo, hi) whose tokens rank r writes (and contributes to the all-gather)."""
    return (rank * n_pages) // world, ((rank + 1) * n_pages) // world


def allgather_pages(pool: torch.Tensor, page_ids: torch.Tensor, rank: int, world: int, group=None):
    """Fill every rank's pool with all ranks' pages: rank r owns pages page_ids[lo_r:hi_r] (physical ids of
    the prompt's logical pages, pages_of_rank split); after the call every rank's `pool` ([num_blocks,
    page, ...]) holds every listed page.  Ranks own nearly equal page counts; the exchange is one
    all-gather of the largest share per rank (padded), then a scatter into place on every rank."""
    import torch.distributed as dist
    n = page_ids.numel()
    shares = [pages_of_rank(n, r, world) for r in range(world)]
    width = max(hi - lo for lo, hi in shares)
    lo, hi = shares[rank]
    mine = torch.zeros((width,) + tuple(pool.shape[1:]), dtype=pool.dtype, device=pool.device)
    if hi > lo:
        mine[: hi - lo] = pool[page_ids[lo:hi].long()]
    parts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    for r, (l, h) in enumerate(shares):
        if h > l:
            pool[page_ids[l:h].long()] = parts[r][: h - l]
    return pool
