"""Context-parallel decode: one decode batch whose caches are spread over G ranks.

Rank r holds a contiguous, page-aligned range of every sequence's tokens (ranks in ascending order of their
ranges).  A step is three local phases around two all-gathers:

  1. ``candidates``: indexer scores and top-k over the rank's own range (the usual calls, on a batch whose
     sequences are the rank's ranges), turned into (score, global position) pairs;
  2. all-gather of the candidates; ``attend``: the global top-k over all ranks' candidates (the usual
     top-k on rows of G*k candidates), the winners inside this rank's range, and the usual decode attention
     over them, giving this rank's partial (o_r, lse_r);
  3. all-gather of the partials; ``merge``: the log-sum-exp combine.

The selected set equals the single-GPU selection (every global winner is in its own range's top-k, and
ties resolve to the lower global position on both levels), and the merge is the cross-block reduction of
split attention ("Engineering Practices for Day-0 Adaptation of Million-Token Context Models on Domestic
AI Chips", Four Key Layers 3) taken across GPUs.  Every step runs in libdsa's kernels; torch moves the
exchanged buffers (torch.distributed all-gathers over NCCL, or stacking when ranks are run one after
another in one process).
"""
from __future__ import annotations

import copy

import numpy as np
import torch

from . import binding as B
from .pipeline import DeviceBatch


def shard_ranges(seq_lens, world: int, page_size: int = 64):
    """(lo, hi) int32 arrays [world, num_seqs]: rank r holds tokens [lo[r, b], hi[r, b]) of sequence b, the
    pages floor(r*P/world) .. floor((r+1)*P/world) - 1 of its P pages (the last page may be partial).  Every
    sequence needs at least `world` pages, so that no rank's range is empty."""
    seq_lens = np.asarray(seq_lens, dtype=np.int64)
    pages = (seq_lens + page_size - 1) // page_size
    if np.any(pages < world):
        raise ValueError(f"context-parallel decode over {world} ranks needs at least {world} pages per sequence")
    r = np.arange(world + 1, dtype=np.int64)[:, None]
    bounds = np.minimum((r * pages[None, :]) // world * page_size, seq_lens[None, :])
    return bounds[:-1].astype(np.int32), bounds[1:].astype(np.int32)


def local_workload(wl, rank: int, world: int):
    """The rank's view of a decode workload: the same query inputs and pools, a block table holding only
    its pages of each sequence, and its range lengths as sequence lengths (the query row is then the last
    local token, so every local token is visible to it).  Returns (workload, lo, hi)."""
    if not np.all(wl.q_lens == 1):
        raise ValueError("context-parallel decode takes decode batches: one query row per sequence")
    lo, hi = shard_ranges(wl.seq_lens, world, wl.page_size)
    lo, hi = lo[rank], hi[rank]
    p0, p1 = lo // wl.page_size, (hi + wl.page_size - 1) // wl.page_size
    width = int((p1 - p0).max())
    bt = np.zeros((wl.num_seqs, width), dtype=np.int32)
    for b in range(wl.num_seqs):
        bt[b, : p1[b] - p0[b]] = wl.block_table[b, p0[b]: p1[b]]
    loc = copy.copy(wl)
    loc.seq_lens = (hi - lo).astype(np.int32)
    loc.block_table = bt
    return loc, lo, hi


class CPDecodeRank:
    """One rank's state for context-parallel decode steps: its local batch (shared pools and query inputs
    may be passed in as `inputs`, device tensors as DeviceBatch.upload_inputs returns them), its range
    bounds and the buffers of the exchanged candidates and partials."""

    def __init__(self, wl, rank: int, world: int, device="cuda", inputs=None):
        self.rank, self.world = rank, world
        dev = torch.device(device)
        loc, lo, hi = local_workload(wl, rank, world)
        base = dict(inputs) if inputs is not None else DeviceBatch.upload_inputs(wl, dev)
        base.update(block_table=torch.from_numpy(loc.block_table).to(dev),
                    seq_lens=torch.from_numpy(loc.seq_lens).to(dev),
                    cu_q=torch.from_numpy(loc.cu_q.astype(np.int32)).to(dev))
        self.db = DeviceBatch(loc, device=dev, decode=True, inputs=base)
        self.T, self.k, self.H, self.Dv = loc.total_q, loc.topk, loc.H, loc.Dv
        self.lo = torch.from_numpy(lo).to(dev)
        self.hi = torch.from_numpy(hi).to(dev)
        T, k, G = self.T, self.k, world
        self.cand_score = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.cand_gidx = torch.empty((T, k), dtype=torch.int32, device=dev)
        # the global selection runs the usual top-k on T rows of G*k candidates
        self.ld_rows = (G * k + 3) // 4 * 4
        self.rows = torch.empty((T, self.ld_rows), dtype=torch.float32, device=dev)
        self.rows_bt = torch.zeros((T, (G * k + 63) // 64), dtype=torch.int32, device=dev)
        self.rows_len = torch.full((T,), G * k, dtype=torch.int32, device=dev)
        self.rows_cu = torch.arange(T + 1, dtype=torch.int32, device=dev)
        self.rows_batch = B.make_batch(self.rows_bt, self.rows_len, self.rows_cu, num_blocks=1, page_size=64,
                                       total_q=T, max_q_per_seq=1, max_seq_len=G * k)
        self.rows_ws_bytes = B.dsa_workspace_size(B.DSA_OP_TOPK, self.rows_batch, k)
        self.rows_ws = torch.zeros(self.rows_ws_bytes, dtype=torch.uint8, device=dev)
        self.sel = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.local_idx = torch.empty((T, k), dtype=torch.int32, device=dev)

    # phase 1 -------------------------------------------------------------------------------------------
    def candidates(self, stream=None):
        """(cand_score [T, k], cand_gidx [T, k]): this range's top-k as (score, global position)."""
        self.db.indexer(stream)
        self.db.topk(stream)
        B.dsa_cp_candidates(self.db.scores, self.db.ld, self.db.idx, self.T, self.k, self.lo, self.cand_score,
                            self.cand_gidx, stream)
        return self.cand_score, self.cand_gidx

    # phase 2 -------------------------------------------------------------------------------------------
    def attend(self, g_score, g_gidx, stream=None):
        """From all ranks' candidates ([G, T, k] each): the global top-k, its part inside this range, and the
        decode attention over that part.  Returns (o_r [T, H, Dv] bf16, lse_r [T, H])."""
        G, T, k = self.world, self.T, self.k
        B.dsa_cp_rows(g_score, G, T, k, self.rows, self.ld_rows, stream)
        B.dsa_topk(self.rows, self.ld_rows, self.rows_batch, k, self.sel, self.rows_ws, self.rows_ws_bytes, stream)
        B.dsa_cp_select_local(self.sel, g_gidx, G, T, k, self.lo, self.hi, self.local_idx, stream)
        self.db.attention(stream, idx=self.local_idx)
        return self.db.out, self.db.lse

    # phase 3 -------------------------------------------------------------------------------------------
    def merge(self, g_out, g_lse, out, lse, stream=None):
        """out [T, H, Dv] bf16, lse [T, H] from all ranks' partials ([G, T, H, Dv] and [G, T, H])."""
        B.dsa_cp_merge(g_out, B.DSA_BF16, g_lse, self.world, self.T, self.H, self.Dv, out, lse, stream)
        return out, lse

    def selected_positions(self):
        """This rank's part of the last step's global top-k, as global positions (numpy, ragged per row)."""
        loc = self.local_idx.cpu().numpy()
        lo = self.lo.cpu().numpy()
        return [loc[t][loc[t] >= 0].astype(np.int64) + int(lo[t]) for t in range(self.T)]


def cp_decode_step(rank_state, all_gather, out, lse, stream=None):
    """One context-parallel decode step of this rank.  `all_gather(t)` returns the [G, ...] stack of every
    rank's `t` (e.g. torch.distributed.all_gather_into_tensor over NCCL); every rank calls this function
    together, with the same collective order."""
    cs, cg = rank_state.candidates(stream)
    g_score, g_gidx = all_gather(cs), all_gather(cg)
    o_r, lse_r = rank_state.attend(g_score, g_gidx, stream)
    g_out, g_lse = all_gather(o_r), all_gather(lse_r)
    return rank_state.merge(g_out, g_lse, out, lse, stream)


def cp_decode_emulated(ranks, out, lse, stream=None):
    """All ranks' steps in one process, one rank after another on one device (no rank ever waits on
    another): the all-gathers are stacks of the ranks' buffers.  Returns (out, lse)."""
    cands = [r.candidates(stream) for r in ranks]
    with torch.cuda.stream(stream) if stream is not None else _null():
        g_score = torch.stack([c[0] for c in cands])
        g_gidx = torch.stack([c[1] for c in cands])
    parts = []
    for r in ranks:
        o_r, lse_r = r.attend(g_score, g_gidx, stream)
        with torch.cuda.stream(stream) if stream is not None else _null():
            parts.append((o_r.clone(), lse_r.clone()))
    with torch.cuda.stream(stream) if stream is not None else _null():
        g_out = torch.stack([p[0] for p in parts])
        g_lse = torch.stack([p[1] for p in parts])
    return ranks[0].merge(g_out, g_lse, out, lse, stream)


class _null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False
