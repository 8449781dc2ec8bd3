"""Device-resident batch and the three-call path (indexer -> top-k -> sparse attention).

`DeviceBatch` uploads a host `Workload` (see workloads.py) into device memory with torch
(plumbing only) and owns the output buffers and one workspace; `run()` enqueues the
three C-ABI calls on one stream.  Nothing here computes any part of the method.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B


def _dev(a, device):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)


def check_inputs_finite(wl) -> None:
    """Optional host pre-check of a workload's inputs: the library requires finite values (and positive key
    scales) and does not test them on the device.  Raises ValueError naming the first offending array.
    bf16 and fp32 values are checked by their exponent bits, E4M3 codes by the two NaN codes (0x7F, 0xFF)."""
    def bad(name, mask):
        if np.any(mask):
            raise ValueError(f"input {name} holds {int(np.count_nonzero(mask))} non-finite value(s)")

    fp8 = wl.kind == "mla"
    for name in ("q", "kv_pool", "v_pool", "qI", "kI_pool", "w", "kS_pool"):
        a = getattr(wl, name, None)
        if a is None:
            continue
        a = np.asarray(a)
        if a.dtype == np.uint16:                                   # bf16 bits
            bad(name, (a & 0x7F80) == 0x7F80)
        elif a.dtype == np.uint8 and fp8:                          # e4m3 codes
            bad(name, (a & 0x7F) == 0x7F)
        else:
            bad(name, ~np.isfinite(a.astype(np.float32, copy=False)))
    if getattr(wl, "kS_pool", None) is not None and np.any(np.asarray(wl.kS_pool) <= 0):
        raise ValueError("input kS_pool holds a key scale <= 0")


class DeviceBatch:
    """One workload resident in HBM plus its outputs.

    scores [total_q, ld] f32, idx [total_q, k] int32, out [total_q, H, Dv] (bf16 or f32),
    lse [total_q, H] f32.  `decode` picks dsa_sparse_attn_decode (every sequence has one
    query row) over dsa_sparse_attn_prefill; default: decode when that holds.
    """

    def __init__(self, wl, device="cuda", decode=None, inputs=None, check_finite=False):
        self.wl = wl
        self.device = torch.device(device)
        dv = self.device
        mla = wl.kind == "mla"
        self.mla = mla
        self.dt = B.DSA_BF16 if mla else B.DSA_F32
        self.idx_dt = B.DSA_FP8_E4M3 if mla else B.DSA_F32
        if check_finite:
            check_inputs_finite(wl)
        if inputs is None:
            inputs = self.upload_inputs(wl, dv)
        self.inputs = inputs
        for k_, v_ in inputs.items():
            setattr(self, k_, v_)
        self.ld = int((wl.max_seq_len + 3) // 4 * 4)
        T = wl.total_q
        self.batch = B.make_batch(self.block_table, self.seq_lens, self.cu_q, num_blocks=wl.num_blocks,
                                  page_size=wl.page_size, total_q=T, max_q_per_seq=wl.max_q_per_seq,
                                  max_seq_len=wl.max_seq_len)
        self.scores = torch.empty((T, self.ld), dtype=torch.float32, device=dv)
        self.idx = torch.empty((T, wl.topk), dtype=torch.int32, device=dv)
        self.out = torch.empty((T, wl.H, wl.Dv), dtype=torch.bfloat16 if mla else torch.float32, device=dv)
        self.lse = torch.empty((T, wl.H), dtype=torch.float32, device=dv)
        if decode is None:
            decode = bool(np.all(wl.q_lens == 1))
        self.decode = decode
        op_attn = B.DSA_OP_ATTN_DECODE if decode else B.DSA_OP_ATTN_PREFILL
        self.ws_bytes = max(B.dsa_workspace_size(B.DSA_OP_INDEXER, self.batch),
                            B.dsa_workspace_size(B.DSA_OP_TOPK, self.batch, wl.topk),
                            B.dsa_workspace_size(B.DSA_OP_INDEXER_TOPK, self.batch, wl.topk),
                            B.dsa_workspace_size(op_attn, self.batch, wl.topk, wl.H, wl.Dv))
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dv)

    @staticmethod
    def upload_inputs(wl, dv):
        """Device copies of every input array of the workload (the cache pools included)."""
        return dict(
            q=_dev(wl.q, dv), kv_pool=_dev(wl.kv_pool, dv), v_pool=_dev(wl.v_pool, dv), qI=_dev(wl.qI, dv),
            kI_pool=_dev(wl.kI_pool, dv), kS_pool=_dev(wl.kS_pool, dv), w=_dev(wl.w, dv),
            block_table=_dev(wl.block_table.astype(np.int32), dv), seq_lens=_dev(wl.seq_lens.astype(np.int32), dv),
            cu_q=_dev(wl.cu_q.astype(np.int32), dv))

    # individual steps --------------------------------------------------------------------------
    def indexer(self, stream=None):
        wl = self.wl
        B.dsa_indexer_scores(self.qI, self.idx_dt, self.w, self.kI_pool, self.idx_dt, self.kS_pool, wl.Hi, wl.Di,
                             self.batch, self.scores, self.ld, self.ws, self.ws_bytes, stream)

    def append_and_indexer(self, kv_new, k_new, k_dt, stream=None):
        """The decode step's cache update fused with the indexer: writes the batch's new tokens (kv_new
        [T, 576] bf16 bits, k_new [T, 128] of k_dt) into this batch's pools, then scores."""
        wl = self.wl
        B.dsa_indexer_scores_append(kv_new, self.dt, k_new, k_dt, self.kv_pool, self.qI, self.idx_dt, self.w,
                                    self.kI_pool, self.idx_dt, self.kS_pool, wl.Hi, wl.Di, self.batch, self.scores,
                                    self.ld, self.ws, self.ws_bytes, stream)

    def indexer_topk(self, stream=None):
        """Scores and selection in one call (the selection fused into the scoring): the same scores and idx
        as indexer() followed by topk()."""
        wl = self.wl
        B.dsa_indexer_topk(self.qI, self.idx_dt, self.w, self.kI_pool, self.idx_dt, self.kS_pool, wl.Hi, wl.Di,
                           self.batch, wl.topk, self.scores, self.ld, self.idx, self.ws, self.ws_bytes, stream)

    def topk(self, stream=None, scores=None):
        B.dsa_topk(self.scores if scores is None else scores, self.ld, self.batch, self.wl.topk, self.idx, self.ws,
                   self.ws_bytes, stream)

    def attention(self, stream=None, idx=None, k=None):
        wl = self.wl
        fn = B.dsa_sparse_attn_decode if self.decode else B.dsa_sparse_attn_prefill
        fn(self.q, self.dt, self.kv_pool, self.v_pool, wl.H, wl.Dqk, wl.Dv, wl.softmax_scale,
           self.idx if idx is None else idx, wl.topk if k is None else k, self.batch, self.out, self.lse, self.ws,
           self.ws_bytes, stream)

    def reuse_select(self, prev_idx, prev_lens, max_new, stream=None):
        """Decode index reuse: candidates = an earlier selection prev_idx [T, k] (made at prev_lens [T]
        tokens) plus the positions added since (at most max_new per row), scored at those positions only,
        the k best kept.  Returns the index array [T, k] for attention(); the candidate list and scores stay
        in cand and cand_scores."""
        wl, dv, T, k = self.wl, self.device, self.wl.total_q, self.wl.topk
        m = (k + max_new + 3) // 4 * 4                      # slots past k + max_new stay -1
        if getattr(self, "_reuse_m", None) != m:
            self.cand = torch.empty((T, m), dtype=torch.int32, device=dv)
            self.cand_scores = torch.empty((T, m), dtype=torch.float32, device=dv)
            self._cand_bt = torch.zeros((T, (m + 63) // 64), dtype=torch.int32, device=dv)
            self._cand_len = torch.full((T,), m, dtype=torch.int32, device=dv)
            self._cand_cu = torch.arange(T + 1, dtype=torch.int32, device=dv)
            self.cand_batch = B.make_batch(self._cand_bt, self._cand_len, self._cand_cu, num_blocks=1,
                                           page_size=wl.page_size, total_q=T, max_q_per_seq=1, max_seq_len=m)
            self._cand_ws_bytes = B.dsa_workspace_size(B.DSA_OP_TOPK, self.cand_batch, k)
            self._cand_ws = torch.zeros(self._cand_ws_bytes, dtype=torch.uint8, device=dv)
            self._cand_sel = torch.empty((T, k), dtype=torch.int32, device=dv)
            self.idx_reuse = torch.empty((T, k), dtype=torch.int32, device=dv)
            self._reuse_m = m
        B.dsa_reuse_candidates(prev_idx, k, prev_lens, m - k, self.batch, self.cand, self.ws, self.ws_bytes, stream)
        B.dsa_indexer_scores_at(self.qI, self.idx_dt, self.w, self.kI_pool, self.idx_dt, self.kS_pool, wl.Hi, wl.Di,
                                self.batch, self.cand, m, self.cand_scores, self.ws, self.ws_bytes, stream)
        B.dsa_topk(self.cand_scores, m, self.cand_batch, k, self._cand_sel, self._cand_ws, self._cand_ws_bytes, stream)
        B.dsa_gather_positions(self._cand_sel, k, self.cand, m, T, self.idx_reuse, stream)
        return self.idx_reuse

    def block_select(self, kb, stream=None):
        """Block-granular selection from the current scores: page scores, the kb best pages per row (the
        usual top-k on a batch of the rows' page lists) and their token positions.  Returns the index
        array [total_q, kb * page_size] for attention(idx=..., k=kb * page_size); the page scores, page
        counts and kept pages stay in blk_scores, blk_lens and blk_idx."""
        wl, dv, T, P = self.wl, self.device, self.wl.total_q, self.wl.page_size
        max_pages = (wl.max_seq_len + P - 1) // P
        if getattr(self, "_blk_kb", None) != kb:
            self.ld_blk = (max_pages + 3) // 4 * 4
            self.blk_scores = torch.empty((T, self.ld_blk), dtype=torch.float32, device=dv)
            self.blk_lens = torch.empty((T,), dtype=torch.int32, device=dv)
            self._blk_bt = torch.zeros((T, (max_pages + P - 1) // P), dtype=torch.int32, device=dv)
            self._blk_cu = torch.arange(T + 1, dtype=torch.int32, device=dv)
            self.blk_batch = B.make_batch(self._blk_bt, self.blk_lens, self._blk_cu, num_blocks=1, page_size=P,
                                          total_q=T, max_q_per_seq=1 if T else 0, max_seq_len=max(max_pages, 1))
            self._blk_ws_bytes = B.dsa_workspace_size(B.DSA_OP_TOPK, self.blk_batch, kb)
            self._blk_ws = torch.zeros(self._blk_ws_bytes, dtype=torch.uint8, device=dv)
            self.blk_idx = torch.empty((T, kb), dtype=torch.int32, device=dv)
            self.idx_blk = torch.empty((T, kb * P), dtype=torch.int32, device=dv)
            op_attn = B.DSA_OP_ATTN_DECODE if self.decode else B.DSA_OP_ATTN_PREFILL
            need = B.dsa_workspace_size(op_attn, self.batch, kb * P, wl.H, wl.Dv)
            if need > self.ws_bytes:
                self.ws_bytes = need
                self.ws = torch.zeros(need, dtype=torch.uint8, device=dv)
            self._blk_kb = kb
        B.dsa_block_scores(self.scores, self.ld, self.batch, self.blk_scores, self.ld_blk, self.blk_lens, stream)
        B.dsa_topk(self.blk_scores, self.ld_blk, self.blk_batch, kb, self.blk_idx, self._blk_ws, self._blk_ws_bytes,
                   stream)
        B.dsa_expand_blocks(self.blk_idx, kb, self.batch, self.idx_blk, stream)
        return self.idx_blk

    # Batches where the fused scores + selection call is the faster form of the first two steps (measured on
    # one B200): many rows longer than one CTA's shared-memory slice of the plain top-k (the mixed batch's
    # 57K-65K-candidate chunk rows: 22.3 ms against 26.4 ms).  For decode batches, prefill prompts of up to a few
    # ten thousand tokens and a single million-token row the two separate calls are faster.
    FUSED_MIN_ROWS = 1024
    FUSED_MIN_LEN = 49153
    FUSED_LONG_ROW = 262144

    def prefers_fused(self):
        # measured on one B200: the fused call wins for big batches of long rows (the mixed batch: 16.7 ms
        # against 19.9) and for very long rows (one 1M-token decode row: 74.6 us against 83.9); the two calls
        # win for decode batches of 4K-32K tokens (38.3 us against 46.2) and the 16k prefill (2.56 ms against 3.48)
        return (self.wl.total_q >= self.FUSED_MIN_ROWS and self.wl.max_seq_len >= self.FUSED_MIN_LEN) or \
            self.wl.max_seq_len >= self.FUSED_LONG_ROW

    def run(self, stream=None, fused=None):
        """One pass of the path: scores, selection, attention.  fused=True takes scores and selection in one
        call (dsa_indexer_topk), False the two calls; None picks by prefers_fused()."""
        if fused is None:
            fused = self.prefers_fused()
        if fused:
            self.indexer_topk(stream)
        else:
            self.indexer(stream)
            self.topk(stream)
        self.attention(stream)

    def check_status(self, stream=None):
        B.dsa_read_device_status(self.ws, stream)
