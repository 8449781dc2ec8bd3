"""Thin ctypes binding of libdsa (include/dsa.h).

Argument marshalling only: every step runs in the library's CUDA kernels.  The functions
keep the C names and take torch tensors (device memory) or raw integer pointers; streams
default to torch's current stream.  If the shared library is missing the first call raises
-- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, DSA_ERR_DEVICE_CHECK, \
    DSA_ERR_TIMEOUT = range(7)
DSA_F32, DSA_BF16, DSA_FP8_E4M3 = 0, 1, 2
DSA_OP_INDEXER, DSA_OP_TOPK, DSA_OP_ATTN_PREFILL, DSA_OP_ATTN_DECODE, DSA_OP_CACHE_APPEND, DSA_OP_INDEXER_TOPK = \
    0, 1, 2, 3, 4, 5

EXPORTS = ("dsa_workspace_size", "dsa_indexer_scores", "dsa_topk", "dsa_sparse_attn_prefill",
           "dsa_sparse_attn_decode", "dsa_read_device_status", "dsa_status_string", "dsa_last_error",
           "dsa_version", "dsa_launch_count", "dsa_topk_noalloc", "dsa_cache_append", "dsa_selftest_wait_timeout",
           "dsa_cp_candidates", "dsa_cp_rows", "dsa_cp_select_local", "dsa_cp_merge", "dsa_block_scores",
           "dsa_expand_blocks", "dsa_reuse_candidates", "dsa_indexer_scores_at", "dsa_gather_positions",
           "dsa_indexer_scores_append", "dsa_indexer_topk")


class dsa_batch_t(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("block_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("cu_q", ctypes.c_void_p),
        ("total_q", ctypes.c_int32),
        ("max_q_per_seq", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32),
    ]


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Load libdsa and declare its signatures (once)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libdsa.so not found at {path}; build it with "
                           f"`python -m sparse_attention_long_dsa_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    B = ctypes.POINTER(dsa_batch_t)
    sig = {
        "dsa_workspace_size": [I32, B, I32, I32, I32, ctypes.POINTER(SZ)],
        "dsa_indexer_scores": [P, I32, P, P, I32, P, I32, I32, B, P, I64, P, SZ, P],
        "dsa_topk": [P, I64, B, I32, P, P, SZ, P],
        "dsa_indexer_topk": [P, I32, P, P, I32, P, I32, I32, B, I32, P, I64, P, P, SZ, P],
        "dsa_topk_noalloc": [P, I64, B, I32, P, P],
        "dsa_sparse_attn_prefill": [P, I32, P, P, I32, I32, I32, F, P, I32, B, P, P, P, SZ, P],
        "dsa_sparse_attn_decode": [P, I32, P, P, I32, I32, I32, F, P, I32, B, P, P, P, SZ, P],
        "dsa_cache_append": [P, I32, P, I32, I32, I32, B, P, P, P, P, SZ, P],
        "dsa_selftest_wait_timeout": [ctypes.c_uint64, P, SZ, P],
        "dsa_block_scores": [P, I64, B, P, I64, P, P],
        "dsa_reuse_candidates": [P, I32, P, I32, B, P, P, SZ, P],
        "dsa_indexer_scores_append": [P, I32, P, I32, P, P, I32, P, P, I32, P, I32, I32, B, P, I64, P, SZ, P],
        "dsa_indexer_scores_at": [P, I32, P, P, I32, P, I32, I32, B, P, I32, P, P, SZ, P],
        "dsa_gather_positions": [P, I32, P, I32, I32, P, P],
        "dsa_expand_blocks": [P, I32, B, P, P],
        "dsa_cp_candidates": [P, I64, P, I32, I32, P, P, P, P],
        "dsa_cp_rows": [P, I32, I32, I32, P, I64, P],
        "dsa_cp_select_local": [P, P, I32, I32, I32, P, P, P, P],
        "dsa_cp_merge": [P, I32, P, I32, I32, I32, I32, P, P, P],
        "dsa_read_device_status": [P, P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    for name in ("dsa_status_string",):
        getattr(lib, name).argtypes = [ctypes.c_int]
        getattr(lib, name).restype = ctypes.c_char_p
    lib.dsa_launch_count.argtypes = []
    lib.dsa_launch_count.restype = ctypes.c_uint64
    for name in ("dsa_last_error", "dsa_version"):
        getattr(lib, name).argtypes = []
        getattr(lib, name).restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != DSA_OK:
        lib = load()
        raise DSAError(status, where, f"{lib.dsa_status_string(status).decode()}: {lib.dsa_last_error().decode()}")


def _ptr(t) -> Optional[int]:
    """Address of a tensor's data, or an integer address passed through.  A tensor must be a dense CUDA tensor:
    the kernels read and write its bytes in the layout include/dsa.h gives, so a host tensor would hand them a
    host address and a strided view would be read as if it were dense."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise DSAError(DSA_ERR_INVALID_ARG, "argument",
                       f"a {tuple(t.shape)} tensor on {t.device}; the library takes device memory")
    if not t.is_contiguous():
        raise DSAError(DSA_ERR_INVALID_ARG, "argument",
                       f"a strided {tuple(t.shape)} tensor (strides {tuple(t.stride())}); the library takes dense arrays")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_batch(block_table, seq_lens, cu_q, *, num_blocks: int, page_size: int, total_q: int,
               max_q_per_seq: int, max_seq_len: int) -> dsa_batch_t:
    """dsa_batch_t from device int32 tensors (block_table [B, max_blocks], seq_lens [B], cu_q [B+1])."""
    return dsa_batch_t(num_seqs=int(seq_lens.shape[0]), page_size=page_size, num_blocks=num_blocks,
                       max_blocks_per_seq=int(block_table.shape[1]), block_table=_ptr(block_table),
                       seq_lens=_ptr(seq_lens), cu_q=_ptr(cu_q), total_q=total_q, max_q_per_seq=max_q_per_seq,
                       max_seq_len=max_seq_len)


def dsa_workspace_size(op: int, batch: dsa_batch_t, k: int = 0, H: int = 0, Dv: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(load().dsa_workspace_size(op, ctypes.byref(batch), k, H, Dv, ctypes.byref(out)), "dsa_workspace_size")
    return out.value


def dsa_indexer_scores(q_idx, q_dt: int, w, k_idx_pool, k_dt: int, k_scale_pool, Hi: int, Di: int,
                       batch: dsa_batch_t, scores, ld_scores: int, ws, ws_bytes: int, stream=None):
    _check(load().dsa_indexer_scores(_ptr(q_idx), q_dt, _ptr(w), _ptr(k_idx_pool), k_dt, _ptr(k_scale_pool), Hi, Di,
                                     ctypes.byref(batch), _ptr(scores), ld_scores, _ptr(ws), ws_bytes,
                                     _stream(stream)), "dsa_indexer_scores")


def dsa_topk(scores, ld_scores: int, batch: dsa_batch_t, k: int, idx, ws, ws_bytes: int, stream=None):
    _check(load().dsa_topk(_ptr(scores), ld_scores, ctypes.byref(batch), k, _ptr(idx), _ptr(ws), ws_bytes,
                           _stream(stream)), "dsa_topk")


def dsa_indexer_topk(q_idx, q_dt: int, w, k_idx_pool, k_dt: int, k_scale_pool, Hi: int, Di: int,
                     batch: dsa_batch_t, k: int, scores, ld_scores: int, idx, ws, ws_bytes: int, stream=None):
    """Indexer scores and the top-k selection in one call (the selection fused into the scoring)."""
    _check(load().dsa_indexer_topk(_ptr(q_idx), q_dt, _ptr(w), _ptr(k_idx_pool), k_dt, _ptr(k_scale_pool), Hi, Di,
                                   ctypes.byref(batch), k, _ptr(scores), ld_scores, _ptr(idx), _ptr(ws), ws_bytes,
                                   _stream(stream)), "dsa_indexer_topk")


def dsa_topk_noalloc(scores, ld_scores: int, batch: dsa_batch_t, k: int, idx, stream=None):
    """Top-k with the library's built-in scratch instead of a caller workspace (no device allocation)."""
    _check(load().dsa_topk_noalloc(_ptr(scores), ld_scores, ctypes.byref(batch), k, _ptr(idx), _stream(stream)),
           "dsa_topk_noalloc")


def dsa_sparse_attn_prefill(q, dt: int, kv_pool, v_pool, H: int, Dqk: int, Dv: int, softmax_scale: float, idx,
                            k: int, batch: dsa_batch_t, out, lse, ws, ws_bytes: int, stream=None):
    _check(load().dsa_sparse_attn_prefill(_ptr(q), dt, _ptr(kv_pool), _ptr(v_pool), H, Dqk, Dv, softmax_scale,
                                          _ptr(idx), k, ctypes.byref(batch), _ptr(out), _ptr(lse), _ptr(ws),
                                          ws_bytes, _stream(stream)), "dsa_sparse_attn_prefill")


def dsa_sparse_attn_decode(q, dt: int, kv_pool, v_pool, H: int, Dqk: int, Dv: int, softmax_scale: float, idx,
                           k: int, batch: dsa_batch_t, out, lse, ws, ws_bytes: int, stream=None):
    _check(load().dsa_sparse_attn_decode(_ptr(q), dt, _ptr(kv_pool), _ptr(v_pool), H, Dqk, Dv, softmax_scale,
                                         _ptr(idx), k, ctypes.byref(batch), _ptr(out), _ptr(lse), _ptr(ws),
                                         ws_bytes, _stream(stream)), "dsa_sparse_attn_decode")


def dsa_cache_append(kv_new, kv_dt: int, k_new, k_dt: int, Dqk: int, Di: int, batch: dsa_batch_t, kv_pool, k_idx_pool,
                     k_scale_pool, ws, ws_bytes: int, stream=None):
    _check(load().dsa_cache_append(_ptr(kv_new), kv_dt, _ptr(k_new), k_dt, Dqk, Di, ctypes.byref(batch), _ptr(kv_pool),
                                   _ptr(k_idx_pool), _ptr(k_scale_pool), _ptr(ws), ws_bytes, _stream(stream)),
           "dsa_cache_append")


def dsa_selftest_wait_timeout(budget_cycles: int, ws, ws_bytes: int, stream=None):
    _check(load().dsa_selftest_wait_timeout(budget_cycles, _ptr(ws), ws_bytes, _stream(stream)),
           "dsa_selftest_wait_timeout")


def dsa_indexer_scores_append(kv_new, kv_dt: int, k_new, k_new_dt: int, kv_pool, q_idx, q_dt: int, w, k_idx_pool,
                              k_dt: int, k_scale_pool, Hi: int, Di: int, batch: dsa_batch_t, scores, ld_scores: int,
                              ws, ws_bytes: int, stream=None):
    _check(load().dsa_indexer_scores_append(_ptr(kv_new), kv_dt, _ptr(k_new), k_new_dt, _ptr(kv_pool), _ptr(q_idx),
                                            q_dt, _ptr(w), _ptr(k_idx_pool), k_dt, _ptr(k_scale_pool), Hi, Di,
                                            ctypes.byref(batch), _ptr(scores), ld_scores, _ptr(ws), ws_bytes,
                                            _stream(stream)), "dsa_indexer_scores_append")


def dsa_reuse_candidates(prev_idx, k: int, prev_lens, max_new: int, batch: dsa_batch_t, cand, ws, ws_bytes: int,
                         stream=None):
    _check(load().dsa_reuse_candidates(_ptr(prev_idx), k, _ptr(prev_lens), max_new, ctypes.byref(batch), _ptr(cand),
                                       _ptr(ws), ws_bytes, _stream(stream)), "dsa_reuse_candidates")


def dsa_indexer_scores_at(q_idx, q_dt: int, w, k_idx_pool, k_dt: int, k_scale_pool, Hi: int, Di: int,
                          batch: dsa_batch_t, cand, m: int, cand_scores, ws, ws_bytes: int, stream=None):
    _check(load().dsa_indexer_scores_at(_ptr(q_idx), q_dt, _ptr(w), _ptr(k_idx_pool), k_dt, _ptr(k_scale_pool), Hi, Di,
                                        ctypes.byref(batch), _ptr(cand), m, _ptr(cand_scores), _ptr(ws), ws_bytes,
                                        _stream(stream)), "dsa_indexer_scores_at")


def dsa_gather_positions(sel, k: int, cand, m: int, T: int, idx, stream=None):
    _check(load().dsa_gather_positions(_ptr(sel), k, _ptr(cand), m, T, _ptr(idx), _stream(stream)),
           "dsa_gather_positions")


def dsa_block_scores(scores, ld_scores: int, batch: dsa_batch_t, blk_scores, ld_blk: int, blk_lens, stream=None):
    _check(load().dsa_block_scores(_ptr(scores), ld_scores, ctypes.byref(batch), _ptr(blk_scores), ld_blk,
                                   _ptr(blk_lens), _stream(stream)), "dsa_block_scores")


def dsa_expand_blocks(blk_idx, kb: int, batch: dsa_batch_t, idx, stream=None):
    _check(load().dsa_expand_blocks(_ptr(blk_idx), kb, ctypes.byref(batch), _ptr(idx), _stream(stream)),
           "dsa_expand_blocks")


def dsa_cp_candidates(scores, ld_scores: int, idx, T: int, k: int, offsets, cand_score, cand_gidx, stream=None):
    _check(load().dsa_cp_candidates(_ptr(scores), ld_scores, _ptr(idx), T, k, _ptr(offsets), _ptr(cand_score),
                                    _ptr(cand_gidx), _stream(stream)), "dsa_cp_candidates")


def dsa_cp_rows(g_score, G: int, T: int, k: int, rows, ld_rows: int, stream=None):
    _check(load().dsa_cp_rows(_ptr(g_score), G, T, k, _ptr(rows), ld_rows, _stream(stream)), "dsa_cp_rows")


def dsa_cp_select_local(sel, g_gidx, G: int, T: int, k: int, lo, hi, local_idx, stream=None):
    _check(load().dsa_cp_select_local(_ptr(sel), _ptr(g_gidx), G, T, k, _ptr(lo), _ptr(hi), _ptr(local_idx),
                                      _stream(stream)), "dsa_cp_select_local")


def dsa_cp_merge(part_out, dt: int, part_lse, G: int, T: int, H: int, Dv: int, out, lse, stream=None):
    _check(load().dsa_cp_merge(_ptr(part_out), dt, _ptr(part_lse), G, T, H, Dv, _ptr(out), _ptr(lse),
                               _stream(stream)), "dsa_cp_merge")


def dsa_read_device_status(ws, stream=None):
    _check(load().dsa_read_device_status(_ptr(ws), _stream(stream)), "dsa_read_device_status")


def dsa_version() -> str:
    return load().dsa_version().decode()


def dsa_launch_count() -> int:
    return int(load().dsa_launch_count())
