"""GPU parity of the fused scores + selection call (dsa_indexer_topk) against the CPU oracle.

The call must give exactly what dsa_indexer_scores followed by dsa_topk give: the same score bits and the
same index set (positions ascending, -1 padded).  On integer-grid inputs every score is exact in fp32, so
the selection must equal the oracle's bit for bit; on random inputs it must equal dsa_topk's selection
over the same fp32 scores (the selection itself is exact).  Shapes: small batches (every row, ragged page
tails, rows shorter and longer than k), the decode batch, the 1M-token planted row and the mixed batch at
full size (sampled rows), plus a row of all-equal scores that forces the selection's refinement passes.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import check_scores, sample_rows
from sparse_attention_long_dsa_b200 import binding as B
from sparse_attention_long_dsa_b200 import workloads as W
from sparse_attention_long_dsa_b200.pipeline import DeviceBatch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    torch.cuda.init()


def _fused(wl):
    db = DeviceBatch(wl)
    db.indexer_topk()
    torch.cuda.synchronize()
    db.check_status()
    return db


def _separate_idx(db):
    """dsa_topk over the fused call's own scores (same fp32 values)."""
    idx = torch.full_like(db.idx, -7)
    B.dsa_topk(db.scores, db.ld, db.batch, db.wl.topk, idx, db.ws, db.ws_bytes)
    torch.cuda.synchronize()
    return idx


def _check_rows_vs_oracle(wl, db, rows):
    ref = oracle.run_rows(wl, rows, want_attention=False)
    gi = db.idx.cpu().numpy()
    for r in rows:
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, r)
        sc = db.scores[r, : pos + 1].cpu().numpy()
        check_scores(wl, r, sc, ref[r]["scores"])
        assert np.array_equal(gi[r], ref[r]["idx"]), f"row {r}: fused top-k differs from the oracle"


@pytest.mark.parametrize("topk", [1, 100, 2048])
def test_fused_small_batches_every_row_grid(topk):
    seq_lens = [70, 300, 2100, 2600, 5000, 129]
    q_lens = [70, 37, 300, 5, 1, 1]
    wl = W.make_workload("fused_small", kind="mla", seed=201 + topk, seq_lens=seq_lens, q_lens=q_lens, topk=topk,
                         grid=True)
    db = _fused(wl)
    _check_rows_vs_oracle(wl, db, list(range(wl.total_q)))


def test_fused_matches_separate_calls_random():
    seq_lens = [4097, 12000, 300, 33000, 2049]
    wl = W.make_workload("fused_rand", kind="mla", seed=205, seq_lens=seq_lens, q_lens=[1, 3, 1, 2, 1], topk=2048)
    db = _fused(wl)
    sc_fused = db.scores.clone()
    sep = DeviceBatch(wl)
    sep.indexer()
    torch.cuda.synchronize()
    for r in range(wl.total_q):
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, r)
        assert torch.equal(sc_fused[r, : pos + 1], sep.scores[r, : pos + 1]), f"row {r}: scores differ"
    assert torch.equal(db.idx, _separate_idx(db))


def test_fused_f32_tiny_every_row():
    wl = W.tiny_f32(grid=True)
    db = _fused(wl)
    _check_rows_vs_oracle(wl, db, list(range(wl.total_q)))


def test_fused_all_equal_scores_take_the_lowest_positions():
    """Every score 0 (zero weights): the whole row falls in one bin, past the survivor capacity, so the
    selection resolves every key bit by counting passes and keeps the lowest k positions."""
    wl = W.make_workload("fused_ties", kind="mla", seed=206, seq_lens=[30000, 70000, 9000], q_lens=[1, 1, 2],
                         topk=2048)
    wl.w = np.zeros_like(wl.w)
    db = _fused(wl)
    gi = db.idx.cpu().numpy()
    for r in range(wl.total_q):
        assert np.array_equal(gi[r], np.arange(2048)), f"row {r}"


def test_fused_decode_batch_full_size():
    wl = W.decode_batch(grid=True)
    db = _fused(wl)
    _check_rows_vs_oracle(wl, db, sample_rows(wl, extra=6))
    assert torch.equal(db.idx, _separate_idx(db))


def test_fused_decode_batch_random_matches_separate_calls():
    wl = W.decode_batch()
    db = _fused(wl)
    assert torch.equal(db.idx, _separate_idx(db))


def test_fused_1m_planted_selects_the_planted_set():
    wl = W.decode_1m_planted()
    db = _fused(wl)
    got = db.idx[0].cpu().numpy()
    assert np.array_equal(got, np.sort(wl.planted)), "fused selection differs from the planted set"
    assert torch.equal(db.idx, _separate_idx(db))


def test_fused_mixed_batch_full_size_grid():
    wl = W.mixed_batch(grid=True)
    db = _fused(wl)
    rows = sample_rows(wl, extra=4)
    _check_rows_vs_oracle(wl, db, rows)
    # every row against dsa_topk over the same scores
    assert torch.equal(db.idx, _separate_idx(db))


def test_fused_long_rows_gather_matches_separate_calls():
    """Rows of 256K candidates or more in a batch of at most 16 rows: the survivors are collected over every SM
    (one range per CTA) before one CTA per row finishes the selection."""
    wl = W.make_workload("fused_long", kind="mla", seed=208, seq_lens=[300000, 270000, 5000], q_lens=[1, 1, 1],
                         topk=2048, attention=False)
    db = _fused(wl)
    assert torch.equal(db.idx, _separate_idx(db))


def test_fused_long_row_with_clustered_top_keys():
    """A 300,000-token row whose 2048 best keys sit at its start: a gathering range keeps at most a fixed number
    of survivors, so the range holding them overflows and the selection streams the row itself."""
    wl = W.make_workload("fused_cluster", kind="mla", seed=207, seq_lens=[300000], q_lens=[1], topk=2048,
                         planted_k=2048, attention=False)
    n, P = 300000, wl.kI_pool.shape[1]
    pos = np.arange(n)
    phys = wl.block_table[0, pos // P].astype(np.int64) * P + pos % P
    order = np.concatenate([wl.planted, np.setdiff1d(pos, wl.planted)])     # planted keys first
    kflat = wl.kI_pool.reshape(-1, wl.kI_pool.shape[-1])
    kflat[phys] = kflat[phys][order]
    sflat = wl.kS_pool.reshape(-1)
    sflat[phys] = sflat[phys][order]
    db = _fused(wl)
    assert np.array_equal(db.idx[0].cpu().numpy(), np.arange(2048))
    assert torch.equal(db.idx, _separate_idx(db))


def test_fused_long_row_all_equal_scores():
    """Every score 0 on a 300,000-token row: the threshold bin holds the whole row, past the survivor capacity,
    so the gathered survivors are not used and the selection resolves every key bit by counting passes."""
    wl = W.make_workload("fused_long_ties", kind="mla", seed=209, seq_lens=[300000], q_lens=[1], topk=2048,
                         attention=False)
    wl.w = np.zeros_like(wl.w)
    db = _fused(wl)
    assert np.array_equal(db.idx[0].cpu().numpy(), np.arange(2048))
