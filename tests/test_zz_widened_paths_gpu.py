"""GPU parity of the paths beyond the three core calls, run after the core parity tests: batches with
sequences that own no query rows and empty batches, the cache append, the bounded-wait self-test,
context-parallel decode (ranks emulated one after another on this GPU) and block-granular selection, each
against the CPU oracle through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from parity import check_attention, compare_rows
from sparse_attention_long_dsa_b200 import binding as B
from sparse_attention_long_dsa_b200 import workloads as W
from sparse_attention_long_dsa_b200.pipeline import DeviceBatch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    torch.cuda.init()


def _run(wl, decode=None):
    db = DeviceBatch(wl, decode=decode)
    db.run()
    torch.cuda.synchronize()
    db.check_status()
    return db


# --------------------------------------------------------------------------------------- ragged batches
@pytest.mark.parametrize("grid", [True, False])
def test_sequences_without_query_rows(grid):
    """Sequences that own no query rows, first, between others and last, beside a whole 64-token prompt,
    a one-token sequence and rows past the 2048-token top-k: every row against the oracle."""
    wl = W.make_workload("ragged_empty", kind="mla", seed=107, seq_lens=[100, 64, 2100, 1, 700, 130, 3000, 90],
                         q_lens=[0, 64, 0, 1, 3, 0, 2, 0], topk=2048, grid=grid)
    db = _run(wl)
    compare_rows(wl, db, list(range(wl.total_q)))


def test_empty_batch_launches_nothing():
    wl = W.make_workload("empty", kind="mla", seed=108, seq_lens=[50, 300], q_lens=[0, 0], topk=2048)
    db = DeviceBatch(wl)
    n0 = B.dsa_launch_count()
    db.run()
    torch.cuda.synchronize()
    assert B.dsa_launch_count() == n0
    assert db.out.numel() == 0 and db.idx.numel() == 0


# --------------------------------------------------------------------------------------- cache append
def _e4m3_ties_row():
    """448 (so the scale is 1) and every value halfway between two adjacent E4M3 magnitudes (126 of
    them, all exact in bf16), padded with 1.0 to 128 entries."""
    mags = oracle.E4M3[:0x7F]
    mid = (mags[:-1] + mags[1:]) / 2
    return np.concatenate([[448.0], mid, [1.0]]).astype(np.float32)


def _append_inputs(T, rng, k_bf16):
    """(kv_new as int16 bf16 bits, keys as passed to the call, their format) for T new tokens."""
    kv_new = W.bf16_encode(rng.standard_normal((T, 576)).astype(np.float32)).view(np.int16)
    k = (rng.standard_normal((T, 128)) * 10.0 ** rng.uniform(-3, 3, (T, 1))).astype(np.float32)
    k[0] = 0.0                                                      # all-zero key: scale 1
    k[1] = 0.0
    k[1, 17] = -3.0                                                 # one non-zero entry
    k[2] = _e4m3_ties_row()                                         # scale 1: the ties themselves round
    k[3] = -k[2]
    if k_bf16:
        kb = W.bf16_encode(k)
        assert np.array_equal(oracle.bf16_decode(kb[2]), k[2])     # the ties survive the bf16 encoding
        return kv_new, kb.view(np.int16), "bf16"
    return kv_new, k, "f32"


def _dev_copy(a, dev):
    a = np.ascontiguousarray(a)
    return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a.copy()).to(dev)


@pytest.mark.parametrize("k_bf16", [False, True])
def test_cache_append_matches_oracle(k_bf16):
    """New tokens written into shuffled pages: a whole 70-token prompt, a 3-token chunk, single decode
    tokens; latent rows and scales bit-exact, FP8 codes bit-exact (a zero code's sign aside), every
    other token of the pools untouched."""
    wl = W.make_workload("append", kind="mla", seed=109, seq_lens=[70, 300, 2100, 1, 65], q_lens=[70, 3, 1, 1, 2],
                         topk=64, spare_blocks=3)
    dev = torch.device("cuda")
    rng = np.random.default_rng(110 + k_bf16)
    kv_new, k_in, fmt = _append_inputs(wl.total_q, rng, k_bf16)
    bt, sl, cu = (_dev_copy(a.astype(np.int32), dev) for a in (wl.block_table, wl.seq_lens, wl.cu_q))
    batch = B.make_batch(bt, sl, cu, num_blocks=wl.num_blocks, page_size=64, total_q=wl.total_q,
                         max_q_per_seq=wl.max_q_per_seq, max_seq_len=wl.max_seq_len)
    kv_pool, kI_pool, kS_pool = _dev_copy(wl.kv_pool, dev), _dev_copy(wl.kI_pool, dev), _dev_copy(wl.kS_pool, dev)
    ws = torch.zeros(B.dsa_workspace_size(B.DSA_OP_CACHE_APPEND, batch), dtype=torch.uint8, device=dev)
    n0 = B.dsa_launch_count()
    B.dsa_cache_append(_dev_copy(kv_new, dev), B.DSA_BF16, _dev_copy(k_in, dev), B.DSA_BF16 if k_bf16 else B.DSA_F32,
                       576, 128, batch, kv_pool, kI_pool, kS_pool, ws, ws.numel())
    torch.cuda.synchronize()
    B.dsa_read_device_status(ws)
    assert B.dsa_launch_count() == n0 + 1
    k_oracle = k_in.view(np.uint16) if k_bf16 else k_in
    ekv, ekI, ekS = oracle.cache_append(wl, kv_new.view(np.uint16), k_oracle, fmt)
    assert np.array_equal(kv_pool.cpu().numpy().view(np.uint16), ekv)
    assert np.array_equal(kS_pool.cpu().numpy().view(np.uint32), ekS.view(np.uint32))
    zero = lambda c: np.where((c & 0x7F) == 0, 0, c)
    assert np.array_equal(zero(kI_pool.cpu().numpy()), zero(ekI))


def test_cache_append_reports_bad_block_ids():
    """A block id outside the pool: those tokens are skipped and the status word says so; the rest of
    the batch is written."""
    wl = W.make_workload("append_bad", kind="mla", seed=111, seq_lens=[130, 64], q_lens=[2, 1], topk=64)
    bt_host = wl.block_table.astype(np.int32).copy()
    bt_host[0, 2] = wl.num_blocks + 5                               # positions 128, 129 of sequence 0
    dev = torch.device("cuda")
    bt, sl, cu = (_dev_copy(a.astype(np.int32), dev) for a in (bt_host, wl.seq_lens, wl.cu_q))
    batch = B.make_batch(bt, sl, cu, num_blocks=wl.num_blocks, page_size=64, total_q=wl.total_q,
                         max_q_per_seq=wl.max_q_per_seq, max_seq_len=wl.max_seq_len)
    kv_pool, kI_pool, kS_pool = _dev_copy(wl.kv_pool, dev), _dev_copy(wl.kI_pool, dev), _dev_copy(wl.kS_pool, dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    kv_new, k_in, _ = _append_inputs(wl.total_q + 4, np.random.default_rng(112), False)
    B.dsa_cache_append(_dev_copy(kv_new[: wl.total_q], dev), B.DSA_BF16, _dev_copy(k_in[4:], dev), B.DSA_F32, 576, 128,
                       batch, kv_pool, kI_pool, kS_pool, ws, 256)
    with pytest.raises(B.DSAError) as e:
        B.dsa_read_device_status(ws)
    assert e.value.status == B.DSA_ERR_DEVICE_CHECK
    changed = np.argwhere((kI_pool.cpu().numpy() != wl.kI_pool).any(axis=2)).tolist()
    blk, slot = oracle.token_slots(bt_host[1], np.array([63]), 64)
    assert changed == [[int(blk[0]), int(slot[0])]]                 # only sequence 1's token was written


# --------------------------------------------------------------------------------------- bounded waits
def test_bounded_wait_gives_up_and_reports_timeout():
    """A device wait on a barrier that nothing completes (the wait routine of the tensor-core kernels, with a
    budget of 2e7 SM cycles) gives up and raises the timeout bit; reading the status clears it, and the
    context still runs a batch that matches the oracle."""
    import time
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    B.dsa_selftest_wait_timeout(20_000_000, ws, 256)
    with pytest.raises(B.DSAError) as e:
        B.dsa_read_device_status(ws)
    assert e.value.status == B.DSA_ERR_TIMEOUT
    assert time.time() - t0 < 60
    B.dsa_read_device_status(ws)                                    # cleared by the read
    wl = W.make_workload("after_timeout", kind="mla", seed=113, seq_lens=[300, 2100], q_lens=[1, 1], topk=2048,
                         grid=True)
    db = _run(wl)
    compare_rows(wl, db, list(range(wl.total_q)))


# --------------------------------------------------------------------------------------- context parallel
def _cp_run(wl, world):
    from sparse_attention_long_dsa_b200 import context_parallel as CP
    dev = torch.device("cuda")
    inputs = DeviceBatch.upload_inputs(wl, dev)
    ranks = [CP.CPDecodeRank(wl, r, world, device=dev, inputs=inputs) for r in range(world)]
    out = torch.empty((wl.total_q, wl.H, wl.Dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.total_q, wl.H), dtype=torch.float32, device=dev)
    CP.cp_decode_emulated(ranks, out, lse)
    torch.cuda.synchronize()
    for r in ranks:
        r.db.check_status()
    sel = [np.sort(np.concatenate([r.selected_positions()[t] for r in ranks])) for t in range(wl.total_q)]
    return sel, out.float().cpu().numpy(), lse.cpu().numpy()


def _cp_check(wl, rows, sel, out, lse):
    """Global selection exact; attention against the oracle on that set.  Each rank's partial output is
    rounded to bf16 before the merge, so the output carries two bf16 roundings (2^-9 relative each) on
    top of the single-GPU path's error: max-abs 3e-2, mean-rel 1e-2; lse 1e-3."""
    ref = oracle.run_rows(wl, rows)
    for t in rows:
        exp = ref[t]["idx"][ref[t]["idx"] >= 0]
        assert np.array_equal(sel[t], exp), f"row {t}: context-parallel selection differs from the oracle"
        o = ref[t]["out"]
        assert np.abs(out[t] - o).max() <= 3e-2, f"row {t}: max-abs {np.abs(out[t] - o).max():.3e}"
        assert np.abs(out[t] - o).sum() / np.abs(o).sum() <= 1e-2
        assert np.abs(lse[t] - ref[t]["lse"]).max() <= 1e-3


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_decode_emulated_ranks(world):
    """A decode batch spread over `world` ranks run one after another on this GPU (no rank waits on
    another; the all-gathers are stacks): the merged result equals the single-GPU selection and attention."""
    wl = W.make_workload("cp_gpu", kind="mla", seed=114, seq_lens=[5000, 9000, 2600], q_lens=[1, 1, 1], topk=2048,
                         grid=True)
    sel, out, lse = _cp_run(wl, world)
    _cp_check(wl, range(wl.total_q), sel, out, lse)


def test_context_parallel_decode_1m_planted():
    """The million-token decode spread over four ranges: the merged selection is exactly the planted set."""
    wl = W.decode_1m_planted()
    sel, out, lse = _cp_run(wl, 4)
    assert np.array_equal(sel[0], np.sort(wl.planted))
    _cp_check(wl, [0], sel, out, lse)


# --------------------------------------------------------------------------------------- block-granular selection
def _block_case(kind, grid):
    if kind == "prefill":
        return W.make_workload("blocks", kind="mla", seed=115, seq_lens=[70, 300, 2100, 2600], q_lens=[70, 37, 300, 5],
                               topk=2048, grid=grid)
    return W.make_workload("blocks_decode", kind="mla", seed=116, seq_lens=[1, 64, 65, 2049, 9000, 15000],
                           q_lens=[1] * 6, topk=2048, grid=grid)


@pytest.mark.parametrize("kind,grid,kb", [("prefill", True, 8), ("prefill", False, 8), ("decode", True, 32),
                                          ("decode", False, 5)])
def test_block_selection_matches_oracle(kind, grid, kb):
    """Page scores bit-exact (a max of the same fp32 scores), kept pages and their positions exact (the
    oracle decides on the GPU's fp32 scores), attention over that set within the MLA tolerances."""
    wl = _block_case(kind, grid)
    db = DeviceBatch(wl)
    db.indexer()
    idx = db.block_select(kb)
    db.attention(idx=idx, k=kb * 64)
    torch.cuda.synchronize()
    db.check_status()
    sc = db.scores.cpu().numpy()
    blk = db.blk_scores.cpu().numpy()
    lens = db.blk_lens.cpu().numpy()
    got = idx.cpu().numpy()
    out, lse = db.out.float().cpu().numpy(), db.lse.cpu().numpy()
    for r in range(wl.total_q):
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, r)
        s = sc[r, : pos + 1].astype(np.float64)
        bs = oracle.block_scores_row(s, 64)
        assert lens[r] == bs.size and np.array_equal(blk[r, : bs.size].astype(np.float64), bs), f"row {r}: page scores"
        exp = oracle.block_topk_row(s, kb, 64)
        assert np.array_equal(got[r], exp), f"row {r}: block selection differs"
        ref_o, ref_l = oracle.sparse_attention_row(wl, r, exp)
        check_attention(wl, r, out[r], lse[r], ref_o, ref_l)


# --------------------------------------------------------------------------------------- decode index reuse
@pytest.mark.parametrize("grid", [True, False])
def test_decode_index_reuse_matches_oracle(grid):
    """An earlier selection (this step's own, cut to the positions before prev_len) plus the positions
    added since: the candidate list exact, the scores at the candidates within the indexer tolerance
    (bit-exact on the integer grid), the kept positions exact (the oracle decides on the GPU's fp32
    candidate scores), attention over them within the MLA tolerances."""
    from parity import SCORE_REL, abs_case
    seq_lens = np.array([300, 2100, 5000, 9000])
    delta = np.array([1, 7, 64, 300])                                # tokens added since the earlier selection
    wl = W.make_workload("reuse", kind="mla", seed=117, seq_lens=seq_lens, q_lens=[1] * 4, topk=2048, grid=grid)
    db = _run(wl)
    prev_lens = seq_lens - delta
    prev = db.idx.clone()
    prev_lens_d = torch.from_numpy(prev_lens.astype(np.int32)).cuda()
    prev[prev >= prev_lens_d[:, None]] = -1
    idx = db.reuse_select(prev, prev_lens_d, int(delta.max()))
    db.attention(idx=idx)
    torch.cuda.synchronize()
    db.check_status()
    cand, cs, got = db.cand.cpu().numpy(), db.cand_scores.cpu().numpy(), idx.cpu().numpy()
    out, lse = db.out.float().cpu().numpy(), db.lse.cpu().numpy()
    prev_h = prev.cpu().numpy()
    acase = abs_case(wl)
    m = cand.shape[1]
    for r in range(wl.total_q):
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, r)
        exp_c = oracle.reuse_candidates(prev_h[r], int(prev_lens[r]), pos)
        exp_c = np.concatenate([exp_c, np.full(m - exp_c.size, -1)])
        assert np.array_equal(cand[r], exp_c), f"row {r}: candidate list differs"
        osc = oracle.candidate_scores_row(wl, r, exp_c)
        fin = np.isfinite(osc)
        assert np.array_equal(np.isfinite(cs[r]), fin), f"row {r}: empty candidate slots differ"
        if grid:
            assert np.array_equal(cs[r][fin].astype(np.float64), osc[fin]), f"row {r}: grid scores inexact"
        else:
            A = oracle.candidate_scores_row(acase, r, exp_c)
            assert np.all(np.abs(cs[r][fin] - osc[fin]) <= SCORE_REL["mla"] * A[fin] + 1e-30), f"row {r}: scores"
        exp = oracle.candidate_topk(cs[r].astype(np.float64), exp_c, wl.topk)
        assert np.array_equal(got[r], exp), f"row {r}: kept positions differ"
        ref_o, ref_l = oracle.sparse_attention_row(wl, r, exp)
        check_attention(wl, r, out[r], lse[r], ref_o, ref_l)


# --------------------------------------------------------------------------------------- append fused with the indexer
def _own_pools(wl, dev):
    inputs = DeviceBatch.upload_inputs(wl, dev)
    inputs["kv_pool"] = torch.from_numpy(np.ascontiguousarray(wl.kv_pool).view(np.int16)).to(dev)
    return inputs


@pytest.mark.parametrize("shape", ["decode", "chunk"])
def test_append_fused_with_indexer_matches_separate_calls(shape):
    """The fused call (inside the indexer's first kernel for <= 256 rows; a separate launch for the 305-row
    chunk) leaves the same pools and scores, bit for bit, as dsa_cache_append followed by dsa_indexer_scores,
    and the pools equal the oracle's append."""
    if shape == "decode":
        seq_lens, q_lens = [300, 2100, 5000, 65], [1, 1, 1, 1]
    else:
        seq_lens, q_lens = [2100, 700], [300, 5]
    wl = W.make_workload("fused_append", kind="mla", seed=118, seq_lens=seq_lens, q_lens=q_lens, topk=2048)
    dev = torch.device("cuda")
    kv_new, k_in, fmt = _append_inputs(wl.total_q, np.random.default_rng(119), False)
    kv_d, k_d = _dev_copy(kv_new, dev), _dev_copy(k_in, dev)
    a = DeviceBatch(wl, inputs=_own_pools(wl, dev))
    b = DeviceBatch(wl, inputs=_own_pools(wl, dev))
    a.append_and_indexer(kv_d, k_d, B.DSA_F32)
    B.dsa_cache_append(kv_d, B.DSA_BF16, k_d, B.DSA_F32, 576, 128, b.batch, b.kv_pool, b.kI_pool, b.kS_pool, b.ws,
                       b.ws_bytes)
    b.indexer()
    torch.cuda.synchronize()
    a.check_status()
    b.check_status()
    for name in ("kv_pool", "kI_pool", "kS_pool"):
        assert torch.equal(getattr(a, name), getattr(b, name)), f"{name} differs between fused and separate calls"
    for r in range(wl.total_q):
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, r)
        assert torch.equal(a.scores[r, : pos + 1], b.scores[r, : pos + 1]), f"row {r}: scores differ"
    ekv, ekI, ekS = oracle.cache_append(wl, kv_new.view(np.uint16), k_in, fmt)
    assert np.array_equal(a.kv_pool.cpu().numpy().view(np.uint16), ekv)
    assert np.array_equal(a.kS_pool.cpu().numpy().view(np.uint32), ekS.view(np.uint32))
    zero = lambda c: np.where((c & 0x7F) == 0, 0, c)
    assert np.array_equal(zero(a.kI_pool.cpu().numpy()), zero(ekI))


# --------------------------------------------------------------------------------------- zig-zag prefill
@pytest.mark.parametrize("world", [2, 3])
def test_zigzag_prefill_ranks_match_one_batch(world):
    """Each rank's zig-zag share of a prompt, run as its own batch, gives its rows exactly the scores, picks,
    outputs and lse that the whole prompt run as one batch gives them (every step is per row)."""
    from sparse_attention_long_dsa_b200 import prefill_parallel as PP
    wl = W.make_workload("zz_gpu", kind="mla", seed=120, seq_lens=[3000], q_lens=[2600], topk=2048, grid=True)
    whole = _run(wl)
    for rank in range(world):
        loc, rows = PP.local_prefill_workload(wl, rank, world)
        db = _run(loc)
        rt = torch.from_numpy(rows).cuda()
        assert torch.equal(db.idx, whole.idx[rt]), f"rank {rank}: picks differ"
        assert torch.equal(db.out, whole.out[rt]) and torch.equal(db.lse, whole.lse[rt]), f"rank {rank}: attention"
        for i in range(0, loc.total_q, 97):
            _, pos = oracle.row_location(loc.seq_lens, loc.cu_q, i)
            assert torch.equal(db.scores[i, : pos + 1], whole.scores[int(rows[i]), : pos + 1]), f"rank {rank} row {i}"
