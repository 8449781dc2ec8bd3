"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Small cases run every row and span several tiles plus ragged tails; the five full-size
workloads run in the same launch configuration the benchmark times and are checked on
sampled rows (rows are independent, so a sampled row is a complete check of that row), and every row's
selection against the top-k's defining properties on the GPU's own scores.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import check_attention, check_topk_every_row, compare_rows, sample_rows
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


# --------------------------------------------------------------------------------------- fp32 path
@pytest.mark.parametrize("grid", [False, True])
def test_tiny_f32_every_row(grid):
    wl = W.tiny_f32(grid=grid)
    db = _run(wl)
    compare_rows(wl, db, list(range(wl.total_q)))


def test_tiny_f32_conditional_and_full_parity_agree_when_sets_match():
    wl = W.tiny_f32()
    db = _run(wl)
    gi = db.idx.cpu().numpy()
    res = oracle.run_rows(wl, range(wl.total_q))
    same = [r for r in range(wl.total_q) if np.array_equal(gi[r], res[r]["idx"])]
    assert len(same) >= wl.total_q * 0.9
    go, gl = db.out.cpu().numpy(), db.lse.cpu().numpy()
    for r in same:
        check_attention(wl, r, go[r], gl[r], res[r]["out"], res[r]["lse"])


# --------------------------------------------------------------------------------------- MLA, small
EDGE_LENS = [1, 2, 63, 64, 65, 127, 128, 129, 200, 2047, 2048, 2049, 3001]


@pytest.mark.parametrize("grid", [True, False])
def test_mla_small_prefill_every_row(grid):
    seq_lens = [70, 300, 2100, 2600]
    q_lens = [70, 37, 300, 5]                # whole prompt, a chunk, a long chunk, a short tail
    wl = W.make_workload("small_prefill", kind="mla", seed=101, seq_lens=seq_lens, q_lens=q_lens, topk=2048,
                         grid=grid)
    db = _run(wl)
    compare_rows(wl, db, list(range(wl.total_q)))


def test_repeated_launches_are_bitwise_identical():
    """The whole path is deterministic: the same batch run again (the first launch included) gives the
    same bits.  Catches ordering races between the CTAs of a pair, which show up as run-to-run
    differences in a few value blocks long before they break a tolerance."""
    seq_lens = [70, 300, 2100, 2600]
    q_lens = [70, 37, 300, 5]
    wl = W.make_workload("small_prefill", kind="mla", seed=101, seq_lens=seq_lens, q_lens=q_lens, topk=2048,
                         grid=True)
    db = DeviceBatch(wl)
    runs = []
    for _ in range(5):
        db.run()
        torch.cuda.synchronize()
        db.check_status()
        runs.append((db.idx.clone(), db.out.clone(), db.lse.clone()))
    for i, (ix, o, l) in enumerate(runs[1:], 1):
        assert torch.equal(ix, runs[0][0]), f"launch {i}: top-k differs from the first launch"
        bad = torch.nonzero((o != runs[0][1]).flatten(1).any(dim=1)).flatten().tolist()
        assert not bad, f"launch {i}: attention output differs from the first launch in rows {bad[:8]}"
        assert torch.equal(l, runs[0][2]), f"launch {i}: lse differs from the first launch"


@pytest.mark.parametrize("grid", [True, False])
def test_mla_small_decode_every_row(grid):
    wl = W.make_workload("small_decode", kind="mla", seed=102, seq_lens=EDGE_LENS, q_lens=[1] * len(EDGE_LENS),
                         topk=2048, grid=grid)
    db = _run(wl)
    assert db.decode
    compare_rows(wl, db, list(range(wl.total_q)))


@pytest.mark.parametrize("topk", [1, 100, 640, 2048])
def test_mla_topk_sizes(topk):
    wl = W.make_workload("small_k", kind="mla", seed=103 + topk, seq_lens=[2500, 700, 64], q_lens=[3, 2, 1],
                         topk=topk, grid=True)
    db = _run(wl)
    compare_rows(wl, db, list(range(wl.total_q)))


def test_mla_prefill_entry_on_decode_batch():
    """A decode-shaped batch through the prefill entry gives the same results as the decode entry."""
    wl = W.make_workload("dec", kind="mla", seed=104, seq_lens=[3000, 129, 4097], q_lens=[1, 1, 1], topk=2048)
    a = _run(wl, decode=True)
    b = _run(wl, decode=False)
    assert torch.equal(a.idx, b.idx)
    out_a, out_b = a.out.float(), b.out.float()
    assert (out_a - out_b).abs().max().item() <= 2e-2


def test_block_table_permutation_is_bit_invariant():
    wl = W.make_workload("perm", kind="mla", seed=105, seq_lens=[2200, 900], q_lens=[4, 1], topk=2048)
    a = _run(wl)
    perm = np.random.default_rng(3).permutation(wl.num_blocks)
    inv = np.argsort(perm)
    wl.kv_pool = np.ascontiguousarray(wl.kv_pool[inv])
    wl.kI_pool = np.ascontiguousarray(wl.kI_pool[inv])
    wl.kS_pool = np.ascontiguousarray(wl.kS_pool[inv])
    wl.block_table = perm[wl.block_table].astype(np.int32)
    b = _run(wl)
    T = wl.total_q
    for r in range(T):
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, r)
        assert torch.equal(a.scores[r, : pos + 1], b.scores[r, : pos + 1])
    assert torch.equal(a.idx, b.idx)
    assert torch.equal(a.out, b.out) and torch.equal(a.lse, b.lse)


# --------------------------------------------------------------------------------------- top-k alone
def _topk_alone(rows_scores, k):
    """GPU top-k on given fp32 score rows (one sequence per row, decode-shaped), expected =
    the oracle's selection on exactly the same fp32 values."""
    n = [len(s) for s in rows_scores]
    B_ = len(n)
    ld = (max(n) + 3) // 4 * 4
    sc = np.zeros((B_, ld), np.float32)
    for i, s in enumerate(rows_scores):
        sc[i, : len(s)] = s
    maxb = (max(n) + 63) // 64
    dev = torch.device("cuda")
    bt = torch.zeros((B_, maxb), dtype=torch.int32, device=dev)
    sl = torch.tensor(n, dtype=torch.int32, device=dev)
    cu = torch.arange(B_ + 1, dtype=torch.int32, device=dev)
    batch = B.make_batch(bt, sl, cu, num_blocks=1, page_size=64, total_q=B_, max_q_per_seq=1, max_seq_len=max(n))
    ws_bytes = B.dsa_workspace_size(B.DSA_OP_TOPK, batch, k)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    scd = torch.from_numpy(sc).to(dev)
    idx = torch.full((B_, k), -7, dtype=torch.int32, device=dev)
    B.dsa_topk(scd, ld, batch, k, idx, ws, ws_bytes)
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    for i, s in enumerate(rows_scores):
        exp = oracle.topk_row(np.asarray(s, np.float32).astype(np.float64), k)
        assert np.array_equal(got[i], exp), f"row {i} (n={len(s)}): first diff at {np.flatnonzero(got[i] != exp)[:5]}"


@pytest.mark.parametrize("k", [1, 7, 2048])
def test_topk_alone_ties_and_lengths(k):
    rng = np.random.default_rng(k)
    rows = []
    for n in [1, 5, k, k + 1, 3000, 49152, 49153, 70001]:
        rows.append(rng.integers(-3, 4, n).astype(np.float32))                     # heavy ties
        rows.append(rng.standard_normal(n).astype(np.float32))                      # distinct
    rows.append(np.zeros(5000, np.float32))                                          # all equal
    z = np.zeros(3000, np.float32); z[::2] = -0.0                                    # +-0 ties
    rows.append(z)
    rows.append(np.concatenate([np.full(100, 1e30, np.float32), -np.abs(rng.standard_normal(60000)).astype(np.float32)]))
    _topk_alone(rows, k)


@pytest.mark.parametrize("max_len", [131072, 300000])
def test_topk_alone_many_rows_past_one_cta(max_len):
    # more rows than half the SMs, all longer than one CTA's shared-memory slice: the rows are taken by
    # 2-CTA clusters up to 98304 candidates and by the multi-launch long-row path beyond, in one call
    rng = np.random.default_rng(max_len)
    rows = []
    for i, n in enumerate(rng.integers(49153, max_len + 1, 150)):
        n = int(max_len) if i == 0 else int(n)
        rows.append(rng.integers(-40, 40, n).astype(np.float32) if i % 2 else rng.standard_normal(n).astype(np.float32))
    _topk_alone(rows, 2048)


def test_topk_alone_long_row():
    rng = np.random.default_rng(9)
    rows = [rng.standard_normal(1 << 20).astype(np.float32),
            rng.integers(-50, 50, 300000).astype(np.float32)]
    _topk_alone(rows, 2048)


# --------------------------------------------------------------------------------------- full-size workloads
@pytest.mark.parametrize("grid", [False, True])
def test_decode_batch(grid):
    wl = W.decode_batch(grid=grid)
    db = _run(wl)
    compare_rows(wl, db, sample_rows(wl, extra=4))
    check_topk_every_row(wl, db.scores, db.idx)


def test_prefill_16k():
    wl = W.prefill_16k()
    db = _run(wl)
    compare_rows(wl, db, sample_rows(wl, extra=24))
    check_topk_every_row(wl, db.scores, db.idx)


def test_decode_1m_planted():
    wl = W.decode_1m_planted()
    db = _run(wl)
    got = db.idx.cpu().numpy()[0]
    assert np.array_equal(got, wl.planted.astype(np.int32)), "GPU top-k is not the planted set"
    compare_rows(wl, db, [0])
    check_topk_every_row(wl, db.scores, db.idx)


def test_mixed_batch():
    wl = W.mixed_batch()
    db = _run(wl)
    assert not db.decode
    compare_rows(wl, db, sample_rows(wl, extra=16))
    check_topk_every_row(wl, db.scores, db.idx)


# --------------------------------------------------------------------------------------- ABI on device
def test_errors_leave_outputs_untouched():
    wl = W.make_workload("err", kind="mla", seed=106, seq_lens=[300], q_lens=[2], topk=64)
    db = DeviceBatch(wl)
    db.idx.fill_(-5)
    with pytest.raises(B.DSAError) as e:
        B.dsa_topk(db.scores, db.ld, db.batch, 0, db.idx, db.ws, db.ws_bytes)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
    with pytest.raises(B.DSAError) as e:
        B.dsa_topk(db.scores, db.ld, db.batch, 64, db.idx, db.ws, 16)
    assert e.value.status == B.DSA_ERR_WORKSPACE
    with pytest.raises(B.DSAError) as e:
        B.dsa_sparse_attn_decode(db.q, B.DSA_BF16, db.kv_pool, None, 128, 576, 512, 0.07, db.idx, 64, db.batch,
                                 db.out, db.lse, db.ws, db.ws_bytes)
    assert e.value.status == B.DSA_ERR_INVALID_ARG          # two query rows in one sequence
    torch.cuda.synchronize()
    assert bool((db.idx == -5).all())
