"""dsa_topk_noalloc: the top-k entry point for callers that cannot allocate device memory (for
example an operator plugin that is handed only a stream, or a latency-critical path where an
allocation and its implicit device synchronisation are not allowed).  It keeps its scratch in an
array inside the library instead of a caller workspace; its output must equal dsa_topk's exactly,
call after call (the array keeps the previous call's contents).

Collected last on purpose (file name), so that a run stopping at the first failure has already run
every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_dsa_b200 import binding as B

pytestmark = pytest.mark.gpu


def _batch(lengths):
    """One query row per sequence (decode-shaped), row i has lengths[i] candidates."""
    dev = torch.device("cuda")
    n = [int(x) for x in lengths]
    maxb = (max(n) + 63) // 64
    bt = torch.zeros((len(n), maxb), dtype=torch.int32, device=dev)
    sl = torch.tensor(n, dtype=torch.int32, device=dev)
    cu = torch.arange(len(n) + 1, dtype=torch.int32, device=dev)
    batch = B.make_batch(bt, sl, cu, num_blocks=1, page_size=64, total_q=len(n), max_q_per_seq=1, max_seq_len=max(n))
    return batch, (bt, sl, cu)


def _scores(lengths, seed):
    rng = np.random.default_rng(seed)
    ld = (max(lengths) + 3) // 4 * 4
    sc = np.zeros((len(lengths), ld), np.float32)
    for i, n in enumerate(lengths):
        if i % 3 == 0:
            sc[i, :n] = rng.integers(-5, 6, n)                    # many ties
        else:
            sc[i, :n] = rng.standard_normal(n)
    return torch.from_numpy(sc).cuda(), ld


@pytest.mark.parametrize("k", [64, 2048])
def test_noalloc_topk_matches_workspace_topk_on_consecutive_calls(k):
    torch.cuda.init()
    # short rows (one CTA each) and long rows (the multi-CTA path that uses the scratch)
    lengths = [1, 63, 2047, 2048, 2049, 40000, 49152, 49153, 70001, 300000, 1 << 20]
    keep = []
    for call, seed in enumerate((11, 12)):
        scores, ld = _scores(lengths, seed + k)
        batch, keep = _batch(lengths)
        ref = torch.full((len(lengths), k), -9, dtype=torch.int32, device="cuda")
        ws_bytes = B.dsa_workspace_size(B.DSA_OP_TOPK, batch, k)
        ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
        B.dsa_topk(scores, ld, batch, k, ref, ws, ws_bytes)
        got = torch.full((len(lengths), k), -7, dtype=torch.int32, device="cuda")
        B.dsa_topk_noalloc(scores, ld, batch, k, got)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}: rows differ {torch.nonzero((got != ref).any(dim=1)).flatten().tolist()}"
        # and directly against the oracle's selection on the same fp32 scores (exact: same values both sides)
        sc = scores.cpu().numpy()
        g = got.cpu().numpy()
        for i, n in enumerate(lengths):
            assert np.array_equal(g[i], oracle.topk_row(sc[i, :n].astype(np.float64), k)), f"call {call}, row {i}"


def test_noalloc_topk_rejects_oversized_batches():
    lengths = [100] * 257                                             # one row over the built-in limit
    batch, keep = _batch(lengths)
    scores = torch.zeros((257, 100), dtype=torch.float32, device="cuda")
    idx = torch.zeros((257, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(B.DSAError) as e:
        B.dsa_topk_noalloc(scores, 100, batch, 8, idx)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
    assert "256 rows" in B.load().dsa_last_error().decode()


def test_noalloc_topk_rejects_rows_past_the_candidate_limit_and_writes_nothing():
    n = (1 << 20) + 1                                                 # one candidate over the built-in limit
    batch, keep = _batch([n, 10])
    ld = (n + 3) // 4 * 4
    scores = torch.zeros((2, ld), dtype=torch.float32, device="cuda")
    idx = torch.full((2, 16), -5, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    with pytest.raises(B.DSAError) as e:
        B.dsa_topk_noalloc(scores, ld, batch, 16, idx)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
    assert "max_seq_len" in B.load().dsa_last_error().decode()
    torch.cuda.synchronize()
    assert bool((idx == -5).all()), "a rejected call must enqueue nothing"
