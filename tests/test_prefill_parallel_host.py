"""Zig-zag prefill over several ranks, on the CPU: the row split, the local batches (every local row sits at
its prompt position and the oracle gives it the prompt's result) and the one all-gather that fills the
pools, as two gloo ranks."""
import datetime
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sparse_attention_long_dsa_b200 import prefill_parallel as PP  # noqa: E402
from sparse_attention_long_dsa_b200 import workloads as W  # noqa: E402


def test_zigzag_chunks_by_hand():
    # 10 rows, 2 ranks: chunk bounds 0, 2, 5, 7, 10
    assert PP.zigzag_chunks(10, 2) == [[(0, 2), (7, 10)], [(2, 5), (5, 7)]]
    for n, g in [(16384, 4), (1000, 3), (7, 3)]:
        rows = sorted(r for rank in PP.zigzag_chunks(n, g) for lo, hi in rank for r in range(lo, hi))
        assert rows == list(range(n))


def test_zigzag_balances_causal_work():
    n, g = 16384, 4
    work = [sum(sum(range(lo + 1, hi + 1)) for lo, hi in rank) for rank in PP.zigzag_chunks(n, g)]
    assert max(work) / min(work) < 1.001


@pytest.mark.parametrize("world", [2, 3])
def test_local_rows_reproduce_the_prompt_rows(world):
    wl = W.make_workload("zz", kind="mla", seed=41, seq_lens=[700], q_lens=[300], topk=128, grid=True)
    p0 = 700 - 300
    seen = []
    for rank in range(world):
        loc, rows = PP.local_prefill_workload(wl, rank, world)
        seen += rows.tolist()
        for i in range(0, loc.total_q, 37):
            _, pos = oracle.row_location(loc.seq_lens, loc.cu_q, i)
            assert pos == p0 + rows[i]
            a = oracle.run_rows(loc, [i])[i]
            b = oracle.run_rows(wl, [int(rows[i])])[int(rows[i])]
            for key in ("scores", "idx", "out", "lse"):
                assert np.array_equal(a[key], b[key]), (rank, i, key)
    assert sorted(seen) == list(range(300))


def _gloo_pages(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(5)
        full = torch.from_numpy(rng.standard_normal((12, 4, 3)).astype(np.float32))
        page_ids = torch.tensor([7, 2, 9, 0, 11, 4, 5], dtype=torch.int32)      # the prompt's pages
        pool = torch.full_like(full, -1.0)
        lo, hi = PP.pages_of_rank(page_ids.numel(), rank, world)
        pool[page_ids[lo:hi].long()] = full[page_ids[lo:hi].long()]            # only this rank's pages written
        PP.allgather_pages(pool, page_ids, rank, world)
        listed = page_ids.long()
        others = torch.ones(12, dtype=torch.bool)
        others[listed] = False
        results[rank] = bool(torch.equal(pool[listed], full[listed])) and bool((pool[others] == -1.0).all())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_fill_the_pool():
    world = 2
    port = 35500 + (os.getpid() % 2000)
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_gloo_pages, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
        assert dict(results) == {0: True, 1: True}
