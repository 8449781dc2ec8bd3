"""Multi-rank host logic of bench.py on CPU with gloo (world size 2): every rank runs its own batch
(weak scaling, no data-path collective), the job's time is the slowest rank's, the whole-job value counts
every rank's tokens, and the per-rank batches are different draws of the same shape."""
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


def _rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from sparse_attention_long_dsa_b200 import workloads as W

        class A:
            workload = "decode_batch"
        # each rank's own timed region: rank 1 is the slow one
        ms = {0: 100.0, 1: 125.0}[rank]
        job_ms = bench.slowest_rank_ms(ms, world, "cpu")
        wl = W.decode_batch(seed=bench._seed(A, rank))
        value = bench.job_tokens_per_s(wl.total_q, world, job_ms / 10)
        # the ranks' batches: same shape, different draws
        shapes = torch.tensor([wl.total_q, wl.num_seqs, int(wl.seq_lens.sum())], dtype=torch.int64)
        gathered = [torch.zeros_like(shapes) for _ in range(world)]
        dist.all_gather(gathered, shapes)
        results[rank] = {"job_ms": job_ms, "value": value, "seq_lens": wl.seq_lens.tolist(),
                         "shapes": [g.tolist() for g in gathered]}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_slowest_rank_time_and_weak_scaling_value():
    world = 2
    port = 29500 + (os.getpid() % 2000)
    with mp.Manager() as mgr:
        results = mgr.dict()
        ctx = mp.get_context("spawn")
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
        res = dict(results)
    assert set(res) == {0, 1}
    # both ranks agree on the job's time: the slowest rank's
    assert res[0]["job_ms"] == res[1]["job_ms"] == 125.0
    # whole-job throughput: both ranks' 32 query rows per step over the slowest rank's step time
    assert res[0]["value"] == pytest.approx(2 * 32 / (12.5e-3))
    # weak scaling: same batch shape on every rank, different contexts (different seeds)
    assert res[0]["shapes"][0][:2] == res[0]["shapes"][1][:2] == [32, 32]
    assert res[0]["seq_lens"] != res[1]["seq_lens"]
    assert np.all(np.asarray(res[0]["seq_lens"]) >= 4096) and np.all(np.asarray(res[1]["seq_lens"]) <= 32768)
