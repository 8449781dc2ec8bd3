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
        # a clock record that rejects rank 0's timed region re-measures on every rank (same collectives)
        calls = []

        def fake_time_steps(replicas, stream, steps, warmup, world_, dev, sampler, selection):
            calls.append(1)
            throttled = rank == 0 and len(calls) == 1
            return 1.0, {}, 0, {"sm_mhz": 1965.0, "sm_max_mhz": 1965,
                                "reasons": ["hw_thermal_slowdown"] if throttled else []}

        bench._time_steps = fake_time_steps
        checked = bench._time_steps_checked(None, None, 1, 1, world, "cpu", None, "auto")
        results[rank] = {"job_ms": job_ms, "value": value, "seq_lens": wl.seq_lens.tolist(),
                         "shapes": [g.tolist() for g in gathered], "timed_regions": len(calls),
                         "rejected_first": checked[3].get("rejected_first")}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_slowest_rank_time_and_weak_scaling_value():
    world = 2
    port = 29500 + (os.getpid() % 2000)
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
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
    # rank 0's throttled region was measured again on both ranks; rank 0 keeps the rejected record
    assert res[0]["timed_regions"] == res[1]["timed_regions"] == 2
    assert res[0]["rejected_first"]["reasons"] == ["hw_thermal_slowdown"]
    assert res[1]["rejected_first"]["reasons"] == []


# ----------------------------------------------------------------------------- overlapped e2e leg
def _fake_cuda(step_ms):
    """Stand-ins for the CUDA stream/event calls the overlapped e2e leg makes, so that its multi-rank
    agreement logic runs on CPU: every recorded event advances a clock by `step_ms`."""
    import contextlib

    class Ev:
        clock = 0.0

        def __init__(self, enable_timing=False):
            self.t = None

        def record(self, stream=None):
            Ev.clock += step_ms
            self.t = Ev.clock

        def elapsed_time(self, other):
            return other.t - self.t

    class St:
        cuda_stream = 0

        def wait_event(self, ev):
            pass

    empty = torch.empty
    torch.empty = lambda *a, pin_memory=False, **k: empty(*a, **k)
    torch.cuda.Stream = lambda device=None: St()
    torch.cuda.Event = Ev
    torch.cuda.stream = lambda s: contextlib.nullcontext()
    torch.cuda.synchronize = lambda device=None: None


class _FakeBatch:
    def __init__(self):
        self.inputs = {n: torch.zeros(4, 3) for n in ("q", "qI", "w", "block_table", "seq_lens", "cu_q")}
        self.out = torch.zeros(2, 8, dtype=torch.bfloat16)
        self.lse = torch.zeros(2, 8)
        self.n = 0

    def run(self, stream):
        self.n += 1
        self.out.fill_(self.n)
        self.lse.fill_(self.n)


def _e2e_rank_main(rank, world, port, results, sets_per_rank):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import types
        import bench
        _fake_cuda(step_ms=1.0 + rank)                         # rank 1 is the slower one
        # the packed copy-in buffers and their batches: plain CPU buffers around the fake batches
        bench._packed_step_inputs = lambda wl, reps, dev: (torch.zeros(512, dtype=torch.uint8),
                                                             [torch.zeros(512, dtype=torch.uint8) for _ in reps],
                                                             list(reps))
        args = types.SimpleNamespace(steps=6, warmup=3)
        wl = types.SimpleNamespace(total_q=32)
        sets = [_FakeBatch() for _ in range(sets_per_rank[rank])]
        res = bench.run_e2e_overlapped(args, wl, sets, "cpu", world)
        results[rank] = None if res is None else {"ms_per_step": res["ms_per_step"], "value": res["value"]}
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("sets_per_rank", [(2, 2), (2, 1)])
def test_overlapped_e2e_ranks_agree(sets_per_rank):
    """Both ranks report the slowest rank's time, or both drop the overlapped leg when one rank cannot
    run it (so that neither waits in a collective the other never enters)."""
    world = 2
    port = 31500 + (os.getpid() % 2000) + 7 * sets_per_rank[1]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_e2e_rank_main, args=(r, world, port, results, sets_per_rank))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
        res = dict(results)
    assert set(res) == {0, 1}
    if sets_per_rank == (2, 1):
        assert res[0] is None and res[1] is None
    else:
        assert res[0] == res[1]
        # the timed region spans 3 events per step for 6 steps plus the closing one; rank 1's events are
        # 2 ms apart (rank 0's 1 ms), so the job's time is rank 1's: 19 * 2 ms over 6 steps
        assert res[0]["ms_per_step"] == pytest.approx(19 * 2.0 / 6)
        assert res[0]["value"] == pytest.approx(2 * 32 / (res[0]["ms_per_step"] / 1e3))
