"""Context-parallel decode on the CPU: the range split, the local batches and the exchange schedule of
`context_parallel`, with every local step done by the oracle (test-only rank objects), against the
single-GPU oracle.  The CUDA kernels of the same steps are checked in tests/test_zz_widened_paths_gpu.py."""
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
from sparse_attention_long_dsa_b200 import context_parallel as CP  # noqa: E402
from sparse_attention_long_dsa_b200 import workloads as W  # noqa: E402


def test_shard_ranges_by_hand():
    lo, hi = CP.shard_ranges([640, 130, 200], 2)
    # 10 pages -> 5 + 5; 3 pages -> 1 + 2; 4 pages (last partial) -> 2 + 2
    assert lo.tolist() == [[0, 0, 0], [320, 64, 128]]
    assert hi.tolist() == [[320, 64, 128], [640, 130, 200]]
    lo, hi = CP.shard_ranges([700], 3)                 # 11 pages -> 3, 4, 4
    assert lo[:, 0].tolist() == [0, 192, 448] and hi[:, 0].tolist() == [192, 448, 700]
    with pytest.raises(ValueError):
        CP.shard_ranges([100], 3)                      # 2 pages over 3 ranks


def test_local_workload_slices_the_block_table():
    wl = W.make_workload("cp_host", kind="mla", seed=21, seq_lens=[300, 700], q_lens=[1, 1], topk=64)
    loc, lo, hi = CP.local_workload(wl, 1, 2)
    # sequence 0: 5 pages -> rank 1 has pages 2..4 (tokens 128..299); sequence 1: 11 pages -> pages 5..10
    assert lo.tolist() == [128, 320] and hi.tolist() == [300, 700]
    assert loc.seq_lens.tolist() == [172, 380]
    assert loc.block_table[0, :3].tolist() == wl.block_table[0, 2:5].tolist()
    assert loc.block_table[1, :6].tolist() == wl.block_table[1, 5:11].tolist()
    assert loc.max_seq_len == 380 and loc.total_q == 2
    # local token j of sequence b is global token lo[b] + j: same (block, slot)
    for b, j in [(0, 0), (0, 171), (1, 5), (1, 379)]:
        gb, gs = oracle.token_slots(wl.block_table[b], np.array([lo[b] + j]), 64)
        lb, ls = oracle.token_slots(loc.block_table[b], np.array([j]), 64)
        assert (gb[0], gs[0]) == (lb[0], ls[0])


class OracleRank:
    """A rank whose local steps are done by the oracle on CPU tensors: the same three phases as
    CP.CPDecodeRank (candidates, attend, merge), in fp64."""

    def __init__(self, wl, rank, world):
        self.loc, self.lo, self.hi = CP.local_workload(wl, rank, world)
        self.world, self.T, self.k = world, wl.total_q, wl.topk

    def candidates(self, stream=None):
        cs = np.full((self.T, self.k), -np.inf)
        cg = np.full((self.T, self.k), -1, dtype=np.int64)
        for t in range(self.T):
            sc = oracle.indexer_scores_row(self.loc, t).astype(np.float32).astype(np.float64)
            idx = oracle.topk_row(sc, self.k)
            ok = idx >= 0
            cs[t, ok] = sc[idx[ok]]
            cg[t, ok] = idx[ok] + self.lo[t]
        return torch.from_numpy(cs), torch.from_numpy(cg)

    def attend(self, g_score, g_gidx, stream=None):
        G, T, k = self.world, self.T, self.k
        gs, gg = g_score.numpy(), g_gidx.numpy()
        o = np.zeros((T, self.loc.H, self.loc.Dv))
        lse = np.full((T, self.loc.H), -np.inf)
        self.sel = np.full((T, k), -1, dtype=np.int64)
        for t in range(T):
            rows = np.concatenate([gs[r, t] for r in range(G)])
            gid = np.concatenate([gg[r, t] for r in range(G)])
            pick = oracle.topk_row(rows, k)
            g = np.where(pick >= 0, gid[np.maximum(pick, 0)], -1)
            self.sel[t] = g
            mine = (g >= self.lo[t]) & (g < self.hi[t])
            local = np.where(mine, g - self.lo[t], -1)
            o[t], lse[t] = oracle.sparse_attention_row(self.loc, t, local)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(self, g_out, g_lse, out, lse, stream=None):
        for t in range(self.T):
            o_t, l_t = oracle.combine([g_out[r, t].numpy() for r in range(self.world)],
                                      [g_lse[r, t].numpy() for r in range(self.world)])
            out[t] = torch.from_numpy(o_t)
            lse[t] = torch.from_numpy(l_t)
        return out, lse


def _cp_case():
    # integer grid: many tied scores, so the tie rule is exercised across ranges
    return W.make_workload("cp", kind="mla", seed=22, seq_lens=[1000, 2600, 700], q_lens=[1, 1, 1], topk=256,
                           grid=True)


def _check_against_single_gpu_oracle(wl, sel, out, lse):
    ref = oracle.run_rows(wl, range(wl.total_q))
    for t in range(wl.total_q):
        got = np.sort(sel[t][sel[t] >= 0])
        exp = ref[t]["idx"][ref[t]["idx"] >= 0]
        assert np.array_equal(got, exp), f"row {t}: global selection differs"
        assert np.abs(out[t] - ref[t]["out"]).max() < 1e-9
        assert np.abs(lse[t] - ref[t]["lse"]).max() < 1e-9


@pytest.mark.parametrize("world", [2, 3])
def test_emulated_ranks_match_single_gpu_oracle(world):
    wl = _cp_case()
    ranks = [OracleRank(wl, r, world) for r in range(world)]
    out = torch.zeros((wl.total_q, wl.H, wl.Dv), dtype=torch.float64)
    lse = torch.zeros((wl.total_q, wl.H), dtype=torch.float64)
    CP.cp_decode_emulated(ranks, out, lse)
    _check_against_single_gpu_oracle(wl, ranks[0].sel, out.numpy(), lse.numpy())


def _gloo_rank(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        wl = _cp_case()
        me = OracleRank(wl, rank, world)

        def all_gather(t):
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t.contiguous())
            return torch.stack(parts)

        out = torch.zeros((wl.total_q, wl.H, wl.Dv), dtype=torch.float64)
        lse = torch.zeros((wl.total_q, wl.H), dtype=torch.float64)
        CP.cp_decode_step(me, all_gather, out, lse)
        results[rank] = {"sel": me.sel.tolist(), "out": out.numpy().tobytes(), "lse": lse.numpy().tobytes()}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_single_gpu_oracle():
    world = 2
    port = 33500 + (os.getpid() % 2000)
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_gloo_rank, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
        res = dict(results)
    wl = _cp_case()
    shape = (wl.total_q, wl.H, wl.Dv)
    outs = [np.frombuffer(res[r]["out"], dtype=np.float64).reshape(shape) for r in range(world)]
    lses = [np.frombuffer(res[r]["lse"], dtype=np.float64).reshape(wl.total_q, wl.H) for r in range(world)]
    assert res[0]["sel"] == res[1]["sel"] and np.array_equal(outs[0], outs[1]) and np.array_equal(lses[0], lses[1])
    _check_against_single_gpu_oracle(wl, np.array(res[0]["sel"]), outs[0], lses[0])
