#!/usr/bin/env python
"""Benchmark of the DSA sparse-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode_batch] [--impl ours|reference]

One step = one pass of the whole path (indexer scores -> top-k -> sparse attention) over one
batch of the workload, through the C ABI.  The default workload is the decode batch (32
sequences, contexts U[4096, 32768], 128 heads x 576 bf16 MLA latent cache, 64 x 128 e4m3
indexer, top-k 2048); the metric is query tokens per second.  Prints ONE JSON line (rank 0).

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a device synchronise,
timed with CUDA events on the launching stream; the max over ranks is reported.  Inputs rotate
over several device replicas so that more than L2 (126 MB) is touched between two reads of the
same replica.  Per-stage CUDA events inside the timed region give the dominant kernel's average
duration for the roofline entry.  `e2e` repeats the timing through the same public calls with
each step's per-step inputs copied from pinned host memory and the results read back: once step
after step on one stream (`e2e.serial`), then with the copies of neighbouring steps overlapping the
compute on separate streams (the reported `e2e.value`, when every rank could run that leg).

Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no data-path collective).
`--impl reference` times the CPU oracle (the plain fp64 restatement of the method) on a bounded
sample of the same workload on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------------------------------------- work accounting
def work_of(wl):
    """Algorithmic bytes and flops per stage for one step (each cached byte the definition must
    read counted once; the scores/idx round trip between stages is reported separately)."""
    T = wl.total_q
    rows_n = []
    for b in range(wl.num_seqs):
        lo, hi = int(wl.cu_q[b]), int(wl.cu_q[b + 1])
        n0 = int(wl.seq_lens[b]) - (hi - lo)
        rows_n.append(np.arange(hi - lo) + n0 + 1)
    n = np.concatenate(rows_n) if rows_n else np.zeros(0)
    sel = np.minimum(n, wl.topk).astype(np.float64)
    mla = wl.kind == "mla"
    kb = (wl.Di * (1 if mla else 4) + (4 if mla else 0))            # indexer key bytes per token
    row_b = wl.Dqk * (2 if mla else 4) + (0 if mla else wl.Dv * 4)   # latent (+V) bytes per token
    el = 2 if mla else 4
    idx_bytes = float(np.sum(wl.seq_lens.astype(np.float64)) * kb + T * wl.Hi * (wl.Di * (1 if mla else 4) + 4))
    idx_flops = float(np.sum(n) * 2 * wl.Hi * wl.Di)
    topk_bytes = float(np.sum(n) * 4 + T * wl.topk * 4)
    attn_rows = float(np.sum(sel))
    # decode: every row is its own sequence, each selected row is read once per query row
    attn_bytes = attn_rows * row_b + T * wl.H * (wl.Dqk * el + wl.Dv * el)
    attn_flops = attn_rows * 2 * wl.H * (wl.Dqk + wl.Dv)
    return dict(indexer=dict(bytes=idx_bytes, flops=idx_flops), topk=dict(bytes=topk_bytes, flops=0.0),
                attention=dict(bytes=attn_bytes, flops=attn_flops), tokens=T, selected_rows=attn_rows)


def step_roofline(work, peaks, ms_per_step):
    """Roofline of one whole step: T_roof = max(fp8 flops / P_fp8 + bf16 flops / P_bf16, bytes / BW) over
    the indexer and the attention (the scores / idx round trip between stages is not credited), with
    the measured HBM copy bandwidth, the burst bf16 GEMM peak and FP8 at twice bf16; frac = T_roof over
    the measured step time."""
    bf16 = peaks["bf16_tflops"] * 1e12
    fp8 = 2.0 * bf16
    bw = peaks["hbm_gbs"] * 1e9
    nbytes = work["indexer"]["bytes"] + work["attention"]["bytes"]
    t_flops = work["indexer"]["flops"] / fp8 + work["attention"]["flops"] / bf16
    t_bytes = nbytes / bw
    t = max(t_flops, t_bytes)
    return {"t_roof_us": t * 1e6, "bound": "hbm" if t_bytes >= t_flops else "tensor", "frac": t / (ms_per_step / 1e3),
            "bytes": nbytes, "flops_fp8": work["indexer"]["flops"], "flops_bf16": work["attention"]["flops"],
            "peaks": "hbm_gbs, bf16_tflops (burst), fp8 = 2 x bf16"}


# ---------------------------------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML for SM clock and throttle reasons in a background thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index, period=0.005):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self.period = period
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return None
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if len(win) < 3:
            win = self.samples
            window = "warmup+timed"
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        bits = 0
        for s in win:
            bits |= s[2]
        reasons = [name for b, name in self.REASONS.items() if bits & b and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(win), "window": window}


# ---------------------------------------------------------------------------------------------- ours
# ---------------------------------------------------------------------------------------------- multi-rank
def slowest_rank_ms(ms, world, device):
    """The job's time for a timed region is its slowest rank's: MAX all-reduce of this rank's CUDA-event
    milliseconds (a no-op on one rank).  `device` is where the collective's tensor lives (the rank's GPU
    under NCCL, the CPU under gloo)."""
    if world > 1:
        import torch
        t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    return ms


# a timed region whose clock record shows one of these is not a valid number: it is measured once more
REJECTED_CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")
# reasons that explain an SM clock below its maximum (kept, noted in the record)
POWER_CLOCK_REASONS = ("sw_power_cap", "hw_power_brake_slowdown")


def clocks_rejected(clocks):
    """Whether a timed region's clock record invalidates its number: a hardware or thermal slowdown was active,
    or the median SM clock sat below 80 % of its maximum with no power-cap reason to explain it (a clock left
    locked).  A missing record (no NVML) rejects nothing."""
    if not clocks or clocks.get("sm_mhz") is None:
        return False
    reasons = clocks.get("reasons") or []
    if any(r in REJECTED_CLOCK_REASONS for r in reasons):
        return True
    mx = clocks.get("sm_max_mhz")
    return bool(mx) and clocks["sm_mhz"] < 0.8 * mx and not any(r in POWER_CLOCK_REASONS for r in reasons)


def any_rank(flag, world, device):
    """True on every rank when it is true on one (MAX all-reduce; a no-op on one rank), so that all ranks take
    the same timed regions."""
    if world > 1:
        import torch
        t = torch.tensor([1.0 if flag else 0.0], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return bool(t.item() > 0)
    return bool(flag)


def _time_steps_checked(replicas, stream, steps, warmup, world, dev, sampler, selection):
    """_time_steps, measured once more when the clock record of the timed region rejects it (on any rank); the
    record then keeps the first region's clocks under `rejected_first`."""
    res = _time_steps(replicas, stream, steps, warmup, world, dev, sampler, selection)
    if any_rank(clocks_rejected(res[3]), world, dev):
        first = res[3]
        res = _time_steps(replicas, stream, steps, warmup, world, dev, sampler, selection)
        clocks = dict(res[3] or {})
        clocks["rejected_first"] = first
        res = (res[0], res[1], res[2], clocks)
    return res


def job_tokens_per_s(tokens_per_rank_step, world, ms_per_step):
    """Whole-job throughput under weak scaling: every rank processes its own batch of the same shape."""
    return world * tokens_per_rank_step / (ms_per_step / 1e3)


def _fused_for(db, selection):
    """Whether a step takes the fused scores + selection call: by the pipeline's shape rule ("auto"), or forced."""
    return db.prefers_fused() if selection == "auto" else selection == "fused"


def _run_step(db, stream, args):
    """One pass of the path through the pipeline (its shape rule picks the selection form unless forced)."""
    selection = getattr(args, "selection", "auto")
    if selection == "auto":
        db.run(stream)
    else:
        db.run(stream, fused=selection == "fused")


STAGES_TIMING = ("a second pass of the same steps with CUDA events between the stages (events end the "
                 "programmatic-launch overlap of neighbouring kernels, so the stages sum to more than ms_per_step)")


def _time_steps(replicas, stream, steps, warmup, world, dev, sampler=None, selection="auto"):
    """W untimed warm-up steps, then K steps bracketed by a barrier and a device synchronise, timed with
    CUDA events on the launching stream around the whole region only: an event recorded between two
    kernels ends the programmatic-launch overlap of the second with the first, so per-stage events inside
    the headline region would slow the step they measure.  The per-stage times come from a second pass of
    the same K steps with events between the stages (their sum therefore exceeds the headline step).
    Returns the slowest rank's total milliseconds, the per-stage averages, the library launches of the
    headline region and its clock summary."""
    import torch
    from sparse_attention_long_dsa_b200 import binding as B
    stages = ("indexer", "topk", "attention")

    def step(db, ev=None):
        # the first two steps as the pipeline runs them: one fused call for batches where that is faster
        # (its time is then reported under "indexer", "topk" holding the empty interval), else two calls
        fused = _fused_for(db, selection)
        if ev is not None:
            ev[0].record(stream)
        if fused:
            db.indexer_topk(stream)
        else:
            db.indexer(stream)
        if ev is not None:
            ev[1].record(stream)
        if not fused:
            db.topk(stream)
        if ev is not None:
            ev[2].record(stream)
        db.attention(stream)
        if ev is not None:
            ev[3].record(stream)

    with torch.cuda.stream(stream):
        for i in range(warmup):
            step(replicas[i % len(replicas)])
    torch.cuda.synchronize(dev)
    for db in replicas:
        db.check_status(stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    launches0 = B.dsa_launch_count()
    w0 = time.perf_counter()
    t_start.record(stream)
    for i in range(steps):
        step(replicas[i % len(replicas)])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    w1 = time.perf_counter()
    launches = B.dsa_launch_count() - launches0
    if world > 1:
        torch.distributed.barrier()
    for db in replicas:
        db.check_status(stream)
    total_ms = t_start.elapsed_time(t_end)
    # the stage breakdown: the same steps again, events between the stages
    for i in range(steps):
        step(replicas[i % len(replicas)], evs[i])
    torch.cuda.synchronize(dev)
    for db in replicas:
        db.check_status(stream)
    stage_ms = {s: [] for s in stages}
    for e in evs:
        for j, s in enumerate(stages):
            stage_ms[s].append(e[j].elapsed_time(e[j + 1]))
    stage_avg = {s: float(np.mean(v)) for s, v in stage_ms.items()}
    total_ms = slowest_rank_ms(total_ms, world, dev)
    clocks = sampler.summary(w0, w1) if sampler is not None else None
    return total_ms, stage_avg, int(launches), clocks


def time_widened(replicas, stream, dev, reps=50):
    """Per-call device times (CUDA events, inputs rotating over the replicas) of the decode step's variants
    against the calls they replace: the fused scores + selection (dsa_indexer_topk) against
    dsa_indexer_scores + dsa_topk; the cache append fused into the indexer (dsa_indexer_scores_append)
    against dsa_indexer_scores alone and against dsa_cache_append + dsa_indexer_scores; the block-granular
    selection (32 pages of 64) and the decode index reuse (the previous selection plus the newest token)
    against the full top-k.  Times in microseconds."""
    import torch
    from sparse_attention_long_dsa_b200 import binding as B
    wl = replicas[0].wl
    T = wl.total_q
    g = torch.Generator(device="cpu").manual_seed(7)
    kv_new = (torch.randn((T, wl.Dqk), generator=g) * 1.0).to(torch.bfloat16).to(dev)
    k_new = torch.randn((T, wl.Di), generator=g).to(dev)
    prev_lens = [torch.clamp(db.seq_lens - 1, min=1) for db in replicas]
    for db in replicas:
        db.indexer(stream)
        db.topk(stream)
    torch.cuda.synchronize(dev)
    prev_idx = [db.idx.clone() for db in replicas]

    def t(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for i in range(len(replicas)):
                fn(i)
            e0.record(stream)
            for i in range(reps):
                fn(i % len(replicas))
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps * 1e3

    def append_sep(i):
        db = replicas[i]
        B.dsa_cache_append(kv_new, B.DSA_BF16, k_new, B.DSA_F32, wl.Dqk, wl.Di, db.batch, db.kv_pool, db.kI_pool,
                           db.kS_pool, db.ws, db.ws_bytes, stream)
        db.indexer(stream)

    res = {
        "indexer": t(lambda i: replicas[i].indexer(stream)),
        "topk": t(lambda i: replicas[i].topk(stream)),
        "indexer_topk_fused": t(lambda i: replicas[i].indexer_topk(stream)),
        "cache_append_then_indexer": t(append_sep),
        "indexer_with_fused_append": t(lambda i: replicas[i].append_and_indexer(kv_new, k_new, B.DSA_F32, stream)),
        "block_select_32_pages": t(lambda i: replicas[i].block_select(32, stream)),
        "index_reuse_select": t(lambda i: replicas[i].reuse_select(prev_idx[i], prev_lens[i], 1, stream)),
    }
    for db in replicas:
        db.check_status(stream)
    res["unit"] = "us per call (device, CUDA events)"
    return res


# the other MLA workloads timed by the default run, each a 1-GPU figure of its own
EXTRA_WORKLOADS = ("prefill_16k", "decode_1m_planted", "mixed_batch")


def run_extra_workload(name, args, dev, stream, sampler):
    """One more workload of the same path, timed like the headline (inputs larger than L2, one device
    replica), reported with its own stage times, the roofline of its dominant stage against the burst peaks
    and the whole step's roofline."""
    import torch
    from sparse_attention_long_dsa_b200 import workloads as W
    from sparse_attention_long_dsa_b200.pipeline import DeviceBatch

    wl = W.BENCH_WORKLOADS[name](seed=_seed_of(name, 0))
    work = work_of(wl)
    db = DeviceBatch(wl, device=dev)
    # enough steps for a timed region of about 0.2 s (clock samples under load), at least --extra-steps
    probe_ms, _, _, _ = _time_steps([db], stream, 1, args.warmup, 1, dev, None, args.selection)
    steps = int(min(2000, max(args.extra_steps, math.ceil(200.0 / max(probe_ms, 1e-3)))))
    total_ms, stage_avg, launches, clocks = _time_steps_checked([db], stream, steps, 1, 1, dev, sampler, args.selection)
    ms_per_step = total_ms / steps
    peaks, peak_src = load_peaks()
    decode = bool(np.all(wl.q_lens == 1))
    dom = max(stage_avg, key=stage_avg.get)
    res = {"metric": "sparse-attn decode tokens/s" if decode else "sparse-attn prefill tokens/s",
           "value": job_tokens_per_s(work["tokens"], 1, ms_per_step), "unit": "tokens/s", "steps": steps,
           "warmup": args.warmup, "ms_per_step": ms_per_step, "stages_ms": stage_avg, "stages_timing": STAGES_TIMING,
           "roofline": roofline_entry(dom, stage_avg[dom], work, peaks, peak_src, name, decode),
           "stage_rooflines": {s: roofline_entry(s, stage_avg[s], work, peaks, peak_src, name, decode)
                               for s in ("indexer", "attention")},
           "step_roofline": step_roofline(work, peaks, ms_per_step), "gpu_launches": launches, "clocks": clocks,
           "selection": "dsa_indexer_topk (fused; stages_ms.indexer holds scores + selection)"
           if _fused_for(db, args.selection) else "dsa_indexer_scores + dsa_topk",
           "config": workload_config(wl, replicas=1, l2="inputs larger than L2 (one device replica)")}
    # both forms of the first two steps, for the choice between them
    def t2(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            fn()
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n
    n2 = max(3, min(50, steps))
    res["scores_and_selection_ms"] = {
        "dsa_indexer_scores + dsa_topk": t2(lambda: (db.indexer(stream), db.topk(stream)), n2),
        "dsa_indexer_topk (fused)": t2(lambda: db.indexer_topk(stream), n2)}
    db.check_status(stream)
    del db
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local_rank):
    import torch
    from sparse_attention_long_dsa_b200 import binding as B
    from sparse_attention_long_dsa_b200 import workloads as W
    from sparse_attention_long_dsa_b200.pipeline import DeviceBatch

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    B.load()
    wl = W.BENCH_WORKLOADS[args.workload](**({} if args.workload == "tiny_f32" else {"seed": _seed(args, rank)}))
    work = work_of(wl)
    replicas = []
    for r in range(args.replicas):
        replicas.append(DeviceBatch(wl, device=dev))
    stream = torch.cuda.Stream(device=dev)

    sampler = ClockSampler(local_rank)
    sampler.start()
    total_ms, stage_avg, launches, clocks = _time_steps_checked(replicas, stream, args.steps, args.warmup, world, dev,
                                                                sampler, args.selection)
    ms_per_step = total_ms / args.steps
    value = job_tokens_per_s(work["tokens"], world, ms_per_step)

    # e2e: per-step inputs from pinned host memory, results read back, same public calls; first one step
    # after another on one stream, then overlapped across steps (copy-in, compute and copy-out of
    # neighbouring steps on three streams), which is reported when every rank could run it
    e2e_serial = run_e2e(args, wl, replicas[0], stream, dev, world)
    e2e = run_e2e_overlapped(args, wl, replicas[:2], dev, world)
    if e2e is None:
        e2e = dict(e2e_serial)
    else:
        e2e["serial"] = {"value": e2e_serial["value"], "ms_per_step": e2e_serial["ms_per_step"]}

    peaks, peak_src = load_peaks()
    dom = max(stage_avg, key=stage_avg.get)
    decode = bool(np.all(wl.q_lens == 1))
    roof = roofline_entry(dom, stage_avg[dom], work, peaks, peak_src, args.workload, decode)
    res = {
        "metric": "sparse-attn decode tokens/s" if wl.kind == "mla" and np.all(wl.q_lens == 1)
        else "sparse-attn prefill tokens/s",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16+e4m3" if wl.kind == "mla" else "f32", "data": "synthetic",
        "config": workload_config(wl, replicas=args.replicas),
        "stages_ms": stage_avg, "stages_timing": STAGES_TIMING, "roofline": roof, "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks, "impl": "ours",
        "selection": "dsa_indexer_topk (fused; stages_ms.indexer holds scores + selection)"
        if _fused_for(replicas[0], args.selection) else "dsa_indexer_scores + dsa_topk",
    }
    if wl.kind == "mla":
        res["step_roofline"] = step_roofline(work, peaks, ms_per_step)
    if world == 1 and args.workload == "decode_batch" and not args.no_widened:
        res["widened"] = time_widened(replicas, stream, dev)
    del replicas
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    # the other MLA workloads (1 GPU only: under torchrun the ranks would each repeat them)
    extras = [] if (world > 1 or args.workload != "decode_batch") else \
        [w for w in (args.extra_workloads.split(",") if args.extra_workloads else []) if w]
    if extras:
        res["workloads"] = {}
        for name in extras:
            res["workloads"][name] = run_extra_workload(name, args, dev, stream, sampler)
    sampler.stop()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    return res


def _seed_of(workload, rank):
    base = {"decode_batch": 20260002, "prefill_16k": 20260003, "decode_1m_planted": 20260004,
            "mixed_batch": 20260005, "prefill_4k": 20260003}[workload]
    return base + 1000 * rank


def _seed(args, rank):
    return _seed_of(args.workload, rank)


def workload_config(wl, replicas=1, l2=None):
    d = {"workload": wl.name, "batch_seqs": wl.num_seqs, "query_rows": wl.total_q,
         "context": f"{int(wl.seq_lens.min())}..{int(wl.seq_lens.max())}", "topk": wl.topk, "heads": wl.H,
         "d_qk": wl.Dqk, "d_v": wl.Dv, "indexer": f"{wl.Hi}x{wl.Di} {'e4m3' if wl.kind == 'mla' else 'f32'}",
         "page": wl.page_size,
         "l2": l2 or f"{replicas} rotating device replicas of all inputs (> L2 touched between reuses)"}
    return d


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum per launch) of the dominant kernel from one
# ncu capture (profiles/), valid only while what decides that kernel's traffic is as it was captured: the
# source regions below (the file's declarations, the kernel's body and its launch, the shared headers) hash to
# the recorded key.  The plan kernel (whose output the GPU tests hold bit-identical) and the split-combine
# kernels and their launches are left out: they are separate launches with traffic of their own.
# A region is (file, first line pattern or None for the file's start, end line pattern or None for its end,
# whether the end line is included).
MEASURED_TRAFFIC = {
    ("attention", "decode_batch"): {
        "bytes": 84242432 + 3617792,
        "regions": (("attn_mla_tc.cu", None, r"^// -+ plan$", False),
                    ("attn_mla_tc.cu", r"^// -+ main$", r"^// -+ combine$", False),
                    ("attn_mla_tc.cu", r"^// -+ host$", r'DSA_LAUNCH_PDL\("attn_mla_kernel"', True),
                    ("tc.cuh", None, None, False),
                    ("common.cuh", None, None, False)),
        "sha256_16": "ba526663a2be75ee"},
}


def _source_region(text, start, end, end_included):
    """The lines of `text` from the first line matching `start` up to the next line matching `end`."""
    lines = text.split("\n")
    i = 0 if start is None else next(n for n, l in enumerate(lines) if re.search(start, l))
    if end is None:
        j = len(lines)
    else:
        j = next(n for n in range(i + 1, len(lines)) if re.search(end, lines[n])) + (1 if end_included else 0)
    return "\n".join(lines[i:j])


def traffic_key(regions):
    import hashlib
    m = hashlib.sha256()
    for f, start, end, incl in regions:
        with open(os.path.join(ROOT, "sparse_attention_long_dsa_b200", "csrc", f), encoding="utf-8") as fh:
            m.update(_source_region(fh.read(), start, end, incl).encode())
    return m.hexdigest()[:16]


def measured_traffic(stage, workload):
    rec = MEASURED_TRAFFIC.get((stage, workload))
    if rec is None:
        return None
    try:
        key = traffic_key(rec["regions"])
    except (StopIteration, OSError, UnicodeDecodeError):   # a marker line or a file is gone: not the captured sources
        return None
    return rec["bytes"] if key == rec["sha256_16"] else None


def roofline_entry(stage, ms, work, peaks, src, workload, decode):
    """Decode stages are HBM-bound (bytes / HBM copy bandwidth); prefill attention and indexer are
    tensor-bound (flops / the burst dense peak: bf16 for attention, 2x bf16 for the FP8 indexer; each stage
    is timed as one call of milliseconds, not as a seconds-long loop)."""
    w = work[stage]
    secs = ms / 1e3
    tag = f"{src} (MEASURED_PEAKS.json)" if src == "measured" else "fallback"
    if decode or stage == "topk":
        ach = w["bytes"] / secs / 1e9
        peak = peaks["hbm_gbs"]
        return {"kernel": stage, "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                "peak_source": f"{tag} hbm_gbs", "algorithmic_bytes_per_launch": w["bytes"],
                "avg_launch_ms": ms, "traffic": measured_traffic(stage, workload),
                "tflops": w["flops"] / secs / 1e12}
    ach = w["flops"] / secs / 1e12
    fp8 = stage == "indexer"
    peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    return {"kernel": stage, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
            "peak_source": f"{tag} bf16_tflops (burst)" + (" x2 (fp8 = 2x bf16 dense ratio)" if fp8 else ""),
            "algorithmic_flops_per_launch": w["flops"], "avg_launch_ms": ms,
            "traffic": measured_traffic(stage, workload),
            "gbs": w["bytes"] / secs / 1e9}


def run_e2e(args, wl, db, stream, dev, world):
    import torch
    per_step = {}
    for name in ("q", "qI", "w", "block_table", "seq_lens", "cu_q"):
        t = db.inputs[name]
        per_step[name] = (torch.empty(t.shape, dtype=t.dtype, pin_memory=True), t)
        per_step[name][0].copy_(t.cpu())
    out_h = torch.empty(db.out.shape, dtype=db.out.dtype, pin_memory=True)
    lse_h = torch.empty(db.lse.shape, dtype=db.lse.dtype, pin_memory=True)
    h2d = sum(h.numel() * h.element_size() for h, _ in per_step.values())
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()

    def step():
        for h, d in per_step.values():
            d.copy_(h, non_blocking=True)
        _run_step(db, stream, args)
        out_h.copy_(db.out, non_blocking=True)
        lse_h.copy_(db.lse, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize(dev)
    ms = slowest_rank_ms(a.elapsed_time(b), world, dev)
    value = job_tokens_per_s(wl.total_q, world, ms / args.steps)
    return {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": ms / args.steps}


def run_e2e_overlapped(args, wl, sets, dev, world):
    """The e2e leg with neighbouring steps overlapped: step i copies its inputs in on one stream, runs
    the three calls on a second and reads its results back on a third, using device set i % 2 (two
    device replicas, so a step's copy-in never overwrites inputs the previous step is still reading,
    and its results never overwrite outputs still being read back).  Every step still moves its own
    inputs and results across PCIe inside the timed region.  Returns None (on every rank) if any rank
    could not run it, so that all ranks take the same collective steps."""
    import torch
    ok, res = True, None
    if len(sets) < 2:
        ok = False
    try:
        if ok:
            res = _e2e_overlapped_local(args, wl, sets, dev)
    except Exception as ex:                                 # keep the bench line: the serial leg stands
        print(f"[bench] overlapped e2e leg failed: {type(ex).__name__}: {ex}", file=sys.stderr)
        ok = False
    if world > 1:
        t = torch.tensor([1 if ok else 0], dtype=torch.int32, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MIN)
        ok = bool(t.item())
        torch.distributed.barrier()
    if not ok:
        return None
    ms = slowest_rank_ms(res["ms"], world, dev)
    return {"value": job_tokens_per_s(wl.total_q, world, ms / args.steps), "unit": "tokens/s",
            "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"], "ms_per_step": ms / args.steps,
            "pipeline": "copy-in (one packed copy), compute and copy-out of neighbouring steps overlapped on three "
                        "streams, two device input/output sets"}


def _packed_step_inputs(wl, replicas, dev):
    """A step's inputs (q, qI, w and the batch descriptor's arrays) packed into one pinned host buffer, and for
    each replica a batch whose per-step inputs are views into one device buffer of the same layout (its pools
    stay the replica's), so that a step's copy-in is a single copy."""
    import torch
    from sparse_attention_long_dsa_b200.pipeline import DeviceBatch
    arrays = {"q": wl.q, "qI": wl.qI, "w": wl.w, "block_table": wl.block_table.astype(np.int32),
              "seq_lens": wl.seq_lens.astype(np.int32), "cu_q": wl.cu_q.astype(np.int32)}
    tdt = {np.dtype(np.uint16): torch.int16, np.dtype(np.uint8): torch.uint8, np.dtype(np.float32): torch.float32,
           np.dtype(np.int32): torch.int32}
    layout, total = {}, 0
    for n, a in arrays.items():
        a = np.ascontiguousarray(a)
        layout[n] = (total, a)
        total += (a.nbytes + 255) // 256 * 256
    host = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    hn = host.numpy()
    for n, (o, a) in layout.items():
        hn[o: o + a.nbytes] = a.reshape(-1).view(np.uint8)
    batches, bufs = [], []
    for db in replicas:
        dbuf = torch.empty(total, dtype=torch.uint8, device=dev)
        inputs = dict(db.inputs)
        for n, (o, a) in layout.items():
            inputs[n] = dbuf[o: o + a.nbytes].view(tdt[a.dtype]).view(a.shape)
        batches.append(DeviceBatch(wl, device=dev, decode=db.decode, inputs=inputs))
        bufs.append(dbuf)
    return host, bufs, batches


def _e2e_overlapped_local(args, wl, replicas, dev):
    import torch
    host_in, dev_in, sets = _packed_step_inputs(wl, replicas[:2], dev)
    host_out = [(torch.empty(db.out.shape, dtype=db.out.dtype, pin_memory=True),
                 torch.empty(db.lse.shape, dtype=db.lse.dtype, pin_memory=True)) for db in sets]
    h2d = host_in.numel()
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    in_done = [torch.cuda.Event() for _ in range(2)]       # set j's inputs are on the device
    cmp_done = [torch.cuda.Event() for _ in range(2)]      # set j's calls finished (inputs free, outputs ready)
    out_done = [torch.cuda.Event() for _ in range(2)]      # set j's outputs are on the host (outputs free)

    def run(n):
        for i in range(n):
            j = i % 2
            db = sets[j]
            if i >= 2:
                s_in.wait_event(cmp_done[j])
            with torch.cuda.stream(s_in):
                dev_in[j].copy_(host_in, non_blocking=True)
            in_done[j].record(s_in)
            s_cmp.wait_event(in_done[j])
            if i >= 2:
                s_cmp.wait_event(out_done[j])
            _run_step(db, s_cmp, args)
            cmp_done[j].record(s_cmp)
            s_out.wait_event(cmp_done[j])
            with torch.cuda.stream(s_out):
                host_out[j][0].copy_(db.out, non_blocking=True)
                host_out[j][1].copy_(db.lse, non_blocking=True)
            out_done[j].record(s_out)

    run(max(4, args.warmup))
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    run(args.steps)
    s_out.wait_event(cmp_done[(args.steps - 1) % 2])
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    last = (args.steps - 1) % 2
    if not (torch.equal(host_out[last][0], sets[last].out.cpu()) and torch.equal(host_out[last][1], sets[last].lse.cpu())):
        raise RuntimeError("read-back of the last step does not match its device results")
    return {"ms": t0.elapsed_time(t1), "h2d": int(h2d), "d2h": int(d2h)}


# ---------------------------------------------------------------------------------------------- oracle timing
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return 1


def cpu_baseline(wl, budget_s=15.0, rows=None):
    """The oracle as it stands, timed on host cores over a bounded sample of rows of the workload."""
    import oracle
    order = list(range(wl.total_q)) if rows is None else rows
    rng = np.random.default_rng(0)
    if rows is None and len(order) > 64:
        order = sorted(rng.choice(wl.total_q, 64, replace=False).tolist())
    done, t0, passes = 0, time.perf_counter(), 0
    while time.perf_counter() - t0 < budget_s:
        for r in order:
            oracle.run_rows(wl, [r])
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        passes += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "tokens/s", "cores": _blas_threads(), "host_cores": os.cpu_count(),
            "threads": "one Python thread walks the rows; numpy's BLAS calls inside it use up to `cores` threads",
            "kind": "oracle",
            "sample": f"{done} query-row evaluations over {len(order)} rows of {wl.name} (full path per row: "
                      f"scores, top-k, attention), {dt:.1f} s wall"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from sparse_attention_long_dsa_b200 import workloads as W
    import oracle
    wl = W.BENCH_WORKLOADS[args.workload](**({} if args.workload == "tiny_f32" else {"seed": _seed(args, 0)}))
    rows_per_step = 2 if wl.total_q > 1 else 1
    rng = np.random.default_rng(1)

    def step(i):
        rs = [(i * rows_per_step + j) % wl.total_q for j in range(rows_per_step)]
        oracle.run_rows(wl, rs)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = rows_per_step * args.steps / dt
    cores = _blas_threads()
    line = {"metric": "sparse-attn decode tokens/s" if np.all(wl.q_lens == 1) else "sparse-attn prefill tokens/s",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": workload_config(wl, replicas=args.replicas), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "host_cores": os.cpu_count(),
                             "threads": "one Python thread walks the rows; numpy's BLAS calls inside it use up to "
                                        "`cores` threads", "kind": "oracle",
                             "sample": f"{rows_per_step} query rows of {wl.name} per step (bounded sample)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


# ---------------------------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode_batch",
                    choices=["decode_batch", "prefill_16k", "prefill_4k", "decode_1m_planted", "mixed_batch", "tiny_f32"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--replicas", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--extra-workloads", default=",".join(EXTRA_WORKLOADS),
                    help="comma-separated MLA workloads timed after the decode batch at N=1 ('' for none)")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--no-widened", action="store_true", help="skip the timing of the decode step's variants")
    ap.add_argument("--selection", default="auto", choices=["auto", "fused", "separate"],
                    help="scores + selection as one fused call, two calls, or by the pipeline's shape rule")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    distributed = world > 1 and args.impl == "ours"
    if distributed:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        # ranks meet first after drawing their workloads (tens of seconds each, drawn at the same time); a
        # collective left waiting longer than this ends with an error instead of holding the GPUs
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        else:
            res = run_ours(args, rank, world, local_rank)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if distributed:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
