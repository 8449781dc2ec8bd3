"""Host-side accounting of bench.py (no GPU): the algorithmic bytes and flops credited per stage follow the
definitions (each causal indexer key once, each selected latent row once, plus q, w and out), and the
whole-step roofline combines them as max(fp8 / P_fp8 + bf16 / P_bf16, bytes / BW)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_attention_long_dsa_b200 import workloads as W  # noqa: E402


def test_work_of_two_decode_rows_by_hand():
    # contexts 100 and 3000, one query each (the last token), top-k 2048
    wl = W.make_workload("acct", kind="mla", seed=1, seq_lens=[100, 3000], q_lens=[1, 1], topk=2048)
    w = bench.work_of(wl)
    keys = 100 + 3000                                  # causal indexer keys, 128 e4m3 + 4-byte scale each
    assert w["indexer"]["bytes"] == keys * 132 + 2 * 64 * (128 + 4)      # + qI rows and w
    assert w["indexer"]["flops"] == keys * 2 * 64 * 128
    rows = 100 + 2048                                  # selected latent rows (all 100 of the short context)
    assert w["selected_rows"] == rows
    assert w["attention"]["bytes"] == rows * 1152 + 2 * 128 * (576 * 2 + 512 * 2)   # + q and out, bf16
    assert w["attention"]["flops"] == rows * 2 * 128 * (576 + 512)
    assert w["topk"]["bytes"] == keys * 4 + 2 * 2048 * 4


def test_step_roofline_tensor_and_hbm_bound():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0, "bf16_tflops_sustained": 90.0}
    work = {"indexer": {"bytes": 1e9, "flops": 2e12}, "topk": {"bytes": 5e9, "flops": 0.0},
            "attention": {"bytes": 1e9, "flops": 1e12}}
    r = bench.step_roofline(work, peaks, 40.0)
    # fp8 at 200 TF/s: 10 ms; bf16: 10 ms; bytes 2 GB (top-k's round trip not credited) at 1 TB/s: 2 ms
    assert r["bound"] == "tensor" and r["t_roof_us"] == pytest.approx(20e3) and r["frac"] == pytest.approx(0.5)
    work["attention"]["bytes"] = 29e9
    r = bench.step_roofline(work, peaks, 60.0)
    assert r["bound"] == "hbm" and r["t_roof_us"] == pytest.approx(30e3) and r["frac"] == pytest.approx(0.5)


def _csrc_copy(tmp_path, edit=None):
    """A copy of the attention kernel's sources under tmp_path (laid out like the package), one file edited."""
    import shutil
    d = tmp_path / "sparse_attention_long_dsa_b200" / "csrc"
    d.mkdir(parents=True)
    src = os.path.join(bench.ROOT, "sparse_attention_long_dsa_b200", "csrc")
    for f in ("attn_mla_tc.cu", "tc.cuh", "common.cuh"):
        shutil.copy(os.path.join(src, f), d / f)
    if edit is not None:
        f, old, new = edit
        text = (d / f).read_text()
        assert text.count(old) == 1, old
        (d / f).write_text(text.replace(old, new))
    return str(tmp_path)


@pytest.mark.parametrize("edit,kept", [
    (None, True),
    # the combine kernels and their launch, and the plan kernel, are launches of their own
    (("attn_mla_tc.cu", "constexpr int kCombineRegSplits = 8;", "constexpr int kCombineRegSplits = 4;"), True),
    (("attn_mla_tc.cu", "constexpr int kAttPlanThreads = 256;", "constexpr int kAttPlanThreads = 128;"), True),
    # the kernel's declarations, its body, its launch and the shared headers decide its traffic
    (("attn_mla_tc.cu", "constexpr int kAttNBuf = 3;", "constexpr int kAttNBuf = 2;"), False),
    (("attn_mla_tc.cu", "const int pairs = std::min(max_pairs, units);", "const int pairs = max_pairs;"), False),
    (("attn_mla_tc.cu", "// ------------------------------------------------------------------------------------------------ main",
      "// main"), False),                                                            # a marker gone
])
def test_measured_traffic_follows_the_captured_kernel(tmp_path, monkeypatch, edit, kept):
    rec = bench.MEASURED_TRAFFIC[("attention", "decode_batch")]
    assert bench.measured_traffic("attention", "decode_batch") in (rec["bytes"], None)
    base = bench.traffic_key(rec["regions"])
    monkeypatch.setattr(bench, "ROOT", _csrc_copy(tmp_path, edit))
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("attention", "decode_batch"), dict(rec, sha256_16=base))
    assert (bench.measured_traffic("attention", "decode_batch") == rec["bytes"]) == kept
    assert bench.measured_traffic("attention", "prefill_16k") is None                # no capture recorded


@pytest.mark.parametrize("clocks,rejected", [
    (None, False),                                                                   # no NVML: nothing to judge
    ({"sm_mhz": None, "sm_max_mhz": 1965, "reasons": []}, False),
    ({"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": []}, False),
    ({"sm_mhz": 1330.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}, False),     # power cap: kept, noted
    ({"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"]}, True),
    ({"sm_mhz": 1800.0, "sm_max_mhz": 1965, "reasons": ["sw_thermal_slowdown"]}, True),
    ({"sm_mhz": 1500.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap", "hw_thermal_slowdown"]}, True),
    ({"sm_mhz": 1100.0, "sm_max_mhz": 1965, "reasons": []}, True),                   # well below max, no reason
    ({"sm_mhz": 1700.0, "sm_max_mhz": 1965, "reasons": []}, False),
])
def test_clock_record_rejection(clocks, rejected):
    assert bench.clocks_rejected(clocks) == rejected


def test_rejected_timed_region_is_measured_once_more(monkeypatch):
    records = [{"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"]},
               {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"]},
               {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": []}]
    calls = []

    def fake(replicas, stream, steps, warmup, world, dev, sampler, selection):
        calls.append(len(calls))
        return 10.0 + len(calls), {"attention": 1.0}, 6, records[len(calls) - 1]

    monkeypatch.setattr(bench, "_time_steps", fake)
    ms, stages, launches, clocks = bench._time_steps_checked(None, None, 1, 3, 1, "cpu", None, "auto")
    # once more, not more: the second region is reported (still rejected: the record says so)
    assert len(calls) == 2 and ms == 12.0 and launches == 6
    assert clocks["reasons"] == ["hw_slowdown"] and clocks["rejected_first"] == records[0]
    calls.clear()
    records[0] = records[2]
    ms, _, _, clocks = bench._time_steps_checked(None, None, 1, 3, 1, "cpu", None, "auto")
    assert len(calls) == 1 and ms == 11.0 and "rejected_first" not in clocks
