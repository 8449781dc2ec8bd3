"""Comparison rules between the CUDA path and the CPU oracle.

Tolerances, derived from the arithmetic of each step:
* scores, fp32 path: |g - o| <= 2e-5 * A(s); FP8 path: |g - o| <= 1e-4 * A(s), where
  A(s) = kS[s] * sum_j |w_j| * sum_d |qI_jd * kI_sd| bounds every partial sum (fp32
  accumulation of ~200 terms in any order, and tensor-core FP8 accumulation).
  Integer-grid inputs: bit-exact.
* top-k: bit-exact on integer-grid inputs and on the top-k-only test (same fp32 scores on
  both sides); otherwise |G| = |O| and every position in the symmetric difference has an
  oracle score within 1e-3 * max(|tau|, 1e-6 * max|I|) of the oracle's k-th score tau.
* attention on the same index set: fp32 max-abs 1e-5 (out and lse); bf16 max-abs 2e-2
  and mean-rel (sum|g-o| / sum|o|) 1e-2 on out, max-abs 1e-3 on lse.
"""
import copy

import numpy as np

import oracle

SCORE_REL = {"f32": 2e-5, "mla": 1e-4}
TOPK_GAP = 1e-3


def abs_case(case):
    c = copy.copy(case)
    if case.kind == "mla":
        c.qI = case.qI & np.uint8(0x7F)
        c.kI_pool = case.kI_pool & np.uint8(0x7F)
    else:
        c.qI = np.abs(case.qI)
        c.kI_pool = np.abs(case.kI_pool)
    c.w = np.abs(case.w)
    return c


def check_scores(case, row, gpu, ref, acase=None):
    gpu = np.asarray(gpu, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if case.grid:
        bad = np.flatnonzero(gpu != ref)
        assert bad.size == 0, f"row {row}: {bad.size} inexact grid scores, first at {bad[:5]}"
        return
    A = oracle.indexer_scores_row(acase or abs_case(case), row)
    err = np.abs(gpu - ref)
    lim = SCORE_REL[case.kind] * A + 1e-30
    bad = np.flatnonzero(err > lim)
    assert bad.size == 0, f"row {row}: {bad.size} scores out of tolerance, worst rel {np.max(err / (A + 1e-30)):.3e}"


def check_topk(case, row, gpu_idx, ref_scores, exact=None):
    gpu_idx = np.asarray(gpu_idx)
    k = gpu_idx.size
    ref_idx = oracle.topk_row(ref_scores, k)
    if exact is None:
        exact = case.grid
    if exact:
        assert np.array_equal(gpu_idx, ref_idx), f"row {row}: top-k differs at {np.flatnonzero(gpu_idx != ref_idx)[:8]}"
        return
    # structure: ascending valid prefix, -1 padding, positions in range
    n = ref_scores.size
    valid = gpu_idx[gpu_idx >= 0]
    assert np.all(gpu_idx[valid.size:] == -1), f"row {row}: -1 padding not at the end"
    assert np.all(np.diff(valid) > 0) and (valid.size == 0 or (valid[0] >= 0 and valid[-1] < n)), f"row {row}: order"
    rv = ref_idx[ref_idx >= 0]
    assert valid.size == rv.size == min(n, k), f"row {row}: {valid.size} selected, expected {min(n, k)}"
    diff = np.setxor1d(valid, rv)
    if diff.size:
        tau = np.sort(ref_scores)[::-1][k - 1]
        lim = TOPK_GAP * max(abs(tau), 1e-6 * np.abs(ref_scores).max())
        worst = np.abs(ref_scores[diff] - tau).max()
        assert worst <= lim, f"row {row}: {diff.size} differing picks, worst gap {worst:.3e} > {lim:.3e}"


def check_attention(case, row, gpu_out, gpu_lse, ref_out, ref_lse):
    g = np.asarray(gpu_out, dtype=np.float64)
    gl = np.asarray(gpu_lse, dtype=np.float64)
    if case.kind == "f32":
        assert np.max(np.abs(g - ref_out)) <= 1e-5, f"row {row}: out max-abs {np.max(np.abs(g - ref_out)):.3e}"
        assert np.max(np.abs(gl - ref_lse)) <= 1e-5, f"row {row}: lse max-abs {np.max(np.abs(gl - ref_lse)):.3e}"
    else:
        mx = np.max(np.abs(g - ref_out))
        mr = np.sum(np.abs(g - ref_out)) / max(np.sum(np.abs(ref_out)), 1e-30)
        assert mx <= 2e-2, f"row {row}: out max-abs {mx:.3e}"
        assert mr <= 1e-2, f"row {row}: out mean-rel {mr:.3e}"
        assert np.max(np.abs(gl - ref_lse)) <= 1e-3, f"row {row}: lse max-abs {np.max(np.abs(gl - ref_lse)):.3e}"


def sample_rows(case, extra=8, seed=0):
    """Rows at sequence edges (first / last row of each sequence, around 2047/2048) plus random ones."""
    rows = set()
    for b in range(case.num_seqs):
        lo, hi = int(case.cu_q[b]), int(case.cu_q[b + 1])
        if hi > lo:
            rows.update({lo, hi - 1})
            n0 = int(case.seq_lens[b]) - (hi - lo)
            for p in (63, 64, 2046, 2047, 2048, 2049):
                r = lo + p - n0
                if lo <= r < hi:
                    rows.add(r)
    rng = np.random.default_rng(seed)
    if case.total_q:
        rows.update(int(r) for r in rng.integers(0, case.total_q, extra))
    return sorted(rows)


def compare_rows(case, db, rows, check_out=True):
    """Full-path parity for the given rows of a DeviceBatch that has run."""
    gs = db.scores.cpu().numpy() if case.total_q * db.ld < (1 << 28) else None
    gi = db.idx.cpu().numpy()
    go = db.out.float().cpu().numpy() if check_out else None
    gl = db.lse.cpu().numpy() if check_out else None
    acase = None if case.grid else abs_case(case)
    ref = oracle.run_rows(case, rows, want_attention=False)
    for r in rows:
        _, pos = oracle.row_location(case.seq_lens, case.cu_q, r)
        g_sc = gs[r, : pos + 1] if gs is not None else db.scores[r, : pos + 1].cpu().numpy()
        check_scores(case, r, g_sc, ref[r]["scores"], acase)
        check_topk(case, r, gi[r], ref[r]["scores"])
        if check_out:
            o, l = oracle.sparse_attention_row(case, r, gi[r])      # attention on the GPU's own index set
            check_attention(case, r, go[r], gl[r], o, l)
    return ref
