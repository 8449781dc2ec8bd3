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


def candidates_per_row(case):
    """n(row) = pos(row) + 1 for every query row (a sequence's rows are its last q_len tokens)."""
    b = case.row_seq()
    first = np.asarray(case.cu_q[:-1], np.int64)[b]
    q_len = np.asarray(case.q_lens, np.int64)[b]
    return np.asarray(case.seq_lens, np.int64)[b] - q_len + (np.arange(case.total_q) - first) + 1


def check_topk_every_row(case, scores, idx, rows_per_chunk=256):
    """The selection of every row against properties that fix the top-k of the given scores exactly: min(n, k)
    entries, ascending, in [0, n), -1 only after them; no unselected score above the smallest selected one; and
    among the keys tied at that score, the selected ones before the unselected ones (ties go to the lower
    position; -0 and +0 compare equal).  `scores` [T, ld] and `idx` [T, k] are torch tensors on any device (the
    GPU's own scores: the rule is checked on the values the selection saw); rows go in chunks to bound memory."""
    import torch
    n_all = candidates_per_row(case)
    T, k = idx.shape
    dev = idx.device
    for r0 in range(0, T, rows_per_chunk):
        r1 = min(T, r0 + rows_per_chunk)
        n = torch.as_tensor(n_all[r0:r1], device=dev)
        L = int(n_all[r0:r1].max())
        pos = torch.arange(L, device=dev)
        live = pos[None, :] < n[:, None]
        S = torch.where(live, scores[r0:r1, :L].float(), torch.tensor(float("-inf"), device=dev))
        I = idx[r0:r1].long()
        valid = I >= 0
        want = torch.clamp(n, max=k)
        where = f"rows {r0}..{r1 - 1}"
        assert torch.equal(valid.sum(1), want), f"{where}: wrong number of selected positions"
        assert torch.equal(valid, torch.arange(k, device=dev)[None, :] < want[:, None]), f"{where}: -1 inside"
        assert bool((I < n[:, None]).all()), f"{where}: a position past the row's candidates"
        assert bool(((I[:, 1:] > I[:, :-1]) | ~valid[:, 1:]).all()), f"{where}: positions not ascending"
        # how often each position is selected (the -1 entries land in a spare column L)
        cnt = torch.zeros((r1 - r0, L + 1), dtype=torch.int32, device=dev)
        cnt.scatter_add_(1, torch.where(valid, I, torch.full_like(I, L)), torch.ones_like(I, dtype=torch.int32))
        assert bool((cnt[:, :L] <= 1).all()), f"{where}: a position selected twice"
        sel = cnt[:, :L] > 0
        full = n <= k                                          # every candidate selected: nothing to rank
        inf = torch.tensor(float("inf"), device=dev)
        tau = torch.where(sel, S, inf).min(1).values
        unsel = live & ~sel
        top_out = torch.where(unsel, S, -inf).max(1).values
        bad = ~full & (top_out > tau)
        assert not bool(bad.any()), f"{where}: an unselected score above the threshold (row {r0 + int(bad.nonzero()[0])})"
        tied = S == tau[:, None]
        last_sel = torch.where(sel & tied, pos[None, :], torch.full_like(pos, -1)[None, :]).max(1).values
        first_out = torch.where(unsel & tied, pos[None, :], torch.full_like(pos, L)[None, :]).min(1).values
        bad = ~full & (last_sel > first_out)
        assert not bool(bad.any()), f"{where}: a tie at the threshold went to a higher position (row {r0 + int(bad.nonzero()[0])})"
