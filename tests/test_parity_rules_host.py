"""The GPU parity rules (`tests/parity.py`) on the CPU: they accept the oracle's own results and results that
differ only within the stated tolerance (fp32 rounding of scores, bf16 rounding of the attention output, a
swap between keys tied at the k-th score), and reject a result with one planted error (no GPU).

The GPU tests feed the kernels' outputs to these rules, so a rule that let a wrong score, a wrong index, a
misplaced -1 or a shifted output through would make every GPU parity test vacuous there.
"""
import numpy as np
import pytest

import oracle
import parity
from sparse_attention_long_dsa_b200 import workloads as W


def _case(kind, grid):
    if kind == "mla":
        return W.make_workload("rules", kind="mla", seed=91, seq_lens=[300, 150], q_lens=[2, 2], topk=32, grid=grid,
                               H=4, Dqk=40, Dv=32, Hi=3, Di=16)
    return W.make_workload("rules", kind="f32", seed=92, seq_lens=[300, 150], q_lens=[2, 2], topk=32, grid=grid,
                           H=3, Dqk=16, Dv=12, Hi=2, Di=8)


def _fails(fn, *a, **kw):
    with pytest.raises(AssertionError):
        fn(*a, **kw)


def _bf16(x):
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("kind", ["f32", "mla"])
def test_score_rule(kind):
    case = _case(kind, grid=False)
    acase = parity.abs_case(case)
    for row in range(case.total_q):
        ref = oracle.indexer_scores_row(case, row)
        A = oracle.indexer_scores_row(acase, row)
        parity.check_scores(case, row, ref, ref, acase)
        parity.check_scores(case, row, ref.astype(np.float32), ref, acase)          # fp32 rounding passes
        bad = ref.copy()
        s = int(np.argmax(A))
        bad[s] += 2 * parity.SCORE_REL[case.kind] * A[s]                           # twice the bound at one key
        _fails(parity.check_scores, case, row, bad, ref, acase)
        _fails(parity.check_scores, case, row, ref[:-1], ref, acase)               # causal bound one short


def test_score_rule_is_exact_on_the_grid():
    case = _case("mla", grid=True)
    ref = oracle.indexer_scores_row(case, 0)
    parity.check_scores(case, 0, ref, ref)
    bad = ref.copy()
    j = int(np.flatnonzero(ref != 0)[0])
    bad[j] = np.nextafter(np.float32(ref[j]), np.float32(np.inf))                  # one fp32 ulp
    _fails(parity.check_scores, case, 0, bad, ref)


def test_topk_rule_exact():
    case = _case("mla", grid=True)
    for row in range(case.total_q):
        sc = oracle.indexer_scores_row(case, row)
        ref = oracle.topk_row(sc, case.topk)
        parity.check_topk(case, row, ref, sc)
        order = np.lexsort((np.arange(sc.size), -sc))
        # the first unselected key in the top-k order (ties included) swapped in for the last selected one
        outside = int(order[case.topk])
        bad = np.sort(np.concatenate([ref[ref != order[case.topk - 1]], [outside]]))
        _fails(parity.check_topk, case, row, bad, sc)


def test_topk_rule_with_tolerance():
    case = _case("f32", grid=False)
    k = case.topk
    for row in range(case.total_q):
        sc = oracle.indexer_scores_row(case, row)
        ref = oracle.topk_row(sc, k)
        parity.check_topk(case, row, ref, sc)
        order = np.lexsort((np.arange(sc.size), -sc))
        # a key tied with the k-th score (made so) may stand in for it
        tied = sc.copy()
        tied[order[k]] = tied[order[k - 1]]
        swap = np.sort(np.concatenate([ref[ref != order[k - 1]], [order[k]]]))
        parity.check_topk(case, row, swap, tied)
        # the worst key in place of the k-th is a real error
        worst = np.sort(np.concatenate([ref[ref != order[k - 1]], [order[-1]]]))
        _fails(parity.check_topk, case, row, worst, sc)
        _fails(parity.check_topk, case, row, ref[::-1].copy(), sc)                  # not ascending
        pad = ref.copy()
        pad[0] = -1
        _fails(parity.check_topk, case, row, pad, sc)                             # -1 before the end
        out_of_range = ref.copy()
        out_of_range[-1] = sc.size                                                 # one past the causal bound
        _fails(parity.check_topk, case, row, out_of_range, sc)


def test_topk_rule_counts_short_rows():
    """A row with fewer candidates than k selects all of them, then -1."""
    case = _case("f32", grid=False)
    sc = np.arange(10, dtype=np.float64)
    ref = oracle.topk_row(sc, 16)
    parity.check_topk(case, 0, ref, sc)
    short = ref.copy()
    short[9] = -1
    _fails(parity.check_topk, case, 0, short, sc)


@pytest.mark.parametrize("kind", ["f32", "mla"])
def test_attention_rule(kind):
    case = _case(kind, grid=False)
    for row in range(case.total_q):
        sc = oracle.indexer_scores_row(case, row)
        idx = oracle.topk_row(sc, case.topk)
        o, l = oracle.sparse_attention_row(case, row, idx)
        parity.check_attention(case, row, o, l, o, l)
        if case.kind == "mla":
            parity.check_attention(case, row, _bf16(o), l.astype(np.float32), o, l)   # bf16 output passes
            shift = 0.03
        else:
            parity.check_attention(case, row, o.astype(np.float32), l.astype(np.float32), o, l)
            shift = 2e-5
        one = o.copy()
        one[1, 3] += shift                                                         # one element off
        _fails(parity.check_attention, case, row, one, l, o, l)
        lse = l.copy()
        lse[0] += 2e-3 if case.kind == "mla" else 2e-5
        _fails(parity.check_attention, case, row, o, lse, o, l)
        # attention over another index set (the last selected key dropped)
        o2, l2 = oracle.sparse_attention_row(case, row, idx[:-1])
        _fails(parity.check_attention, case, row, o2, l2, o, l)


def test_attention_rule_mean_relative_bound():
    """A uniform 2 % scale of an output no larger than 0.5 stays under the max-abs bound (0.01 <= 0.02) but fails
    the mean-relative one."""
    case = _case("mla", grid=False)
    sc = oracle.indexer_scores_row(case, 0)
    o, l = oracle.sparse_attention_row(case, 0, oracle.topk_row(sc, case.topk))
    small = 0.5 * o / np.abs(o).max()
    parity.check_attention(case, 0, small, l, small, l)
    with pytest.raises(AssertionError, match="mean-rel"):
        parity.check_attention(case, 0, small * 1.02, l, small, l)


def _scored_case(tied):
    """A 4-row case, its scores (garbage past each row's candidates, as the kernels leave them) and the
    oracle's selection of every row."""
    import torch
    case = W.make_workload("rows", kind="f32", seed=93, seq_lens=[300, 150, 20], q_lens=[2, 2, 1], topk=32,
                           H=3, Dqk=16, Dv=12, Hi=2, Di=8)
    rng = np.random.default_rng(94 if tied else 95)
    ld = 304
    sc = (rng.integers(-2, 3, (case.total_q, ld)) if tied else rng.standard_normal((case.total_q, ld))).astype(np.float32)
    if tied:
        sc[0, ::7] = -0.0                                                       # -0 ties +0
    n = parity.candidates_per_row(case)
    idx = np.stack([oracle.topk_row(sc[r, : n[r]].astype(np.float64), case.topk) for r in range(case.total_q)])
    sc[np.arange(ld)[None, :] >= n[:, None]] = 1e30                            # never read
    return case, torch.from_numpy(sc), torch.from_numpy(idx), n


def test_candidates_per_row_by_hand():
    case, _, _, n = _scored_case(False)
    assert n.tolist() == [299, 300, 149, 150, 20]


@pytest.mark.parametrize("tied", [False, True])
def test_every_row_rule_accepts_the_definition(tied):
    case, sc, idx, _ = _scored_case(tied)
    for chunk in (1, 2, 256):
        parity.check_topk_every_row(case, sc, idx, rows_per_chunk=chunk)


def test_every_row_rule_rejects_planted_errors():
    import torch
    case, sc, idx, n = _scored_case(True)
    k = case.topk
    r = 2                                                                         # 149 candidates, k = 32
    s = sc[r, : n[r]].double().numpy()
    sel = idx[r].numpy()
    tau = s[sel].min()
    out = np.setdiff1d(np.arange(n[r]), sel)

    def planted(fn):
        bad = idx.clone()
        fn(bad[r])
        with pytest.raises(AssertionError):
            parity.check_topk_every_row(case, sc, bad)

    lower = out[s[out] < tau][0]                       # a key strictly below the threshold
    tied_out = out[s[out] == tau]                      # keys tied at the threshold left out (higher positions)
    last_tied_in = sel[s[sel] == tau].max()
    assert tied_out.size and tied_out.min() > last_tied_in

    def swap(row, old, new):
        v = row.numpy()
        v[v == old] = new
        v.sort()

    planted(lambda row: swap(row, sel[np.argmin(s[sel])], lower))                # below the threshold
    planted(lambda row: swap(row, last_tied_in, tied_out.max()))                 # tie to a higher position
    planted(lambda row: row.__setitem__(k - 1, -1))                              # one short
    planted(lambda row: row.__setitem__(0, -1))                                  # -1 first
    planted(lambda row: row.__setitem__(k - 1, int(n[r])))                       # past the candidates
    planted(lambda row: row.__setitem__(1, int(row[0])))                         # one position twice
    planted(lambda row: row.copy_(torch.flip(row, [0])))                         # descending
    # a row with fewer candidates than k must select all of them
    bad = idx.clone()
    bad[4, 19] = -1
    with pytest.raises(AssertionError):
        parity.check_topk_every_row(case, sc, bad)
