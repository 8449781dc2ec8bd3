"""The fused selection's algorithm, run on the CPU step by step as `select_stream_kernel` takes it, against the
oracle's top-k (no GPU).

The kernel splits a row into C contiguous slices (one CTA each).  The leading 11 bits of the order-preserving
key come from a row histogram (the indexer's, or a counting pass); while the keys at or above the threshold
digit would not fit the survivor capacity, counting passes over the slices fix the next digit (11, 11, 10
bits), each from the sum of the slices' histograms; when every bit is fixed, only the first `need` keys equal to
the threshold (the earlier slices' first) are kept.  Each slice keeps its survivors in position order; the
remaining digits are fixed on the survivors, stopping once the prefix's bin holds exactly the keys still needed;
each slice then writes every survivor above the prefix and the row's first `need` equal to it, offset by the
counts of the slices before it.  The GPU tests check the kernel itself against the oracle; this checks that the
steps compose to the top-k's definition (score descending, position ascending; -0 == +0) under ties, all-equal
rows, signed zeros, tiny magnitudes, keys that differ only in their last bits, small capacities that force every
counting pass, and 1 to 16 slices.  (Dropping the last digit pass, taking one equal key too many, halving a
digit's bins or offsetting a slice by all of the earlier slices' equal keys each fail it.)  The decode top-k
(`topk_rows_smem_kernel`) is checked the same way.
"""
import numpy as np
import pytest

import oracle


def _okey(scores):
    """fp32 -> u32 key whose unsigned order is the float order, -0 folded onto +0."""
    u = np.asarray(scores, np.float32).view(np.uint32).astype(np.uint64)
    u = np.where(u == 0x80000000, 0, u)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


def _find_bin(h, need):
    """Bin holding the need-th key from the top, and the count of keys in higher bins."""
    above = np.concatenate([np.cumsum(h[::-1])[::-1][1:], [0]])     # keys in bins above each bin
    d = int(np.flatnonzero((above < need) & (above + h >= need)).max())
    return d, int(above[d])


def _select(scores, k, C, cap, use_hist):
    n = scores.size
    keys = _okey(scores)
    if n <= k:
        return np.array([j if j < n else -1 for j in range(k)], np.int32)
    per = ((n + C - 1) // C + 3) & ~3
    slices = [(min(n, r * per), min(n, min(n, r * per) + per)) for r in range(C)]
    P = M = 0
    above, need, bin_cnt, shift = 0, k, n, 32
    local_eq = [0] * C
    if use_hist:
        d, ab = _find_bin(np.bincount((keys >> 21).astype(np.int64), minlength=2048), need)
        P, M, above, need, shift = d << 21, 0xFFE00000, ab, need - ab, 21
        bin_cnt = int(((keys & M) == P).sum())

    def digit_pass(parts, shift):
        nbits = 10 if shift == 10 else 11
        ns, nb = shift - nbits, 1 << nbits
        hs = [np.bincount(((p[(p & M) == P] >> ns) & (nb - 1)).astype(np.int64), minlength=nb) for p in parts]
        return ns, nb, hs

    # counting passes over the slices while the survivors would not fit
    while shift > 0 and (shift == 32 or above + bin_cnt > cap):
        ns, nb, hs = digit_pass([keys[lo:hi] for lo, hi in slices], shift)
        d, ab = _find_bin(sum(hs), need)
        P, M = P | (d << ns), M | ((nb - 1) << ns)
        above, need, bin_cnt, shift = above + ab, need - ab, int(sum(hs)[d]), ns
        local_eq = [int(h[d]) for h in hs]
    full = shift == 0
    eq_before = np.concatenate([[0], np.cumsum(local_eq)[:-1]])
    # storing pass: each slice's survivors in position order
    surv = []
    for r, (lo, hi) in enumerate(slices):
        km = keys[lo:hi] & M
        eq = km == P
        keep = km > P
        if full:
            keep |= eq & (eq_before[r] + np.cumsum(eq) - 1 < need)
        else:
            keep |= eq
        assert keep.sum() <= cap
        surv.append((keys[lo:hi][keep], np.arange(lo, hi)[keep]))
    # remaining digits on the survivors
    while shift > 0 and bin_cnt != need:
        ns, nb, hs = digit_pass([s for s, _ in surv], shift)
        d, ab = _find_bin(sum(hs), need)
        P, M = P | (d << ns), M | ((nb - 1) << ns)
        above, need, bin_cnt, shift = above + ab, need - ab, int(sum(hs)[d]), ns
    # ordered write per slice, offset by the earlier slices' counts
    out = np.full(k, -1, np.int32)
    gt_n = [int(((s & M) > P).sum()) for s, _ in surv]
    eq_n = [int(((s & M) == P).sum()) for s, _ in surv]
    for r, (s, pos) in enumerate(surv):
        eq_seen = sum(eq_n[:r])
        base = sum(g + max(0, min(e, need - sum(eq_n[:c]))) for c, (g, e) in enumerate(zip(gt_n[:r], eq_n[:r])))
        km = s & M
        eq = km == P
        take = (km > P) | (eq & (eq_seen + np.cumsum(eq) - 1 < need))
        sel = pos[take]
        out[base: base + sel.size] = sel[: max(0, k - base)]
    return out


def _rows(seed):
    rng = np.random.default_rng(seed)
    for n in (5, 100, 2049, 3000, 9000, 20000):
        yield rng.standard_normal(n).astype(np.float32)
        yield rng.integers(-3, 4, n).astype(np.float32)                 # heavy ties
        yield rng.integers(0, n // 300 + 2, n).astype(np.float32)       # ~300 keys per level: a tied threshold
                                                                         # with keys above it in every slice
        yield np.zeros(n, np.float32)                                    # all equal
        z = np.zeros(n, np.float32)
        z[::2] = -0.0                                                    # signed zeros tie
        yield z
        yield (rng.standard_normal(n) * 1e-30).astype(np.float32)       # tiny magnitudes
        # consecutive floats in [1, 2), shuffled: the keys agree on their top bits and differ in the last ones,
        # so the threshold is found only by the final 10-bit digit
        yield rng.permutation(np.float32(1.0) + np.arange(n, dtype=np.float32) * np.float32(2.0 ** -23))


@pytest.mark.parametrize("k", [1, 7, 100, 2048])
def test_selection_steps_reproduce_the_topk_definition(k):
    rng = np.random.default_rng(1000 + k)
    for t, s in enumerate(_rows(k)):
        C = int(rng.choice([1, 2, 4, 16]))
        cap = max(k, int(rng.choice([k, 2 * k, 8192])))                 # small capacities force counting passes
        got = _select(s, k, C, cap, use_hist=bool(t % 2))
        exp = oracle.topk_row(s.astype(np.float64), k)
        assert np.array_equal(got, exp), f"case {t}: n={s.size} k={k} C={C} cap={cap}"


def _topk_slices(scores, k, C):
    """The steps of `topk_rows_smem_kernel` (a row in C slices of a cluster): 11-, 11- and 10-bit digits, each
    chosen from the sum of the slices' histograms of the keys matching the prefix; the passes stop as soon as the
    threshold bin holds exactly the keys still needed, and the keys are then compared on the digits fixed so far;
    each slice writes its keys above the threshold and its share of the row's first keys equal to it, in position
    order, offset by the slices before it."""
    n = scores.size
    keys = _okey(scores)
    if n <= k:
        return np.array([j if j < n else -1 for j in range(k)], np.int32)
    per = ((n + C - 1) // C + 3) & ~3
    slices = [(min(n, r * per), min(n, min(n, r * per) + per)) for r in range(C)]
    prefix = pmask = 0
    k_rem = k
    for shift, nb in ((21, 2048), (10, 2048), (0, 1024)):
        hist = sum(np.bincount(((keys[lo:hi][(keys[lo:hi] & pmask) == prefix] >> shift) & (nb - 1)).astype(np.int64),
                               minlength=nb) for lo, hi in slices)
        d, ab = _find_bin(hist, k_rem)
        prefix, pmask, k_rem = prefix | (d << shift), pmask | ((nb - 1) << shift), k_rem - ab
        if hist[d] == k_rem:
            break
    out = np.full(k, -1, np.int32)
    counts = [(int(((keys[lo:hi] & pmask) > prefix).sum()), int(((keys[lo:hi] & pmask) == prefix).sum()))
              for lo, hi in slices]
    for r, (lo, hi) in enumerate(slices):
        out_base = eq_base = 0
        for g, e in counts[:r]:
            out_base += g + (min(e, k_rem - eq_base) if k_rem > eq_base else 0)
            eq_base += e
        km = keys[lo:hi] & pmask
        eq = km == prefix
        take = (km > prefix) | (eq & (eq_base + np.cumsum(eq) - 1 < k_rem))
        sel = np.arange(lo, hi)[take]
        out[out_base: out_base + sel.size] = sel[: max(0, k - out_base)]
    return out


@pytest.mark.parametrize("k", [1, 7, 100, 2048])
def test_topk_slice_steps_reproduce_the_topk_definition(k):
    rng = np.random.default_rng(2000 + k)
    for t, s in enumerate(_rows(k + 1)):
        C = int(rng.choice([1, 2, 4, 8]))
        got = _topk_slices(s, k, C)
        exp = oracle.topk_row(s.astype(np.float64), k)
        assert np.array_equal(got, exp), f"case {t}: n={s.size} k={k} C={C}"
