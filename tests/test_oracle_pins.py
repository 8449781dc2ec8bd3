"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks one oracle function against hand-worked values (tests/golden),
exact rational arithmetic, a torch library routine, or an independent brute
force, chosen so that a plausible slip (a dropped scale, a wrong causal bound,
a reversed tie-break, a transposed operand) fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_dsa_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _single_row_case(qI, kI, w, kS=None, q=None, kv=None, v=None, topk=4, scale=1.0, page=64):
    """One sequence whose last token is the only query; tokens laid out contiguously."""
    qI = np.asarray(qI, np.float32)
    kI = np.asarray(kI, np.float32)
    n = kI.shape[0]
    nb = (n + page - 1) // page
    def paged(a):
        a = np.asarray(a, np.float32)
        out = np.zeros((nb * page,) + a.shape[1:], np.float32)
        out[:n] = a
        return out.reshape((nb, page) + a.shape[1:])
    return SimpleNamespace(
        kind="f32", page_size=page, seq_lens=np.array([n], np.int32), cu_q=np.array([0, 1], np.int32),
        block_table=np.arange(nb, dtype=np.int32)[None, :], qI=qI[None], w=np.asarray(w, np.float32)[None],
        kI_pool=paged(kI), kS_pool=None if kS is None else paged(kS),
        q=None if q is None else np.asarray(q, np.float32)[None], kv_pool=None if kv is None else paged(kv),
        v_pool=None if v is None else paged(v), Dqk=None if kv is None else np.asarray(kv).shape[1],
        Dv=None if v is None else np.asarray(v).shape[1], topk=topk, softmax_scale=scale)


# ----------------------------------------------------------------------------- storage formats

def test_e4m3_table_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = oracle.E4M3
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), ~finite)
    assert np.array_equal(ours[finite], ref[finite])


def test_e4m3_definition_points():
    # largest finite, one, smallest subnormal, smallest normal, negative one, zero / minus zero
    assert oracle.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert oracle.e4m3_decode(np.array([0x38]))[0] == 1.0
    assert oracle.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert oracle.e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6
    assert oracle.e4m3_decode(np.array([0xB8]))[0] == -1.0
    assert oracle.e4m3_decode(np.array([0x00]))[0] == 0.0
    assert math.copysign(1.0, oracle.e4m3_decode(np.array([0x80]))[0]) == -1.0


def test_bf16_decode_matches_torch():
    bits = np.random.default_rng(1).integers(0, 1 << 16, 4096, dtype=np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]                       # finite only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_decode(bits), ref)


def test_generator_encoders_match_torch():
    x = np.random.default_rng(2).standard_normal(20000).astype(np.float32) * 60
    x = np.concatenate([x, [448.0, -448.0, 2 ** -9, 2 ** -10, 3 * 2 ** -11, 0.0, 240.0, 241.0, 232.0]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(W.e4m3_encode(x), ref)
    ref16 = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(W.bf16_encode(x), ref16)


# ----------------------------------------------------------------------------- layout

def test_row_location_hand():
    seq_lens = np.array([10, 3, 7], np.int32)
    cu_q = np.array([0, 1, 4, 6], np.int32)          # q_lens 1, 3, 2
    got = [oracle.row_location(seq_lens, cu_q, r) for r in range(6)]
    assert got == [(0, 9), (1, 0), (1, 1), (1, 2), (2, 5), (2, 6)]


def test_token_slots_hand():
    table = np.array([5, 2, 9], np.int32)
    blk, slot = oracle.token_slots(table, np.array([0, 63, 64, 130]), 64)
    assert blk.tolist() == [5, 5, 2, 9] and slot.tolist() == [0, 63, 0, 2]


# ----------------------------------------------------------------------------- indexer

@pytest.mark.parametrize("case", _golden("indexer_hand.json")["cases"], ids=lambda c: c["name"])
def test_indexer_hand(case):
    c = _single_row_case(case["qI"], case["kI"], case["w"])
    got = oracle.indexer_scores_row(c, 0)
    assert got.tolist() == case["scores"]


def _fraction_score(wl, row, s):
    """Exact rational score from torch's own decoders: sum_j w_j * max(0, sum_d q_jd * kS * k_sd)."""
    b, pos = oracle.row_location(wl.seq_lens, wl.cu_q, row)
    assert s <= pos
    blk = int(wl.block_table[b, s // wl.page_size]); slot = s % wl.page_size
    if wl.kind == "mla":
        dec = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        q = dec(wl.qI[row]); k = dec(wl.kI_pool[blk, slot]); ks = Fraction(float(wl.kS_pool[blk, slot]))
    else:
        q = wl.qI[row].astype(np.float64); k = wl.kI_pool[blk, slot].astype(np.float64); ks = Fraction(1)
    tot = Fraction(0)
    for j in range(q.shape[0]):
        d = sum(Fraction(float(q[j, i])) * ks * Fraction(float(k[i])) for i in range(q.shape[1]))
        tot += Fraction(float(wl.w[row, j])) * max(d, Fraction(0))
    return tot


def _small_mla(grid, seed=77, seq_lens=(130, 70), q_lens=(3, 2), topk=16):
    return W.make_workload("pin", kind="mla", seed=seed, seq_lens=list(seq_lens), q_lens=list(q_lens),
                           topk=topk, grid=grid, H=4, Dqk=40, Dv=32, Hi=3, Di=16)


def test_indexer_exact_rationals_random_fp8():
    wl = _small_mla(grid=False)
    rng = np.random.default_rng(5)
    for row in range(wl.total_q):
        sc = oracle.indexer_scores_row(wl, row)
        b, pos = oracle.row_location(wl.seq_lens, wl.cu_q, row)
        assert sc.size == pos + 1                          # causal: s = 0..pos inclusive
        for s in list(rng.choice(pos + 1, 6, replace=False)) + [pos, 0]:
            exact = float(_fraction_score(wl, row, int(s)))
            assert abs(sc[s] - exact) <= 1e-12 * max(1.0, abs(exact))


def test_indexer_integer_grid_is_exact():
    wl = _small_mla(grid=True)
    for row in range(wl.total_q):
        sc = oracle.indexer_scores_row(wl, row)
        for s in range(0, sc.size, 7):
            assert Fraction(float(sc[s])) == _fraction_score(wl, row, s)


def test_indexer_f32_rationals():
    wl = W.make_workload("pinf", kind="f32", seed=3, seq_lens=[90], q_lens=[5], topk=8, H=2, Dqk=8, Dv=8,
                         Hi=2, Di=8, shuffle=True)
    for row in range(wl.total_q):
        sc = oracle.indexer_scores_row(wl, row)
        for s in (0, 17, sc.size - 1):
            exact = float(_fraction_score(wl, row, s))
            assert abs(sc[s] - exact) <= 1e-12 * max(1.0, abs(exact))


def test_indexer_positive_homogeneity_in_key_scale():
    wl = _small_mla(grid=False)
    base = oracle.indexer_scores_row(wl, 2)
    wl.kS_pool = wl.kS_pool * np.float32(4.0)
    assert np.array_equal(oracle.indexer_scores_row(wl, 2), 4.0 * base)


# ----------------------------------------------------------------------------- top-k

@pytest.mark.parametrize("case", _golden("topk_hand.json")["cases"])
def test_topk_hand(case):
    assert oracle.topk_row(np.array(case["scores"]), case["k"]).tolist() == case["idx"]


def _topk_threshold_scan(scores, k):
    """Independent selection: tau = k-th largest value (np.partition); keep everything above
    tau, then the lowest positions equal to tau until k are taken."""
    n = len(scores)
    if n <= k:
        return list(range(n)) + [-1] * (k - n)
    tau = np.partition(scores, n - k)[n - k]
    above = [s for s in range(n) if scores[s] > tau]
    equal = [s for s in range(n) if scores[s] == tau]
    return sorted(above + equal[: k - len(above)])


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(11)
    for trial in range(300):
        n = int(rng.integers(1, 200))
        k = int(rng.integers(1, 80))
        scores = rng.integers(-4, 5, n).astype(np.float64) * (0.5 if trial % 2 else 1.0)
        assert oracle.topk_row(scores, k).tolist() == _topk_threshold_scan(scores, k)


def test_topk_brute_force_distinct():
    rng = np.random.default_rng(12)
    for _ in range(100):
        n = int(rng.integers(1, 5000)); k = int(rng.integers(1, 600))
        scores = rng.standard_normal(n)
        assert oracle.topk_row(scores, k).tolist() == _topk_threshold_scan(scores, k)


# ----------------------------------------------------------------------------- attention

def test_attention_hand():
    g = _golden("attention_hand.json")
    a = g["attention"]
    o, lse = oracle.attention(np.array(a["q"]), np.array(a["K"])[a["idx"]], np.array(a["V"])[a["idx"]], a["scale"])
    assert np.allclose(o, a["out"], rtol=0, atol=1e-14) and np.allclose(lse, a["lse"], rtol=0, atol=1e-14)
    c = g["combine"]
    o, lse = oracle.combine(c["parts"], c["lses"])
    assert np.allclose(o, c["out"], rtol=0, atol=1e-14) and np.allclose(lse, c["lse"], rtol=0, atol=1e-14)


def _tiny_case(topk, grid=False, seed=20260001):
    return W.make_workload("t", kind="f32", seed=seed, seq_lens=[96], q_lens=[96], topk=topk,
                           H=3, Dqk=16, Dv=12, Hi=2, Di=8, shuffle=True, grid=grid, w_dist="uniform")


def test_attention_matches_torch_sdpa_with_mask():
    wl = _tiny_case(topk=10)
    rng = np.random.default_rng(4)
    for row in (0, 5, 40, 95):
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, row)
        idx = np.sort(rng.choice(pos + 1, min(10, pos + 1), replace=False))
        o, lse = oracle.sparse_attention_row(wl, row, idx)
        allpos = np.arange(int(wl.seq_lens[0]))
        blk, slot = wl.block_table[0, allpos // 64], allpos % 64
        K = torch.from_numpy(wl.kv_pool[blk, slot].astype(np.float64))
        V = torch.from_numpy(wl.v_pool[blk, slot].astype(np.float64))
        q = torch.from_numpy(wl.q[row].astype(np.float64))
        mask = torch.zeros(allpos.size, dtype=torch.bool); mask[torch.from_numpy(idx)] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, None, :], K.expand(q.shape[0], -1, -1), V.expand(q.shape[0], -1, -1),
            attn_mask=mask[None, None, :].expand(q.shape[0], 1, -1), scale=wl.softmax_scale)[:, 0, :]
        assert np.allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        logits = wl.softmax_scale * (q @ K.T)[:, torch.from_numpy(idx)]
        assert np.allclose(lse, torch.logsumexp(logits, dim=1).numpy(), rtol=0, atol=1e-12)
        dense = oracle.dense_masked_attention(wl, row, idx)
        assert np.allclose(o, dense, rtol=0, atol=1e-12)


def test_full_topk_reproduces_dense_causal_attention():
    """k >= context: the path (indexer -> top-k -> attention) is dense causal attention."""
    wl = _tiny_case(topk=128)
    res = oracle.run_rows(wl, range(wl.total_q))
    allpos = np.arange(96)
    blk, slot = wl.block_table[0, allpos // 64], allpos % 64
    K = torch.from_numpy(wl.kv_pool[blk, slot].astype(np.float64))
    V = torch.from_numpy(wl.v_pool[blk, slot].astype(np.float64))
    q = torch.from_numpy(wl.q.astype(np.float64)).permute(1, 0, 2)          # [H, T, D]
    H = q.shape[0]
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, K.expand(H, -1, -1), V.expand(H, -1, -1), is_causal=True, scale=wl.softmax_scale).permute(1, 0, 2)
    for row in range(96):
        assert res[row]["idx"][: row + 1].tolist() == list(range(row + 1))
        assert np.allclose(res[row]["out"], ref[row].numpy(), rtol=0, atol=1e-12)


def test_topk_one_selects_argmax_value():
    wl = _tiny_case(topk=1)
    res = oracle.run_rows(wl, [50, 77])
    for row, r in res.items():
        sc = r["scores"]
        best = int(np.flatnonzero(sc == sc.max())[0])
        assert r["idx"].tolist() == [best]
        K, V = oracle.gather_kv(wl, 0, np.array([best]))
        assert np.allclose(r["out"], np.broadcast_to(V[0], r["out"].shape), rtol=0, atol=1e-15)


def test_equal_logits_average_values():
    wl = _tiny_case(topk=12)
    wl.q = np.zeros_like(wl.q)
    r = oracle.run_rows(wl, [60])[60]
    K, V = oracle.gather_kv(wl, 0, r["idx"])
    assert np.allclose(r["out"], np.broadcast_to(V.mean(axis=0), r["out"].shape), rtol=0, atol=1e-14)
    assert np.allclose(r["lse"], math.log(12), rtol=0, atol=1e-14)


def test_split_and_combine_equals_whole():
    wl = _tiny_case(topk=40)
    rng = np.random.default_rng(8)
    r = oracle.run_rows(wl, [90])[90]
    idx = r["idx"][r["idx"] >= 0]
    cut = rng.permutation(idx.size)
    parts, lses = [], []
    for sub in (idx[cut[:7]], idx[cut[7:25]], idx[cut[25:]], np.array([], np.int64)):
        o, l = oracle.sparse_attention_row(wl, 90, sub)
        parts.append(o); lses.append(l)
    o, lse = oracle.combine(parts, lses)
    assert np.allclose(o, r["out"], rtol=0, atol=1e-13) and np.allclose(lse, r["lse"], rtol=0, atol=1e-13)


def test_block_table_permutation_invariance():
    wl = _small_mla(grid=False)
    ref = oracle.run_rows(wl, range(wl.total_q))
    perm = np.random.default_rng(9).permutation(wl.num_blocks)     # new physical id of old block
    inv = np.argsort(perm)
    wl.kv_pool = wl.kv_pool[inv]; wl.kI_pool = wl.kI_pool[inv]; wl.kS_pool = wl.kS_pool[inv]
    wl.block_table = perm[wl.block_table].astype(np.int32)
    got = oracle.run_rows(wl, range(wl.total_q))
    for row in ref:
        for key in ("scores", "idx", "out", "lse"):
            assert np.array_equal(ref[row][key], got[row][key])


def _bf16_bits_by_torch(x):
    """bf16 bit patterns of x through torch's own fp32 -> bf16 cast (the values used here are exact)."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_mla_value_slice_hand():
    """MLA layout: keys are the whole latent row, values its leading Dv entries.  The rope dims carry values
    that a trailing slice, the whole row, or a dropped rope term in the keys would turn into other outputs."""
    g = _golden("mla_attention_hand.json")
    P, Dqk = g["page_size"], g["Dqk"]
    kv = np.zeros((1, P, Dqk), np.float32)
    kv[0, : len(g["kv"])] = g["kv"]
    case = SimpleNamespace(kind="mla", page_size=P, seq_lens=np.array([len(g["kv"])], np.int32),
                           cu_q=np.array([0, 1], np.int32), block_table=np.zeros((1, 1), np.int32),
                           q=_bf16_bits_by_torch(np.array(g["q"], np.float32)[None]), kv_pool=_bf16_bits_by_torch(kv),
                           v_pool=None, Dqk=Dqk, Dv=g["Dv"], softmax_scale=math.log(3.0))
    for c in g["cases"]:
        o, lse = oracle.sparse_attention_row(case, 0, np.array(c["idx"]))
        assert o.shape == (2, g["Dv"])
        assert np.allclose(o, c["out"], rtol=0, atol=1e-14)
        assert np.allclose(lse, c["lse"], rtol=0, atol=1e-14)


def test_mla_attention_matches_torch_sdpa_on_bf16_rows():
    """The oracle's MLA attention (its own bf16 decoder, paged lookup and value slice) against torch's fp64
    SDPA over the same rows decoded by torch's bf16 view: K = the whole latent row, V = its first Dv
    entries, a boolean mask for the selected set."""
    wl = _small_mla(grid=False)
    assert wl.Dqk > wl.Dv and wl.v_pool is None
    for row in range(wl.total_q):
        b, pos = oracle.row_location(wl.seq_lens, wl.cu_q, row)
        r = oracle.run_rows(wl, [row])[row]
        idx = r["idx"][r["idx"] >= 0]
        allpos = np.arange(int(wl.seq_lens[b]))
        blk, slot = wl.block_table[b, allpos // wl.page_size], allpos % wl.page_size
        lat = torch.from_numpy(np.ascontiguousarray(wl.kv_pool[blk, slot]).view(np.int16)).view(torch.bfloat16)
        lat = lat.to(torch.float64)
        q = torch.from_numpy(np.ascontiguousarray(wl.q[row]).view(np.int16)).view(torch.bfloat16).to(torch.float64)
        K, V = lat, lat[:, : wl.Dv]
        H = q.shape[0]
        mask = torch.zeros(allpos.size, dtype=torch.bool)
        mask[torch.from_numpy(idx)] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, None, :], K.expand(H, -1, -1), V.expand(H, -1, -1),
            attn_mask=mask[None, None, :].expand(H, 1, -1), scale=wl.softmax_scale)[:, 0, :]
        assert np.allclose(r["out"], ref.numpy(), rtol=0, atol=1e-12)
        lse_ref = torch.logsumexp(wl.softmax_scale * (q @ K.T)[:, torch.from_numpy(idx)], dim=1)
        assert np.allclose(r["lse"], lse_ref.numpy(), rtol=0, atol=1e-12)


def test_lse_is_log_normaliser():
    wl = _tiny_case(topk=20)
    r = oracle.run_rows(wl, [70])[70]
    q = wl.q[70].astype(np.float64)
    K, V = oracle.gather_kv(wl, 0, r["idx"])
    z = wl.softmax_scale * q @ K.T
    assert np.allclose(np.exp(z - r["lse"][:, None]).sum(axis=1), 1.0, rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- planted long-context case

def test_planted_long_context_selection():
    """1,048,576-token decode: the 2048 planted positions are exactly the oracle's top-k,
    with the lowest planted score at least twice the highest other score."""
    wl = W.decode_1m_planted(attention=False)
    sc = oracle.indexer_scores_row(wl, 0)
    idx = oracle.topk_row(sc, 2048)
    assert np.array_equal(idx, wl.planted)
    others = np.delete(sc, wl.planted)
    assert sc[wl.planted].min() > 2.0 * max(others.max(), 0.0)


# ----------------------------------------------------------------------------- cache append (FP8 key quantiser)

def _e4m3_midpoints():
    """Every value halfway between two adjacent finite E4M3 magnitudes (exact in fp32), with the
    fp32 neighbours on either side of each."""
    mags = oracle.E4M3[:0x7F].astype(np.float32)
    mid = ((mags[:-1].astype(np.float64) + mags[1:]) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (mags[:-1].astype(np.float64) + mags[1:]) / 2)
    return np.concatenate([mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(np.inf))])


def test_e4m3_encoder_matches_torch_cast():
    """Round to nearest, ties to even, signed zero: torch's fp32 -> float8_e4m3fn cast on |v| <= 448
    (ties between every adjacent pair of codes, the subnormal range, random values, +-0)."""
    rng = np.random.default_rng(5)
    pos = np.concatenate([_e4m3_midpoints(), oracle.E4M3[:0x7F].astype(np.float32),
                          rng.uniform(0, 448, 20000).astype(np.float32),
                          (rng.uniform(0, 2 ** -6, 5000)).astype(np.float32),
                          np.array([0.0, 1e-30, 2 ** -10, 3 * 2 ** -11, 448.0], np.float32)])
    v = np.concatenate([pos, -pos])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode_rne(v.astype(np.float64)), ref)


def test_e4m3_encoder_saturates():
    codes = oracle.e4m3_encode_rne(np.array([448.0, 460.0, 464.0, 500.0, 1e9, -470.0, -1e30]))
    assert codes.tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_quantize_index_key_hand():
    g = _golden("cache_append_hand.json")
    for row in g["rows"]:
        codes, scale = oracle.quantize_index_key(np.array(row["k"], np.float32))
        assert codes.tolist() == row["codes"], row["note"]
        exact = Fraction(row["scale"])
        # the fp32 value nearest to the exact scale: no fp32 neighbour is closer
        assert scale.dtype == np.float32
        for nb in (np.nextafter(scale, np.float32(0)), np.nextafter(scale, np.float32(np.inf))):
            assert abs(Fraction(float(scale)) - exact) <= abs(Fraction(float(nb)) - exact)


def test_quantize_index_key_error_bound_and_range():
    """Dequantised keys are within half a grid step of the key (a step is 2^-3 of the binade for
    normal codes, 2^-9 for subnormal ones, both times the scale), and the largest |k| maps to 448."""
    rng = np.random.default_rng(6)
    for i in range(300):
        k = (rng.standard_normal(128) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        if i % 7 == 0:
            k[rng.integers(0, 128, 40)] = 0.0
        codes, scale = oracle.quantize_index_key(k)
        deq = oracle.E4M3[codes] * float(scale)
        q = np.abs(k.astype(np.float64)) / float(scale)
        step = np.where(q >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(q, 2.0 ** -6))) - 3), 2.0 ** -9)
        assert np.all(np.abs(deq - k) <= 0.5 * step * float(scale) * (1 + 1e-6) + 1e-300)
        assert np.all((codes & 0x7F) <= 0x7E)
        assert (codes[np.argmax(np.abs(k))] & 0x7F) == 0x7E


def test_cache_append_places_tokens_by_hand():
    """Two sequences, shuffled blocks: row 0, 1 are positions 68, 69 of sequence 0 (its block 1 =
    physical 0, slots 4 and 5); row 2 is position 4 of sequence 1 (its block 0 = physical 1, slot 4).
    Nothing else changes."""
    rng = np.random.default_rng(7)
    NB, P = 4, 64
    case = SimpleNamespace(page_size=P, seq_lens=np.array([70, 5], np.int32), cu_q=np.array([0, 2, 3], np.int32),
                           block_table=np.array([[3, 0], [1, 2]], np.int32),
                           kv_pool=rng.integers(0, 1 << 16, (NB, P, 576)).astype(np.uint16),
                           kI_pool=rng.integers(0, 256, (NB, P, 128)).astype(np.uint8),
                           kS_pool=rng.uniform(0.1, 1, (NB, P)).astype(np.float32))
    kv_new = rng.integers(0, 1 << 16, (3, 576)).astype(np.uint16)
    kI_new = np.stack([np.full(128, 448.0), np.zeros(128), np.full(128, -2.0)]).astype(np.float32)
    kv, kI, kS = oracle.cache_append(case, kv_new, kI_new, "f32")
    where = {0: (0, 4), 1: (0, 5), 2: (1, 4)}
    touched = np.zeros((NB, P), bool)
    for r, (blk, slot) in where.items():
        touched[blk, slot] = True
        assert np.array_equal(kv[blk, slot], kv_new[r])
    assert kI[0, 4].tolist() == [0x7E] * 128 and kS[0, 4] == np.float32(1.0)
    assert kI[0, 5].tolist() == [0] * 128 and kS[0, 5] == np.float32(1.0)
    assert kI[1, 4].tolist() == [0xFE] * 128 and kS[1, 4] == np.float32(2.0 / 448.0)
    assert np.array_equal(kv[~touched], case.kv_pool[~touched])
    assert np.array_equal(kI[~touched], case.kI_pool[~touched])
    assert np.array_equal(kS[~touched], case.kS_pool[~touched])


# ----------------------------------------------------------------------------- block-granular selection

def test_block_topk_hand():
    g = _golden("block_topk_hand.json")
    for c in g["cases"]:
        sc = np.array(c["scores"], dtype=np.float64)
        assert oracle.block_scores_row(sc, c["page"]).tolist() == c["block_scores"], c["note"]
        assert oracle.block_topk_row(sc, c["kb"], c["page"]).tolist() == c["positions"], c["note"]


def test_block_topk_brute_force():
    """Independent brute force: page maxima by a Python loop, pages ranked by sorting (-max, page)."""
    rng = np.random.default_rng(31)
    for it in range(300):
        n = int(rng.integers(1, 400))
        page = int(rng.choice([1, 2, 4, 64]))
        kb = int(rng.integers(1, 12))
        sc = (rng.integers(-5, 6, n) if it % 2 else rng.standard_normal(n)).astype(np.float64)
        maxima = [max(sc[p:p + page]) for p in range(0, n, page)]
        ranked = sorted(range(len(maxima)), key=lambda p: (-maxima[p], p))[:kb]
        exp = []
        for p in sorted(ranked):
            exp += [x if x < n else -1 for x in range(p * page, p * page + page)]
        exp += [-1] * (kb * page - len(exp))
        assert oracle.block_topk_row(sc, kb, page).tolist() == exp


def test_block_topk_reduces_to_token_topk():
    """One-token pages select exactly the token top-k; with every page selected the result is every
    candidate in order, the token path's layout for k >= n."""
    rng = np.random.default_rng(32)
    for _ in range(100):
        n = int(rng.integers(1, 300))
        sc = rng.integers(-3, 4, n).astype(np.float64)
        kb = int(rng.integers(1, 40))
        assert np.array_equal(oracle.block_topk_row(sc, kb, 1), oracle.topk_row(sc, kb))
        nb = (n + 63) // 64
        assert np.array_equal(oracle.block_topk_row(sc, nb, 64), oracle.topk_row(sc, nb * 64))


# ----------------------------------------------------------------------------- decode index reuse

def test_reuse_candidates_and_selection_by_hand():
    # an earlier selection {2, 5, 9} (one -1 slot) made at 12 tokens; the query now sits at position 14
    cands = oracle.reuse_candidates(np.array([2, 5, 9, -1]), 12, 14)
    assert cands.tolist() == [2, 5, 9, -1, 12, 13, 14]
    sc = np.array([0.5, 3.0, 3.0, -np.inf, 1.0, 3.0, -2.0])
    # k = 3: the three 3.0's (slots 1, 2, 5 -> positions 5, 9, 13)
    assert oracle.candidate_topk(sc, cands, 3).tolist() == [5, 9, 13]
    # k = 2: the tie at 3.0 goes to the earlier slots (positions 5 and 9)
    assert oracle.candidate_topk(sc, cands, 2).tolist() == [5, 9]
    # k = 8 >= 7 candidates: every slot in slot order (the empty slot stays -1), then -1 padding
    assert oracle.candidate_topk(sc, cands, 8).tolist() == [2, 5, 9, -1, 12, 13, 14, -1]


def test_reuse_with_every_position_is_the_full_selection():
    """When the earlier selection held every earlier position, reuse selects exactly what a full top-k
    selects (the candidates are then all positions, in order)."""
    wl = _tiny_case(topk=20)
    for row in (30, 70, 95):
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, row)
        prev = np.arange(0, pos - 3)
        cands = oracle.reuse_candidates(prev, pos - 3, pos)
        sc = oracle.candidate_scores_row(wl, row, cands)
        full = oracle.indexer_scores_row(wl, row)
        assert np.array_equal(sc, full)
        assert np.array_equal(oracle.candidate_topk(sc, cands, 20), oracle.topk_row(full, 20))


def test_reuse_of_the_same_step_is_idempotent():
    """Reusing a selection made at the same position with no new tokens returns that selection."""
    wl = _tiny_case(topk=16)
    for row in (10, 40, 95):
        full = oracle.indexer_scores_row(wl, row)
        sel = oracle.topk_row(full, 16)
        _, pos = oracle.row_location(wl.seq_lens, wl.cu_q, row)
        cands = oracle.reuse_candidates(sel, pos + 1, pos)
        got = oracle.candidate_topk(oracle.candidate_scores_row(wl, row, cands), cands, 16)
        assert np.array_equal(np.sort(got[got >= 0]), sel[sel >= 0])


def test_reuse_empty_slots_score_minus_infinity_and_are_never_chosen():
    """An earlier selection's -1 slots carry no token: they score -inf, so even when every real candidate
    scores below zero (a negative indexer weight) none of them is passed over for an empty slot."""
    # one head, one active dim, weight -1: token s has key (s + 1, 0), so I[s] = -ReLU(s + 1) = -(s + 1)
    case = _single_row_case(qI=[[1.0, 0.0]], kI=[[s + 1.0, 0.0] for s in range(6)], w=[-1.0])
    assert oracle.indexer_scores_row(case, 0).tolist() == [-1.0, -2.0, -3.0, -4.0, -5.0, -6.0]
    # an earlier selection {0, 2} with two empty slots, made at 4 tokens; the query sits at position 5
    cands = oracle.reuse_candidates(np.array([0, 2, -1, -1]), 4, 5)
    assert cands.tolist() == [0, 2, -1, -1, 4, 5]
    sc = oracle.candidate_scores_row(case, 0, cands)
    assert sc.tolist() == [-1.0, -3.0, -np.inf, -np.inf, -5.0, -6.0]
    # k = 4: the four real candidates, in slot order
    assert oracle.candidate_topk(sc, cands, 4).tolist() == [0, 2, 4, 5]
    # k = 3: the three best (-1, -3, -5)
    assert oracle.candidate_topk(sc, cands, 3).tolist() == [0, 2, 4]
