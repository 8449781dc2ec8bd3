"""Plausible mistakes planted in the oracle, each caught by a pin (CPU, no GPU).

Every entry below plants one slip in a copy of the oracle's source held in memory (a wrong exponent bias or
subnormal scale, a dropped ReLU, weight or key scale, an off-by-one causal bound, a reversed tie-break, the
value slice taken from the wrong end of the latent row, a missing softmax scale, an inverted combine weight,
...), runs the pin named beside it from `tests/test_oracle_pins.py` against that copy, and expects the pin to
fail.  The oracle on disk is never modified; the pins pass on it in their own file.  A change to the oracle's
text that moves one of these snippets fails `test_every_snippet_is_in_the_oracle_once`, so the table is kept
in step with the oracle.
"""
import inspect
import types

import pytest

import oracle
import test_oracle_pins as pins

_SRC = inspect.getsource(oracle.dsa_oracle)

# (what the slip is, text in the oracle, the slip, the pin that catches it)
_MISTAKES = [
    # storage formats
    ("e4m3 exponent bias 8", "* 2.0 ** (e - 7)", "* 2.0 ** (e - 8)", "test_e4m3_table_matches_torch"),
    ("e4m3 subnormal step 2^-10", "t[code] = sign * m * 2.0 ** -9", "t[code] = sign * m * 2.0 ** -10",
     "test_e4m3_table_matches_torch"),
    ("e4m3 subnormals with an implicit one", "t[code] = sign * m * 2.0 ** -9",
     "t[code] = sign * (1 + m / 8.0) * 2.0 ** -6", "test_e4m3_table_matches_torch"),
    ("e4m3 without NaN", "if e == 0xF and m == 0x7:", "if False:", "test_e4m3_table_matches_torch"),
    ("e4m3 mantissa over 16", "(1.0 + m / 8.0)", "(1.0 + m / 16.0)", "test_e4m3_table_matches_torch"),
    ("bf16 shifted by 15", "<< np.uint32(16)", "<< np.uint32(15)", "test_bf16_decode_matches_torch"),
    ("e4m3 encoder ties to odd", "% 2 == 0)", "% 2 == 1)", "test_e4m3_encoder_matches_torch_cast"),
    ("e4m3 encoder drops the sign", "np.where(np.signbit(v), code | 0x80, code)", "np.where(False, code | 0x80, code)",
     "test_e4m3_encoder_matches_torch_cast"),
    ("e4m3 encoder ties to the larger magnitude",
     "code = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(nearest, axis=-1))",
     "code = np.where(nearest.sum(axis=-1) > 1, nearest.shape[-1] - 1 - np.argmax(nearest[..., ::-1], axis=-1), "
     "np.argmax(nearest, axis=-1))", "test_e4m3_encoder_matches_torch_cast"),
    # paged layout
    ("query position off by one", "pos = int(seq_lens[b]) - q_len + (row - int(cu_q[b]))",
     "pos = int(seq_lens[b]) - q_len + (row - int(cu_q[b])) - 1", "test_row_location_hand"),
    ("query row found on the wrong side", 'side="right") - 1)', 'side="left") - 1)', "test_row_location_hand"),
    ("block and slot swapped",
     "return block_table_row[positions // page_size].astype(np.int64), positions % page_size",
     "return block_table_row[positions % page_size].astype(np.int64), positions // page_size",
     "test_token_slots_hand"),
    # cache append
    ("key scale over 240", "scale = np.float32(amax / np.float32(E4M3_MAX))",
     "scale = np.float32(amax / np.float32(240.0))", "test_quantize_index_key_hand"),
    ("key multiplied by its scale", "return e4m3_encode_rne((k32 / scale).astype(np.float64)), scale",
     "return e4m3_encode_rne((k32 * scale).astype(np.float64)), scale", "test_quantize_index_key_hand"),
    ("zero key keeps scale 0", "        scale = np.float32(1.0)\n", "        scale = np.float32(0.0)\n",
     "test_quantize_index_key_hand"),
    ("token written one slot over", "        kv_pool[blk, slot] = np.asarray(kv_new[row])",
     "        kv_pool[blk, (slot + 1) % case.page_size] = np.asarray(kv_new[row])",
     "test_cache_append_places_tokens_by_hand"),
    ("key scale not stored", "        kS_pool[blk, slot] = scale\n", "        kS_pool[blk, slot] = 1.0\n",
     "test_cache_append_places_tokens_by_hand"),
    # indexer scores
    ("indexer without ReLU", "out[lo: lo + s.size] = np.maximum(dots, 0.0) @ w", "out[lo: lo + s.size] = dots @ w",
     "test_indexer_hand"),
    ("indexer ReLU after the weights", "out[lo: lo + s.size] = np.maximum(dots, 0.0) @ w",
     "out[lo: lo + s.size] = np.maximum(dots @ w, 0.0)", "test_indexer_hand"),
    ("indexer |x| for ReLU", "out[lo: lo + s.size] = np.maximum(dots, 0.0) @ w",
     "out[lo: lo + s.size] = np.abs(dots) @ w", "test_indexer_hand"),
    ("indexer head weights dropped", "out[lo: lo + s.size] = np.maximum(dots, 0.0) @ w",
     "out[lo: lo + s.size] = np.maximum(dots, 0.0).sum(axis=1)", "test_indexer_hand"),
    ("indexer key scale dropped",
     "            kI = kI * np.asarray(case.kS_pool[blk, slot], dtype=np.float64)[:, None]\n", "            pass\n",
     "test_indexer_exact_rationals_random_fp8"),
    ("causal bound excludes the query's own token", "    n = pos + 1\n    qI", "    n = pos\n    qI",
     "test_indexer_hand"),
    # top-k and its variants
    ("ties to the higher position", "order = np.lexsort((pos, -scores))", "order = np.lexsort((-pos, -scores))",
     "test_topk_hand"),
    ("lowest scores kept", "order = np.lexsort((pos, -scores))", "order = np.lexsort((pos, scores))",
     "test_topk_hand"),
    ("selection in score order", "sel = np.sort(order[:k])", "sel = order[:k]", "test_topk_hand"),
    ("one index short", "sel = np.sort(order[:k])", "sel = np.sort(order[:k - 1])", "test_topk_hand"),
    ("path selects k - 1", 'r["idx"] = topk_row(sc, case.topk)', 'r["idx"] = topk_row(sc, case.topk - 1)',
     "test_topk_one_selects_argmax_value"),
    ("page score = mean", "return padded.reshape(nb, page_size).max(axis=1)",
     "return np.where(np.isfinite(padded), padded, 0).reshape(nb, page_size).mean(axis=1)",
     "test_block_topk_hand"),
    ("page score = first token", "return padded.reshape(nb, page_size).max(axis=1)",
     "return padded.reshape(nb, page_size)[:, 0]", "test_block_topk_hand"),
    ("last page past the context kept", "out[i * page_size: (i + 1) * page_size] = np.where(pos < n, pos, -1)",
     "out[i * page_size: (i + 1) * page_size] = pos", "test_block_topk_hand"),
    ("reuse skips the first new token", "np.arange(prev_len, pos + 1, dtype=np.int64)",
     "np.arange(prev_len + 1, pos + 1, dtype=np.int64)", "test_reuse_candidates_and_selection_by_hand"),
    ("reuse leaves out the query's token", "np.arange(prev_len, pos + 1, dtype=np.int64)",
     "np.arange(prev_len, pos, dtype=np.int64)", "test_reuse_candidates_and_selection_by_hand"),
    ("empty reuse slots score 0", "return np.where(cands >= 0, full[np.maximum(cands, 0)], -np.inf)",
     "return np.where(cands >= 0, full[np.maximum(cands, 0)], 0.0)",
     "test_reuse_empty_slots_score_minus_infinity_and_are_never_chosen"),
    ("reuse returns slots, not positions",
     "return np.where(slots >= 0, cands[np.maximum(slots, 0)], -1).astype(np.int32)",
     "return slots.astype(np.int32)", "test_reuse_candidates_and_selection_by_hand"),
    # gather and attention
    ("MLA value = trailing latent dims", "        V = rows[:, : case.Dv]\n    else:\n        V = _real(case.v_pool",
     "        V = rows[:, -case.Dv:]\n    else:\n        V = _real(case.v_pool", "test_mla_value_slice_hand"),
    ("MLA value = whole latent row", "        V = rows[:, : case.Dv]\n    else:\n        V = _real(case.v_pool",
     "        V = rows\n    else:\n        V = _real(case.v_pool", "test_mla_value_slice_hand"),
    ("key cut to the value width", "    K = rows[:, : case.Dqk]\n    if case.v_pool",
     "    K = rows[:, : case.Dv]\n    if case.v_pool", "test_attention_matches_torch_sdpa_with_mask"),
    ("-1 indices gathered", "    idx = idx[idx >= 0]\n    blk, slot = token_slots(case.block_table[b], idx",
     "    blk, slot = token_slots(case.block_table[b], idx", "test_full_topk_reproduces_dense_causal_attention"),
    ("query's rope dims dropped", '    q = _real(case.q[row], fm["q"])                         # [H, Dqk]\n    K, V',
     '    q = _real(case.q[row], fm["q"]).copy(); q[:, case.Dv:] = 0\n    K, V',
     "test_attention_matches_torch_sdpa_with_mask"),
    ("softmax scale dropped", "    z = scale * (q @ K.T)  ", "    z = (q @ K.T)  ",
     "test_attention_matches_torch_sdpa_with_mask"),
    ("softmax scale square-rooted", "    z = scale * (q @ K.T)  ", "    z = np.sqrt(scale) * (q @ K.T)  ",
     "test_attention_matches_torch_sdpa_with_mask"),
    ("base-2 exponent", "    p = np.exp(z - m)\n", "    p = np.exp2(z - m)\n", "test_attention_hand"),
    ("output not normalised", "    o = (p @ V) / l\n", "    o = (p @ V)\n", "test_attention_hand"),
    ("lse without the maximum", "    lse = (m + np.log(l))[:, 0]", "    lse = (np.log(l))[:, 0]", "test_attention_hand"),
    ("lse in base 2", "    lse = (m + np.log(l))[:, 0]", "    lse = (m + np.log2(l))[:, 0]", "test_attention_hand"),
    ("empty set lse = 0", "return np.zeros((H, V.shape[1])), np.full(H, -np.inf)",
     "return np.zeros((H, V.shape[1])), np.zeros(H)", "test_split_and_combine_equals_whole"),
    # split combine
    ("combine weights inverted", "wts = np.where(np.isfinite(L), np.exp(L - safe), 0.0)",
     "wts = np.where(np.isfinite(L), np.exp(safe - L), 0.0)", "test_attention_hand"),
    ("combined lse without the maximum",
     "lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)",
     "lse = np.where(tot > 0, np.log(np.where(tot > 0, tot, 1.0)), -np.inf)", "test_attention_hand"),
    ("parts averaged", 'o = np.einsum("sh,shd->hd", wts, O) / np.where(tot > 0, tot, 1.0)[:, None]',
     "o = O.mean(axis=0)", "test_attention_hand"),
]


def _mutant(old, new):
    m = types.ModuleType("oracle_with_a_planted_mistake")
    exec(compile(_SRC.replace(old, new), "<oracle with a planted mistake>", "exec"), m.__dict__)
    return m


def _run_pin(name):
    """Call a pin with each of its parametrised values (the pins take no fixtures)."""
    f = getattr(pins, name)
    marks = [m for m in getattr(f, "pytestmark", []) if m.name == "parametrize"]
    if not marks:
        f()
        return
    (mark,) = marks
    for value in mark.args[1]:
        f(**{mark.args[0]: value})


def test_every_snippet_is_in_the_oracle_once():
    for what, old, _, pin in _MISTAKES:
        assert _SRC.count(old) == 1, what
        assert callable(getattr(pins, pin)), pin


def test_an_unmodified_copy_passes_every_pin_used(monkeypatch):
    """The control: the in-memory copy itself, with nothing planted, passes each pin, so a failure above is the
    planted mistake's."""
    monkeypatch.setattr(pins, "oracle", _mutant("", ""))
    for pin in sorted({m[3] for m in _MISTAKES}):
        _run_pin(pin)


@pytest.mark.parametrize("what,old,new,pin", _MISTAKES, ids=[m[0] for m in _MISTAKES])
def test_pin_catches_planted_mistake(what, old, new, pin, monkeypatch):
    assert _SRC.count(old) == 1
    monkeypatch.setattr(pins, "oracle", _mutant(old, new))
    with pytest.raises(Exception):
        _run_pin(pin)
