"""CPU oracle for DSA sparse attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the C-ABI library
and its Python binding) never calls it and has no CPU fallback.

It is a plain, slow, obviously correct restatement of what the path
computes, in float64, one query row at a time.  It shares no code with the
CUDA side: it decodes the storage formats itself (OCP FP8 E4M3 from its
bit-level definition, bf16 from its bit layout), resolves the paged layout
itself, and uses numpy only for matmuls, sorting and elementwise math.

What each step follows (page titles and sections of the source pages):

* Paged cache lookup -- "Day-0 Adaptation: Running Trillion-Parameter
  Models on Domestic AI Accelerators", 3.2 KV Cache Layout: the cache is cut
  into fixed-size blocks and a block table maps logical to physical blocks;
  "Engineering Practices for Day-0 Adaptation of Million-Token Context
  Models on Domestic AI Chips", Four Key Layers 2 (64- or 128-token blocks).
* Indexer score -- "Day-0 Adaptation for LLMs: Implementing Sparse
  Attention and Low-Precision Weights", III.1 Index Selection Path (a
  lightweight scoring network relates each query to historical tokens,
  scored at higher precision than attention; mixed-precision boundaries in
  V keep index scoring in BF16/FP32).  The pages leave the scorer's form
  open; this library takes it as
      I(t, s) = sum_j w[t, j] * ReLU(qI[t, j] . kI[s]),   s <= pos(t),
  where kI[s] = kS[s] * e4m3(kI8[s]) is the dequantised indexer key.
* Top-k -- same page III.1 and the decode sketch (score -> topk(score, k)):
  the k highest scores, ties to the lower token index; every candidate when
  a query has at most k of them.
* Sparse attention -- same page, decode sketch (gather the selected rows,
  then exact attention over them) and "Day-0 Model Adaptation Depends on
  the Compute Software Stack", Operator Library Abstraction (query vectors,
  key-value pairs and index lists in, aggregated context vector out).
  Written here as plain two-pass softmax: m = max z, p = exp(z - m),
  o = sum p V / sum p, lse = m + ln(sum p).
* Split combine -- "Engineering Practices ...", Four Key Layers 3 (partial
  results over candidate KV blocks followed by a cross-block reduction).
* Block-granular selection -- "Day-0 Adaptation: Running Trillion-Parameter
  Models on Domestic AI Accelerators", 3.1 (the selection operator's top-k
  counts key-value blocks): a page's score is taken as the largest token
  score in it (the pages do not say how token scores make a block score),
  the best kb pages are kept with ties to the lower page, and attention runs
  over all their causal tokens.  An approximation of the token-granular
  path, with this oracle of its own.
* Decode index reuse -- "Day-0 Adaptation: Running Trillion-Parameter Models
  on Domestic AI Accelerators", 3.3 (the decode path keeps its indices
  incrementally and reuses the previous step's result): the candidates of a
  step are an earlier selection plus every token added since, scored by the
  same indexer at those positions only, and the k best are kept (ties to the
  lower position).  An approximation of a full selection, exact on its own
  definition.
* Cache append -- "Engineering Practices ...", Four Key Layers 3 (the decode
  step writes the new token into the KV cache, merged with its attention
  launch) and 2 (the block table places a token in its block); the indexer
  key is stored as FP8 E4M3 with one scale per token ("Day-0 Adaptation for
  LLMs ...", III.1: low-precision index scoring).  The pages do not spell the
  quantiser out; this library takes scale = max|k| / 448 (1 for an all-zero
  key) and code = the E4M3 value nearest to k / scale, ties to the even code,
  clamped to +-448, both divisions in fp32.

Every function is pinned by tests/test_oracle_pins.py against values fixed
by hand or by independent arithmetic (exact rationals, torch library
routines, brute force).
"""
from __future__ import annotations

import math
from typing import Iterable, Sequence

import numpy as np

# ----------------------------------------------------------------------------
# storage formats
# ----------------------------------------------------------------------------

def _e4m3_table() -> np.ndarray:
    """Value of every OCP FP8 E4M3 byte: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; no infinities."""
    t = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            t[code] = math.nan
        elif e == 0:
            t[code] = sign * m * 2.0 ** -9
        else:
            t[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


E4M3 = _e4m3_table()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3[np.asarray(codes, dtype=np.uint8).astype(np.int64)]


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns are the upper half of an fp32 word."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def _real(arr: np.ndarray, fmt: str) -> np.ndarray:
    if fmt == "f32":
        return np.asarray(arr, dtype=np.float64)
    if fmt == "bf16":
        return bf16_decode(arr)
    if fmt == "e4m3":
        return e4m3_decode(arr)
    raise ValueError(fmt)


E4M3_MAX = 448.0
_E4M3_NONNEG = E4M3[:0x7F]          # codes 0x00..0x7E: the finite non-negative values, increasing


def e4m3_encode_rne(v) -> np.ndarray:
    """E4M3 code of each real v: the finite value nearest to v, on a tie the code whose last
    mantissa bit is 0, magnitudes beyond 448 clamped to 448; the sign bit is v's (so a
    negative v that rounds to zero gives -0).  Brute force over all 127 magnitudes."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    d = np.abs(a[..., None] - _E4M3_NONNEG)                 # [..., 127] distance to every magnitude
    nearest = d == d.min(axis=-1, keepdims=True)            # one code, or two adjacent ones on a tie
    even = nearest & (np.arange(_E4M3_NONNEG.size) % 2 == 0)
    code = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(nearest, axis=-1))
    return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)


# ----------------------------------------------------------------------------
# paged layout
# ----------------------------------------------------------------------------

def row_location(seq_lens: np.ndarray, cu_q: np.ndarray, row: int):
    """(sequence, absolute position) of query row `row`: a sequence's rows are its last
    q_len tokens, so row cu_q[b] + i sits at seq_lens[b] - q_len[b] + i."""
    b = int(np.searchsorted(cu_q, row, side="right") - 1)
    q_len = int(cu_q[b + 1] - cu_q[b])
    pos = int(seq_lens[b]) - q_len + (row - int(cu_q[b]))
    return b, pos


def token_slots(block_table_row: np.ndarray, positions: np.ndarray, page_size: int):
    """Logical token positions -> (physical block, slot) through the block table."""
    positions = np.asarray(positions, dtype=np.int64)
    return block_table_row[positions // page_size].astype(np.int64), positions % page_size


def _formats(case):
    if case.kind == "f32":
        return dict(q="f32", kv="f32", qI="f32", kI="f32")
    return dict(q="bf16", kv="bf16", qI="e4m3", kI="e4m3")


# ----------------------------------------------------------------------------
# step 0: appending new tokens to the paged cache
# ----------------------------------------------------------------------------

def quantize_index_key(k):
    """(codes, scale) of one indexer key: scale = max|k| / 448 in fp32 (1 when that is 0),
    codes = e4m3(k / scale) with the quotient taken in fp32."""
    k32 = np.asarray(k, dtype=np.float32)
    amax = np.float32(np.max(np.abs(k32))) if k32.size else np.float32(0.0)
    scale = np.float32(amax / np.float32(E4M3_MAX))
    if scale == 0:
        scale = np.float32(1.0)
    return e4m3_encode_rne((k32 / scale).astype(np.float64)), scale


def cache_append(case, kv_new, kI_new, kI_fmt: str):
    """The pools after the batch's query rows are written as new tokens.  Row cu_q[b] + i is the
    token at position seq_lens[b] - q_len[b] + i of sequence b (the same rows the other steps
    treat as queries); its latent row is copied bit for bit into kv_pool, its indexer key is
    quantised into kI_pool (codes) and kS_pool (scale), all at the token's (block, slot).
    Returns new arrays (kv_pool, kI_pool, kS_pool); the inputs are not modified."""
    kv_pool = np.array(case.kv_pool, copy=True)
    kI_pool = np.array(case.kI_pool, copy=True)
    kS_pool = np.array(case.kS_pool, copy=True)
    T = int(case.cu_q[-1])
    for row in range(T):
        b, pos = row_location(case.seq_lens, case.cu_q, row)
        blk, slot = token_slots(case.block_table[b], np.array([pos]), case.page_size)
        blk, slot = int(blk[0]), int(slot[0])
        kv_pool[blk, slot] = np.asarray(kv_new[row])
        codes, scale = quantize_index_key(_real(kI_new[row], kI_fmt))
        kI_pool[blk, slot] = codes
        kS_pool[blk, slot] = scale
    return kv_pool, kI_pool, kS_pool


# ----------------------------------------------------------------------------
# step 1: indexer scores
# ----------------------------------------------------------------------------

def indexer_scores_row(case, row: int, chunk: int = 1 << 16) -> np.ndarray:
    """I[s] for s = 0..pos(row) (fp64):
    I[s] = sum_j w[row, j] * max(0, sum_d qI[row, j, d] * kI[s, d]),
    with kI[s] = kS[s] * e4m3(kI8[s]) (kS absent: kI is the fp32 key itself)."""
    fm = _formats(case)
    b, pos = row_location(case.seq_lens, case.cu_q, row)
    n = pos + 1
    qI = _real(case.qI[row], fm["qI"])                      # [Hi, Di]
    w = np.asarray(case.w[row], dtype=np.float64)           # [Hi]
    out = np.empty(n, dtype=np.float64)
    for lo in range(0, n, chunk):
        s = np.arange(lo, min(n, lo + chunk))
        blk, slot = token_slots(case.block_table[b], s, case.page_size)
        kI = _real(case.kI_pool[blk, slot], fm["kI"])       # [m, Di]
        if case.kS_pool is not None:
            kI = kI * np.asarray(case.kS_pool[blk, slot], dtype=np.float64)[:, None]
        dots = kI @ qI.T                                    # [m, Hi]
        out[lo: lo + s.size] = np.maximum(dots, 0.0) @ w
    return out


# ----------------------------------------------------------------------------
# step 2: top-k
# ----------------------------------------------------------------------------

def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    """The k best positions under the order (score descending, position ascending),
    returned ascending and padded with -1 to length k; all positions when n <= k."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.size
    pos = np.arange(n)
    if n <= k:
        sel = pos
    else:
        order = np.lexsort((pos, -scores))   # last key is primary
        sel = np.sort(order[:k])
    out = np.full(k, -1, dtype=np.int32)
    out[: sel.size] = sel
    return out


def block_scores_row(scores: np.ndarray, page_size: int) -> np.ndarray:
    """Score of each page of a row's candidates: the largest token score in it (the last page may be
    partial)."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.size
    nb = (n + page_size - 1) // page_size
    padded = np.full(nb * page_size, -np.inf)
    padded[:n] = scores
    return padded.reshape(nb, page_size).max(axis=1)


def block_topk_row(scores: np.ndarray, kb: int, page_size: int) -> np.ndarray:
    """Block-granular selection: the kb best pages by block score (ties to the lower page, every page when
    there are at most kb), each expanded to its token positions.  Selected page i (in ascending page order)
    fills entries [i*page_size, (i+1)*page_size) with its positions, -1 past the last candidate; unused
    entries are -1.  Length kb*page_size."""
    n = np.asarray(scores).size
    pages = topk_row(block_scores_row(scores, page_size), kb)
    out = np.full(kb * page_size, -1, dtype=np.int32)
    for i, p in enumerate(pages):
        if p < 0:
            continue
        pos = p * page_size + np.arange(page_size)
        out[i * page_size: (i + 1) * page_size] = np.where(pos < n, pos, -1)
    return out


def reuse_candidates(prev_idx: np.ndarray, prev_len: int, pos: int) -> np.ndarray:
    """Candidates of a decode step that reuses an earlier selection: that selection's positions (made when
    the sequence held prev_len tokens) followed by every position added since, prev_len .. pos.  -1 entries
    of the earlier selection stay as -1 slots."""
    prev_idx = np.asarray(prev_idx, dtype=np.int64)
    return np.concatenate([prev_idx, np.arange(prev_len, pos + 1, dtype=np.int64)])


def candidate_scores_row(case, row: int, cands: np.ndarray) -> np.ndarray:
    """Indexer scores of one query row at the given candidate positions (-1 gives -inf), from the full
    scorer: the same definition, evaluated only where asked."""
    cands = np.asarray(cands, dtype=np.int64)
    full = indexer_scores_row(case, row)
    return np.where(cands >= 0, full[np.maximum(cands, 0)], -np.inf)


def candidate_topk(cand_scores: np.ndarray, cands: np.ndarray, k: int) -> np.ndarray:
    """The k best candidates by score (ties to the earlier candidate slot, which is the lower position when
    the candidates are in ascending position order), returned as positions in slot order, -1 padded."""
    slots = topk_row(cand_scores, k)
    cands = np.asarray(cands, dtype=np.int64)
    return np.where(slots >= 0, cands[np.maximum(slots, 0)], -1).astype(np.int32)


# ----------------------------------------------------------------------------
# step 3: sparse attention over the selected rows
# ----------------------------------------------------------------------------

def gather_kv(case, b: int, idx: np.ndarray):
    """Selected latent rows: K[i] = kv[idx_i, :Dqk]; V[i] = kv[idx_i, :Dv] for MLA (the value
    is the leading part of the shared latent row) or v[idx_i] when V is stored apart.
    -1 entries are dropped."""
    fm = _formats(case)
    idx = np.asarray(idx, dtype=np.int64)
    idx = idx[idx >= 0]
    blk, slot = token_slots(case.block_table[b], idx, case.page_size)
    rows = _real(case.kv_pool[blk, slot], fm["kv"])
    K = rows[:, : case.Dqk]
    if case.v_pool is None:
        V = rows[:, : case.Dv]
    else:
        V = _real(case.v_pool[blk, slot], fm["kv"])
    return K, V


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Exact softmax attention of every head of q [H, D] over the rows K [m, D], V [m, Dv]:
    two passes (max, then normalised sum).  Empty set: o = 0, lse = -inf."""
    H = q.shape[0]
    if K.shape[0] == 0:
        return np.zeros((H, V.shape[1])), np.full(H, -np.inf)
    z = scale * (q @ K.T)                                   # [H, m]
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ V) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def sparse_attention_row(case, row: int, idx: np.ndarray):
    fm = _formats(case)
    b, _ = row_location(case.seq_lens, case.cu_q, row)
    q = _real(case.q[row], fm["q"])                         # [H, Dqk]
    K, V = gather_kv(case, b, idx)
    return attention(q, K, V, case.softmax_scale)


def combine(parts: Sequence, lses: Sequence):
    """Merge partial results over disjoint key subsets: lse = log sum_i exp(lse_i),
    o = sum_i exp(lse_i - lse) * o_i (partials with lse_i = -inf contribute nothing)."""
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lses])     # [S, H]
    O = np.stack([np.asarray(x, dtype=np.float64) for x in parts])    # [S, H, Dv]
    mx = L.max(axis=0)
    safe = np.where(np.isfinite(mx), mx, 0.0)
    wts = np.where(np.isfinite(L), np.exp(L - safe), 0.0)             # [S, H]
    tot = wts.sum(axis=0)
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    o = np.einsum("sh,shd->hd", wts, O) / np.where(tot > 0, tot, 1.0)[:, None]
    return o, lse


# ----------------------------------------------------------------------------
# whole path, row by row
# ----------------------------------------------------------------------------

def run_rows(case, rows: Iterable[int], want_scores: bool = True, want_attention: bool = True) -> dict:
    """Scores, top-k and attention of the given query rows (attention on another implementation's index set
    is `sparse_attention_row` called with that set)."""
    res = {}
    for row in rows:
        row = int(row)
        r = {}
        sc = indexer_scores_row(case, row)
        if want_scores:
            r["scores"] = sc
        r["idx"] = topk_row(sc, case.topk)
        if want_attention:
            r["out"], r["lse"] = sparse_attention_row(case, row, r["idx"])
        res[row] = r
    return res


def dense_masked_attention(case, row: int, idx: np.ndarray):
    """Second formulation used only to pin `attention`: logits over every cached position of
    the row's sequence, -inf outside the selected set, softmax over the full axis."""
    fm = _formats(case)
    b, pos = row_location(case.seq_lens, case.cu_q, row)
    n_all = int(case.seq_lens[b])
    allpos = np.arange(n_all)
    blk, slot = token_slots(case.block_table[b], allpos, case.page_size)
    rows = _real(case.kv_pool[blk, slot], fm["kv"])
    K = rows[:, : case.Dqk]
    V = rows[:, : case.Dv] if case.v_pool is None else _real(case.v_pool[blk, slot], fm["kv"])
    q = _real(case.q[row], fm["q"])
    logits = case.softmax_scale * (q @ K.T)
    mask = np.zeros(n_all, dtype=bool)
    sel = np.asarray(idx, dtype=np.int64)
    mask[sel[sel >= 0]] = True
    logits = np.where(mask[None, :], logits, -np.inf)
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    return (e / e.sum(axis=1, keepdims=True)) @ V
