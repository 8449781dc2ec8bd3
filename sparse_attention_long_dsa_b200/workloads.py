"""Seeded synthetic inputs for the DSA sparse-attention path.

This module only *draws* inputs: random values, their storage encodings
(bf16 bits, OCP FP8 e4m3 bytes with a per-token fp32 scale), paged block
tables and the planted structure of the long-context case.  It holds none
of the method's arithmetic (no scoring, selection or attention), so both
the CPU oracle tests and the CUDA path can take their inputs from here
without sharing any compute code.

Shapes follow the pages' workloads ("Day-0 Adaptation: Running
Trillion-Parameter Models on Domestic AI Accelerators", section 3.1/3.2:
a query tensor, a paged key cache addressed through a block table, a top-k
count) with the MLA dimensions and distributions this library is built for:

* latent KV rows of 576 bf16 (512 shared K/V + 64 rope), 128 query heads,
  softmax scale 1/sqrt(192);
* indexer keys of 128 e4m3 bytes with one fp32 scale per token, indexer
  queries of 64 heads x 128 e4m3, per-head weights w;
* 64-token pages, shuffled physical block ids.

Every array is generated chunk-wise from ``numpy.random.default_rng`` with a
seed derived from (workload seed, stream name, chunk number), so results do
not depend on the number of host threads used to produce them.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "make_workload", "bf16_encode", "e4m3_encode",
    "tiny_f32", "decode_batch", "prefill_16k", "prefill_4k", "decode_1m_planted", "mixed_batch",
    "BENCH_WORKLOADS",
]

MLA_H, MLA_DQK, MLA_DV = 128, 576, 512
IDX_H, IDX_D = 64, 128
PAGE = 64
E4M3_MAX = 448.0

_CHUNK = 1 << 22
_THREADS = 8


# ----------------------------------------------------------------------------
# storage encodings (input quantisation, not part of the method)
# ----------------------------------------------------------------------------

def bf16_encode(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even.  Inputs are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Real values -> OCP FP8 E4M3 bytes: bias 7, 3 mantissa bits, subnormal step 2^-9,
    round to nearest even, saturating at +-448 (the largest finite e4m3 value)."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.uint8) << np.uint8(7)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # exponent of a (a = f * 2^ex with f in [0.5, 1)), clamped to the normal range
    _, ex = np.frexp(np.maximum(a, 2.0 ** -10))
    e = np.clip(ex - 1, -6, 8).astype(np.float64)
    quantum = np.exp2(e - 3.0)
    m = np.minimum(np.round(a / quantum) * quantum, E4M3_MAX)   # np.round: half to even
    _, ex2 = np.frexp(np.maximum(m, 2.0 ** -10))
    e2 = (ex2 - 1).astype(np.int64)
    normal = m >= 2.0 ** -6
    mant = np.where(normal, np.round((m / np.exp2(e2.astype(np.float64)) - 1.0) * 8.0), 0.0).astype(np.int64)
    code_n = ((e2 + 7) << 3) | mant
    code_s = np.round(m / 2.0 ** -9).astype(np.int64)
    code = np.where(normal, code_n, code_s).astype(np.uint8)
    return code | sign


def _e4m3_encode_chunked(x: np.ndarray) -> np.ndarray:
    """e4m3_encode over a large array, element for element the same codes, computed in pieces of
    2^20 values on the thread pool (small temporaries, several cores)."""
    x = np.ascontiguousarray(x)
    out = np.empty(x.shape, dtype=np.uint8)
    fx, fo = x.reshape(-1), out.reshape(-1)
    step = 1 << 20

    def work(lo):
        fo[lo: lo + step] = e4m3_encode(fx[lo: lo + step])

    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(work, range(0, fx.size, step)))
    return out


# ----------------------------------------------------------------------------
# chunked, thread-parallel draws
# ----------------------------------------------------------------------------

def _stream_seed(seed: int, name: str) -> int:
    h = 1469598103934665603
    for ch in name.encode():
        h = ((h ^ ch) * 1099511628211) & ((1 << 63) - 1)
    return (seed * 1000003 + h) & ((1 << 63) - 1)


def _fill(seed: int, name: str, n: int, draw) -> np.ndarray:
    """Fill a flat array of n values chunk-wise; `draw(rng, m)` returns m values."""
    base = _stream_seed(seed, name)
    first = draw(np.random.default_rng([base, 0]), min(_CHUNK, n))
    out = np.empty(n, dtype=first.dtype)
    out[: first.size] = first

    def work(c):
        lo = c * _CHUNK
        m = min(_CHUNK, n - lo)
        out[lo: lo + m] = draw(np.random.default_rng([base, c]), m)

    nchunks = (n + _CHUNK - 1) // _CHUNK
    if nchunks > 1:
        with ThreadPoolExecutor(_THREADS) as ex:
            list(ex.map(work, range(1, nchunks)))
    return out


def _normal_f32(seed, name, shape, std=1.0):
    n = int(np.prod(shape))
    a = _fill(seed, name, n, lambda r, m: r.standard_normal(m, dtype=np.float32))
    if std != 1.0:
        a *= np.float32(std)
    return a.reshape(shape)


def _normal_bf16(seed, name, shape):
    n = int(np.prod(shape))
    return _fill(seed, name, n, lambda r, m: bf16_encode(r.standard_normal(m, dtype=np.float32))).reshape(shape)


def _uniform_f32(seed, name, shape):
    n = int(np.prod(shape))
    return _fill(seed, name, n, lambda r, m: r.random(m, dtype=np.float32)).reshape(shape)


def _grid_int(seed, name, shape, lo, hi):
    n = int(np.prod(shape))
    return _fill(seed, name, n, lambda r, m: r.integers(lo, hi + 1, m, dtype=np.int8)).reshape(shape)


def _quantise_tokens(k: np.ndarray):
    """Per-token e4m3 quantisation of indexer keys k[..., Di] (fp32):
    scale = max|k| / 448 (1.0 for an all-zero token), code = e4m3(k / scale)."""
    amax = np.abs(k).max(axis=-1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0).astype(np.float32)
    codes = np.empty(k.shape, dtype=np.uint8)
    flat_k = k.reshape(-1, k.shape[-1])
    flat_s = scale.reshape(-1)
    flat_c = codes.reshape(-1, k.shape[-1])
    step = max(1, (1 << 20) // k.shape[-1])

    def work(lo):
        hi = min(lo + step, flat_k.shape[0])
        flat_c[lo:hi] = e4m3_encode(flat_k[lo:hi].astype(np.float64) / flat_s[lo:hi, None].astype(np.float64))

    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(work, range(0, flat_k.shape[0], step)))
    return codes, scale


# ----------------------------------------------------------------------------
# the workload container
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    """One batch of the path's inputs, host-resident (numpy).

    kind "f32": q [T,H,Dqk] f32, kv_pool [NB,P,Dqk] f32 (keys), v_pool [NB,P,Dv] f32,
                qI [T,Hi,Di] f32, kI_pool [NB,P,Di] f32, kS_pool None.
    kind "mla": q [T,H,576] bf16 bits (uint16), kv_pool [NB,P,576] bf16 bits, v_pool None
                (V = first Dv entries of the latent row), qI [T,Hi,Di] e4m3 bytes,
                kI_pool [NB,P,Di] e4m3 bytes, kS_pool [NB,P] f32.
    Common: w [T,Hi] f32, block_table [B,max_blocks] int32, seq_lens [B], cu_q [B+1].
    Query rows of sequence b are its LAST q_len[b] tokens: row cu_q[b]+i sits at
    absolute position seq_lens[b] - q_len[b] + i, and its own KV is already cached.
    """
    name: str
    kind: str
    seed: int
    page_size: int
    H: int
    Dqk: int
    Dv: int
    Hi: int
    Di: int
    topk: int
    softmax_scale: float
    seq_lens: np.ndarray
    q_lens: np.ndarray
    cu_q: np.ndarray
    block_table: np.ndarray
    num_blocks: int
    q: np.ndarray
    kv_pool: np.ndarray
    v_pool: Optional[np.ndarray]
    qI: np.ndarray
    kI_pool: np.ndarray
    kS_pool: Optional[np.ndarray]
    w: np.ndarray
    grid: bool = False
    planted: Optional[np.ndarray] = None
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.size)

    @property
    def total_q(self) -> int:
        return int(self.cu_q[-1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.seq_lens.size else 0

    @property
    def max_q_per_seq(self) -> int:
        return int(self.q_lens.max()) if self.q_lens.size else 0

    def row_seq(self) -> np.ndarray:
        """Sequence id of every query row."""
        return np.repeat(np.arange(self.num_seqs, dtype=np.int32), self.q_lens)


def make_workload(name: str, *, kind: str, seed: int, seq_lens, q_lens, topk: int,
                  page_size: int = PAGE, H: int = MLA_H, Dqk: int = MLA_DQK, Dv: int = MLA_DV,
                  Hi: int = IDX_H, Di: int = IDX_D, softmax_scale: Optional[float] = None,
                  shuffle: bool = True, grid: bool = False, w_dist: str = "normal",
                  spare_blocks: int = 0, planted_k: int = 0, planted_gain: float = 16.0,
                  attention: bool = True) -> Workload:
    """Draw one workload.  `grid=True` draws the integer-grid twin: indexer queries and
    keys in {-2..2}, w in (1/16)*{-16..16}, key scales 2^e with e in [-2, 2], so every
    indexer score is exactly representable in fp32 whatever the summation order."""
    if kind not in ("f32", "mla"):
        raise ValueError(kind)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    q_lens = np.asarray(q_lens, dtype=np.int32)
    assert seq_lens.shape == q_lens.shape and np.all(q_lens <= seq_lens) and np.all(q_lens >= 0)
    B = seq_lens.size
    P = page_size
    cu_q = np.zeros(B + 1, dtype=np.int32)
    cu_q[1:] = np.cumsum(q_lens)
    T = int(cu_q[-1])
    nblk = (seq_lens + P - 1) // P
    NB = int(nblk.sum()) + spare_blocks
    max_blocks = max(1, int(nblk.max()) if B else 1)
    rng = np.random.default_rng(_stream_seed(seed, "layout"))
    phys = rng.permutation(NB).astype(np.int32) if shuffle else np.arange(NB, dtype=np.int32)
    block_table = np.zeros((B, max_blocks), dtype=np.int32)
    off = 0
    for b in range(B):
        block_table[b, : nblk[b]] = phys[off: off + nblk[b]]
        off += int(nblk[b])
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(192.0) if kind == "mla" else 1.0 / math.sqrt(Dqk)

    # attention operands
    if not attention:
        q = kv_pool = v_pool = None
    elif kind == "f32":
        q = _normal_f32(seed, "q", (T, H, Dqk))
        kv_pool = _normal_f32(seed, "k", (NB, P, Dqk))
        v_pool = _normal_f32(seed, "v", (NB, P, Dv))
    else:
        q = _normal_bf16(seed, "q", (T, H, Dqk))
        kv_pool = _normal_bf16(seed, "kv", (NB, P, Dqk))
        v_pool = None

    # indexer operands
    if grid:
        qI_real = _grid_int(seed, "qI", (T, Hi, Di), -2, 2).astype(np.float32)
        kI_real = _grid_int(seed, "kI", (NB, P, Di), -2, 2).astype(np.float32)
        w = (_grid_int(seed, "w", (T, Hi), -16, 16).astype(np.float32) / np.float32(16.0))
        if kind == "f32":
            qI, kI_pool, kS_pool = qI_real, kI_real, None
        else:
            qI = _e4m3_encode_chunked(qI_real)
            kI_pool = _e4m3_encode_chunked(kI_real)
            kS_pool = np.exp2(_grid_int(seed, "kS", (NB, P), -2, 2).astype(np.float32)).astype(np.float32)
    else:
        if w_dist == "uniform":
            w = _uniform_f32(seed, "w", (T, Hi))
        else:
            w = _normal_f32(seed, "w", (T, Hi), std=1.0 / 8.0)    # variance 1/64
        if kind == "f32":
            qI = _normal_f32(seed, "qI", (T, Hi, Di))
            kI_pool = _normal_f32(seed, "kI", (NB, P, Di))
            kS_pool = None
        else:
            qI = _e4m3_encode_chunked(_normal_f32(seed, "qI", (T, Hi, Di)))
            k_real = _normal_f32(seed, "kI", (NB, P, Di))
            planted = None
            if planted_k:
                k_real, planted = _plant(seed, k_real, qI, w, block_table, seq_lens, q_lens, cu_q,
                                         P, planted_k, planted_gain)
            kI_pool, kS_pool = _quantise_tokens(k_real)

    wl = Workload(name=name, kind=kind, seed=seed, page_size=P, H=H, Dqk=Dqk, Dv=Dv, Hi=Hi, Di=Di,
                  topk=topk, softmax_scale=float(softmax_scale), seq_lens=seq_lens, q_lens=q_lens,
                  cu_q=cu_q, block_table=block_table, num_blocks=NB, q=q, kv_pool=kv_pool,
                  v_pool=v_pool, qI=qI, kI_pool=kI_pool, kS_pool=kS_pool, w=w, grid=grid)
    if kind == "mla" and not grid and planted_k:
        wl.planted = planted
    return wl


def _e4m3_value_table() -> np.ndarray:
    # decoding table for building the planted direction only (input construction);
    # the oracle keeps its own decoder.
    codes = np.arange(256, dtype=np.int64)
    s = np.where(codes & 0x80, -1.0, 1.0)
    e = (codes >> 3) & 0xF
    m = codes & 7
    v = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    return s * v


def _plant(seed, k_real, qI, w, block_table, seq_lens, q_lens, cu_q, P, count, gain):
    """Long-context planted structure (sequence 0, its last query row): `count` random
    positions get indexer keys gain * (v + small noise) with v = sum of the query's
    positively weighted indexer heads, so that exactly those positions score highest."""
    rng = np.random.default_rng(_stream_seed(seed, "plant"))
    n = int(seq_lens[0])
    pos = np.sort(rng.choice(n, size=count, replace=False)).astype(np.int64)
    row = int(cu_q[1]) - 1
    table = _e4m3_value_table()
    qv = table[qI[row].astype(np.int64)]                  # [Hi, Di]
    wr = w[row].astype(np.float64)
    v = (np.clip(wr, 0.0, None)[:, None] * qv).sum(axis=0)
    rms = float(np.sqrt(np.mean(v * v))) or 1.0
    noise = rng.standard_normal((count, v.size)) * (0.05 * rms)
    keys = (gain * (v[None, :] + noise)).astype(np.float32)
    blk = block_table[0, pos // P]
    slot = pos % P
    k_real[blk, slot] = keys
    return k_real, pos


# ----------------------------------------------------------------------------
# the five benchmark workloads
# ----------------------------------------------------------------------------

def tiny_f32(grid: bool = False) -> Workload:
    """Tiny fp32 causal prefill: 1 sequence of 256 tokens, every token a query; 4 heads of
    dim 64 with K and V separate (one shared K head, one V head), indexer 2 heads x 32 with
    w ~ U(0,1), top-k 32; contiguous cache (identity block table, 4 pages of 64)."""
    return make_workload("tiny_f32" + ("_grid" if grid else ""), kind="f32", seed=20260001,
                         seq_lens=[256], q_lens=[256], topk=32, H=4, Dqk=64, Dv=64, Hi=2, Di=32,
                         shuffle=False, grid=grid, w_dist="uniform")


def decode_batch(seed: int = 20260002, grid: bool = False) -> Workload:
    """Decode batch: 32 sequences, one query each, contexts ~ U[4096, 32768]."""
    rng = np.random.default_rng(_stream_seed(seed, "ctx"))
    ctx = rng.integers(4096, 32768 + 1, size=32).astype(np.int32)
    return make_workload("decode_batch", kind="mla", seed=seed, seq_lens=ctx,
                         q_lens=np.ones(32, np.int32), topk=2048, grid=grid)


def prefill_16k(seed: int = 20260003, grid: bool = False) -> Workload:
    """Prefill: one 16384-token causal prompt, every token a query."""
    return make_workload("prefill_16k", kind="mla", seed=seed, seq_lens=[16384], q_lens=[16384],
                         topk=2048, grid=grid)


def prefill_4k(seed: int = 20260003, grid: bool = False) -> Workload:
    """The prefill workload at a quarter of the length (4096-token causal prompt): small enough for a
    full profiler capture, the same shapes otherwise."""
    return make_workload("prefill_4k", kind="mla", seed=seed, seq_lens=[4096], q_lens=[4096], topk=2048, grid=grid)


def decode_1m_planted(seed: int = 20260004, attention: bool = True) -> Workload:
    """Long-context decode: one query over a 1,048,576-token paged cache, with 2048
    planted positions whose indexer keys align with the query."""
    return make_workload("decode_1m_planted", kind="mla", seed=seed, seq_lens=[1 << 20], q_lens=[1],
                         topk=2048, planted_k=2048, attention=attention)


def mixed_batch(seed: int = 20260005, grid: bool = False) -> Workload:
    """Mixed continuous batch: 16 decode sequences (contexts ~ U[8192, 131072]) followed
    by 2 chunked-prefill requests of 8192 rows appended to a 57,344-token prefix."""
    rng = np.random.default_rng(_stream_seed(seed, "ctx"))
    ctx = rng.integers(8192, 131072 + 1, size=16).astype(np.int32)
    seq_lens = np.concatenate([ctx, np.array([65536, 65536], np.int32)])
    q_lens = np.concatenate([np.ones(16, np.int32), np.array([8192, 8192], np.int32)])
    return make_workload("mixed_batch", kind="mla", seed=seed, seq_lens=seq_lens, q_lens=q_lens,
                         topk=2048, grid=grid)


BENCH_WORKLOADS = {
    "tiny_f32": tiny_f32,
    "decode_batch": decode_batch,
    "prefill_16k": prefill_16k,
    "prefill_4k": prefill_4k,
    "decode_1m_planted": decode_1m_planted,
    "mixed_batch": mixed_batch,
}
