"""The seeded input generator (no GPU): the same seed gives the same arrays whatever the number of host
threads that draw them, different seeds give different draws, and the decode-batch recipe has the shapes and
ranges it is documented with."""
import numpy as np

from sparse_attention_long_dsa_b200 import workloads as W


def _arrays(wl):
    return {n: getattr(wl, n) for n in ("q", "kv_pool", "qI", "kI_pool", "kS_pool", "w", "block_table", "seq_lens")}


def test_draws_do_not_depend_on_the_thread_count(monkeypatch):
    mk = lambda: W.make_workload("det", kind="mla", seed=77, seq_lens=[5000, 9000], q_lens=[1, 3], topk=256)
    monkeypatch.setattr(W, "_CHUNK", 1 << 16)           # several chunks per array
    monkeypatch.setattr(W, "_THREADS", 1)
    a = _arrays(mk())
    monkeypatch.setattr(W, "_THREADS", 7)
    b = _arrays(mk())
    for n in a:
        assert np.array_equal(a[n], b[n]), n


def test_seeds_give_different_draws():
    a = W.make_workload("s", kind="mla", seed=1, seq_lens=[300], q_lens=[2], topk=64)
    b = W.make_workload("s", kind="mla", seed=2, seq_lens=[300], q_lens=[2], topk=64)
    assert not np.array_equal(a.q, b.q) and not np.array_equal(a.kI_pool, b.kI_pool)


def test_decode_batch_recipe():
    wl = W.decode_batch()
    assert wl.num_seqs == 32 and wl.total_q == 32 and wl.topk == 2048
    assert wl.seq_lens.min() >= 4096 and wl.seq_lens.max() <= 32768
    assert wl.q.shape == (32, 128, 576) and wl.q.dtype == np.uint16
    assert wl.qI.shape == (32, 64, 128) and wl.qI.dtype == np.uint8
    assert wl.kv_pool.shape[1:] == (64, 576) and wl.kI_pool.shape[1:] == (64, 128)
    # the physical page ids are a permutation of the whole pool
    used = np.concatenate([wl.block_table[b, : (int(wl.seq_lens[b]) + 63) // 64] for b in range(32)])
    assert np.array_equal(np.sort(used), np.arange(wl.num_blocks))
    # w ~ N(0, 1/64): sample standard deviation near 1/8
    assert abs(float(np.std(wl.w)) - 0.125) < 0.01
    assert np.all(wl.kS_pool > 0)
