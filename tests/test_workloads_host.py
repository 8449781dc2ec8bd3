"""The seeded input generator (no GPU): the same seed gives the same arrays whatever the number of host
threads that draw them, different seeds give different draws, the decode-batch recipe has the shapes and
ranges it is documented with, and the other recipes hand the generator their documented configurations."""
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


def _recipe(monkeypatch, fn, **kw):
    """The arguments a workload recipe hands to make_workload (nothing is drawn)."""
    got = {}
    monkeypatch.setattr(W, "make_workload", lambda name, **a: got.update(a, name=name) or got)
    fn(**kw)
    return got


def test_other_recipes(monkeypatch):
    t = _recipe(monkeypatch, W.tiny_f32)
    assert (t["kind"], list(t["seq_lens"]), list(t["q_lens"]), t["topk"]) == ("f32", [256], [256], 32)
    assert (t["H"], t["Dqk"], t["Dv"], t["Hi"], t["Di"]) == (4, 64, 64, 2, 32)
    assert t["shuffle"] is False and t["w_dist"] == "uniform" and t["seed"] == 20260001
    p = _recipe(monkeypatch, W.prefill_16k)
    assert (p["kind"], list(p["seq_lens"]), list(p["q_lens"]), p["topk"]) == ("mla", [16384], [16384], 2048)
    p4 = _recipe(monkeypatch, W.prefill_4k)
    assert (list(p4["seq_lens"]), list(p4["q_lens"]), p4["topk"]) == ([4096], [4096], 2048)
    d = _recipe(monkeypatch, W.decode_1m_planted)
    assert (list(d["seq_lens"]), list(d["q_lens"]), d["topk"], d["planted_k"]) == ([1 << 20], [1], 2048, 2048)
    m = _recipe(monkeypatch, W.mixed_batch)
    sl, ql = np.asarray(m["seq_lens"]), np.asarray(m["q_lens"])
    assert m["kind"] == "mla" and m["topk"] == 2048 and sl.size == ql.size == 18
    assert np.all(ql[:16] == 1) and np.all((sl[:16] >= 8192) & (sl[:16] <= 131072))
    # two chunks of 8192 rows: positions 57,344..65,535 of 65,536-token sequences (the chunk's KV is cached)
    assert list(ql[16:]) == [8192, 8192] and list(sl[16:]) == [65536, 65536]
    assert list(sl[16:] - ql[16:]) == [57344, 57344]
