"""Host-side ABI checks (no GPU): the library loads, exports every declared entry point, and
rejects bad arguments before touching the device."""
import os
import re

import numpy as np
import pytest

from sparse_attention_long_dsa_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_symbol():
    lib = B.load()
    names = _declared()
    assert set(B.EXPORTS) <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    lib = B.load()
    for s in range(7):
        assert lib.dsa_status_string(s)
    assert B.dsa_version() == "0.1.0"


def _batch(**kw):
    d = dict(num_seqs=2, page_size=64, num_blocks=4, max_blocks_per_seq=2, block_table=1 << 20, seq_lens=1 << 21,
             cu_q=1 << 22, total_q=3, max_q_per_seq=2, max_seq_len=100)
    d.update(kw)
    return B.dsa_batch_t(**d)


def test_workspace_size_host_only():
    b = _batch()
    assert B.dsa_workspace_size(B.DSA_OP_INDEXER, b) >= 256
    assert B.dsa_workspace_size(B.DSA_OP_TOPK, b, 2048) >= 256
    big = _batch(max_seq_len=1 << 20, max_blocks_per_seq=1 << 14, total_q=2)
    assert B.dsa_workspace_size(B.DSA_OP_TOPK, big, 2048) > 2 * 2048 * 4


@pytest.mark.parametrize("bad,status", [
    (dict(page_size=128), B.DSA_ERR_UNSUPPORTED),
    (dict(num_seqs=0), B.DSA_ERR_INVALID_ARG),
    (dict(block_table=0), B.DSA_ERR_INVALID_ARG),
    (dict(max_seq_len=129), B.DSA_ERR_INVALID_ARG),        # > max_blocks_per_seq * page_size
    (dict(total_q=5), B.DSA_ERR_INVALID_ARG),             # > num_seqs * max_q_per_seq
    (dict(max_q_per_seq=200), B.DSA_ERR_INVALID_ARG),     # > max_seq_len
])
def test_batch_validation(bad, status):
    with pytest.raises(B.DSAError) as e:
        B.dsa_workspace_size(B.DSA_OP_TOPK, _batch(**bad), 16)
    assert e.value.status == status


def test_compute_calls_reject_before_launch():
    b = _batch()
    P = 1 << 24
    with pytest.raises(B.DSAError) as e:       # unsupported indexer dims
        B.dsa_indexer_scores(P, B.DSA_FP8_E4M3, P, P, B.DSA_FP8_E4M3, P, 32, 128, b, P, 128, P, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
    with pytest.raises(B.DSAError) as e:       # ld_scores too small
        B.dsa_topk(P, 64, b, 16, P, P, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_INVALID_ARG
    with pytest.raises(B.DSAError) as e:       # dtype mix
        B.dsa_indexer_scores(P, B.DSA_F32, P, P, B.DSA_FP8_E4M3, None, 2, 32, b, P, 128, P, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_INVALID_ARG
    with pytest.raises(B.DSAError) as e:       # attention shape outside both paths
        B.dsa_sparse_attn_prefill(P, B.DSA_BF16, P, None, 64, 576, 512, 0.1, P, 16, b, P, P, P, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
    with pytest.raises(B.DSAError) as e:       # misaligned workspace
        B.dsa_topk(P, 128, b, 16, P, P + 8, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_INVALID_ARG
    with pytest.raises(B.DSAError) as e:       # decode with several rows per sequence
        B.dsa_sparse_attn_decode(P, B.DSA_BF16, P, None, 128, 576, 512, 0.1, P, 16, b, P, P, P, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_INVALID_ARG
    assert "one query row" in B.load().dsa_last_error().decode()


def test_nonfinite_scale_rejected():
    b = _batch(total_q=2, max_q_per_seq=1)
    P = 1 << 24
    with pytest.raises(B.DSAError) as e:
        B.dsa_sparse_attn_decode(P, B.DSA_BF16, P, None, 128, 576, 512, float("nan"), P, 16, b, P, P, P, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_INVALID_ARG


def test_empty_batch_is_a_noop_without_a_device():
    """total_q == 0: every compute entry validates the descriptor and returns DSA_OK, enqueueing nothing
    (no device is touched, so this holds on a host without a GPU) and accepting NULL data pointers."""
    b = _batch(total_q=0, max_q_per_seq=0)
    n0 = B.dsa_launch_count()
    B.dsa_indexer_scores(None, B.DSA_FP8_E4M3, None, None, B.DSA_FP8_E4M3, None, 64, 128, b, None, 128, None, 0, 0)
    B.dsa_topk(None, 128, b, 2048, None, None, 0, 0)
    B.dsa_topk_noalloc(None, 128, b, 2048, None, 0)
    B.dsa_sparse_attn_prefill(None, B.DSA_BF16, None, None, 128, 576, 512, 0.07, None, 2048, b, None, None, None, 0, 0)
    B.dsa_sparse_attn_decode(None, B.DSA_BF16, None, None, 128, 576, 512, 0.07, None, 2048, b, None, None, None, 0, 0)
    B.dsa_cache_append(None, B.DSA_BF16, None, B.DSA_F32, 576, 128, b, None, None, None, None, 0, 0)
    assert B.dsa_launch_count() == n0
    with pytest.raises(B.DSAError) as e:      # the descriptor itself is still checked
        B.dsa_topk(None, 128, _batch(total_q=0, max_q_per_seq=0, page_size=32), 2048, None, None, 0, 0)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED


def test_cache_append_rejects_before_launch():
    b = _batch()
    P = 1 << 24
    assert B.dsa_workspace_size(B.DSA_OP_CACHE_APPEND, b) == 256
    cases = [
        (dict(Di=64), B.DSA_ERR_UNSUPPORTED),                         # only the MLA pools' key width
        (dict(Dqk=512), B.DSA_ERR_UNSUPPORTED),
        (dict(k_dt=B.DSA_FP8_E4M3), B.DSA_ERR_UNSUPPORTED),           # keys arrive unquantised
        (dict(kv_dt=B.DSA_F32), B.DSA_ERR_UNSUPPORTED),
        (dict(k_scale_pool=None), B.DSA_ERR_INVALID_ARG),
        (dict(k_new=P + 8), B.DSA_ERR_INVALID_ARG),                   # misaligned
        (dict(ws_bytes=128), B.DSA_ERR_WORKSPACE),
    ]
    for bad, status in cases:
        a = dict(kv_new=P, kv_dt=B.DSA_BF16, k_new=P, k_dt=B.DSA_F32, Dqk=576, Di=128, kv_pool=P, k_idx_pool=P,
                 k_scale_pool=P, ws=P, ws_bytes=256)
        a.update(bad)
        with pytest.raises(B.DSAError) as e:
            B.dsa_cache_append(a["kv_new"], a["kv_dt"], a["k_new"], a["k_dt"], a["Dqk"], a["Di"], b, a["kv_pool"],
                               a["k_idx_pool"], a["k_scale_pool"], a["ws"], a["ws_bytes"], 0)
        assert e.value.status == status, bad


def test_host_precheck_rejects_non_finite_inputs():
    """The optional host pre-check names the first array holding a NaN / Inf (bf16 bits, E4M3 NaN codes,
    fp32) or a non-positive key scale; clean workloads pass."""
    from sparse_attention_long_dsa_b200 import workloads as W
    from sparse_attention_long_dsa_b200.pipeline import check_inputs_finite
    wl = W.make_workload("chk", kind="mla", seed=3, seq_lens=[130, 70], q_lens=[2, 1], topk=64)
    check_inputs_finite(wl)
    check_inputs_finite(W.tiny_f32())
    plants = [("q", 0x7FC0), ("kv_pool", 0xFF80), ("qI", 0x7F), ("kI_pool", 0xFF), ("w", np.nan), ("kS_pool", np.inf),
              ("kS_pool", 0.0)]
    for name, val in plants:
        a = getattr(wl, name)
        keep = a.flat[5]
        a.flat[5] = val
        with pytest.raises(ValueError, match=name):
            check_inputs_finite(wl)
        a.flat[5] = keep
    check_inputs_finite(wl)


def test_wait_selftest_rejects_before_launch():
    P = 1 << 24
    for budget, ws_bytes, status in [(0, 256, B.DSA_ERR_INVALID_ARG), (5_000_000_000, 256, B.DSA_ERR_INVALID_ARG),
                                     (1000, 128, B.DSA_ERR_WORKSPACE)]:
        with pytest.raises(B.DSAError) as e:
            B.dsa_selftest_wait_timeout(budget, P, ws_bytes, 0)
        assert e.value.status == status


def test_context_parallel_entries_validate_before_launch():
    P = 1 << 24
    # empty batches are no-ops without a device
    B.dsa_cp_candidates(None, 128, None, 0, 16, None, None, None, 0)
    B.dsa_cp_rows(None, 2, 0, 16, None, 32, 0)
    B.dsa_cp_select_local(None, None, 2, 0, 16, None, None, None, 0)
    B.dsa_cp_merge(None, B.DSA_BF16, None, 2, 0, 128, 512, None, None, 0)
    bad = [
        (lambda: B.dsa_cp_candidates(P, 128, P, 2, 0, P, P, P, 0), B.DSA_ERR_INVALID_ARG),        # k = 0
        (lambda: B.dsa_cp_candidates(P, 128, None, 2, 16, P, P, P, 0), B.DSA_ERR_INVALID_ARG),    # NULL idx
        (lambda: B.dsa_cp_rows(P, 0, 2, 16, P, 32, 0), B.DSA_ERR_INVALID_ARG),                     # G = 0
        (lambda: B.dsa_cp_rows(P, 2, 2, 16, P, 31, 0), B.DSA_ERR_INVALID_ARG),                     # ld < G*k
        (lambda: B.dsa_cp_select_local(P, P, 2, 2, 16, None, P, P, 0), B.DSA_ERR_INVALID_ARG),     # NULL lo
        (lambda: B.dsa_cp_merge(P, B.DSA_F32, P, 2, 2, 128, 512, P, P, 0), B.DSA_ERR_UNSUPPORTED),  # f32 parts
        (lambda: B.dsa_cp_merge(P, B.DSA_BF16, P, 2, 2, 128, 6, P, P, 0), B.DSA_ERR_UNSUPPORTED),   # Dv % 4
        (lambda: B.dsa_cp_merge(P + 2, B.DSA_BF16, P, 2, 2, 128, 512, P, P, 0), B.DSA_ERR_INVALID_ARG),  # align
    ]
    for call, status in bad:
        with pytest.raises(B.DSAError) as e:
            call()
        assert e.value.status == status


def test_block_selection_entries_validate_before_launch():
    b = _batch()                                       # max_seq_len 100 -> 2 pages
    P = 1 << 24
    B.dsa_block_scores(None, 128, _batch(total_q=0, max_q_per_seq=0), None, 4, None, 0)      # empty: no-op
    B.dsa_expand_blocks(None, 2, _batch(total_q=0, max_q_per_seq=0), None, 0)
    bad = [
        (lambda: B.dsa_block_scores(P, 64, b, P, 4, P, 0), B.DSA_ERR_INVALID_ARG),          # ld_scores < 100
        (lambda: B.dsa_block_scores(P, 128, b, P, 1, P, 0), B.DSA_ERR_INVALID_ARG),         # ld_blk < 2 pages
        (lambda: B.dsa_block_scores(P, 128, b, P, 6, P, 0), B.DSA_ERR_INVALID_ARG),         # ld_blk % 4
        (lambda: B.dsa_block_scores(P, 128, b, P + 4, 4, P, 0), B.DSA_ERR_INVALID_ARG),     # alignment
        (lambda: B.dsa_block_scores(P, 128, b, P, 4, None, 0), B.DSA_ERR_INVALID_ARG),      # NULL blk_lens
        (lambda: B.dsa_expand_blocks(P, 0, b, P, 0), B.DSA_ERR_INVALID_ARG),                # kb = 0
        (lambda: B.dsa_expand_blocks(None, 2, b, P, 0), B.DSA_ERR_INVALID_ARG),
    ]
    for call, status in bad:
        with pytest.raises(B.DSAError) as e:
            call()
        assert e.value.status == status


def test_reuse_entries_validate_before_launch():
    b = _batch(total_q=2, max_q_per_seq=1)
    P = 1 << 24
    empty = _batch(total_q=0, max_q_per_seq=0)
    B.dsa_reuse_candidates(None, 16, None, 4, empty, None, None, 0, 0)
    B.dsa_indexer_scores_at(None, B.DSA_FP8_E4M3, None, None, B.DSA_FP8_E4M3, None, 64, 128, empty, None, 20, None,
                            None, 0, 0)
    B.dsa_gather_positions(None, 16, None, 20, 0, None, 0)
    bad = [
        (lambda: B.dsa_reuse_candidates(P, 16, P, 4, _batch(), P, P, 256, 0), B.DSA_ERR_INVALID_ARG),   # 2 rows/seq
        (lambda: B.dsa_reuse_candidates(P, 0, P, 4, b, P, P, 256, 0), B.DSA_ERR_INVALID_ARG),           # k = 0
        (lambda: B.dsa_reuse_candidates(P, 16, P, 4, b, P, P, 128, 0), B.DSA_ERR_WORKSPACE),
        (lambda: B.dsa_indexer_scores_at(P, B.DSA_F32, P, P, B.DSA_F32, None, 2, 32, b, P, 20, P, P, 256, 0),
         B.DSA_ERR_UNSUPPORTED),
        (lambda: B.dsa_indexer_scores_at(P, B.DSA_FP8_E4M3, P, P + 4, B.DSA_FP8_E4M3, P, 64, 128, b, P, 20, P, P, 256, 0),
         B.DSA_ERR_INVALID_ARG),
        (lambda: B.dsa_gather_positions(P, 16, None, 20, 2, P, 0), B.DSA_ERR_INVALID_ARG),
    ]
    for call, status in bad:
        with pytest.raises(B.DSAError) as e:
            call()
        assert e.value.status == status


def test_fused_append_validates_before_launch():
    b = _batch(total_q=2, max_q_per_seq=1)
    P = 1 << 24
    F8, BF, F32 = B.DSA_FP8_E4M3, B.DSA_BF16, B.DSA_F32
    B.dsa_indexer_scores_append(None, BF, None, F32, None, None, F8, None, None, F8, None, 64, 128,
                                _batch(total_q=0, max_q_per_seq=0), None, 128, None, 0, 0)          # empty: no-op
    bad = [
        (dict(k_new_dt=F8), B.DSA_ERR_UNSUPPORTED),
        (dict(Hi=32), B.DSA_ERR_UNSUPPORTED),
        (dict(kv_pool=None), B.DSA_ERR_INVALID_ARG),
        (dict(ld=64), B.DSA_ERR_INVALID_ARG),                # < max_seq_len 100
        (dict(k_new=P + 8), B.DSA_ERR_INVALID_ARG),          # alignment
        (dict(ws_bytes=16), B.DSA_ERR_WORKSPACE),
    ]
    for over, status in bad:
        a = dict(kv_new=P, k_new=P, k_new_dt=F32, kv_pool=P, Hi=64, ld=128, ws_bytes=1 << 20)
        a.update(over)
        with pytest.raises(B.DSAError) as e:
            B.dsa_indexer_scores_append(a["kv_new"], BF, a["k_new"], a["k_new_dt"], a["kv_pool"], P, F8, P, P, F8, P,
                                        a["Hi"], 128, b, P, a["ld"], P, a["ws_bytes"], 0)
        assert e.value.status == status, over


def test_fused_selection_workspace_holds_the_gather_buffers_for_long_rows():
    """dsa_indexer_topk on a batch of at most 16 rows whose longest row has 262,144 candidates or more also
    gathers each row's survivors over the SMs first: its workspace then holds 160 slots of 512 (key, position)
    pairs and their counts, and only then."""
    gather = 160 * 512 * 8 + 768            # pairs (256-byte rounded) + 160 counts (rounded to 768)
    def ws(total_q, max_seq_len):
        b = _batch(num_seqs=total_q, total_q=total_q, max_q_per_seq=1, max_seq_len=max_seq_len,
                   max_blocks_per_seq=(max_seq_len + 63) // 64)
        return B.dsa_workspace_size(B.DSA_OP_INDEXER_TOPK, b, 2048)
    assert ws(1, 262144) - ws(1, 262143) == gather
    assert ws(16, 1 << 20) - ws(16, 262143) == gather
    assert ws(17, 1 << 20) == ws(17, 262143)               # more rows: one cluster per row, no gather


def test_binding_rejects_host_and_strided_tensors_before_the_library():
    """A host tensor would give the kernels a host address and a strided view would be read as dense: the
    binding refuses both before anything reaches the library (nothing is launched)."""
    import torch
    b = _batch()
    n0 = B.dsa_launch_count()
    with pytest.raises(B.DSAError, match="device memory") as e:
        B.dsa_topk(torch.zeros(4, 128), 128, b, 16, 1 << 20, 1 << 21, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_INVALID_ARG

    class _StridedCuda:                                   # stands in for a CUDA view (no device here)
        is_cuda = True
        shape = (4, 128)

        def is_contiguous(self):
            return False

        def stride(self):
            return (1, 4)

    with pytest.raises(B.DSAError, match="dense") as e:
        B.dsa_topk(_StridedCuda(), 128, b, 16, 1 << 20, 1 << 21, 1 << 20, 0)
    assert e.value.status == B.DSA_ERR_INVALID_ARG
    assert B.dsa_launch_count() == n0
