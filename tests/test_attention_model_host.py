"""The MLA attention kernel's numerical scheme, run on the CPU step by step, against the oracle's exact
attention (no GPU).

`attn_mla_kernel` walks the selected rows in 64-token chunks.  For each head two threads hold the chunk's two
32-token halves and share one running maximum (log2 units).  O is rescaled only when the chunk's maximum exceeds
the reference maximum by more than 2^8, so between rescales the unnormalised weights p = 2^(z - m_ref) may reach
2^8.  P is rounded to bf16 for the P V product, which accumulates in fp32, while l sums the unrounded p.  The
result is O / l and lse = (m_ref + log2 l) ln 2.  The GPU tests hold the kernel to the oracle within the bf16
tolerance (`tests/parity.py`: out max-abs 2e-2 and mean-rel 1e-2, lse max-abs 1e-3).  This checks that the
scheme itself meets it, with a maximum that stays flat, rises slowly (within 2^8: no rescale), rises in jumps
(rescales) or falls, with masked positions, and with the bf16 inputs of the MLA layout (values = the first Dv
latent dims; the score profile rides on a rope dim past them).
"""
import numpy as np
import pytest

import oracle

LOG2E = 1.4426950408889634


def _bf16(x):
    """Round fp32 to bf16 (nearest, ties to even) and back."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def _kernel_scheme(q, K, V, scale, valid, chunk=64, rescale_log2=8.0):
    """q [H, D], K [m, D], V [m, Dv] (bf16 values), valid [m] -> (o [H, Dv], lse [H]) as the kernel computes."""
    H, m = q.shape[0], K.shape[0]
    z = (q.astype(np.float32) @ K.astype(np.float32).T).astype(np.float32) * np.float32(scale * LOG2E)   # log2 units
    z = np.where(valid[None, :], z, -np.inf).astype(np.float32)
    O = np.zeros((H, V.shape[1]), np.float32)
    l = np.zeros(H, np.float32)
    m_ref = np.full(H, -np.inf, np.float32)
    for c0 in range(0, m, chunk):
        zc = z[:, c0:c0 + chunk]
        m_new = np.maximum(m_ref, zc.max(axis=1))
        if c0 == 0:
            m_ref = m_new
        else:
            grow = m_new > m_ref + rescale_log2
            alpha = np.where(grow, np.exp2(m_ref - m_new), 1.0).astype(np.float32)
            O *= alpha[:, None]
            l *= alpha
            m_ref = np.where(grow, m_new, m_ref)
        m_use = np.where(np.isfinite(m_ref), m_ref, 0.0).astype(np.float32)
        p = np.exp2(zc - m_use[:, None]).astype(np.float32)          # masked: 2^-inf = 0
        l += p.sum(axis=1, dtype=np.float32)
        O += _bf16(p) @ V[c0:c0 + chunk].astype(np.float32)
    o = np.where(l[:, None] > 0, O / np.where(l > 0, l, 1)[:, None], 0.0)
    lse = np.where(l > 0, (m_ref + np.log2(np.where(l > 0, l, 1))) / LOG2E, -np.inf)
    return o, lse


@pytest.mark.parametrize("profile,seed", [("flat", 11), ("slow_rise", 12), ("jumps", 13), ("fall", 14)])
def test_kernel_scheme_meets_the_bf16_tolerance(profile, seed):
    rng = np.random.default_rng(seed)
    H, D, Dv, m = 8, 64, 48, 2048                                    # MLA layout: values = first Dv dims
    scale = 1.0 / np.sqrt(D)
    q = _bf16(rng.standard_normal((H, D)))
    lat = rng.standard_normal((m, D))
    # score profile along the selected rows: how the running maximum evolves over the chunks
    t = np.arange(m) / m
    shift = {"flat": 0.0 * t, "slow_rise": 10.0 * t, "jumps": 30.0 * np.floor(8 * t), "fall": 20.0 * (1 - t)}[profile]
    # the profile rides on the last latent dim, a rope dim past the values (as in the MLA layout), so the
    # values keep their N(0, 1) magnitudes while the scores rise, jump or fall
    lat[:, D - 1] = shift * np.sqrt(D) / max(1e-9, float(np.abs(q[:, D - 1]).max()))
    K = _bf16(lat)
    V = K[:, :Dv]
    valid = rng.random(m) > 0.1                                      # masked (-1) positions
    o, lse = _kernel_scheme(q, K, V, scale, valid)
    ref_o, ref_lse = oracle.attention(q.astype(np.float64), K[valid].astype(np.float64), V[valid].astype(np.float64),
                                      scale)
    err = np.abs(o - ref_o)
    assert err.max() <= 2e-2
    assert err.sum() / np.abs(ref_o).sum() <= 1e-2
    assert np.abs(lse - ref_lse).max() <= 1e-3


def test_kernel_scheme_rescales_only_past_the_threshold():
    """With the maximum rising by less than 2^8 over the whole row, no rescale happens and the weights exceed 1;
    the result is the same as with a rescale at every chunk, to fp32 rounding."""
    rng = np.random.default_rng(5)
    H, D, m = 4, 32, 512
    q = _bf16(rng.standard_normal((H, D)))
    K = _bf16(rng.standard_normal((m, D)))
    V = K[:, :24]
    valid = np.ones(m, bool)
    o_lazy, lse_lazy = _kernel_scheme(q, K, V, 1.0 / np.sqrt(D), valid)
    o_eager, lse_eager = _kernel_scheme(q, K, V, 1.0 / np.sqrt(D), valid, rescale_log2=0.0)
    assert np.abs(o_lazy - o_eager).max() <= 4e-3
    assert np.abs(lse_lazy - lse_eager).max() <= 1e-5
