"""Pins for the rolling block K/V cache oracle: the fill phase equals the
streaming-chunk mask of the attention definition, hand-enumerated visible sets
for fill and post-eviction steady state, the single-chunk window, eviction and
sink effects, and storage-order invariance.

Source: flashdreams.accelerated developer guide, "Generic Multi Head Attention
Interface" (streaming example, cache storage [B, sink + window, H, d]); user
guide, "Cache lifecycle" (write before query; test fill and post-eviction).
"""

from __future__ import annotations

import numpy as np
import pytest

from oracle import MASK_CHUNK, MASK_NONE, attention_fwd
from oracle import rolling_cache as rc


def _stream(T, Hq, Hkv, d, seed):
    g = np.random.default_rng(seed)
    return (g.standard_normal((1, T, Hq, d)), g.standard_normal((1, T, Hkv, d)),
            g.standard_normal((1, T, Hkv, d)))


def test_visible_sets_hand_enumerated():
    # chunk 2, sink 2, window 4 (tokens)
    want = {0: [0, 1], 1: [0, 1, 2, 3], 2: [0, 1, 2, 3, 4, 5], 3: [0, 1, 4, 5, 6, 7],
            4: [0, 1, 6, 7, 8, 9], 7: [0, 1, 12, 13, 14, 15]}
    for c, toks in want.items():
        assert rc.visible_tokens(c, 2, 2, 4).tolist() == toks
    # no sink: a pure sliding window of two chunks
    assert rc.visible_tokens(5, 3, 0, 6).tolist() == [12, 13, 14, 15, 16, 17]


def test_steady_state_holds_sink_plus_window_tokens():
    # chunk 8, sink 16, window 32: from chunk 5 on the window starts past the sinks
    assert len(rc.visible_tokens(4, 8, 16, 32)) == 40
    for c in range(5, 30):
        v = rc.visible_tokens(c, 8, 16, 32)
        assert len(v) == 48 and len(set(v.tolist())) == 48
        assert v[:16].tolist() == list(range(16))
        assert v[-1] == 8 * c + 7


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2)])
def test_fill_phase_equals_chunk_mask_on_the_prefix(Hq, Hkv):
    C, sink, window, d = 5, 5, 20, 16
    q, k, v = _stream(4 * C, Hq, Hkv, d, 1)
    qs = [q[:, c * C:(c + 1) * C] for c in range(4)]
    got = rc.stream_attention(qs, k, v, C, sink, window, 0.25)
    for c in range(4):
        end = (c + 1) * C
        o, lse = attention_fwd(qs[c], k[:, :end], v[:, :end], 0.25, MASK_CHUNK, c * C)
        np.testing.assert_allclose(got[c][0], o, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got[c][1], lse, rtol=1e-12, atol=1e-12)


def test_single_chunk_window_without_sink_is_attention_within_the_chunk():
    C, d = 4, 8
    q, k, v = _stream(3 * C, 2, 2, d, 2)
    qs = [q[:, c * C:(c + 1) * C] for c in range(3)]
    got = rc.stream_attention(qs, k, v, C, 0, C, 0.3)
    for c in range(3):
        o, _ = attention_fwd(qs[c], k[:, c * C:(c + 1) * C], v[:, c * C:(c + 1) * C], 0.3, MASK_NONE, 0)
        np.testing.assert_allclose(got[c][0], o, rtol=1e-12, atol=1e-12)


def test_evicted_tokens_have_no_effect_and_sinks_do():
    C, sink, window, d = 3, 3, 6, 8
    q, k, v = _stream(6 * C, 2, 1, d, 3)
    qs = [q[:, c * C:(c + 1) * C] for c in range(6)]
    base = rc.stream_attention(qs, k, v, C, sink, window, 0.4)
    # token 4 (chunk 1) is out of the window from chunk 3 on
    k2, v2 = k.copy(), v.copy()
    k2[:, 4] += 5.0
    v2[:, 4] -= 3.0
    pert = rc.stream_attention(qs, k2, v2, C, sink, window, 0.4)
    for c in (3, 4, 5):
        np.testing.assert_array_equal(pert[c][0], base[c][0])
    assert not np.allclose(pert[1][0], base[1][0])
    # token 1 is a sink: every chunk sees it
    k3 = k.copy()
    k3[:, 1] += 5.0
    pert = rc.stream_attention(qs, k3, v, C, sink, window, 0.4)
    for c in range(6):
        assert not np.allclose(pert[c][0], base[c][0])


def test_storage_order_does_not_matter():
    C, sink, window, d = 4, 4, 8, 8
    q, k, v = _stream(5 * C, 2, 2, d, 4)
    c = 4
    idx = rc.visible_tokens(c, C, sink, window)
    perm = np.random.default_rng(5).permutation(len(idx))
    o1, l1 = attention_fwd(q[:, c * C:(c + 1) * C], k[:, idx], v[:, idx], 0.35, MASK_NONE, 0)
    o2, l2 = attention_fwd(q[:, c * C:(c + 1) * C], k[:, idx[perm]], v[:, idx[perm]], 0.35, MASK_NONE, 0)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bad", [dict(chunk=0), dict(sink=3), dict(window=6), dict(window=2)])
def test_sizes_must_be_whole_chunks(bad):
    kw = dict(chunk=4, sink=4, window=8)
    kw.update(bad)
    with pytest.raises(ValueError):
        rc.visible_tokens(2, kw["chunk"], kw["sink"], kw["window"])


# ------------------------------------------------------------ after-cache RoPE

def _linear_angles(R, d, base=10000.0):
    """Expanded interleaved table: feature pair r of position p at angle p * base^(-2r/d)."""
    inv = base ** (-np.arange(0, d, 2) / d)
    ang = np.repeat(np.arange(R)[:, None] * inv[None, :], 2, axis=1)
    return ang


def _rot_pairs(x, theta):
    """Interleaved rotation written as complex multiplication (x [.., d], theta [d/2])."""
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * theta)
    y = np.empty_like(x)
    y[..., 0::2], y[..., 1::2] = z.real, z.imag
    return y


def _before(q_chunks, k, v, C, sink, W, scale, ang):
    """Before-cache reference: every token rotated once at its absolute position."""
    from oracle.prologue import ROPE_INTERLEAVED, rope
    T = k.shape[1]
    kr = rope(k, ang[:T], ROPE_INTERLEAVED)
    qr = [rope(q, ang[c * C:(c + 1) * C], ROPE_INTERLEAVED) for c, q in enumerate(q_chunks)]
    return rc.stream_attention(qr, kr, v, C, sink, W, scale)


def test_after_cache_rope_without_eviction_equals_before_cache():
    """No key evicted: cache-relative positions are the absolute ones."""
    q, k, v = _stream(24, 4, 2, 16, seed=41)
    C = 8
    qc = [q[:, c * C:(c + 1) * C] for c in range(3)]
    ang = _linear_angles(24, 16)
    a = rc.stream_attention_after_rope(qc, k, v, C, 0, 24, 0.3, ang, 1)
    b = _before(qc, k, v, C, 0, 24, 0.3, ang)
    for (oa, la), (ob, lb) in zip(a, b):
        np.testing.assert_allclose(oa, ob, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(la, lb, rtol=1e-12, atol=1e-12)


def test_after_cache_rope_window_only_matches_before_cache_after_eviction():
    """RoPE scores depend on position differences only, so a sink-free window
    (cache-relative positions = absolute ones minus a constant) gives the
    before-cache result even after evictions."""
    q, k, v = _stream(40, 2, 2, 16, seed=42)
    C = 8
    qc = [q[:, c * C:(c + 1) * C] for c in range(5)]
    a = rc.stream_attention_after_rope(qc, k, v, C, 0, 16, 0.3, _linear_angles(16, 16), 1)
    b = _before(qc, k, v, C, 0, 16, 0.3, _linear_angles(40, 16))
    for (oa, la), (ob, lb) in zip(a, b):
        np.testing.assert_allclose(oa, ob, rtol=1e-9, atol=1e-9)
        np.testing.assert_allclose(la, lb, rtol=1e-9, atol=1e-9)


def test_after_cache_rope_with_sinks_brute_force():
    """With a sink the cache-relative positions close the gap between the sink
    and the window (unlike before-cache RoPE); checked against a direct loop
    over the visible keys with complex-number rotations."""
    q, k, v = _stream(32, 2, 1, 8, seed=43)
    C, sink, W = 4, 4, 8
    qc = [q[:, c * C:(c + 1) * C] for c in range(8)]
    ang = _linear_angles(12, 8)
    got = rc.stream_attention_after_rope(qc, k, v, C, sink, W, 0.4, ang, 1)
    for c in (2, 5, 7):
        vis = [t for t in range(min(sink, max(0, (c + 1) * C - W)))] + \
              list(range(max(0, (c + 1) * C - W), (c + 1) * C))
        R = len(vis)
        for h in range(2):
            for i in range(C):
                qi = _rot_pairs(qc[c][0, i, h], ang[R - C + i, 0::2])
                s = np.array([0.4 * qi @ _rot_pairs(k[0, t, 0], ang[j, 0::2]) for j, t in enumerate(vis)])
                w = np.exp(s - s.max())
                o = (w[:, None] * v[0, vis, 0]).sum(0) / w.sum()
                np.testing.assert_allclose(got[c][0][0, i, h], o, rtol=1e-10, atol=1e-12)
    before = _before(qc, k, v, C, sink, W, 0.4, _linear_angles(32, 8))
    assert np.abs(got[7][0] - before[7][0]).max() > 1e-3   # the sink's distance changed
