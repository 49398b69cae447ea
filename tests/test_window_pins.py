"""Pins for the sliding-window mode of the attention oracle (mask 3,
``window=(left, right)``, -1 = unbounded): reductions to the other masks,
PyTorch float64 SDPA with an explicit boolean mask, a pure-Python brute force,
closed forms, and keys outside the window having no effect.

Source: skill page "optimizing-attention-flash", "Sliding window attention"
(flash-attn ``window_size=(left, right)``; (-1, -1) is no window).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import (MASK_CAUSAL, MASK_NONE, MASK_WINDOW, attention_fwd, visible_pairs,
                    visible_range)


def _qkv(B, Lq, Lk, Hq, Hkv, d, seed):
    g = np.random.default_rng(seed)
    return (g.standard_normal((B, Lq, Hq, d)), g.standard_normal((B, Lk, Hkv, d)),
            g.standard_normal((B, Lk, Hkv, d)))


def test_unbounded_window_is_no_mask_and_left_only_is_causal():
    q, k, v = _qkv(1, 9, 20, 2, 1, 8, 1)
    a = attention_fwd(q, k, v, 0.3, MASK_WINDOW, 11, window=(-1, -1))
    b = attention_fwd(q, k, v, 0.3, MASK_NONE, 0)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-13)
    a = attention_fwd(q, k, v, 0.3, MASK_WINDOW, 11, window=(-1, 0))
    b = attention_fwd(q, k, v, 0.3, MASK_CAUSAL, 11)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-13)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-13)


@pytest.mark.parametrize("window,off", [((3, 2), 0), ((0, 5), 4), ((7, -1), 10), ((16, 16), 0)])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 1)])
def test_matches_torch_sdpa_with_a_boolean_mask(window, off, Hq, Hkv):
    B, Lq, Lk, d, scale = 2, 12, 30, 16, 0.25
    q, k, v = _qkv(B, Lq, Lk, Hq, Hkv, d, 2)
    o, lse = attention_fwd(q, k, v, scale, MASK_WINDOW, off, window=window)
    left, right = window
    p = off + np.arange(Lq)[:, None]
    j = np.arange(Lk)[None, :]
    vis = np.ones((Lq, Lk), dtype=bool)
    if left >= 0:
        vis &= j >= p - left
    if right >= 0:
        vis &= j <= p + right
    rep = Hq // Hkv
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).repeat_interleave(rep, dim=2).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).repeat_interleave(rep, dim=2).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(vis),
                                                           scale=scale).permute(0, 2, 1, 3)
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-10, atol=1e-10)
    s = scale * torch.einsum("bhid,bhjd->bhij", qt, kt)
    s = s.masked_fill(~torch.from_numpy(vis), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-10, atol=1e-10)


def test_brute_force_tiny():
    q, k, v = _qkv(1, 4, 9, 1, 1, 3, 3)
    o, lse = attention_fwd(q, k, v, 0.7, MASK_WINDOW, 3, window=(2, 1))
    for i in range(4):
        p = 3 + i
        js = [j for j in range(9) if p - 2 <= j <= p + 1]
        s = [0.7 * math.fsum(q[0, i, 0, c] * k[0, j, 0, c] for c in range(3)) for j in js]
        m = max(s)
        w = [math.exp(x - m) for x in s]
        tot = math.fsum(w)
        for c in range(3):
            want = math.fsum(wj * v[0, j, 0, c] for wj, j in zip(w, js)) / tot
            assert o[0, i, 0, c] == pytest.approx(want, abs=1e-12)
        assert lse[0, 0, i] == pytest.approx(m + math.log(tot), abs=1e-12)


def test_zero_width_window_returns_the_aligned_key():
    q, k, v = _qkv(1, 5, 12, 2, 2, 8, 4)
    o, lse = attention_fwd(q, k, v, 0.5, MASK_WINDOW, 6, window=(0, 0))
    for i in range(5):
        np.testing.assert_allclose(o[0, i], v[0, 6 + i], rtol=1e-14)
        for h in range(2):
            assert lse[0, h, i] == pytest.approx(0.5 * float(q[0, i, h] @ k[0, 6 + i, h]), abs=1e-12)


def test_keys_outside_the_window_have_no_effect():
    q, k, v = _qkv(1, 6, 40, 2, 1, 8, 5)
    a = attention_fwd(q, k, v, 0.4, MASK_WINDOW, 20, window=(4, 3))
    k2, v2 = k.copy(), v.copy()
    for i in range(6):
        lo, hi = visible_range(MASK_WINDOW, i, 6, 40, 20, (4, 3))
        assert (lo, hi) == (16 + i, 24 + i)
    k2[:, :16] += 3.0
    v2[:, 29:] -= 7.0
    b = attention_fwd(q, k2, v2, 0.4, MASK_WINDOW, 20, window=(4, 3))
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_visible_pairs_enumerated():
    # Lq = Lk = 6, offset 0, window (1, 1): rows see 2, 3, 3, 3, 3, 2 keys
    assert visible_pairs(6, 6, MASK_WINDOW, 0, (1, 1)) == 16
    assert visible_pairs(6, 6, MASK_CAUSAL, 0) == 21
    assert visible_pairs(6, 6, MASK_NONE, 0) == 36
