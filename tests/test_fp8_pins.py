"""Pins for the FP8 oracle: the e4m3 cast against a value table built from
the format's definition (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
bits, subnormals at exponent 0, no infinities, 448 the largest finite value),
round-to-nearest-even by brute force, saturation, idempotence of the FP8
attention on values already in e4m3, and the P-rounding bound checked against
a direct simulation of rounding the softmax weights.

Source: developer guide, "OptimizedImplConfig" (quantized_sdpa: unscaled
float8_e4m3fn casts of Q, K, V; FP8 probabilities for P V).
"""

from __future__ import annotations

import numpy as np
import pytest

from oracle import MASK_NONE, attention_fwd
from oracle import fp8


def _e4m3_table():
    vals = set()
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # the NaN encoding of e4m3fn
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals.add(v)
            vals.add(-v)
    return np.array(sorted(vals))


TABLE = _e4m3_table()


def test_table_extremes():
    assert TABLE.max() == 448.0 and TABLE.min() == -448.0
    assert np.min(TABLE[TABLE > 0]) == 2.0 ** -9
    assert len(TABLE) == 2 * 127 - 1  # +-0 coincide


def _nearest_even(x):
    out = np.empty_like(x)
    for i, xi in enumerate(x):
        d = np.abs(TABLE - xi)
        best = np.nonzero(d == d.min())[0]
        if len(best) == 1:
            out[i] = TABLE[best[0]]
        else:  # tie: the value whose mantissa is even
            cand = TABLE[best]
            even = [c for c in cand if c == 0 or int(round(abs(c) / 2.0 ** (np.floor(np.log2(abs(c))) - 3))) % 2 == 0]
            out[i] = even[0]
    return out


def test_cast_rounds_to_nearest_even_within_range():
    g = np.random.default_rng(1)
    x = np.concatenate([g.standard_normal(3000) * s for s in (0.01, 1.0, 30.0)])
    x = x[np.abs(x) <= 448]
    np.testing.assert_array_equal(fp8.e4m3(x), _nearest_even(x))


def test_cast_exact_values_ties_and_saturation():
    np.testing.assert_array_equal(fp8.e4m3(TABLE), TABLE)
    # 1.0625 is halfway between 1.0 (mantissa 0, even) and 1.125: ties to 1.0
    assert fp8.e4m3([1.0625])[0] == 1.0
    assert fp8.e4m3([1.1875])[0] == 1.25   # halfway between 1.125 and 1.25: even is 1.25
    np.testing.assert_array_equal(fp8.e4m3([1e4, -600.0, 449.0]), [448.0, -448.0, 448.0])


def test_fp8_attention_is_attention_of_the_cast_values():
    g = np.random.default_rng(2)
    q, k, v = (g.standard_normal(s) for s in ((1, 7, 2, 16), (1, 11, 1, 16), (1, 11, 1, 16)))
    a = fp8.attention_fp8(q, k, v, 0.3)
    b = attention_fwd(fp8.e4m3(q), fp8.e4m3(k), fp8.e4m3(v), 0.3, MASK_NONE, 0)
    np.testing.assert_array_equal(a[0], b[0])
    c = fp8.attention_fp8(fp8.e4m3(q), fp8.e4m3(k), fp8.e4m3(v), 0.3)
    np.testing.assert_array_equal(a[0], c[0])


def _simulate(q, k, v, scale, shift=0.0):
    """O with P = e4m3(exp(s - m - shift)) and the unrounded row sum, m the row
    max: the rounding the bounds describe, with the reference `shift` nats
    below or above the max."""
    q8, k8, v8 = fp8.e4m3(q), fp8.e4m3(k), fp8.e4m3(v)
    o = np.zeros((q.shape[0], q.shape[1], q.shape[2], q.shape[3]))
    rep = q.shape[2] // k.shape[2]
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            s = scale * q8[b, :, h] @ k8[b, :, h // rep].T
            p = np.exp(s - s.max(axis=1, keepdims=True) - shift)
            o[b, :, h] = (fp8.e4m3(p) @ v8[b, :, h // rep]) / p.sum(axis=1, keepdims=True)
    return o


@pytest.mark.parametrize("seed,scale,shift", [(3, 32 ** -0.5, 0.0), (4, 32 ** -0.5, 0.0),
                                              (5, 1.5, 0.0), (6, 32 ** -0.5, 0.3)])
def test_p_rounding_bound_and_variance_cover_a_simulation(seed, scale, shift):
    """scale 1.5 spreads the scores so most weights fall below e4m3's smallest
    normal (2^-6): the subnormal term of the bound is what covers them."""
    g = np.random.default_rng(seed)
    q, k, v = (g.standard_normal(s) for s in ((1, 9, 2, 32), (1, 400, 2, 32), (1, 400, 2, 32)))
    o_exact, _ = fp8.attention_fp8(q, k, v, scale)
    o_sim = _simulate(q, k, v, scale, shift)
    bound = fp8.p_rounding_bound(q, k, v, scale)
    var = fp8.p_rounding_var(q, k, v, scale)
    err = np.abs(o_sim - o_exact)
    assert np.all(err <= bound + 1e-12)
    assert err.max() > 0  # the rounding is visible, the bound is not vacuous
    ratio = np.mean(err ** 2) / np.mean(var)
    assert 0.02 < ratio <= 1.0, ratio  # the variance bound holds and is not loose by orders


def test_subnormal_weights_need_the_absolute_term():
    g = np.random.default_rng(5)
    q, k, v = (g.standard_normal(s) for s in ((1, 9, 2, 32), (1, 400, 2, 32), (1, 400, 2, 32)))
    o_exact, _, w = attention_fwd(fp8.e4m3(q), fp8.e4m3(k), fp8.e4m3(v), 1.5, MASK_NONE, 0,
                                  return_weights=True)
    rel_only = 2.0 ** -4 * np.einsum("bhrk,bkhd->brhd", w, np.abs(fp8.e4m3(v)))
    err = np.abs(_simulate(q, k, v, 1.5) - o_exact)
    assert np.any(err > rel_only)  # a relative-only bound would not hold here


def test_bound_rows_are_the_rows_of_the_full_bound():
    g = np.random.default_rng(7)
    q, k, v = (g.standard_normal(s) for s in ((2, 20, 4, 16), (2, 30, 2, 16), (2, 30, 2, 16)))
    rows = [0, 7, 19]
    for mask, off in ((0, 0), (1, 10), (2, 5)):
        full = fp8.p_rounding_bound(q, k, v, 0.4, mask, off)
        part = fp8.p_rounding_bound(q, k, v, 0.4, mask, off, rows=rows)
        np.testing.assert_allclose(part, full[:, rows], rtol=1e-12, atol=0)
        fv = fp8.p_rounding_var(q, k, v, 0.4, mask, off)
        pv = fp8.p_rounding_var(q, k, v, 0.4, mask, off, rows=rows)
        np.testing.assert_allclose(pv, fv[:, rows], rtol=1e-12, atol=0)
